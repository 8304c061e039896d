"""Seeded synthetic workloads for paged decode attention.

This module is the ONLY thing the CUDA path and the CPU oracle share.  It
draws inputs -- shapes, N(0,1) values rounded to bf16 by torch, shuffled
physical block ids, context lengths, slot ids of the appended tokens -- and
holds none of the method's arithmetic: no attention, no quantisation, no
gather.  (Slot ids and table rows are plain bookkeeping: logical block i of a
sequence sits in physical block table[i], token t in slot table[t//bs]*bs + t%bs.)

Workloads (shaped like the pages' Llama-3-8B examples; names say what they are):

=====================  ==========================================================
tiny_gqa2_d64          2 seqs, ctx 37 and 80 cached (+1 appended each), 4 q / 2 kv
                       heads, d 64, bs 16, pool of 16 blocks in seeded random order
llama3_8b_b64          64 seqs, 32 q / 8 kv heads, d 128, bf16, bs 16,
                       ctx ~ U{512..4096} (incl. the appended token), pool 1.1x demand
long_context_b8        8 seqs, 32 / 8 heads, d 128, bf16, bs 16, ctx ~ U{32768..131072},
                       split-context partitions of 512 tokens
shared_prefix_4x8      4 prompts x 2048 tokens, each shared by 8 samples through
                       identical physical ids; private tails ~ U{0..256}
shared_prefix_16x8     16 prompts x 8 samples (unique prompt KV > L2), sharers adjacent;
 _interleaved          the same batch with each prompt's sharers 16 rows apart
fp8_mha_b32_bs{16,32,64}  32 seqs, 32 q / 32 kv heads, d 128, E4M3 cache with a
                       per-tensor fp32 scale max|x|/448, ctx 4096
int8_mha_b32_bs{16,32,64} the same shape with an INT8 cache, per-tensor scale max|x|/127
int8_mha_b32_bs16_head  INT8, bs 16, one scale per KV head: max over that head's values / 127
=====================  ==========================================================

Values: q, K, V ~ N(0, 1) drawn in fp32 by ``torch.Generator(device).manual_seed(seed)``
and rounded to bf16 by torch.  Cache slots no sequence owns (the tail of a
partially filled last block, and every block no table references) hold a NaN
sentinel, so any read of them into a result shows up.  Table entries past a
sequence's last block are -1.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import torch

BF16_NAN = 0x7FC1          # bf16 quiet NaN with a payload: the "never read this" sentinel
E4M3_NAN = 0x7F            # E4M3 NaN code
INT8_UNUSED = -128         # an INT8 code the symmetric encoder never writes
QUANT_MAX = {"e4m3": 448.0, "int8": 127.0}   # largest code magnitude: scale = max|x| / QUANT_MAX

CONFIGS = {
    "tiny_gqa2_d64": dict(B=2, h_q=4, h_kv=2, d=64, bs=16, cache="bf16", ctx_cached=(37, 80),
                          num_blocks=16, partition=0),
    "llama3_8b_b64": dict(B=64, h_q=32, h_kv=8, d=128, bs=16, cache="bf16", ctx_range=(512, 4096),
                          pool_factor=1.1, partition=2048),
    "long_context_b8": dict(B=8, h_q=32, h_kv=8, d=128, bs=16, cache="bf16",
                            ctx_range=(32768, 131072), pool_factor=1.0, partition=512),
    "shared_prefix_4x8": dict(prompts=4, samples=8, prompt_len=2048, tail_range=(0, 256), h_q=32,
                              h_kv=8, d=128, bs=16, cache="bf16", partition=512),
    # 16 prompts x 8 samples: ~134 MB of unique prompt KV, more than L2; sharers adjacent in the
    # batch ("grouped", the order pa_alloc_order_by_prefix gives) or spread over it
    "shared_prefix_16x8": dict(prompts=16, samples=8, prompt_len=2048, tail_range=(0, 256), h_q=32,
                               h_kv=8, d=128, bs=16, cache="bf16", partition=512),
    "shared_prefix_16x8_interleaved": dict(prompts=16, samples=8, prompt_len=2048, tail_range=(0, 256), h_q=32,
                                           h_kv=8, d=128, bs=16, cache="bf16", partition=512,
                                           order="interleaved"),
    "fp8_mha_b32_bs16": dict(B=32, h_q=32, h_kv=32, d=128, bs=16, cache="e4m3", ctx_fixed=4096,
                             pool_factor=1.0, partition=1024),
    "fp8_mha_b32_bs32": dict(B=32, h_q=32, h_kv=32, d=128, bs=32, cache="e4m3", ctx_fixed=4096,
                             pool_factor=1.0, partition=1024),
    "fp8_mha_b32_bs64": dict(B=32, h_q=32, h_kv=32, d=128, bs=64, cache="e4m3", ctx_fixed=4096,
                             pool_factor=1.0, partition=1024),
    "int8_mha_b32_bs16": dict(B=32, h_q=32, h_kv=32, d=128, bs=16, cache="int8", ctx_fixed=4096,
                              pool_factor=1.0, partition=1024),
    "int8_mha_b32_bs32": dict(B=32, h_q=32, h_kv=32, d=128, bs=32, cache="int8", ctx_fixed=4096,
                              pool_factor=1.0, partition=1024),
    "int8_mha_b32_bs64": dict(B=32, h_q=32, h_kv=32, d=128, bs=64, cache="int8", ctx_fixed=4096,
                              pool_factor=1.0, partition=1024),
    "int8_mha_b32_bs16_head": dict(B=32, h_q=32, h_kv=32, d=128, bs=16, cache="int8", ctx_fixed=4096,
                                   pool_factor=1.0, partition=1024, scales="head"),
}


@dataclass
class DecodeCase:
    """One decode step of a batch: caches hold every token but the last of each sequence;
    ``key_new``/``value_new`` are the appended tokens and ``slot_mapping`` their slots."""
    name: str
    B: int
    h_q: int
    h_kv: int
    d: int
    bs: int
    num_blocks: int
    cache: str                      # "bf16", "e4m3" or "int8"
    partition: int
    scale: float
    q: torch.Tensor                 # bf16 [B, h_q, d]
    key_new: torch.Tensor           # bf16 [B, h_kv, d]
    value_new: torch.Tensor         # bf16 [B, h_kv, d]
    slot_mapping: torch.Tensor      # int64 [B]
    block_tables: torch.Tensor      # int32 [B, max_blocks]
    context_lens: torch.Tensor      # int32 [B], including the appended token
    # bf16 caches: filled directly [NB, h_kv, bs, d]; quantised caches: None (each side fills
    # its own from fill_rows / fill_slots with its own quantiser)
    k_cache: Optional[torch.Tensor] = None
    v_cache: Optional[torch.Tensor] = None
    fill_k_rows: Optional[torch.Tensor] = None   # bf16 [n_fill, h_kv, d]
    fill_v_rows: Optional[torch.Tensor] = None
    fill_slots: Optional[torch.Tensor] = None    # int64 [n_fill]
    k_scale: float = 1.0            # per-tensor scales, or (scales="head") fp32 [h_kv] CPU tensors
    v_scale: float = 1.0
    meta: dict = field(default_factory=dict)

    @property
    def quantised(self) -> bool:
        return self.cache in QUANT_MAX

    @property
    def per_head_scales(self) -> bool:
        return isinstance(self.k_scale, torch.Tensor)

    @property
    def max_context_len(self) -> int:
        return int(self.context_lens.max().item()) if self.B else 0

    @property
    def elem_bytes(self) -> int:
        return 1 if self.quantised else 2

    def kv_bytes(self) -> int:
        """K+V bytes the step must read: sum of ctx * h_kv * d * elem * 2."""
        return int(self.context_lens.to(torch.int64).sum().item()) * self.h_kv * self.d * self.elem_bytes * 2


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _randn_bf16(shape, g, device) -> torch.Tensor:
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)


def _cpu_gen(seed: int) -> torch.Generator:
    g = torch.Generator()
    g.manual_seed(seed)
    return g


def _tables_from_order(order: list, blocks_per_seq: list, max_blocks: int) -> torch.Tensor:
    """Hand consecutive ids of ``order`` to the sequences in turn; -1 pads each row."""
    tab = torch.full((len(blocks_per_seq), max_blocks), -1, dtype=torch.int32)
    pos = 0
    for s, n in enumerate(blocks_per_seq):
        tab[s, :n] = torch.tensor(order[pos:pos + n], dtype=torch.int32)
        pos += n
    return tab


def _owned_slot_mask(tables: torch.Tensor, cached: torch.Tensor, num_blocks: int, bs: int) -> torch.Tensor:
    """bool [num_blocks, bs]: True where a cached (pre-append) token lives."""
    mask = torch.zeros(num_blocks, bs, dtype=torch.bool)
    for s in range(tables.shape[0]):
        n = int(cached[s])
        full, rem = divmod(n, bs)
        ids = tables[s, :full].to(torch.int64)
        mask[ids] = True
        if rem:
            mask[int(tables[s, full]), :rem] = True
    return mask


def make_case(name: str, seed: int = 0, device="cpu", **over) -> DecodeCase:
    """Build one workload.  ``over`` replaces any config entry (e.g. B=4 for a reduced case)."""
    if name not in CONFIGS:
        raise KeyError(name)
    cfg = dict(CONFIGS[name])
    cfg.update(over)
    device = torch.device(device)
    gc = _cpu_gen(seed)                    # structure (lengths, block order) always from the CPU stream

    if "prompts" in cfg:
        return _make_shared_prefix(name, cfg, seed, device, gc)

    B, h_q, h_kv, d, bs = cfg["B"], cfg["h_q"], cfg["h_kv"], cfg["d"], cfg["bs"]
    if "ctx_cached" in cfg:
        cached = torch.tensor(cfg["ctx_cached"][:B], dtype=torch.int64)
    elif "ctx_fixed" in cfg:
        cached = torch.full((B,), cfg["ctx_fixed"] - 1, dtype=torch.int64)
    else:
        lo, hi = cfg["ctx_range"]
        cached = torch.randint(lo, hi + 1, (B,), generator=gc, dtype=torch.int64) - 1
    ctx = cached + 1
    blocks_per_seq = [int(-(-int(c) // bs)) for c in ctx]
    demand = sum(blocks_per_seq)
    if "num_blocks" in cfg:
        nb = cfg["num_blocks"]
    else:
        nb = int(math.ceil(cfg.get("pool_factor", 1.0) * demand))
    if nb < demand:
        raise ValueError("pool of %d blocks cannot hold %d" % (nb, demand))
    max_blocks = max(blocks_per_seq) if blocks_per_seq else 1
    order = torch.randperm(nb, generator=gc).tolist()
    tables = _tables_from_order(order, blocks_per_seq, max_blocks)
    slots = torch.tensor([int(tables[s, int(cached[s]) // bs]) * bs + int(cached[s]) % bs
                          for s in range(B)], dtype=torch.int64)

    g = _gen(seed, device)
    q = _randn_bf16((B, h_q, d), g, device)
    k_new = _randn_bf16((B, h_kv, d), g, device)
    v_new = _randn_bf16((B, h_kv, d), g, device)
    owned = _owned_slot_mask(tables, cached, nb, bs)

    case = DecodeCase(name=name, B=B, h_q=h_q, h_kv=h_kv, d=d, bs=bs, num_blocks=nb, cache=cfg["cache"],
                      partition=cfg["partition"], scale=1.0 / math.sqrt(d), q=q, key_new=k_new,
                      value_new=v_new, slot_mapping=slots.to(device), block_tables=tables.to(device),
                      context_lens=ctx.to(torch.int32).to(device),
                      meta=dict(seed=seed, cached=cached.tolist()))
    pool_k = _randn_bf16((nb, h_kv, bs, d), g, device)
    pool_v = _randn_bf16((nb, h_kv, bs, d), g, device)
    hole = (~owned).to(device)[:, None, :, None].expand(nb, h_kv, bs, d)
    if cfg["cache"] == "bf16":
        nan = torch.tensor(BF16_NAN, dtype=torch.int16).view(torch.bfloat16).to(device)
        case.k_cache = torch.where(hole, nan, pool_k)
        case.v_cache = torch.where(hole, nan, pool_v)
    else:
        # quantised: each side quantises the owned rows itself (pool layout -> rows + slot ids).
        ids = owned.reshape(-1).nonzero().flatten()                 # slot ids of owned tokens
        blk, off = ids // bs, ids % bs
        kr = pool_k.permute(0, 2, 1, 3)[blk.to(device), off.to(device)]   # [n, h_kv, d]
        vr = pool_v.permute(0, 2, 1, 3)[blk.to(device), off.to(device)]
        case.fill_k_rows, case.fill_v_rows = kr.contiguous(), vr.contiguous()
        case.fill_slots = ids.to(torch.int64).to(device)
        set_scales(case, cfg.get("scales", "tensor"))
    return case


def set_scales(case: DecodeCase, granularity: str = "tensor") -> DecodeCase:
    """Scales of a quantised case from its fill rows and appended rows: max|x| / QUANT_MAX over
    every K (resp. V) value of the workload ("tensor", floats) or over each KV head's values
    ("head", fp32 [h_kv] CPU tensors)."""
    qmax = QUANT_MAX[case.cache]
    out = []
    for rows, new in ((case.fill_k_rows, case.key_new), (case.fill_v_rows, case.value_new)):
        a = torch.cat([rows.float().abs().reshape(-1, case.h_kv, case.d),
                       new.float().abs().reshape(-1, case.h_kv, case.d)]).cpu()
        if granularity == "head":
            out.append((a.amax(dim=(0, 2)) / qmax).to(torch.float32))
        elif granularity == "tensor":
            out.append(float((a.max() / qmax).item()))
        else:
            raise ValueError(granularity)
    case.k_scale, case.v_scale = out
    return case


def empty_quant_pool(case: DecodeCase, device=None) -> tuple[torch.Tensor, torch.Tensor]:
    """Two code pools [NB, h_kv, bs, d] filled with a code the cache write never produces:
    uint8 E4M3 NaN for "e4m3", int8 -128 for "int8"."""
    device = device if device is not None else case.q.device
    shape = (case.num_blocks, case.h_kv, case.bs, case.d)
    if case.cache == "int8":
        fill, dt = INT8_UNUSED, torch.int8
    else:
        fill, dt = E4M3_NAN, torch.uint8
    return (torch.full(shape, fill, dtype=dt, device=device), torch.full(shape, fill, dtype=dt, device=device))


def _make_shared_prefix(name, cfg, seed, device, gc) -> DecodeCase:
    """P prompts of L tokens, S samples each; the samples' tables repeat the prompt's physical
    ids (refcount S), then list private tail blocks.  L is block aligned, so tails start in
    fresh blocks and the appended token lands in a private block."""
    P, S, L = cfg["prompts"], cfg["samples"], cfg["prompt_len"]
    h_q, h_kv, d, bs = cfg["h_q"], cfg["h_kv"], cfg["d"], cfg["bs"]
    B = P * S
    lo, hi = cfg["tail_range"]
    tails = torch.randint(lo, hi + 1, (B,), generator=gc, dtype=torch.int64)
    cached = L + tails                       # prompt + generated tail, before this step
    ctx = cached + 1
    pblocks = -(-L // bs)
    private = [int(-(-int(c) // bs)) - pblocks for c in ctx]
    nb = P * pblocks + sum(private)
    order = torch.randperm(nb, generator=gc).tolist()
    max_blocks = pblocks + max(private)
    tables = torch.full((B, max_blocks), -1, dtype=torch.int32)
    pos = P * pblocks
    for p in range(P):
        pids = torch.tensor(order[p * pblocks:(p + 1) * pblocks], dtype=torch.int32)
        for j in range(S):
            s = p * S + j
            tables[s, :pblocks] = pids
            n = private[s]
            tables[s, pblocks:pblocks + n] = torch.tensor(order[pos:pos + n], dtype=torch.int32)
            pos += n
    if cfg.get("order") == "interleaved":
        # batch row r holds sample r // P of prompt r % P: a prompt's sharers are P rows apart
        perm = torch.tensor([p * S + j for j in range(S) for p in range(P)])
        tables, cached, ctx = tables[perm], cached[perm], ctx[perm]
    slots = torch.tensor([int(tables[s, int(cached[s]) // bs]) * bs + int(cached[s]) % bs
                          for s in range(B)], dtype=torch.int64)
    owned = _owned_slot_mask(tables, cached, nb, bs)
    g = _gen(seed, device)
    q = _randn_bf16((B, h_q, d), g, device)
    k_new = _randn_bf16((B, h_kv, d), g, device)
    v_new = _randn_bf16((B, h_kv, d), g, device)
    pool_k = _randn_bf16((nb, h_kv, bs, d), g, device)
    pool_v = _randn_bf16((nb, h_kv, bs, d), g, device)
    hole = (~owned).to(device)[:, None, :, None].expand(nb, h_kv, bs, d)
    nan = torch.tensor(BF16_NAN, dtype=torch.int16).view(torch.bfloat16).to(device)
    return DecodeCase(name=name, B=B, h_q=h_q, h_kv=h_kv, d=d, bs=bs, num_blocks=nb, cache="bf16",
                      partition=cfg["partition"], scale=1.0 / math.sqrt(d), q=q, key_new=k_new,
                      value_new=v_new, slot_mapping=slots.to(device), block_tables=tables.to(device),
                      context_lens=ctx.to(torch.int32).to(device),
                      k_cache=torch.where(hole, nan, pool_k), v_cache=torch.where(hole, nan, pool_v),
                      meta=dict(seed=seed, cached=cached.tolist(), prompts=P, samples=S,
                                prompt_blocks=pblocks, unique_tokens=P * L + int(tails.sum()) + B))


def random_rows(n: int, h_kv: int, d: int, seed: int, device="cpu") -> tuple[torch.Tensor, torch.Tensor]:
    """K and V rows ~ N(0,1) in bf16, [n, h_kv, d] each (for cache-write cases)."""
    g = _gen(seed, torch.device(device))
    return _randn_bf16((n, h_kv, d), g, device), _randn_bf16((n, h_kv, d), g, device)


# ---------------------------------------------------------------------------- serving traces
# Request-length traces for the memory-utilisation measurement (host only).  Each request has a
# prompt length and an output length; the context window bounds prompt + output.  The pages give
# no length distribution, so the recipes are plain seeded uniforms whose names say what they are.
TRACES = {
    # a chat-like mix in a 2048-token window: prompts U{32..512}, outputs U{16..1024}
    "chat_w2048_b64": dict(requests=512, slots=64, window=2048, prompt=(32, 512), output=(16, 1024), bs=16),
    # the same mix, 8 concurrent requests (the pages' "8 concurrent requests" setting)
    "chat_w2048_b8": dict(requests=64, slots=8, window=2048, prompt=(32, 512), output=(16, 1024), bs=16),
    # long answers in a 4096-token window: prompts U{256..1024}, outputs U{512..3072}
    "long_w4096_b32": dict(requests=128, slots=32, window=4096, prompt=(256, 1024), output=(512, 3072), bs=16),
}


@dataclass
class Trace:
    name: str
    prompts: list           # prompt length of request i
    outputs: list           # output length of request i (>= 1)
    slots: int              # concurrent request slots (continuous batching)
    window: int             # context window: the contiguous scheme reserves this per request
    bs: int


def make_trace(name: str, seed: int = 0, **over) -> Trace:
    cfg = dict(TRACES[name])
    cfg.update(over)
    g = _cpu_gen(seed)
    n = cfg["requests"]
    p = torch.randint(cfg["prompt"][0], cfg["prompt"][1] + 1, (n,), generator=g).tolist()
    o = torch.randint(cfg["output"][0], cfg["output"][1] + 1, (n,), generator=g).tolist()
    if any(a + b > cfg["window"] for a, b in zip(p, o)):
        raise ValueError("a request exceeds the window")
    return Trace(name=name, prompts=p, outputs=o, slots=cfg["slots"], window=cfg["window"], bs=cfg["bs"])


# ------------------------------------------------------------------ prompts sharing a prefix
# Prompt token ids for the prefix-caching measurement: a system prompt, then one of a few long
# documents, then a short question ("vLLM 推理原理…" section 前缀缓存能省掉哪部分工作: fix the
# system text and the document, vary only the final question).  With front_changed=True every
# request's document gets its own first tokens, so only the system prompt can match.
PREFIX_TRACES = {
    "sys256_doc1536x4_q64_n64": dict(requests=64, system=256, docs=4, doc=1536, question=(16, 64), bs=16),
}


def make_prefix_prompts(name: str, seed: int = 0, front_changed: bool = False) -> list:
    cfg = PREFIX_TRACES[name]
    g = _cpu_gen(seed)
    vocab = 32000
    system = torch.randint(0, vocab, (cfg["system"],), generator=g).tolist()
    docs = [torch.randint(0, vocab, (cfg["doc"],), generator=g).tolist() for _ in range(cfg["docs"])]
    prompts = []
    for i in range(cfg["requests"]):
        doc = list(docs[int(torch.randint(0, cfg["docs"], (1,), generator=g))])
        if front_changed:
            doc[:8] = torch.randint(0, vocab, (8,), generator=g).tolist()
        nq = int(torch.randint(cfg["question"][0], cfg["question"][1] + 1, (1,), generator=g))
        prompts.append(system + doc + torch.randint(0, vocab, (nq,), generator=g).tolist())
    return prompts


# ---------------------------------------------------------------------------- prefill chunks
# Chunked prefill: every sequence already holds `cached` tokens and appends a chunk of new
# tokens whose query rows attend causally to the whole prefix (the chunk included).
PREFILL_CONFIGS = {
    # 8 sequences, each appending a 512-token chunk to a cached prefix of U{0..3584} tokens
    "prefill_llama3_8b_b8_chunk512": dict(B=8, h_q=32, h_kv=8, d=128, bs=16, cached=(0, 3584), chunk=(512, 512),
                                          pool_factor=1.1),
    # whole prompts of U{256..2048} tokens, nothing cached
    "prefill_llama3_8b_b8_prompt": dict(B=8, h_q=32, h_kv=8, d=128, bs=16, cached=(0, 0), chunk=(256, 2048),
                                        pool_factor=1.1),
}


@dataclass
class PrefillCase:
    name: str
    B: int
    h_q: int
    h_kv: int
    d: int
    bs: int
    num_blocks: int
    scale: float
    q: torch.Tensor                 # bf16 [T, h_q, d]: the chunks' query rows, stacked
    key_new: torch.Tensor           # bf16 [T, h_kv, d]: the chunks' K rows
    value_new: torch.Tensor
    slot_mapping: torch.Tensor      # int64 [T]
    query_start: torch.Tensor       # int32 [B + 1]
    context_lens: torch.Tensor      # int32 [B], including the chunk
    block_tables: torch.Tensor      # int32 [B, max_blocks]
    k_cache: torch.Tensor           # bf16 [NB, h_kv, bs, d] holding the cached prefixes (NaN elsewhere)
    v_cache: torch.Tensor
    meta: dict = field(default_factory=dict)

    @property
    def max_query_len(self) -> int:
        return int((self.query_start[1:] - self.query_start[:-1]).max().item()) if self.B else 0

    def attention_flops(self) -> int:
        """4 d (p + 1) per query row and head (Q K^T and P V over the p + 1 visible tokens)."""
        qs = self.query_start.cpu().tolist()
        ctx = self.context_lens.cpu().tolist()
        tot = 0
        for s in range(self.B):
            n = qs[s + 1] - qs[s]
            first = ctx[s] - n + 1                  # tokens seen by the chunk's first row
            tot += n * first + n * (n - 1) // 2
        return 4 * self.d * self.h_q * tot


def make_prefill_case(name: str, seed: int = 0, device="cpu", **over) -> PrefillCase:
    cfg = dict(PREFILL_CONFIGS[name])
    cfg.update(over)
    device = torch.device(device)
    gc = _cpu_gen(seed)
    B, h_q, h_kv, d, bs = cfg["B"], cfg["h_q"], cfg["h_kv"], cfg["d"], cfg["bs"]
    cached = torch.randint(cfg["cached"][0], cfg["cached"][1] + 1, (B,), generator=gc, dtype=torch.int64)
    chunk = torch.randint(cfg["chunk"][0], cfg["chunk"][1] + 1, (B,), generator=gc, dtype=torch.int64)
    ctx = cached + chunk
    blocks_per_seq = [int(-(-int(c) // bs)) for c in ctx]
    nb = max(1, int(math.ceil(cfg.get("pool_factor", 1.0) * sum(blocks_per_seq))))
    order = torch.randperm(nb, generator=gc).tolist()
    tables = _tables_from_order(order, blocks_per_seq, max(blocks_per_seq) if blocks_per_seq else 1)
    qs = torch.zeros(B + 1, dtype=torch.int64)
    qs[1:] = torch.cumsum(chunk, 0)
    slots = []
    for s in range(B):
        for t in range(int(cached[s]), int(ctx[s])):
            slots.append(int(tables[s, t // bs]) * bs + t % bs)
    T = int(qs[-1])
    g = _gen(seed, device)
    q = _randn_bf16((T, h_q, d), g, device)
    k_new = _randn_bf16((T, h_kv, d), g, device)
    v_new = _randn_bf16((T, h_kv, d), g, device)
    pool_k = _randn_bf16((nb, h_kv, bs, d), g, device)
    pool_v = _randn_bf16((nb, h_kv, bs, d), g, device)
    owned = _owned_slot_mask(tables, cached, nb, bs)
    hole = (~owned).to(device)[:, None, :, None].expand(nb, h_kv, bs, d)
    nan = torch.tensor(BF16_NAN, dtype=torch.int16).view(torch.bfloat16).to(device)
    return PrefillCase(name=name, B=B, h_q=h_q, h_kv=h_kv, d=d, bs=bs, num_blocks=nb, scale=1.0 / math.sqrt(d),
                       q=q, key_new=k_new, value_new=v_new,
                       slot_mapping=torch.tensor(slots, dtype=torch.int64).to(device),
                       query_start=qs.to(torch.int32).to(device), context_lens=ctx.to(torch.int32).to(device),
                       block_tables=tables.to(device), k_cache=torch.where(hole, nan, pool_k),
                       v_cache=torch.where(hole, nan, pool_v),
                       meta=dict(seed=seed, cached=cached.tolist(), chunk=chunk.tolist()))
