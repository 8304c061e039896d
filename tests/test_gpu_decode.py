"""GPU decode attention against the fp64 oracle, on every workload shape, plus the
invariants the method fixes (through the C ABI)."""
import math

import numpy as np
import pytest
import torch

import workloads
import paged_kv_cache_428_b200 as pa
from paritylib import (check_close, codes, gpu_step, oracle_caches, oracle_out, u16, u8)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _full_parity(orc, case, rows=None, seqs=None, **kw):
    out, kc, vc = gpu_step(case, **kw)
    torch.cuda.synchronize()
    okc, ovc = oracle_caches(case, orc, seqs=seqs)
    if seqs is None:                                       # the step's cache writes are bit-exact
        assert np.array_equal(codes(kc, case.cache), okc) and np.array_equal(codes(vc, case.cache), ovc)
    ref = oracle_out(case, orc, okc, ovc, rows)
    got = out if rows is None else torch.stack([out[s, h] for s, h in rows])
    return check_close(got, ref, case.cache == "e4m3", case.name)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_tiny_gqa2_d64(orc, seed):
    case = workloads.make_case("tiny_gqa2_d64", seed)
    _full_parity(orc, case)
    # decode before the append too (contexts 37 and 80), and with split partitions
    case_b = workloads.make_case("tiny_gqa2_d64", seed)
    case_b.context_lens = torch.tensor(case_b.meta["cached"], dtype=torch.int32)
    case_b.slot_mapping = torch.full_like(case_b.slot_mapping, -1)
    _full_parity(orc, case_b)
    _full_parity(orc, case, partition_size=16)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_llama3_8b_b64_full(orc, seed):
    """The benchmarked workload at full size, in the launch configuration bench.py times."""
    case = workloads.make_case("llama3_8b_b64", seed, device=DEV)
    _full_parity(orc, case)


def test_long_context_b8_sampled(orc):
    case = workloads.make_case("long_context_b8", 0, device=DEV)
    rows = [(s, h) for s in (0, 5) for h in (0, 3, 4, 17, 31)] + [(7, 8), (2, 30)]
    _full_parity(orc, case, rows=rows)


def test_long_context_b8_full_size_all_rows(orc):
    """The long-context workload at full size (8 sequences of U{32768..131072} tokens, 2.7 GB of
    K/V, 512-token partitions: up to 256 per sequence, combined by the separate merge pass),
    every (sequence, query head) row against the oracle, in the launch configuration
    bench.py times."""
    case = workloads.make_case("long_context_b8", 0, device=DEV)
    _full_parity(orc, case)


@pytest.mark.parametrize("seed", [0, 1])
def test_long_context_reduced_all_rows(orc, seed):
    case = workloads.make_case("long_context_b8", seed, B=2, ctx_range=(20000, 40000))
    _full_parity(orc, case)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_shared_prefix_4x8(orc, seed):
    case = workloads.make_case("shared_prefix_4x8", seed, device=DEV)
    _full_parity(orc, case)


@pytest.mark.parametrize("name", ["shared_prefix_16x8", "shared_prefix_16x8_interleaved"])
def test_shared_prefix_16x8_sampled(orc, name):
    case = workloads.make_case(name, 0, device=DEV)
    g = torch.Generator().manual_seed(3)
    seqs = sorted(set(torch.randint(0, case.B, (6,), generator=g).tolist()))
    rows = [(s, h) for s in seqs for h in (0, 9, 31)]
    _full_parity(orc, case, rows=rows)


@pytest.mark.parametrize("bs", [16, 32, 64])
def test_fp8_mha_b32_sampled_full_size(orc, bs):
    case = workloads.make_case("fp8_mha_b32_bs%d" % bs, 0, device=DEV)
    seqs = {0, 13, 31}
    rows = [(s, h) for s in sorted(seqs) for h in (0, 7, 19, 31)]
    _full_parity(orc, case, rows=rows, seqs=seqs)


def test_fp8_mha_b32_bs16_full_size_all_rows(orc):
    """The E4M3 MHA workload at full size (32 sequences x 4096 tokens x 32 KV heads, 1.07 GB of
    codes), every row against the oracle evaluated on its own quantised cache."""
    case = workloads.make_case("fp8_mha_b32_bs16", 0, device=DEV)
    _full_parity(orc, case)


@pytest.mark.parametrize("bs", [16, 32, 64])
@pytest.mark.parametrize("seed", [1, 2])
def test_fp8_mha_reduced_all_rows(orc, bs, seed):
    case = workloads.make_case("fp8_mha_b32_bs%d" % bs, seed, B=3, ctx_fixed=1000)
    _full_parity(orc, case)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("bs", [16, 32, 64])
@pytest.mark.parametrize("g", [1, 2, 4, 8])
@pytest.mark.parametrize("cache", ["bf16", "e4m3", "int8"])
def test_every_kernel_variant(orc, d, bs, g, cache):
    """Small ragged cases over the whole supported shape grid (each template instance)."""
    h_kv = 2
    case = workloads.make_case("llama3_8b_b64", 7 * d + bs + g, B=5, h_q=h_kv * g, h_kv=h_kv, d=d, bs=bs,
                               ctx_range=(1, 700), pool_factor=1.3, partition=128 if bs <= 64 else 0)
    if cache != "bf16":
        case = _as_quant(case, cache)
    _full_parity(orc, case)
    _full_parity(orc, case, partition_size=0)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("bs", [16, 64])
@pytest.mark.parametrize("cache", ["e4m3", "int8"])
def test_per_head_scales(orc, d, bs, cache):
    """Quantised caches with one scale per KV head (pa_*_head_scales) against the oracle; the
    heads' ranges are made to differ by 20x so that a wrong head's scale shows."""
    h_kv, g = 4, 2
    case = workloads.make_case("llama3_8b_b64", 11 * d + bs, B=4, h_q=h_kv * g, h_kv=h_kv, d=d, bs=bs,
                               ctx_range=(1, 600), pool_factor=1.2, partition=128)
    spread = torch.tensor([1.0, 20.0, 0.3, 5.0]).to(case.k_cache.device)[None, :, None, None]
    case.k_cache = (case.k_cache.float() * spread).to(torch.bfloat16)
    case.v_cache = (case.v_cache.float() * spread.flip(1)).to(torch.bfloat16)
    case.key_new = (case.key_new.float() * spread[:, :, :, 0]).to(torch.bfloat16)
    case.value_new = (case.value_new.float() * spread.flip(1)[:, :, :, 0]).to(torch.bfloat16)
    case = _as_quant(case, cache, "head")
    assert case.per_head_scales and float(case.k_scale.max() / case.k_scale.min()) > 10
    _full_parity(orc, case)
    _full_parity(orc, case, partition_size=0)


def _as_quant(case, cache, granularity="tensor"):
    """Turn a bf16 case into a quantised one: the same rows become fill rows."""
    bs = case.bs
    kc, vc = case.k_cache, case.v_cache
    owned = ~torch.isnan(kc.float()).all(dim=3).all(dim=1)            # [nb, bs]
    ids = owned.reshape(-1).nonzero().flatten()
    blk, off = ids // bs, ids % bs
    case.fill_k_rows = kc.permute(0, 2, 1, 3)[blk, off].contiguous()
    case.fill_v_rows = vc.permute(0, 2, 1, 3)[blk, off].contiguous()
    case.fill_slots = ids.to(torch.int64)
    case.cache = cache
    workloads.set_scales(case, granularity)
    case.k_cache = case.v_cache = None
    return case



@pytest.mark.parametrize("bs", [16, 32, 64])
def test_int8_mha_b32_sampled_full_size(orc, bs):
    case = workloads.make_case("int8_mha_b32_bs%d" % bs, 0, device=DEV)
    g = torch.Generator().manual_seed(bs)
    rows = [(int(s), int(h)) for s, h in zip(torch.randint(0, case.B, (48,), generator=g),
                                             torch.randint(0, case.h_q, (48,), generator=g))]
    seqs = sorted({s for s, _ in rows})
    _full_parity(orc, case, rows=rows, seqs=seqs)


@pytest.mark.parametrize("bs", [16, 32, 64])
@pytest.mark.parametrize("seed", [0, 1])
def test_int8_mha_reduced_all_rows(orc, bs, seed):
    case = workloads.make_case("int8_mha_b32_bs%d" % bs, seed, B=3, ctx_fixed=777, h_q=8, h_kv=8)
    _full_parity(orc, case)


def test_int8_per_head_workload_sampled(orc):
    case = workloads.make_case("int8_mha_b32_bs16_head", 0, device=DEV)
    assert case.per_head_scales
    g = torch.Generator().manual_seed(5)
    rows = [(int(s), int(h)) for s, h in zip(torch.randint(0, case.B, (32,), generator=g),
                                             torch.randint(0, case.h_q, (32,), generator=g))]
    _full_parity(orc, case, rows=rows, seqs=sorted({s for s, _ in rows}))


# ---------------------------------------------------------------- invariants and special cases

def _with_appended(case):
    """Write the case's appended tokens into its (device) caches, in place, so that every
    slot below the context length holds data; returns the case."""
    pa.pa_reshape_and_cache(case.key_new.to(DEV), case.value_new.to(DEV), case.k_cache, case.v_cache,
                            case.slot_mapping.to(DEV))
    return case


def _decode(case, kc, vc, tables=None, P=None, ctx=None, mcl=None):
    out = torch.empty((case.B, case.h_q, case.d), dtype=torch.bfloat16, device=DEV)
    tab = (case.block_tables if tables is None else tables).to(DEV)
    cl = (case.context_lens if ctx is None else ctx).to(DEV)
    pa.pa_decode(out, case.q.to(DEV), kc, vc, tab, cl, case.max_context_len if mcl is None else mcl, case.scale,
                 case.partition if P is None else P, case.k_scale, case.v_scale)
    torch.cuda.synchronize()
    return out


def test_permutation_invariance_bitwise():
    case = _with_appended(workloads.make_case("llama3_8b_b64", 4, device=DEV, B=16))
    kc, vc = case.k_cache, case.v_cache
    out1 = _decode(case, kc, vc)
    perm = torch.randperm(case.num_blocks, generator=torch.Generator().manual_seed(1)).to(DEV)
    kc2, vc2 = torch.empty_like(kc), torch.empty_like(vc)
    kc2[perm], vc2[perm] = kc, vc
    tab = case.block_tables
    tab2 = torch.where(tab >= 0, perm[tab.clamp(min=0).long()].to(torch.int32), tab)
    out2 = _decode(case, kc2, vc2, tables=tab2)
    assert torch.isfinite(out1.float()).all()
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))


def test_contiguous_physical_blocks_give_the_same_bits():
    """Identity placement (logical block i in physical block i of each row) vs the shuffled
    pool: the result does not depend on where blocks live."""
    case = _with_appended(workloads.make_case("llama3_8b_b64", 6, device=DEV, B=8))
    out1 = _decode(case, case.k_cache, case.v_cache)
    tab = case.block_tables.cpu()
    nblk = [-(-int(c) // case.bs) for c in case.context_lens.cpu()]
    order = [b for s in range(case.B) for b in tab[s, :nblk[s]].tolist()]
    kc2 = torch.empty_like(case.k_cache)
    vc2 = torch.empty_like(case.v_cache)
    src = torch.tensor(order, device=DEV)
    kc2[: len(order)], vc2[: len(order)] = case.k_cache[src], case.v_cache[src]
    tab2 = torch.full_like(tab, -1)
    pos = 0
    for s in range(case.B):
        tab2[s, :nblk[s]] = torch.arange(pos, pos + nblk[s], dtype=torch.int32)
        pos += nblk[s]
    out2 = _decode(case, kc2, vc2, tables=tab2)
    assert torch.isfinite(out1.float()).all()
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))


def test_shared_vs_privately_copied_prefix_bitwise():
    """Samples reading one refcounted prefix vs samples whose prefix blocks were copied
    with pa_copy_blocks into private blocks: identical blocks and identical outputs."""
    case = _with_appended(workloads.make_case("shared_prefix_4x8", 1, device=DEV))
    kc, vc = case.k_cache, case.v_cache
    out_shared = _decode(case, kc, vc)
    pb = case.meta["prompt_blocks"]
    S = case.meta["samples"]
    tab = case.block_tables.cpu().clone()
    extra = (S - 1) * case.meta["prompts"] * pb
    nb2 = case.num_blocks + extra
    kc2 = torch.cat([kc, torch.empty((extra,) + tuple(kc.shape[1:]), dtype=kc.dtype, device=DEV)])
    vc2 = torch.cat([vc, torch.empty((extra,) + tuple(vc.shape[1:]), dtype=vc.dtype, device=DEV)])
    nxt = case.num_blocks
    pairs = []
    for s in range(case.B):
        if s % S == 0:
            continue                                     # the first sample keeps the originals
        for i in range(pb):
            pairs.append((int(tab[s, i]), nxt))
            tab[s, i] = nxt
            nxt += 1
    pa.pa_copy_blocks([kc2], [vc2], torch.tensor(pairs, dtype=torch.int64, device=DEV))
    for a, b in pairs[:50]:
        assert torch.equal(kc2[a].view(torch.int16), kc2[b].view(torch.int16))
    case.num_blocks = nb2
    out_private = _decode(case, kc2, vc2, tables=tab)
    assert torch.isfinite(out_shared.float()).all()
    assert torch.equal(out_shared.view(torch.int16), out_private.view(torch.int16))


def _mean_abs_v_under_softmax(case, kc, vc):
    """sum_t p_t |V_t| / sum_t p_t per (sequence, query head, dim), by plain torch on the
    gathered rows: the scale of the error that rounding the probabilities to bf16 can cause."""
    g = case.h_q // case.h_kv
    out = torch.empty((case.B, case.h_q, case.d), dtype=torch.float32, device=DEV)
    tab = case.block_tables.to(DEV).long()
    for s in range(case.B):
        n = int(case.context_lens[s])
        blocks = tab[s, : -(-n // case.bs)]
        K = kc[blocks].permute(0, 2, 1, 3).reshape(-1, case.h_kv, case.d)[:n].float()   # [n, h_kv, d]
        V = vc[blocks].permute(0, 2, 1, 3).reshape(-1, case.h_kv, case.d)[:n].float()
        q = case.q[s].to(DEV).float().view(case.h_kv, g, case.d)
        logits = torch.einsum("hgd,nhd->hgn", q, K) * case.scale
        w = torch.softmax(logits, dim=-1)
        out[s] = torch.einsum("hgn,nhd->hgd", w, V.abs()).reshape(case.h_q, case.d)
    return out


def test_split_vs_unsplit_agree():
    """Split vs unsplit context: the same attention ("现代 AI 的“推理加速之谜”…" section 1,
    softmax(q K^T / sqrt(d)) V) evaluated with different partition sizes.

    Bound, derived from the kernel's arithmetic: p.V runs on the tensor cores with the
    probabilities p_t rounded to the operand type of V (bf16, unit roundoff 2^-9), while the
    normaliser l sums the unrounded fp32 p_t.  One evaluation's result therefore differs from
    exact fp32 arithmetic by at most |sum_t (p~_t - p_t) V_t| / sum_t p_t <= 2^-9 * wbar, with
    wbar = sum_t p_t |V_t| / sum_t p_t.  Two partitionings round against different running
    maxima, so their fp32 results differ by at most 2 * 2^-9 * wbar (plus fp32 reordering, the
    1e-6 term); each is then rounded to bf16 (half an ulp, at most 2^-8 |x|), giving
    2^-7 * max(|a|, |b|) + 2^-8 * wbar.  The oracle tolerance (2e-2) is unchanged; this bound
    is about 3e-3 at these magnitudes."""
    case = _with_appended(workloads.make_case("llama3_8b_b64", 2, device=DEV, B=24))
    ref = _decode(case, case.k_cache, case.v_cache, P=0).float()
    wbar = _mean_abs_v_under_softmax(case, case.k_cache, case.v_cache)
    for P in (16, 64, 256, 512, 2048, AUTO):
        got = _decode(case, case.k_cache, case.v_cache, P=P).float()
        assert torch.isfinite(got).all()
        tol = 2.0 ** -7 * torch.maximum(ref.abs(), got.abs()) + 2.0 ** -8 * wbar + 1e-6
        excess = ((got - ref).abs() - tol).max().item()
        assert excess <= 0, (P, excess)


def test_context_hint_smaller_than_real_context(orc):
    """max_context_len only sizes the grid: a longer context is still attended in full."""
    case = workloads.make_case("llama3_8b_b64", 3, B=6, ctx_range=(700, 3000))
    out, kc, vc = gpu_step(case, max_context_len=600)
    okc, ovc = oracle_caches(case, orc)
    check_close(out, oracle_out(case, orc, okc, ovc), False, "short hint")


def test_single_token_context_returns_v0_exactly():
    case = workloads.make_case("tiny_gqa2_d64", 0, device=DEV)
    ctx = torch.tensor([1, 1], dtype=torch.int32)
    out = _decode(case, case.k_cache, case.v_cache, ctx=ctx, P=0)
    tab = case.block_tables.cpu()
    g = case.h_q // case.h_kv
    for s in range(case.B):
        for h in range(case.h_q):
            v0 = case.v_cache[int(tab[s, 0]), h // g, 0]
            assert torch.equal(out[s, h].view(torch.int16), v0.view(torch.int16))


def test_zero_query_gives_mean_of_v(orc):
    case = workloads.make_case("llama3_8b_b64", 8, B=4)
    case.q = torch.zeros_like(case.q)
    out, kc, vc = gpu_step(case)
    okc, ovc = oracle_caches(case, orc)
    ref = oracle_out(case, orc, okc, ovc)
    check_close(out, ref, False, "q=0")


def test_empty_context_gives_zeros():
    case = _with_appended(workloads.make_case("llama3_8b_b64", 9, device=DEV, B=4))
    ctx = case.context_lens.clone()
    ctx[1] = 0
    ctx[3] = 0
    out = _decode(case, case.k_cache, case.v_cache, ctx=ctx)
    assert torch.count_nonzero(out[1].float()) == 0 and torch.count_nonzero(out[3].float()) == 0
    assert torch.isfinite(out.float()).all()


def test_bad_block_id_is_skipped_and_flagged():
    case = _with_appended(workloads.make_case("llama3_8b_b64", 10, device=DEV, B=3))
    tab = case.block_tables.clone()
    tab[1, 2] = case.num_blocks + 7                          # outside the pool
    pa.pa_device_errors(clear=True)
    out = _decode(case, case.k_cache, case.v_cache, tables=tab)
    assert pa.pa_device_errors(clear=True) & pa.PA_DEVERR_BAD_BLOCK
    assert torch.isnan(out[1].float()).all()                  # the damaged sequence is poisoned
    ok = _decode(case, case.k_cache, case.v_cache)
    assert torch.equal(out[0].view(torch.int16), ok[0].view(torch.int16))
    assert torch.equal(out[2].view(torch.int16), ok[2].view(torch.int16))
    assert pa.pa_device_errors(clear=True) == 0


def test_sentinel_slots_never_reach_the_result():
    """Unowned slots hold NaN; outputs stay finite for every partition size."""
    case = _with_appended(workloads.make_case("llama3_8b_b64", 12, device=DEV, B=8))
    for P in (0, 16, 512):
        assert torch.isfinite(_decode(case, case.k_cache, case.v_cache, P=P).float()).all()


def test_workspace_reused_across_calls(orc):
    """One workspace for many calls: the per-group counters of the in-kernel merge are left at
    zero by every call, so consecutive calls with different inputs stay exact."""
    ws = None
    for seed in (31, 32, 33):
        case = workloads.make_case("llama3_8b_b64", seed, B=12, ctx_range=(600, 4000))
        out, kc, vc = gpu_step(case)            # warm the kernels; fresh workspace inside
        if ws is None:
            ws = pa.make_workspace(case.B, case.h_q, case.d, 4096, case.partition, DEV)
        out2 = torch.empty_like(out)
        pa.pa_decode(out2, case.q.to(DEV), kc, vc, case.block_tables.to(DEV), case.context_lens.to(DEV), 4096,
                     case.scale, case.partition, workspace=ws)
        torch.cuda.synchronize()
        okc, ovc = oracle_caches(case, orc)
        check_close(out2, oracle_out(case, orc, okc, ovc), False, "reuse %d" % seed)
        assert torch.equal(out.view(torch.int16), out2.view(torch.int16))
    counters = ws[: case.B * case.h_q * 4].view(torch.int32)
    assert int(counters.abs().sum()) == 0


# ---------------------------------------------------------------- balanced schedule (AUTO)
AUTO = -1


@pytest.mark.parametrize("name,kw", [
    ("tiny_gqa2_d64", {}),
    ("llama3_8b_b64", {}),
    ("llama3_8b_b64", dict(B=3, ctx_range=(1, 90))),          # tiny groups, many per CTA
    ("llama3_8b_b64", dict(B=1, ctx_range=(60000, 60000))),    # one group over every CTA
    ("shared_prefix_4x8", {}),
])
def test_auto_schedule_parity(orc, name, kw):
    case = workloads.make_case(name, 5, device=DEV, **kw)
    _full_parity(orc, case, partition_size=AUTO)


def test_auto_schedule_long_context_sampled(orc):
    case = workloads.make_case("long_context_b8", 1, device=DEV)
    rows = [(s, h) for s in (1, 6) for h in (0, 9, 31)] + [(3, 5)]
    _full_parity(orc, case, rows=rows, partition_size=AUTO)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("bs", [16, 32, 64])
@pytest.mark.parametrize("g", [1, 2, 4, 8])
def test_auto_schedule_every_variant(orc, d, bs, g):
    case = workloads.make_case("llama3_8b_b64", 11 * d + bs + g, B=7, h_q=2 * g, h_kv=2, d=d, bs=bs,
                               ctx_range=(1, 3000), pool_factor=1.2)
    _full_parity(orc, case, partition_size=AUTO)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("bs", [16, 32])
@pytest.mark.parametrize("g", [1, 2, 4, 8])
def test_auto_whole_block_every_variant(orc, d, bs, g):
    """8 KV heads, every (head_dim, block size, group) the whole-block kernel instantiates, on
    PA_PARTITION_AUTO: the per-KV-head balanced kernel here, the whole-block kernel (one CTA
    streams every head of a block) when the child process of test_gpu_cuda_core_variants.py
    sets PA_DECODE_AUTO_WHOLE_BLOCK=1."""
    case = workloads.make_case("llama3_8b_b64", 7 * d + bs + g, B=9, h_q=8 * g, h_kv=8, d=d, bs=bs,
                               ctx_range=(1, 2500), pool_factor=1.2)
    _full_parity(orc, case, partition_size=AUTO)


def test_auto_schedule_e4m3_falls_back(orc):
    case = workloads.make_case("fp8_mha_b32_bs16", 2, B=3, ctx_fixed=1500)
    _full_parity(orc, case, partition_size=AUTO)


def test_auto_schedule_edge_cases(orc):
    case = _with_appended(workloads.make_case("llama3_8b_b64", 14, device=DEV, B=10))
    ctx = case.context_lens.clone()
    ctx[0] = 0
    ctx[4] = 0
    ctx[9] = 1
    out = _decode(case, case.k_cache, case.v_cache, ctx=ctx, P=AUTO)
    assert torch.count_nonzero(out[0].float()) == 0 and torch.count_nonzero(out[4].float()) == 0
    assert torch.isfinite(out.float()).all()
    ref = _decode(case, case.k_cache, case.v_cache, ctx=ctx, P=512)
    tol = 2.0 ** -7 * torch.maximum(ref.float().abs(), out.float().abs()) + 2.0 ** -8
    assert ((out.float() - ref.float()).abs() <= tol).all()
    # a bad block id poisons its own sequence only and is flagged
    tab = case.block_tables.clone()
    tab[6, 3] = case.num_blocks + 1
    pa.pa_device_errors(clear=True)
    bad = _decode(case, case.k_cache, case.v_cache, tables=tab, P=AUTO)
    assert pa.pa_device_errors(clear=True) & pa.PA_DEVERR_BAD_BLOCK
    assert torch.isnan(bad[6].float()).all()
    good = _decode(case, case.k_cache, case.v_cache, P=AUTO)
    for s in (0, 5, 7, 9):
        assert torch.equal(bad[s].view(torch.int16), good[s].view(torch.int16))
    assert pa.pa_device_errors(clear=True) == 0


def test_auto_schedule_permutation_invariance_and_reuse():
    case = _with_appended(workloads.make_case("llama3_8b_b64", 15, device=DEV, B=20))
    ws = pa.make_workspace(case.B, case.h_q, case.d, case.max_context_len, AUTO, DEV)
    out1 = torch.empty((case.B, case.h_q, case.d), dtype=torch.bfloat16, device=DEV)
    for _ in range(3):                                         # the same workspace, three calls
        pa.pa_decode(out1, case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens,
                     case.max_context_len, case.scale, AUTO, workspace=ws)
    perm = torch.randperm(case.num_blocks, generator=torch.Generator().manual_seed(3)).to(DEV)
    kc2, vc2 = torch.empty_like(case.k_cache), torch.empty_like(case.v_cache)
    kc2[perm], vc2[perm] = case.k_cache, case.v_cache
    tab = case.block_tables
    tab2 = torch.where(tab >= 0, perm[tab.clamp(min=0).long()].to(torch.int32), tab)
    out2 = torch.empty_like(out1)
    pa.pa_decode(out2, case.q, kc2, vc2, tab2, case.context_lens, case.max_context_len, case.scale, AUTO, workspace=ws)
    torch.cuda.synchronize()
    assert torch.isfinite(out1.float()).all()
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))
    counters = ws[:64].view(torch.int32)        # the schedule's counters at the front of the workspace
    assert int(counters.abs().sum()) == 0
