"""Helpers of the GPU parity tests: one decode step through the C ABI on the GPU, the same
step in the CPU oracle, and the tolerance checks.  (Test infrastructure: imports oracle.)"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import workloads
import paged_kv_cache_428_b200 as pa

# Tolerances of the decode output against the fp64 oracle (bf16 output, fp32 accumulation).
# bf16 and INT8 caches: 2e-2 absolute and 1e-2 of max|ref|; E4M3: 6e-2 absolute.
BF16_ABS, BF16_REL = 2e-2, 1e-2
E4M3_ABS = 6e-2


def u16(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def u8(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().view(torch.uint8).numpy()


def codes(t: torch.Tensor, cache: str) -> np.ndarray:
    """Cache contents as numpy in the oracle's element type (uint16 bits, uint8 or int8 codes)."""
    if cache == "int8":
        return t.detach().contiguous().cpu().numpy()
    return u8(t) if cache == "e4m3" else u16(t)


def dev_scales(case, dev="cuda"):
    """The case's scales as pa_* arguments: floats, or CUDA fp32 [h_kv] tensors per KV head."""
    if case.per_head_scales:
        return case.k_scale.to(dev), case.v_scale.to(dev)
    return case.k_scale, case.v_scale


def np_scales(case):
    """The case's scales as oracle arguments: floats, or fp32 [h_kv] arrays."""
    if case.per_head_scales:
        return case.k_scale.numpy(), case.v_scale.numpy()
    return case.k_scale, case.v_scale


def gpu_fill_quant(case, dev="cuda"):
    """Quantise the case's pre-existing rows into fresh code pools with pa_reshape_and_cache."""
    kc, vc = workloads.empty_quant_pool(case, dev)
    if case.fill_slots is not None and case.fill_slots.numel():
        pa.pa_reshape_and_cache(case.fill_k_rows.to(dev), case.fill_v_rows.to(dev), kc, vc,
                                case.fill_slots.to(dev), *dev_scales(case, dev))
    return kc, vc



def gpu_step(case, partition_size=None, dev="cuda", max_context_len=None, caches=None):
    """Write the appended tokens, then decode; returns (out bf16 [B,h_q,d], k_cache, v_cache)."""
    P = case.partition if partition_size is None else partition_size
    if caches is not None:
        kc, vc = caches
    elif case.quantised:
        kc, vc = gpu_fill_quant(case, dev)
    else:
        kc, vc = case.k_cache.to(dev).clone(), case.v_cache.to(dev).clone()
    ks, vs = dev_scales(case, dev)
    pa.pa_reshape_and_cache(case.key_new.to(dev), case.value_new.to(dev), kc, vc, case.slot_mapping.to(dev), ks, vs)
    out = torch.empty((case.B, case.h_q, case.d), dtype=torch.bfloat16, device=dev)
    mcl = case.max_context_len if max_context_len is None else max_context_len
    pa.pa_decode(out, case.q.to(dev), kc, vc, case.block_tables.to(dev), case.context_lens.to(dev), mcl,
                 case.scale, P, ks, vs)
    return out, kc, vc


def oracle_caches(case, orc, seqs=None):
    """The oracle's own caches after the step's writes (numpy, pool layout).  With `seqs`,
    only the rows of those sequences are quantised (the rest keeps the sentinel)."""
    ks, vs = np_scales(case)
    if case.quantised:
        shape = (case.num_blocks, case.h_kv, case.bs, case.d)
        if case.cache == "int8":
            kc = np.full(shape, workloads.INT8_UNUSED, np.int8)
        else:
            kc = np.full(shape, workloads.E4M3_NAN, np.uint8)
        vc = kc.copy()
        slots = case.fill_slots.cpu()
        krows, vrows = case.fill_k_rows.cpu(), case.fill_v_rows.cpu()
        if seqs is not None:
            owner = block_owner(case)
            keep = torch.tensor([owner.get(int(s) // case.bs, -1) in seqs for s in slots.tolist()], dtype=torch.bool)
            slots, krows, vrows = slots[keep], krows[keep], vrows[keep]
        orc.reshape_and_cache(u16(krows), u16(vrows), kc, vc, slots.numpy(), h_kv=case.h_kv, d=case.d,
                              bs=case.bs, num_blocks=case.num_blocks, cache=case.cache, k_scale=ks, v_scale=vs)
    else:
        kc, vc = u16(case.k_cache).copy(), u16(case.v_cache).copy()
    orc.reshape_and_cache(u16(case.key_new), u16(case.value_new), kc, vc, case.slot_mapping.cpu().numpy(),
                          h_kv=case.h_kv, d=case.d, bs=case.bs, num_blocks=case.num_blocks, cache=case.cache,
                          k_scale=ks, v_scale=vs)
    return kc, vc


def block_owner(case) -> dict:
    """physical block id -> sequence (first owner) for the case's tables."""
    owner = {}
    tab = case.block_tables.cpu()
    for s in range(case.B):
        n = -(-int(case.context_lens[s]) // case.bs)
        for b in tab[s, :n].tolist():
            owner.setdefault(b, s)
    return owner


def oracle_out(case, orc, kc, vc, rows=None):
    ks, vs = np_scales(case)
    kw = dict(h_kv=case.h_kv, bs=case.bs, scale=case.scale, cache=case.cache, k_scale=ks, v_scale=vs)
    q = u16(case.q)
    tab = case.block_tables.cpu().numpy()
    ctx = case.context_lens.cpu().numpy()
    if rows is None:
        return orc.paged_decode(q, kc, vc, tab, ctx, **kw)
    return orc.paged_decode_rows(rows, q, kc, vc, tab, ctx, **kw)


def check_close(got: torch.Tensor, ref: np.ndarray, fp8: bool, what: str = "") -> dict:
    g = got.detach().float().cpu().numpy().astype(np.float64)
    assert np.isfinite(g).all(), "%s: non-finite output" % what
    err = np.abs(g - ref)
    max_abs = float(err.max()) if err.size else 0.0
    max_ref = float(np.abs(ref).max()) if ref.size else 0.0
    stats = {"max_abs": max_abs, "max_ref": max_ref, "rel": max_abs / max_ref if max_ref else 0.0}
    if fp8:
        assert max_abs <= E4M3_ABS, "%s: %s" % (what, stats)
    else:
        assert max_abs <= BF16_ABS and max_abs <= BF16_REL * max_ref + 1e-30, "%s: %s" % (what, stats)
    return stats
