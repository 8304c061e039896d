"""Pins of the CPU oracle to things other than itself (CPU only).

Each ``pin_*`` function takes an oracle object and asserts against an
independent source: the pages' printed numbers (tests/golden/), torch's own
bf16 / float8_e4m3fn casts and fp64 scaled_dot_product_attention (library
routines), brute-force Python loops with math.fsum, closed-form special cases,
and invariants.  ``test_planted_mistakes_are_caught`` compiles mutated copies
of oracle.c (a dropped term, a flipped sign, a wrong index ...) and checks
that at least one pin fails for each, so the pins are shown to bite.
"""
from __future__ import annotations

import json
import math
import os
import subprocess
import sys
import tempfile
from pathlib import Path

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from workloads import BF16_NAN, E4M3_NAN

GOLDEN = Path(__file__).resolve().parent / "golden"


def _golden(name):
    with open(GOLDEN / name) as f:
        return json.load(f)


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


# ----------------------------------------------------------------------------
# closed forms
# ----------------------------------------------------------------------------

def pin_closed_forms(orc):
    g = _golden("kv_size_closed_forms.json")
    for e in g["per_token"]:
        assert orc.kv_bytes_per_token(e["layers"], e["h_kv"], e["head_dim"], e["elem_bytes"]) == e["bytes"], e
    for e in g["per_sequence"]:
        assert orc.kv_bytes_sequence(e["layers"], e["tokens"], e["h_kv"], e["head_dim"],
                                     e["elem_bytes"]) == e["bytes"], e
    c = g["fp8_doubles_capacity"]
    fp16 = orc.kv_bytes_per_token(c["layers"], c["h_kv"], c["head_dim"], 2)
    fp8 = orc.kv_bytes_per_token(c["layers"], c["h_kv"], c["head_dim"], 1)
    assert fp16 == 2 * fp8
    budget = c["kv_budget_gib"] * 2 ** 30
    # the page rounds; its figures must be within 5 % of the exact token counts
    assert abs(budget // fp16 - c["fp16_tokens_approx"]) / c["fp16_tokens_approx"] < 0.05
    assert abs(budget // fp8 - c["fp8_tokens_approx"]) / c["fp8_tokens_approx"] < 0.05


def test_closed_forms(orc):
    pin_closed_forms(orc)


# ----------------------------------------------------------------------------
# number formats
# ----------------------------------------------------------------------------

def pin_bf16_codec(orc):
    codes = np.arange(1 << 16, dtype=np.uint16)
    want = torch.from_numpy(codes.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    got = orc.bf16_decode(codes)
    same = (got == want) | (np.isnan(got) & np.isnan(want))
    assert same.all()
    # encode: torch's RNE cast on random values, exact ties and carries
    g = torch.Generator().manual_seed(7)
    x = torch.randn(200000, generator=g) * torch.exp(torch.randn(200000, generator=g) * 8)
    base = torch.randint(0, 1 << 15, (4096,), generator=g, dtype=torch.int32) << 16
    ties = (base | 0x8000).view(torch.float32)               # exactly half-way: ties to even
    odd_ties = ((base | 0x10000) | 0x8000).view(torch.float32)
    above = (base | 0x8001).view(torch.float32)
    below = (base | 0x7FFF).view(torch.float32)
    for v in (x, ties, odd_ties, above, below, torch.tensor([3.3895314e38, -3.3895314e38, 1e-40, -0.0])):
        v = v.to(torch.float32)
        want = v.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        got = orc.bf16_encode_rne(v.numpy())
        nan_in = np.isnan(v.numpy())          # NaN payloads are not canonical: compare NaN-ness
        assert np.array_equal(got[~nan_in], want[~nan_in])
        assert np.isnan(orc.bf16_decode(got[nan_in])).all()


def pin_e4m3_codec(orc):
    codes = np.arange(256, dtype=np.uint8)
    want = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = orc.e4m3_decode(codes)
    same = (got == want) | (np.isnan(got) & np.isnan(want))
    assert same.all()
    named = _golden("e4m3_named_values.json")
    for e in named["values"]:
        c = int(e["code"], 16)
        v = orc.e4m3_decode([c])[0]
        assert v == e["value"] and math.copysign(1, v) == math.copysign(1, e["value"])
        assert orc.e4m3_encode_satfinite([e["value"]])[0] == c
    for c in named["nan_codes"]:
        assert np.isnan(orc.e4m3_decode([int(c, 16)])[0])
    # round trip of every finite code
    finite = codes[~np.isnan(want)]
    assert np.array_equal(orc.e4m3_encode_satfinite(orc.e4m3_decode(finite).astype(np.float32)), finite)
    # encode vs torch's RNE cast (torch does not saturate, so clamp to +-448 first: the
    # saturating conversion is RNE of the clamped value)
    g = torch.Generator().manual_seed(11)
    vals = [torch.randn(1 << 20, generator=g) * 40,
            torch.randn(1 << 16, generator=g) * 1e-2,
            torch.randn(1 << 16, generator=g) * 1e3]
    pos = np.sort(np.unique(np.abs(want[~np.isnan(want)])))
    mids = torch.from_numpy(((pos[1:] + pos[:-1]) / 2).astype(np.float32))
    vals += [mids, -mids, torch.nextafter(mids, torch.tensor(1e9)), torch.nextafter(mids, torch.tensor(-1e9)),
             torch.tensor([448.0, 449.0, 463.9, 464.0, 464.1, 479.0, 480.0, 1e30, float("inf"),
                           -float("inf"), -500.0, 0.0, -0.0, 1e-9, -1e-9])]
    for v in vals:
        v = v.to(torch.float32)
        exp = v.clamp(-448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        got = orc.e4m3_encode_satfinite(v.numpy())
        assert np.array_equal(got, exp)


def pin_div_f32(orc):
    g = torch.Generator().manual_seed(3)
    x = torch.randn(100000, generator=g)
    s = 0.0123456
    want = (x / torch.tensor(s, dtype=torch.float32)).numpy()
    assert np.array_equal(orc.div_f32(x.numpy(), s), want)


def _int8_expected(c: int, off: float) -> int:
    """Integer reasoning for x = c + off, |off| <= 1/2: the nearest integer, the even one on a
    tie, then limited to [-127, 127]."""
    if abs(off) < 0.5:
        r = c
    else:
        r = c if c % 2 == 0 else c + (1 if off > 0 else -1)
    return max(-127, min(127, r))


def pin_int8_codec(orc):
    codes = np.arange(-128, 128, dtype=np.int16).astype(np.int8)
    assert np.array_equal(orc.int8_decode(codes), np.arange(-128, 128, dtype=np.float64))
    # brute force around every integer of the range and past both ends (all exact in fp32)
    offs = [-0.5, -0.49999997, -0.25, 0.0, 0.25, 0.49999997, 0.5]
    xs, want = [], []
    for c in range(-140, 141):
        for o in offs:
            x = np.float32(c) + np.float32(o)
            if float(x) - c != o:              # not exactly representable at this magnitude
                continue
            xs.append(x)
            want.append(_int8_expected(c, o))
    got = orc.int8_encode_sat(np.array(xs, np.float32))
    assert np.array_equal(got.astype(np.int64), np.array(want, np.int64))
    special = np.array([np.nan, np.inf, -np.inf, 1e30, -1e30, -127.6, -127.5, -127.4, 127.5, -0.0, 1e-30],
                       np.float32)
    assert orc.int8_encode_sat(special).tolist() == [0, 127, -127, 127, -127, -127, -127, -127, 127, 0, 0]
    # random values against torch's round-half-to-even, clamped
    g = torch.Generator().manual_seed(12)
    v = torch.randn(1 << 18, generator=g) * 60
    exp = torch.round(v).clamp(-127, 127).to(torch.int8).numpy()
    assert np.array_equal(orc.int8_encode_sat(v.numpy()), exp)


def test_bf16_codec(orc):
    pin_bf16_codec(orc)


def test_int8_codec(orc):
    pin_int8_codec(orc)


def test_e4m3_codec(orc):
    pin_e4m3_codec(orc)


def test_div_f32(orc):
    pin_div_f32(orc)


# ----------------------------------------------------------------------------
# decode attention
# ----------------------------------------------------------------------------

def build_paged(contig_k, contig_v, order, bs, num_blocks, sentinel=BF16_NAN):
    """Scatter per-sequence contiguous rows [n_s, h_kv, d] (bf16) into a pool
    [num_blocks, h_kv, bs, d] through tables built from ``order``; every other slot
    holds the sentinel.  Plain index arithmetic written here, independent of the oracle."""
    h_kv, d = contig_k[0].shape[1], contig_k[0].shape[2]
    kp = torch.full((num_blocks, h_kv, bs, d), sentinel, dtype=torch.int16).view(torch.bfloat16)
    vp = kp.clone()
    nblk = [-(-k.shape[0] // bs) for k in contig_k]
    table = torch.full((len(contig_k), max(max(nblk), 1)), -1, dtype=torch.int32)
    pos = 0
    for s, (k, v) in enumerate(zip(contig_k, contig_v)):
        for i in range(nblk[s]):
            phys = order[pos]
            pos += 1
            table[s, i] = phys
            rows = slice(i * bs, min((i + 1) * bs, k.shape[0]))
            n = rows.stop - rows.start
            kp[phys, :, :n, :] = k[rows].transpose(0, 1)
            vp[phys, :, :n, :] = v[rows].transpose(0, 1)
    return kp, vp, table


def sdpa_reference(q, contig_k, contig_v, scale):
    """fp64 torch SDPA per sequence on contiguous rows; GQA by torch's enable_gqa."""
    B, h_q, d = q.shape
    out = torch.zeros(B, h_q, d, dtype=torch.float64)
    for s in range(B):
        n = contig_k[s].shape[0]
        if n == 0:
            continue
        qq = q[s].to(torch.float64)[None, :, None, :]                       # [1, h_q, 1, d]
        kk = contig_k[s].to(torch.float64).transpose(0, 1)[None]           # [1, h_kv, n, d]
        vv = contig_v[s].to(torch.float64).transpose(0, 1)[None]
        o = F.scaled_dot_product_attention(qq, kk, vv, scale=scale, enable_gqa=True)
        out[s] = o[0, :, 0, :]
    return out


def _random_decode(seed, B, h_q, h_kv, d, bs, ctxs=None, extra_blocks=3):
    g = torch.Generator().manual_seed(seed)
    if ctxs is None:
        ctxs = torch.randint(0, 5 * bs, (B,), generator=g).tolist()
    ks = [torch.randn(n, h_kv, d, generator=g).to(torch.bfloat16) for n in ctxs]
    vs = [torch.randn(n, h_kv, d, generator=g).to(torch.bfloat16) for n in ctxs]
    q = torch.randn(B, h_q, d, generator=g).to(torch.bfloat16)
    nb = sum(-(-n // bs) for n in ctxs) + extra_blocks
    order = torch.randperm(nb, generator=g).tolist()
    return q, ks, vs, order, nb, ctxs


def pin_decode_vs_sdpa(orc):
    shapes = [(3, 4, 2, 64, 16), (2, 8, 1, 128, 32), (4, 8, 8, 64, 16), (2, 16, 2, 128, 64), (5, 4, 4, 64, 16)]
    for seed, (B, h_q, h_kv, d, bs) in enumerate(shapes):
        ctxs = None
        if seed == 0:
            ctxs = [0, 1, bs]                       # empty, single token, exactly one block
        if seed == 4:
            ctxs = [bs - 1, bs + 1, 2 * bs + 5, 3 * bs, 1]
        q, ks, vs, order, nb, ctxs = _random_decode(seed, B, h_q, h_kv, d, bs, ctxs)
        kp, vp, table = build_paged(ks, vs, order, bs, nb)
        scale = 1.0 / math.sqrt(d)
        got = orc.paged_decode(_bits(q), _bits(kp), _bits(vp), table.numpy(), np.array(ctxs, np.int32),
                               h_kv=h_kv, bs=bs, scale=scale)
        want = sdpa_reference(q, ks, vs, scale).numpy()
        assert np.isfinite(got).all()
        np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-13)


def pin_decode_brute_force(orc):
    """Tiny GQA case against explicit Python loops with math.fsum (kv head = h // g)."""
    B, h_q, h_kv, d, bs = 2, 4, 2, 8, 4
    q, ks, vs, order, nb, ctxs = _random_decode(5, B, h_q, h_kv, d, bs, ctxs=[5, 11])
    kp, vp, table = build_paged(ks, vs, order, bs, nb)
    scale = 0.37
    got = orc.paged_decode(_bits(q), _bits(kp), _bits(vp), table.numpy(), np.array(ctxs, np.int32),
                           h_kv=h_kv, bs=bs, scale=scale)
    g = h_q // h_kv
    for s in range(B):
        K = ks[s].double().tolist()
        V = vs[s].double().tolist()
        for h in range(h_q):
            qv = q[s, h].double().tolist()
            kv = h // g
            logits = [scale * math.fsum(qv[i] * K[t][kv][i] for i in range(d)) for t in range(ctxs[s])]
            m = max(logits)
            w = [math.exp(x - m) for x in logits]
            den = math.fsum(w)
            ref = [math.fsum(w[t] * V[t][kv][i] for t in range(ctxs[s])) / den for i in range(d)]
            np.testing.assert_allclose(got[s, h], ref, rtol=1e-13, atol=1e-15)


def pin_decode_special_cases(orc):
    d, bs, h_kv, h_q = 64, 16, 2, 4
    g = torch.Generator().manual_seed(9)
    scale = 1.0 / math.sqrt(d)
    # ctx = 1 -> exactly V_0
    q, ks, vs, order, nb, ctxs = _random_decode(1, 1, h_q, h_kv, d, bs, ctxs=[1])
    kp, vp, table = build_paged(ks, vs, order, bs, nb)
    out = orc.paged_decode(_bits(q), _bits(kp), _bits(vp), table.numpy(), np.array(ctxs, np.int32),
                           h_kv=h_kv, bs=bs, scale=scale)
    for h in range(h_q):
        assert np.array_equal(out[0, h], vs[0][0, h // 2].double().numpy())
    # q = 0 -> uniform weights -> mean of V (fsum)
    n = 37
    q0 = torch.zeros(1, h_q, d, dtype=torch.bfloat16)
    _, ks, vs, order, nb, _ = _random_decode(2, 1, h_q, h_kv, d, bs, ctxs=[n])
    kp, vp, table = build_paged(ks, vs, order, bs, nb)
    out = orc.paged_decode(_bits(q0), _bits(kp), _bits(vp), table.numpy(), np.array([n], np.int32),
                           h_kv=h_kv, bs=bs, scale=scale)
    V = vs[0].double()
    for h in range(h_q):
        mean = [math.fsum(V[t, h // 2, i].item() for t in range(n)) / n for i in range(d)]
        np.testing.assert_allclose(out[0, h], mean, rtol=1e-13, atol=1e-15)
    # one dominant logit: q = 8 * K_j  ->  out ~= V_j
    j = 23
    qd = torch.zeros(1, h_q, d, dtype=torch.bfloat16)
    for h in range(h_q):
        qd[0, h] = (ks[0][j, h // 2].float() * 8).to(torch.bfloat16)
    out = orc.paged_decode(_bits(qd), _bits(kp), _bits(vp), table.numpy(), np.array([n], np.int32),
                           h_kv=h_kv, bs=bs, scale=scale)
    for h in range(h_q):
        np.testing.assert_allclose(out[0, h], V[j, h // 2].numpy(), atol=1e-3)


def pin_worked_block_table_example(orc):
    """The pages' example: A's logical blocks live in physical blocks 2, 5, 1, last one partial."""
    ex = _golden("block_table_example.json")
    phys = ex["logical_to_physical"]
    bs, h_q, h_kv, d = 16, 4, 2, 64
    n = 2 * bs + 5                          # three logical blocks, the last partly filled
    g = torch.Generator().manual_seed(21)
    K = torch.randn(n, h_kv, d, generator=g).to(torch.bfloat16)
    Vv = torch.randn(n, h_kv, d, generator=g).to(torch.bfloat16)
    q = torch.randn(1, h_q, d, generator=g).to(torch.bfloat16)
    nb = 8
    order = list(phys) + [b for b in range(nb) if b not in phys]
    kp, vp, table = build_paged([K], [Vv], order, bs, nb)
    assert table[0, :3].tolist() == phys
    scale = 1.0 / math.sqrt(d)
    got = orc.paged_decode(_bits(q), _bits(kp), _bits(vp), table.numpy(), np.array([n], np.int32),
                           h_kv=h_kv, bs=bs, scale=scale)
    want = sdpa_reference(q, [K], [Vv], scale).numpy()
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-13)
    # identity placement (contiguous physical blocks 0,1,2) gives the bit-identical result
    kp2, vp2, table2 = build_paged([K], [Vv], list(range(nb)), bs, nb)
    got2 = orc.paged_decode(_bits(q), _bits(kp2), _bits(vp2), table2.numpy(), np.array([n], np.int32),
                            h_kv=h_kv, bs=bs, scale=scale)
    assert np.array_equal(got, got2)


def pin_permutation_invariance(orc):
    B, h_q, h_kv, d, bs = 4, 8, 2, 64, 16
    q, ks, vs, order, nb, ctxs = _random_decode(13, B, h_q, h_kv, d, bs)
    kp, vp, table = build_paged(ks, vs, order, bs, nb)
    out1 = orc.paged_decode(_bits(q), _bits(kp), _bits(vp), table.numpy(), np.array(ctxs, np.int32),
                            h_kv=h_kv, bs=bs, scale=0.125)
    perm = torch.randperm(nb, generator=torch.Generator().manual_seed(99))
    kp2 = torch.empty_like(kp); vp2 = torch.empty_like(vp)
    kp2[perm] = kp; vp2[perm] = vp
    table2 = torch.where(table >= 0, perm[table.clamp(min=0).long()].to(torch.int32), table)
    out2 = orc.paged_decode(_bits(q), _bits(kp2), _bits(vp2), table2.numpy(), np.array(ctxs, np.int32),
                            h_kv=h_kv, bs=bs, scale=0.125)
    assert np.array_equal(out1, out2)


def pin_fp8_decode(orc):
    """E4M3 cache: the oracle equals fp64 SDPA over the dequantised rows (torch's own float8
    decode times the per-tensor scale)."""
    B, h_q, h_kv, d, bs = 3, 4, 4, 128, 32
    g = torch.Generator().manual_seed(17)
    ctxs = [45, 64, 100]
    codes_k = [torch.randint(0, 256, (n, h_kv, d), generator=g, dtype=torch.uint8) for n in ctxs]
    codes_v = [torch.randint(0, 256, (n, h_kv, d), generator=g, dtype=torch.uint8) for n in ctxs]
    for c in codes_k + codes_v:                       # no NaN codes in live slots
        c[(c & 0x7F) == 0x7F] = 0x7E
    q = torch.randn(B, h_q, d, generator=g).to(torch.bfloat16)
    ksc, vsc = float(np.float32(0.0123)), float(np.float32(0.0071))    # scales are fp32
    nb = sum(-(-n // bs) for n in ctxs) + 2
    order = torch.randperm(nb, generator=g).tolist()
    kp = torch.full((nb, h_kv, bs, d), E4M3_NAN, dtype=torch.uint8)
    vp = kp.clone()
    table = torch.full((B, 4), -1, dtype=torch.int32)
    pos = 0
    for s, n in enumerate(ctxs):
        for i in range(-(-n // bs)):
            phys = order[pos]; pos += 1
            table[s, i] = phys
            r = slice(i * bs, min((i + 1) * bs, n))
            kp[phys, :, :r.stop - r.start] = codes_k[s][r].transpose(0, 1)
            vp[phys, :, :r.stop - r.start] = codes_v[s][r].transpose(0, 1)
    got = orc.paged_decode(_bits(q), kp.numpy(), vp.numpy(), table.numpy(), np.array(ctxs, np.int32),
                           h_kv=h_kv, bs=bs, scale=1 / math.sqrt(d), fp8=True, k_scale=ksc, v_scale=vsc)
    deq_k = [c.view(torch.float8_e4m3fn).to(torch.float64) * ksc for c in codes_k]
    deq_v = [c.view(torch.float8_e4m3fn).to(torch.float64) * vsc for c in codes_v]
    want = sdpa_reference(q, deq_k, deq_v, 1 / math.sqrt(d)).numpy()
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-13)


def _quantised_pool(codes_k, codes_v, ctxs, bs, h_kv, d, g, fill, dtype):
    nb = sum(-(-n // bs) for n in ctxs) + 2
    order = torch.randperm(nb, generator=g).tolist()
    kp = torch.full((nb, h_kv, bs, d), fill, dtype=dtype)
    vp = kp.clone()
    table = torch.full((len(ctxs), max(-(-n // bs) for n in ctxs)), -1, dtype=torch.int32)
    pos = 0
    for s, n in enumerate(ctxs):
        for i in range(-(-n // bs)):
            phys = order[pos]; pos += 1
            table[s, i] = phys
            r = slice(i * bs, min((i + 1) * bs, n))
            kp[phys, :, :r.stop - r.start] = codes_k[s][r].transpose(0, 1)
            vp[phys, :, :r.stop - r.start] = codes_v[s][r].transpose(0, 1)
    return kp, vp, table


def pin_int8_decode_per_head(orc):
    """INT8 cache with a different scale per KV head: the oracle equals fp64 SDPA over the
    rows dequantised by torch (code x the head's scale), and a per-tensor call equals the
    per-head call with equal scales."""
    B, h_q, h_kv, d, bs = 3, 8, 4, 64, 16
    g = torch.Generator().manual_seed(19)
    ctxs = [33, 16, 70]
    codes_k = [torch.randint(-127, 128, (n, h_kv, d), generator=g, dtype=torch.int8) for n in ctxs]
    codes_v = [torch.randint(-127, 128, (n, h_kv, d), generator=g, dtype=torch.int8) for n in ctxs]
    q = torch.randn(B, h_q, d, generator=g).to(torch.bfloat16)
    ksc = np.array([0.011, 0.023, 0.0047, 0.031], np.float32)
    vsc = np.array([0.019, 0.006, 0.027, 0.013], np.float32)
    kp, vp, table = _quantised_pool(codes_k, codes_v, ctxs, bs, h_kv, d, g, -128, torch.int8)
    scale = 1 / math.sqrt(d)
    got = orc.paged_decode(_bits(q), kp.numpy(), vp.numpy(), table.numpy(), np.array(ctxs, np.int32),
                           h_kv=h_kv, bs=bs, scale=scale, cache="int8", k_scale=ksc, v_scale=vsc)
    kt = torch.from_numpy(ksc.astype(np.float64))[None, :, None]
    vt = torch.from_numpy(vsc.astype(np.float64))[None, :, None]
    deq_k = [c.to(torch.float64) * kt for c in codes_k]
    deq_v = [c.to(torch.float64) * vt for c in codes_v]
    want = sdpa_reference(q, deq_k, deq_v, scale).numpy()
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-13)
    one = orc.paged_decode(_bits(q), kp.numpy(), vp.numpy(), table.numpy(), np.array(ctxs, np.int32),
                           h_kv=h_kv, bs=bs, scale=scale, cache="int8", k_scale=0.02, v_scale=0.01)
    same = orc.paged_decode(_bits(q), kp.numpy(), vp.numpy(), table.numpy(), np.array(ctxs, np.int32),
                            h_kv=h_kv, bs=bs, scale=scale, cache="int8", k_scale=[0.02] * h_kv,
                            v_scale=[0.01] * h_kv)
    assert np.array_equal(one, same)


def pin_fp8_decode_per_head(orc):
    """E4M3 cache with per-KV-head scales against fp64 SDPA on torch-dequantised rows."""
    B, h_q, h_kv, d, bs = 2, 4, 2, 64, 16
    g = torch.Generator().manual_seed(23)
    ctxs = [40, 17]
    codes_k = [torch.randint(0, 256, (n, h_kv, d), generator=g, dtype=torch.uint8) for n in ctxs]
    codes_v = [torch.randint(0, 256, (n, h_kv, d), generator=g, dtype=torch.uint8) for n in ctxs]
    for c in codes_k + codes_v:
        c[(c & 0x7F) == 0x7F] = 0x7E
    q = torch.randn(B, h_q, d, generator=g).to(torch.bfloat16)
    ksc = np.array([0.0093, 0.0210], np.float32)
    vsc = np.array([0.0150, 0.0041], np.float32)
    kp, vp, table = _quantised_pool(codes_k, codes_v, ctxs, bs, h_kv, d, g, E4M3_NAN, torch.uint8)
    got = orc.paged_decode(_bits(q), kp.numpy(), vp.numpy(), table.numpy(), np.array(ctxs, np.int32),
                           h_kv=h_kv, bs=bs, scale=0.125, cache="e4m3", k_scale=ksc, v_scale=vsc)
    kt = torch.from_numpy(ksc.astype(np.float64))[None, :, None]
    vt = torch.from_numpy(vsc.astype(np.float64))[None, :, None]
    deq_k = [c.view(torch.float8_e4m3fn).to(torch.float64) * kt for c in codes_k]
    deq_v = [c.view(torch.float8_e4m3fn).to(torch.float64) * vt for c in codes_v]
    want = sdpa_reference(q, deq_k, deq_v, 0.125).numpy()
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-13)


def _prefill_case(seed, B, h_q, h_kv, d, bs, cached_lens, chunk_lens):
    """Contiguous K/V rows of each sequence (cached + chunk), scattered through tables, and the
    chunk's query rows stacked as [T, h_q, d]."""
    g = torch.Generator().manual_seed(seed)
    ctxs = [c + n for c, n in zip(cached_lens, chunk_lens)]
    ks = [torch.randn(n, h_kv, d, generator=g).to(torch.bfloat16) for n in ctxs]
    vs = [torch.randn(n, h_kv, d, generator=g).to(torch.bfloat16) for n in ctxs]
    q = torch.randn(sum(chunk_lens), h_q, d, generator=g).to(torch.bfloat16)
    nb = sum(-(-n // bs) for n in ctxs) + 2
    order = torch.randperm(nb, generator=g).tolist()
    kp, vp, table = build_paged(ks, vs, order, bs, nb)
    qstart = np.concatenate([[0], np.cumsum(chunk_lens)]).astype(np.int32)
    return q, ks, vs, kp, vp, table, qstart, ctxs


def pin_prefill_vs_masked_sdpa(orc):
    """Chunked prefill: row i of a chunk of n rows ending at the sequence's last token attends
    to tokens 0 .. ctx - n + i; against fp64 SDPA with that causal mask on contiguous rows
    (a whole prompt, cached = 0, is plain causal attention)."""
    for seed, (h_q, h_kv, d, bs, cached, chunk) in enumerate([
            (4, 2, 64, 16, [0, 20, 37], [5, 17, 40]),
            (8, 1, 128, 32, [64, 0], [1, 33]),
            (4, 4, 64, 16, [3], [16])]):
        q, ks, vs, kp, vp, table, qstart, ctxs = _prefill_case(seed, len(chunk), h_q, h_kv, d, bs, cached, chunk)
        scale = 1.0 / math.sqrt(d)
        got = orc.paged_prefill(_bits(q), _bits(kp), _bits(vp), table.numpy(), qstart, np.array(ctxs, np.int32),
                                h_kv=h_kv, bs=bs, scale=scale)
        for s_ in range(len(chunk)):
            n, ctx = chunk[s_], ctxs[s_]
            qq = q[qstart[s_]:qstart[s_ + 1]].to(torch.float64).transpose(0, 1)[None]      # [1, h_q, n, d]
            kk = ks[s_].to(torch.float64).transpose(0, 1)[None]
            vv = vs[s_].to(torch.float64).transpose(0, 1)[None]
            mask = torch.arange(ctx)[None, :] <= (ctx - n + torch.arange(n))[:, None]   # [n, ctx]
            want = F.scaled_dot_product_attention(qq, kk, vv, attn_mask=mask, scale=scale, enable_gqa=True)
            np.testing.assert_allclose(got[qstart[s_]:qstart[s_ + 1]], want[0].transpose(0, 1).numpy(),
                                       rtol=1e-12, atol=1e-13)
            if cached[s_] == 0:
                causal = F.scaled_dot_product_attention(qq, kk, vv, is_causal=True, scale=scale, enable_gqa=True)
                np.testing.assert_allclose(got[qstart[s_]:qstart[s_ + 1]], causal[0].transpose(0, 1).numpy(),
                                           rtol=1e-12, atol=1e-13)


def pin_prefill_chunk_of_one_is_decode(orc):
    """A one-token chunk is a decode step: the same row as or_paged_decode."""
    h_q, h_kv, d, bs = 8, 2, 64, 16
    q, ks, vs, kp, vp, table, qstart, ctxs = _prefill_case(41, 3, h_q, h_kv, d, bs, [10, 0, 47], [1, 1, 1])
    kw = dict(h_kv=h_kv, bs=bs, scale=0.3)
    pre = orc.paged_prefill(_bits(q), _bits(kp), _bits(vp), table.numpy(), qstart, np.array(ctxs, np.int32), **kw)
    dec = orc.paged_decode(_bits(q), _bits(kp), _bits(vp), table.numpy(), np.array(ctxs, np.int32), **kw)
    assert np.array_equal(pre, dec)


def pin_decode_rows_subset(orc):
    B, h_q, h_kv, d, bs = 3, 8, 4, 64, 16
    q, ks, vs, order, nb, ctxs = _random_decode(31, B, h_q, h_kv, d, bs, ctxs=[20, 50, 3])
    kp, vp, table = build_paged(ks, vs, order, bs, nb)
    full = orc.paged_decode(_bits(q), _bits(kp), _bits(vp), table.numpy(), np.array(ctxs, np.int32),
                            h_kv=h_kv, bs=bs, scale=0.2)
    rows = [(2, 7), (0, 0), (1, 5)]
    sub = orc.paged_decode_rows(rows, _bits(q), _bits(kp), _bits(vp), table.numpy(), np.array(ctxs, np.int32),
                                h_kv=h_kv, bs=bs, scale=0.2)
    for i, (s, h) in enumerate(rows):
        assert np.array_equal(sub[i], full[s, h])


def test_decode_vs_sdpa(orc):
    pin_decode_vs_sdpa(orc)


def test_decode_brute_force(orc):
    pin_decode_brute_force(orc)


def test_decode_special_cases(orc):
    pin_decode_special_cases(orc)


def test_worked_block_table_example(orc):
    pin_worked_block_table_example(orc)


def test_permutation_invariance(orc):
    pin_permutation_invariance(orc)


def test_fp8_decode(orc):
    pin_fp8_decode(orc)


def test_decode_rows_subset(orc):
    pin_decode_rows_subset(orc)


def test_prefill_vs_masked_sdpa(orc):
    pin_prefill_vs_masked_sdpa(orc)


def test_prefill_chunk_of_one_is_decode(orc):
    pin_prefill_chunk_of_one_is_decode(orc)


def test_int8_decode_per_head(orc):
    pin_int8_decode_per_head(orc)


def test_fp8_decode_per_head(orc):
    pin_fp8_decode_per_head(orc)


# ----------------------------------------------------------------------------
# cache write and block copy
# ----------------------------------------------------------------------------

def pin_reshape_and_cache(orc):
    T, h_kv, d, bs, nb = 9, 4, 64, 16, 6
    g = torch.Generator().manual_seed(4)
    key = (torch.randn(T, h_kv, d, generator=g) * 3).to(torch.bfloat16)
    val = (torch.randn(T, h_kv, d, generator=g) * 3).to(torch.bfloat16)
    slots = torch.tensor([5, 17, -1, 0, 95, 33, 34, -7, 64], dtype=torch.int64)
    kc = torch.full((nb, h_kv, bs, d), BF16_NAN, dtype=torch.int16).view(torch.bfloat16)
    vc = kc.clone()
    kb, vb = _bits(kc).copy(), _bits(vc).copy()
    orc.reshape_and_cache(_bits(key), _bits(val), kb, vb, slots.numpy(), h_kv=h_kv, d=d, bs=bs, num_blocks=nb)
    ek, ev = kc.clone(), vc.clone()
    for t, s in enumerate(slots.tolist()):
        if s >= 0:
            ek[s // bs, :, s % bs, :] = key[t]
            ev[s // bs, :, s % bs, :] = val[t]
    assert np.array_equal(kb, _bits(ek)) and np.array_equal(vb, _bits(ev))
    # E4M3: torch's RNE cast of the fp32 quotient, clamped to the finite range
    ksc, vsc = 0.0137, 0.0211
    kc8 = np.full((nb, h_kv, bs, d), E4M3_NAN, np.uint8)
    vc8 = kc8.copy()
    orc.reshape_and_cache(_bits(key), _bits(val), kc8, vc8, slots.numpy(), h_kv=h_kv, d=d, bs=bs,
                          num_blocks=nb, fp8=True, k_scale=ksc, v_scale=vsc)
    e8k = torch.full((nb, h_kv, bs, d), E4M3_NAN, dtype=torch.uint8)
    e8v = e8k.clone()
    for t, s in enumerate(slots.tolist()):
        if s >= 0:
            qk = (key[t].float() / torch.tensor(ksc, dtype=torch.float32)).clamp(-448, 448)
            qv = (val[t].float() / torch.tensor(vsc, dtype=torch.float32)).clamp(-448, 448)
            e8k[s // bs, :, s % bs, :] = qk.to(torch.float8_e4m3fn).view(torch.uint8)
            e8v[s // bs, :, s % bs, :] = qv.to(torch.float8_e4m3fn).view(torch.uint8)
    assert np.array_equal(kc8, e8k.numpy()) and np.array_equal(vc8, e8v.numpy())
    # saturation is exercised: |x| up to ~4 sigma * 3 / 0.0137 >> 448
    assert (np.abs(key.float().numpy()) / ksc > 448).any()
    # INT8 with a scale per KV head: torch's round-half-to-even of the fp32 quotient, clamped
    kh = np.array([0.031, 0.052, 0.017, 0.09], np.float32)
    vh = np.array([0.044, 0.021, 0.075, 0.012], np.float32)
    kc_i = np.full((nb, h_kv, bs, d), -128, np.int8)
    vc_i = kc_i.copy()
    orc.reshape_and_cache(_bits(key), _bits(val), kc_i, vc_i, slots.numpy(), h_kv=h_kv, d=d, bs=bs,
                          num_blocks=nb, cache="int8", k_scale=kh, v_scale=vh)
    eik = torch.full((nb, h_kv, bs, d), -128, dtype=torch.int8)
    eiv = eik.clone()
    for t, s_ in enumerate(slots.tolist()):
        if s_ >= 0:
            qk = torch.round(key[t].float() / torch.from_numpy(kh)[:, None]).clamp(-127, 127)
            qv = torch.round(val[t].float() / torch.from_numpy(vh)[:, None]).clamp(-127, 127)
            eik[s_ // bs, :, s_ % bs, :] = qk.to(torch.int8)
            eiv[s_ // bs, :, s_ % bs, :] = qv.to(torch.int8)
    assert np.array_equal(kc_i, eik.numpy()) and np.array_equal(vc_i, eiv.numpy())
    assert (np.abs(key.float().numpy()) / kh[None, :, None] > 127).any()     # saturation exercised


def pin_copy_blocks(orc):
    L, nb, h_kv, bs, d = 3, 10, 2, 16, 64
    g = torch.Generator().manual_seed(8)
    ks = [torch.randint(-32768, 32767, (nb, h_kv, bs, d), generator=g, dtype=torch.int16) for _ in range(L)]
    vs = [torch.randint(-32768, 32767, (nb, h_kv, bs, d), generator=g, dtype=torch.int16) for _ in range(L)]
    pairs = np.array([[3, 7], [0, 9], [3, 2]], np.int64)
    kn = [k.numpy().copy() for k in ks]
    vn = [v.numpy().copy() for v in vs]
    orc.copy_blocks(kn, vn, pairs, block_bytes=h_kv * bs * d * 2, num_blocks=nb)
    for l in range(L):
        ek, ev = ks[l].clone(), vs[l].clone()
        for s, t in pairs.tolist():
            ek[t] = ks[l][s]
            ev[t] = vs[l][s]
        assert np.array_equal(kn[l], ek.numpy()) and np.array_equal(vn[l], ev.numpy())
    with pytest.raises(ValueError):
        orc.copy_blocks(kn, vn, np.array([[0, nb]]), block_bytes=h_kv * bs * d * 2, num_blocks=nb)


def test_reshape_and_cache(orc):
    pin_reshape_and_cache(orc)


def test_copy_blocks(orc):
    pin_copy_blocks(orc)


# ----------------------------------------------------------------------------
# the pins bite: planted mistakes in copies of the oracle must fail a pin
# ----------------------------------------------------------------------------

ALL_PINS = [pin_closed_forms, pin_bf16_codec, pin_e4m3_codec, pin_int8_codec, pin_div_f32,
            pin_decode_vs_sdpa, pin_decode_brute_force, pin_decode_special_cases,
            pin_worked_block_table_example, pin_permutation_invariance, pin_fp8_decode,
            pin_int8_decode_per_head, pin_fp8_decode_per_head, pin_decode_rows_subset,
            pin_prefill_vs_masked_sdpa, pin_prefill_chunk_of_one_is_decode,
            pin_reshape_and_cache, pin_copy_blocks]

MUTANTS = {
    "gqa_mapping": ("int kvh = h / g;", "int kvh = h % h_kv;"),
    "dropped_scale": ("logit[t] = scale * dot;", "logit[t] = dot;"),
    "softmax_sign": ("double w = exp(logit[t] - m);", "double w = exp(m - logit[t]);"),
    "dropped_normalisation": ("for (int i = 0; i < d; ++i) out_row[i] /= denom;", ""),
    "table_index": ("int32_t phys = block_tables[(size_t)s * max_blocks_per_seq + t / bs];\n        if (phys < 0",
                    "int32_t phys = block_tables[(size_t)s * max_blocks_per_seq + t % bs];\n        if (phys < 0"),
    "drops_last_token": ("    for (int t = 0; t < n; ++t) {\n        double w", "    for (int t = 0; t < n - 1; ++t) {\n        double w"),
    "kv_swapped": ("out_row[i] += w * cache_elem(v_cache", "out_row[i] += w * cache_elem(k_cache"),
    "e4m3_round_half_up": ("double k = rint(a / quantum);", "double k = floor(a / quantum + 0.5);"),
    "e4m3_subnormal_step": ("quantum = ldexp(1.0, -9);", "quantum = ldexp(1.0, -10);"),
    "e4m3_decode_bias": ("else        v = ldexp(1.0 + m / 8.0, e - 7);", "else        v = ldexp(1.0 + m / 8.0, e - 8);"),
    "bf16_round_half_up": ("if (rest > 0x8000u || (rest == 0x8000u && (keep & 1u))) keep += 1u;",
                           "if (rest >= 0x8000u) keep += 1u;"),
    "cache_head_index": ("size_t dst = cache_index(blk, h, off, i, h_kv, bs, d);",
                         "size_t dst = cache_index(blk, 0, off, i, h_kv, bs, d);"),
    "copy_direction": ("k_caches[l][(uint64_t)dst * block_bytes + b] = k_caches[l][(uint64_t)src * block_bytes + b];",
                       "k_caches[l][(uint64_t)src * block_bytes + b] = k_caches[l][(uint64_t)dst * block_bytes + b];"),
    "closed_form_factor": ("return 2ull * (uint64_t)layers", "return 1ull * (uint64_t)layers"),
    "int8_round_half_up": ("else r = (fmod(f, 2.0) == 0.0) ? f : f + 1.0;", "else r = f + 1.0;"),
    "int8_asymmetric_range": ("if (x <= -127.0f) return -127;", "if (x <= -128.0f) return -128;"),
    "int8_decode_unsigned": ("double or_int8_decode(int8_t c) { return (double)c; }",
                             "double or_int8_decode(int8_t c) { return (double)(uint8_t)c; }"),
    "per_head_scale_index": ("double k_scale = cache_dtype ? (double)k_scales[kvh] : 1.0;",
                             "double k_scale = cache_dtype ? (double)k_scales[0] : 1.0;"),
    "prefill_causal_off_by_one": ("int n = p + 1;                            /* tokens it attends to */",
                                  "int n = p;                                /* tokens it attends to */"),
    "prefill_gqa_mapping": ("const int kh = h / group;", "const int kh = h % h_kv;"),
    "prefill_dropped_scale": ("score[j] = acc * scale;", "score[j] = acc;"),
    "prefill_softmax_sign": ("const double wj = exp(score[j] - top);", "const double wj = exp(top - score[j]);"),
    "prefill_kv_swapped": ("out_row[e] += wj * cache_elem(v_cache", "out_row[e] += wj * cache_elem(k_cache"),
    "prefill_table_index": ("const int32_t blk = block_tables[(size_t)s * max_blocks_per_seq + j / bs];\n        if (blk",
                            "const int32_t blk = block_tables[(size_t)s * max_blocks_per_seq + j % bs];\n        if (blk"),
    "prefill_chunk_position": ("int p = ctx - chunk + i;                  /* absolute position of this query token */",
                               "int p = ctx - chunk;                      /* absolute position of this query token */"),
    "per_head_encode_index": ("or_int8_encode_sat(or_div_f32(vx, v_scales[h]))",
                              "or_int8_encode_sat(or_div_f32(vx, v_scales[0]))"),
}


def _run_pins_against(lib_path: str) -> list:
    """Run every pin against the library at lib_path; return the names that failed."""
    mutant = oracle.Oracle(Path(lib_path))
    failed = []
    for pin in ALL_PINS:
        try:
            pin(mutant)
        except (AssertionError, ValueError):
            failed.append(pin.__name__)
    return failed


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistakes_are_caught(name):
    src = Path(oracle.__file__).with_name("oracle.c").read_text()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, "mutation anchor not found: %r" % old
    with tempfile.TemporaryDirectory() as tmp:
        csrc = Path(tmp) / "oracle.c"
        csrc.write_text(src.replace(old, new))
        lib = Path(tmp) / ("liboracle_%s.so" % name)
        oracle.build(csrc, lib)
        # a child process, so that a mutant that crashes cannot take the suite down
        code = ("import sys, json; sys.path[:0] = [%r, %r]; import test_oracle_pins as t; "
                "print(json.dumps(t._run_pins_against(%r)))"
                % (str(Path(__file__).resolve().parent.parent), str(Path(__file__).resolve().parent), str(lib)))
        r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600)
        assert r.returncode == 0, r.stderr[-2000:]
        failed = json.loads(r.stdout.strip().splitlines()[-1])
        assert failed, "no pin caught the planted mistake %s" % name
