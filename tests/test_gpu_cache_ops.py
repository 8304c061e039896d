"""GPU cache write and block copy: bit-exact against the oracle (through the C ABI)."""
import numpy as np
import pytest
import torch

import workloads
import paged_kv_cache_428_b200 as pa
from paritylib import codes, u16, u8

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _pool(nb, h_kv, bs, d, cache):
    """Device pools of the cache type filled with its never-written sentinel."""
    shape = (nb, h_kv, bs, d)
    if cache in (True, "e4m3"):
        return (torch.full(shape, workloads.E4M3_NAN, dtype=torch.uint8, device=DEV),
                torch.full(shape, workloads.E4M3_NAN, dtype=torch.uint8, device=DEV))
    if cache == "int8":
        return (torch.full(shape, workloads.INT8_UNUSED, dtype=torch.int8, device=DEV),
                torch.full(shape, workloads.INT8_UNUSED, dtype=torch.int8, device=DEV))
    k = torch.full(shape, workloads.BF16_NAN, dtype=torch.int16, device=DEV).view(torch.bfloat16)
    return k, k.clone()


@pytest.mark.parametrize("cache,per_head", [("bf16", False), ("e4m3", False), ("int8", False), ("e4m3", True),
                                            ("int8", True)])
@pytest.mark.parametrize("d,bs", [(64, 16), (128, 16), (128, 32), (128, 64), (64, 64)])
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_reshape_and_cache_bit_exact(orc, cache, per_head, d, bs, seed):
    h_kv, nb = 4, 40
    T = 300 if seed else 37                                   # ragged token counts
    quant = cache != "bf16"
    g = torch.Generator().manual_seed(seed)
    k_rows = (torch.randn(T, h_kv, d, generator=g) * (30 if quant else 1)).to(torch.bfloat16)
    v_rows = (torch.randn(T, h_kv, d, generator=g) * (30 if quant else 1)).to(torch.bfloat16)
    slots = torch.randperm(nb * bs, generator=g)[:T].to(torch.int64)
    slots[::7] = -1                                           # padding tokens are skipped
    if per_head:
        ks_np = np.array([0.05, 0.31, 0.011, 0.9], np.float32)
        vs_np = np.array([0.2, 0.031, 0.47, 0.07], np.float32)
        ks, vs = torch.from_numpy(ks_np).to(DEV), torch.from_numpy(vs_np).to(DEV)
    else:
        ks_np, vs_np = ks, vs = (0.05, 0.031) if quant else (1.0, 1.0)
    kc, vc = _pool(nb, h_kv, bs, d, cache)
    pa.pa_reshape_and_cache(k_rows.to(DEV), v_rows.to(DEV), kc, vc, slots.to(DEV), ks, vs)
    torch.cuda.synchronize()
    ok_, ov_ = (codes(t, cache).copy() for t in _pool(nb, h_kv, bs, d, cache))
    orc.reshape_and_cache(u16(k_rows), u16(v_rows), ok_, ov_, slots.numpy(), h_kv=h_kv, d=d, bs=bs, num_blocks=nb,
                          cache=cache, k_scale=ks_np, v_scale=vs_np)
    assert np.array_equal(codes(kc, cache), ok_) and np.array_equal(codes(vc, cache), ov_)
    if quant:                                                 # saturation was exercised
        qmax = workloads.QUANT_MAX[cache]
        assert (np.abs(k_rows.float().numpy()) / np.asarray(ks_np).reshape(-1)[:, None] > qmax).any()


def test_int8_write_ties_saturation(orc):
    """scale 1: every bf16 value in [-300, 300] is quantised directly -- exact halves (ties to
    even), values past +-127 (saturation), -0 and tiny values."""
    h_kv, d, bs, nb = 2, 64, 16, 64
    allbits = torch.arange(0, 1 << 16, dtype=torch.int32).to(torch.int16).view(torch.bfloat16)
    f = allbits.float()
    vals = allbits[torch.isfinite(f) & (f.abs() <= 300)]
    per_row = h_kv * d
    T = -(-vals.numel() // per_row)
    pad = torch.zeros(T * per_row - vals.numel(), dtype=torch.bfloat16)
    k_rows = torch.cat([vals, pad]).reshape(T, h_kv, d).contiguous()
    v_rows = (-k_rows.float()).to(torch.bfloat16).contiguous()
    assert T <= nb * bs
    slots = torch.randperm(nb * bs, generator=torch.Generator().manual_seed(2))[:T].to(torch.int64)
    kc, vc = _pool(nb, h_kv, bs, d, "int8")
    pa.pa_reshape_and_cache(k_rows.to(DEV), v_rows.to(DEV), kc, vc, slots.to(DEV), 1.0, 1.0)
    ok_ = np.full((nb, h_kv, bs, d), workloads.INT8_UNUSED, np.int8)
    ov_ = ok_.copy()
    orc.reshape_and_cache(u16(k_rows), u16(v_rows), ok_, ov_, slots.numpy(), h_kv=h_kv, d=d, bs=bs, num_blocks=nb,
                          cache="int8", k_scale=1.0, v_scale=1.0)
    assert np.array_equal(codes(kc, "int8"), ok_) and np.array_equal(codes(vc, "int8"), ov_)
    written = ok_[slots.numpy() // bs, :, slots.numpy() % bs, :]
    assert written.min() == -127 and written.max() == 127          # saturation, never -128


def test_e4m3_write_ties_subnormals_saturation(orc):
    """scale 1: every bf16 value is quantised directly, so many values sit exactly half-way
    between E4M3 neighbours (ties to even), below 2^-6 (subnormals) and above 448."""
    h_kv, d, bs, nb = 2, 128, 16, 8
    T = 32
    allbits = torch.arange(0, 1 << 16, dtype=torch.int32).to(torch.int16).view(torch.bfloat16)
    vals = allbits[torch.isfinite(allbits.float())]
    g = torch.Generator().manual_seed(5)
    pick = vals[torch.randint(0, vals.numel(), (2 * T * h_kv * d,), generator=g)]
    k_rows = pick[: T * h_kv * d].reshape(T, h_kv, d).contiguous()
    v_rows = pick[T * h_kv * d:].reshape(T, h_kv, d).contiguous()
    slots = torch.arange(T, dtype=torch.int64) * 3 % (nb * bs)
    kc, vc = _pool(nb, h_kv, bs, d, True)
    pa.pa_reshape_and_cache(k_rows.to(DEV), v_rows.to(DEV), kc, vc, slots.to(DEV), 1.0, 1.0)
    ok_ = np.full((nb, h_kv, bs, d), workloads.E4M3_NAN, np.uint8)
    ov_ = ok_.copy()
    orc.reshape_and_cache(u16(k_rows), u16(v_rows), ok_, ov_, slots.numpy(), h_kv=h_kv, d=d, bs=bs, num_blocks=nb,
                          fp8=True, k_scale=1.0, v_scale=1.0)
    assert np.array_equal(u8(kc), ok_) and np.array_equal(u8(vc), ov_)


def test_reshape_and_cache_strided_rows(orc):
    """K and V taken as views of one packed [T, 3, h_kv, d] tensor (stride 3*h_kv*d)."""
    T, h_kv, d, bs, nb = 50, 8, 128, 16, 20
    g = torch.Generator().manual_seed(3)
    qkv = torch.randn(T, 3, h_kv, d, generator=g).to(torch.bfloat16).to(DEV)
    k, v = qkv[:, 1], qkv[:, 2]
    slots = torch.randperm(nb * bs, generator=g)[:T].to(torch.int64)
    kc, vc = _pool(nb, h_kv, bs, d, False)
    pa.pa_reshape_and_cache(k, v, kc, vc, slots.to(DEV))
    ok_, ov_ = u16(_pool(nb, h_kv, bs, d, False)[0]).copy(), u16(_pool(nb, h_kv, bs, d, False)[1]).copy()
    orc.reshape_and_cache(u16(k.cpu()), u16(v.cpu()), ok_, ov_, slots.numpy(), h_kv=h_kv, d=d, bs=bs, num_blocks=nb)
    assert np.array_equal(u16(kc), ok_) and np.array_equal(u16(vc), ov_)


def test_reshape_and_cache_bad_slot_is_skipped_and_flagged():
    h_kv, d, bs, nb = 2, 64, 16, 4
    k_rows = torch.randn(3, h_kv, d).to(torch.bfloat16).to(DEV)
    kc, vc = _pool(nb, h_kv, bs, d, False)
    before = kc.clone()
    pa.pa_device_errors(clear=True)
    slots = torch.tensor([nb * bs, 5, nb * bs + 100], dtype=torch.int64, device=DEV)   # two past the pool
    pa.pa_reshape_and_cache(k_rows, k_rows, kc, vc, slots)
    assert pa.pa_device_errors(clear=True) & pa.PA_DEVERR_BAD_SLOT
    changed = (u16(kc) != u16(before)).reshape(nb, h_kv, bs, d).any(axis=(1, 3))
    assert changed.sum() == 1 and changed[0, 5]


@pytest.mark.parametrize("fp8", [False, True])
def test_copy_blocks_bit_exact(orc, fp8):
    L, nb, h_kv, bs, d = 4, 30, 8, 16, 128
    g = torch.Generator().manual_seed(11)
    dt = torch.uint8 if fp8 else torch.int16
    lo, hi = (0, 255) if fp8 else (-32768, 32767)
    ks = [torch.randint(lo, hi, (nb, h_kv, bs, d), generator=g, dtype=dt) for _ in range(L)]
    vs = [torch.randint(lo, hi, (nb, h_kv, bs, d), generator=g, dtype=dt) for _ in range(L)]
    pairs = torch.tensor([[3, 17], [0, 29], [3, 5], [12, 4], [7, 7]], dtype=torch.int64)
    view = (lambda t: t) if fp8 else (lambda t: t.view(torch.bfloat16))
    kd = [view(k.to(DEV)) for k in ks]
    vd = [view(v.to(DEV)) for v in vs]
    pa.pa_copy_blocks(kd, vd, pairs.to(DEV))
    torch.cuda.synchronize()
    kn = [k.numpy().copy() for k in ks]
    vn = [v.numpy().copy() for v in vs]
    orc.copy_blocks(kn, vn, pairs.numpy(), block_bytes=h_kv * bs * d * (1 if fp8 else 2), num_blocks=nb)
    for l in range(L):
        assert np.array_equal(kd[l].cpu().view(dt).numpy(), kn[l])
        assert np.array_equal(vd[l].cpu().view(dt).numpy(), vn[l])


def test_copy_blocks_bad_pair_is_skipped_and_flagged():
    nb, h_kv, bs, d = 6, 2, 16, 64
    k = torch.randn(nb, h_kv, bs, d).to(torch.bfloat16).to(DEV)
    v = k.clone()
    before = k.clone()
    pa.pa_device_errors(clear=True)
    pa.pa_copy_blocks([k], [v], torch.tensor([[0, nb], [-1, 2], [1, 3]], dtype=torch.int64, device=DEV))
    assert pa.pa_device_errors(clear=True) & pa.PA_DEVERR_BAD_PAIR
    exp = before.clone()
    exp[3] = before[1]
    assert torch.equal(k.view(torch.int16), exp.view(torch.int16))
