"""GPU cache write and block copy: bit-exact against the oracle (through the C ABI)."""
import numpy as np
import pytest
import torch

import workloads
import paged_kv_cache_428_b200 as pa
from paritylib import u16, u8

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _pool(nb, h_kv, bs, d, fp8):
    shape = (nb, h_kv, bs, d)
    if fp8:
        return (torch.full(shape, workloads.E4M3_NAN, dtype=torch.uint8, device=DEV),
                torch.full(shape, workloads.E4M3_NAN, dtype=torch.uint8, device=DEV))
    k = torch.full(shape, workloads.BF16_NAN, dtype=torch.int16, device=DEV).view(torch.bfloat16)
    return k, k.clone()


@pytest.mark.parametrize("fp8", [False, True])
@pytest.mark.parametrize("d,bs", [(64, 16), (128, 16), (128, 32), (128, 64), (64, 64)])
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_reshape_and_cache_bit_exact(orc, fp8, d, bs, seed):
    h_kv, nb = 4, 40
    T = 300 if seed else 37                                   # ragged token counts
    g = torch.Generator().manual_seed(seed)
    k_rows = (torch.randn(T, h_kv, d, generator=g) * (30 if fp8 else 1)).to(torch.bfloat16)
    v_rows = (torch.randn(T, h_kv, d, generator=g) * (30 if fp8 else 1)).to(torch.bfloat16)
    slots = torch.randperm(nb * bs, generator=g)[:T].to(torch.int64)
    slots[::7] = -1                                           # padding tokens are skipped
    ks, vs = (0.05, 0.031) if fp8 else (1.0, 1.0)
    kc, vc = _pool(nb, h_kv, bs, d, fp8)
    pa.pa_reshape_and_cache(k_rows.to(DEV), v_rows.to(DEV), kc, vc, slots.to(DEV), ks, vs)
    torch.cuda.synchronize()
    conv = u8 if fp8 else u16
    ok_, ov_ = conv(_pool(nb, h_kv, bs, d, fp8)[0]).copy(), conv(_pool(nb, h_kv, bs, d, fp8)[1]).copy()
    orc.reshape_and_cache(u16(k_rows), u16(v_rows), ok_, ov_, slots.numpy(), h_kv=h_kv, d=d, bs=bs, num_blocks=nb,
                          fp8=fp8, k_scale=ks, v_scale=vs)
    assert np.array_equal(conv(kc), ok_) and np.array_equal(conv(vc), ov_)
    if fp8:                                                   # saturation was exercised
        assert (np.abs(k_rows.float().numpy()) / ks > 448).any()


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
