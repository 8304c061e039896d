"""Shared prompts and copy-on-write, end to end: the C++ allocator drives prefill, fork,
decode steps and CoW copies on the GPU; the oracle replays the same operations with the
reference allocator model and its own cache arithmetic.  Ids, copy pairs and caches must
agree exactly; decode outputs within the bf16 tolerance."""
import numpy as np
import pytest
import torch

import workloads
import paged_kv_cache_428_b200 as pa
from oracle.alloc_model import AllocatorModel
from paritylib import check_close, u16

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("seed", [0, 1])
def test_shared_prompt_fork_and_copy_on_write(orc, seed):
    P, S, L, bs, h_q, h_kv, d = 4, 8, 2048, 16, 32, 8, 128
    g = torch.Generator().manual_seed(seed)
    common = torch.randint(1, bs, (P,), generator=g).tolist()     # tokens shared after the prompt
    nb = P * (L // bs + 2) + P * S * 4 + 8
    alloc = pa.BlockAllocator(nb, bs, seed + 11)
    model = AllocatorModel(nb, bs, seed + 11)
    shape = (nb, h_kv, bs, d)
    kc = torch.full(shape, workloads.BF16_NAN, dtype=torch.int16, device=DEV).view(torch.bfloat16)
    vc = kc.clone()
    okc, ovc = u16(kc).copy(), u16(vc).copy()

    def write(rows_k, rows_v, slots):
        pa.pa_reshape_and_cache(rows_k.to(DEV), rows_v.to(DEV), kc, vc, torch.tensor(slots, device=DEV))
        orc.reshape_and_cache(u16(rows_k), u16(rows_v), okc, ovc, np.array(slots, np.int64), h_kv=h_kv, d=d,
                              bs=bs, num_blocks=nb)

    samples = []
    for p in range(P):
        sa, sm = alloc.new_seq(), model.new_seq()
        assert sa == sm
        n = L + common[p]
        slots, pair = alloc.append_n(sa, n)
        mslots, mpair = model.append_n(sm, n)
        assert slots == mslots and pair == mpair == (-1, -1)
        write(torch.randn(n, h_kv, d, generator=g).to(torch.bfloat16),
              torch.randn(n, h_kv, d, generator=g).to(torch.bfloat16), slots)
        group = [sa]
        for _ in range(S - 1):
            c = alloc.fork(sa)
            assert c == model.fork(sm)
            group.append(c)
        samples += group
    partial = alloc.block_table([samples[0]], L // bs + 1)[0][0, L // bs].item()
    assert alloc.refcount(partial) == S                        # the partly filled block is shared by 8

    max_blocks = L // bs + 8
    for step in range(3):
        slots, pairs = alloc.append_batch(samples)
        mres = [model.append_slot(s) for s in samples]
        assert slots == [r[0] for r in mres]
        assert pairs == [r[1] for r in mres if r[1][0] >= 0]
        if step == 0:
            assert len(pairs) == P * (S - 1)                   # n sharers -> n - 1 copies
        else:
            assert pairs == []
        if pairs:
            pt = torch.tensor(pairs, dtype=torch.int64)
            pa.pa_copy_blocks([kc], [vc], pt.to(DEV))
            orc.copy_blocks([okc], [ovc], pt.numpy(), block_bytes=h_kv * bs * d * 2, num_blocks=nb)
        B = len(samples)
        write(torch.randn(B, h_kv, d, generator=g).to(torch.bfloat16),
              torch.randn(B, h_kv, d, generator=g).to(torch.bfloat16), slots)
        tab, lens = alloc.block_table(samples, max_blocks)
        mtab, mlens = model.block_table(samples, max_blocks)
        assert tab.tolist() == mtab and lens.tolist() == mlens
        q = torch.randn(B, h_q, d, generator=g).to(torch.bfloat16)
        out = torch.empty((B, h_q, d), dtype=torch.bfloat16, device=DEV)
        pa.pa_decode(out, q.to(DEV), kc, vc, tab.to(DEV), lens.to(DEV), int(lens.max()), d ** -0.5, 512)
        torch.cuda.synchronize()
        assert np.array_equal(u16(kc), okc) and np.array_equal(u16(vc), ovc)
        ref = orc.paged_decode(u16(q), okc, ovc, tab.numpy(), lens.numpy(), h_kv=h_kv, bs=bs, scale=d ** -0.5)
        check_close(out, ref, False, "cow step %d" % step)
        model.check_invariants()
    st = alloc.stats()
    assert st == model.stats() and st["shared"] == P * (L // bs)   # full prompt blocks stay shared
