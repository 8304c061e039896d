"""The OpenMP build of the oracle (the multi-core CPU baseline of bench.py) computes exactly what
the single-threaded build does: rows are independent and each row's arithmetic is the same, so
the outputs are equal bit for bit."""
import numpy as np
import torch

import oracle
import workloads


def test_openmp_build_matches_single_threaded():
    case = workloads.make_case("llama3_8b_b64", 31, B=6, ctx_range=(40, 700))
    u16 = lambda t: t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
    kc, vc = u16(case.k_cache).copy(), u16(case.v_cache).copy()
    oracle.load().reshape_and_cache(u16(case.key_new), u16(case.value_new), kc, vc, case.slot_mapping.numpy(),
                                    h_kv=case.h_kv, d=case.d, bs=case.bs, num_blocks=case.num_blocks)
    kw = dict(h_kv=case.h_kv, bs=case.bs, scale=case.scale)
    args = (u16(case.q), kc, vc, case.block_tables.numpy(), case.context_lens.numpy())
    one = oracle.load().paged_decode(*args, **kw)
    many = oracle.load(openmp=True).paged_decode(*args, **kw)
    assert np.isfinite(one).all()
    assert np.array_equal(one, many)
    rows = [(s, h) for s in range(case.B) for h in (0, 5, 31)]
    r1 = oracle.load().paged_decode_rows(rows, *args, **kw)
    r2 = oracle.load(openmp=True).paged_decode_rows(rows, *args, **kw)
    assert np.array_equal(r1, r2)
