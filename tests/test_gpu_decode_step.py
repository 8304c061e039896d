"""pa_decode_step (append + decode in one call, the decode launched as a programmatic dependent
of the cache write) against the two calls made separately (bit-identical) and the oracle."""
import numpy as np
import pytest
import torch

import workloads
import paged_kv_cache_428_b200 as pa
from paritylib import check_close, codes, gpu_fill_quant, oracle_caches, oracle_out

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _caches(case):
    if case.quantised:
        return gpu_fill_quant(case, DEV)
    return case.k_cache.to(DEV).clone(), case.v_cache.to(DEV).clone()


@pytest.mark.parametrize("name,kw,P", [
    ("llama3_8b_b64", dict(B=12, ctx_range=(1, 2000)), 512),
    ("llama3_8b_b64", dict(B=12, ctx_range=(1, 2000)), 0),
    ("llama3_8b_b64", dict(B=12, ctx_range=(1, 2000)), pa.PA_PARTITION_AUTO),
    ("long_context_b8", dict(B=2, ctx_range=(9000, 12000)), 512),
    ("fp8_mha_b32_bs16", dict(B=4, ctx_fixed=900, h_q=8, h_kv=8), 256),
    ("int8_mha_b32_bs32", dict(B=4, ctx_fixed=1000, h_q=8, h_kv=8), 512),
    ("tiny_gqa2_d64", dict(), 0),
])
def test_step_equals_separate_calls_and_oracle(orc, name, kw, P):
    case = workloads.make_case(name, 3, **kw)
    mcl = case.max_context_len
    q, kn, vn = case.q.to(DEV), case.key_new.to(DEV), case.value_new.to(DEV)
    sl, tab, ctx = case.slot_mapping.to(DEV), case.block_tables.to(DEV), case.context_lens.to(DEV)
    # separate calls
    kc1, vc1 = _caches(case)
    out1 = torch.empty((case.B, case.h_q, case.d), dtype=torch.bfloat16, device=DEV)
    pa.pa_reshape_and_cache(kn, vn, kc1, vc1, sl, case.k_scale, case.v_scale)
    pa.pa_decode(out1, q, kc1, vc1, tab, ctx, mcl, case.scale, P, case.k_scale, case.v_scale)
    # one step
    kc2, vc2 = _caches(case)
    out2 = torch.empty_like(out1)
    pa.pa_decode_step(kn, vn, sl, out2, q, kc2, vc2, tab, ctx, mcl, case.scale, P, case.k_scale, case.v_scale)
    torch.cuda.synchronize()
    assert pa.pa_device_errors() == 0
    bits = lambda t: t.view(torch.uint8)                 # NaN sentinels: compare bit patterns
    assert torch.equal(bits(kc1), bits(kc2)) and torch.equal(bits(vc1), bits(vc2))
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))
    okc, ovc = oracle_caches(case, orc)
    assert np.array_equal(codes(kc2, case.cache), okc) and np.array_equal(codes(vc2, case.cache), ovc)
    check_close(out2, oracle_out(case, orc, okc, ovc), case.cache == "e4m3", name)


def test_step_rejects_bad_arguments_before_launching():
    case = workloads.make_case("tiny_gqa2_d64", 0)
    kc, vc = case.k_cache.to(DEV).clone(), case.v_cache.to(DEV).clone()
    out = torch.empty((case.B, case.h_q, case.d), dtype=torch.bfloat16, device=DEV)
    before = kc.clone()
    with pytest.raises(pa.PagedKVError):          # partition not a multiple of the block size
        pa.pa_decode_step(case.key_new.to(DEV), case.value_new.to(DEV), case.slot_mapping.to(DEV), out,
                          case.q.to(DEV), kc, vc, case.block_tables.to(DEV), case.context_lens.to(DEV),
                          case.max_context_len, case.scale, 24)
    torch.cuda.synchronize()
    assert torch.equal(before.view(torch.int16), kc.view(torch.int16))   # nothing was written (bit patterns)
