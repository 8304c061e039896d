"""pa_decode_static_ws: decode for callers that may not allocate device memory where they
run (engine plugins inside an enqueue callback, fixed-budget hosts, runtimes that own the
allocator).  It keeps its partials in the library's static per-device array instead of a
caller workspace.  Checked through the C ABI against pa_decode on the same inputs, on two
calls in a row (the second finds the first call's leftovers in the shared array).  This file
is collected last so that a failure here comes after every other test has run."""
import ctypes

import numpy as np
import pytest
import torch

import workloads
import paged_kv_cache_428_b200 as pa
from paritylib import BF16_ABS, BF16_REL

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _static_call(out, case, kc, vc, partition):
    return pa.lib().pa_decode_static_ws(
        out.data_ptr(), case.q.data_ptr(), kc.data_ptr(), vc.data_ptr(), case.block_tables.data_ptr(),
        case.block_tables.shape[1], case.context_lens.data_ptr(), case.B, case.max_context_len, case.h_q,
        case.h_kv, case.d, case.bs, case.num_blocks, ctypes.c_float(case.scale), pa.PA_CACHE_BF16,
        ctypes.c_float(1.0), ctypes.c_float(1.0), partition, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_static_workspace_decode_matches_pa_decode():
    case = workloads.make_case("llama3_8b_b64", 21, device=DEV, B=32)
    kc, vc = case.k_cache, case.v_cache
    pa.pa_reshape_and_cache(case.key_new, case.value_new, kc, vc, case.slot_mapping)
    P = 512
    need = pa.pa_decode_workspace_size(case.B, case.h_q, case.d, case.max_context_len, P)
    assert 0 < need <= pa.PA_STATIC_WS_BYTES
    ref = torch.empty((case.B, case.h_q, case.d), dtype=torch.bfloat16, device=DEV)
    pa.pa_decode(ref, case.q, kc, vc, case.block_tables, case.context_lens, case.max_context_len, case.scale, P)
    r = ref.float().cpu().numpy()
    for call in range(2):
        out = torch.full((case.B, case.h_q, case.d), float("nan"), dtype=torch.bfloat16, device=DEV)
        assert _static_call(out, case, kc, vc, P) == 0
        torch.cuda.synchronize()
        g = out.float().cpu().numpy()
        assert np.isfinite(g).all(), call
        err = float(np.abs(g - r).max())
        assert err <= BF16_ABS and err <= BF16_REL * float(np.abs(r).max()), (call, err)
    assert pa.pa_device_errors(clear=True) == 0


def test_static_workspace_rejects_requests_beyond_its_size():
    case = workloads.make_case("llama3_8b_b64", 22, device=DEV, B=4)
    out = torch.empty((case.B, case.h_q, case.d), dtype=torch.bfloat16, device=DEV)
    # 4 sequences declared as 131072 tokens long with 16-token partitions: far beyond the array
    case.context_lens = case.context_lens.clone()
    huge = pa.pa_decode_workspace_size(case.B, case.h_q, case.d, 131072, 16)
    assert huge > pa.PA_STATIC_WS_BYTES
    rc = pa.lib().pa_decode_static_ws(
        out.data_ptr(), case.q.data_ptr(), case.k_cache.data_ptr(), case.v_cache.data_ptr(),
        case.block_tables.data_ptr(), case.block_tables.shape[1], case.context_lens.data_ptr(), case.B, 131072,
        case.h_q, case.h_kv, case.d, case.bs, case.num_blocks, ctypes.c_float(case.scale), pa.PA_CACHE_BF16,
        ctypes.c_float(1.0), ctypes.c_float(1.0), 16, ctypes.c_void_p(0))
    assert rc == -3                                   # PA_ERR_WORKSPACE, nothing launched
