"""pa_decode_static_ws: decode for callers that may not allocate device memory where they
run (engine plugins inside an enqueue callback, fixed-budget hosts, runtimes that own the
allocator).  It keeps its partials in the library's static per-device array instead of a
caller workspace.  Each case is checked through the C ABI against pa_decode on the same
inputs and against the CPU oracle, on two calls in a row (the second finds the first call's
leftovers in the shared array).  The cases run in one order on purpose: a large call first,
then calls whose partials are fewer or laid out differently, so that stale partials of an
earlier call would show up.  This file is collected last so that a failure here comes after
every other test has run."""
import ctypes

import numpy as np
import pytest
import torch

import workloads
import paged_kv_cache_428_b200 as pa
from paritylib import check_close, dev_scales, gpu_fill_quant, oracle_caches, oracle_out

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _static_call(out, case, kc, vc, partition, ks=1.0, vs=1.0):
    return pa.lib().pa_decode_static_ws(
        out.data_ptr(), case.q.data_ptr(), kc.data_ptr(), vc.data_ptr(), case.block_tables.data_ptr(),
        case.block_tables.shape[1], case.context_lens.data_ptr(), case.B, case.max_context_len, case.h_q,
        case.h_kv, case.d, case.bs, case.num_blocks, ctypes.c_float(case.scale), pa.cache_dtype_code(kc),
        ctypes.c_float(ks), ctypes.c_float(vs), partition,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _check_static(orc, case, partition, label):
    """pa_decode with a caller workspace, then two static-array calls; both compared with it
    and with the oracle within the decode tolerances."""
    case = case if case.q.is_cuda else _to_dev(case)
    if case.quantised:
        kc, vc = gpu_fill_quant(case, DEV)
    else:
        kc, vc = case.k_cache.clone(), case.v_cache.clone()
    ks, vs = dev_scales(case, DEV)
    pa.pa_reshape_and_cache(case.key_new, case.value_new, kc, vc, case.slot_mapping, ks, vs)
    need = pa.pa_decode_workspace_size(case.B, case.h_q, case.d, case.max_context_len, partition)
    assert need <= pa.PA_STATIC_WS_BYTES, (label, need)
    ref = torch.empty((case.B, case.h_q, case.d), dtype=torch.bfloat16, device=DEV)
    pa.pa_decode(ref, case.q, kc, vc, case.block_tables, case.context_lens, case.max_context_len, case.scale,
                 partition, ks, vs)
    okc, ovc = oracle_caches(case, orc)
    oref = oracle_out(case, orc, okc, ovc)
    fp8 = case.cache == "e4m3"
    check_close(ref, oref, fp8, label + " pa_decode")
    r = ref.float().cpu().numpy().astype(np.float64)
    for call in range(2):
        out = torch.full((case.B, case.h_q, case.d), float("nan"), dtype=torch.bfloat16, device=DEV)
        assert _static_call(out, case, kc, vc, partition, ks, vs) == 0, (label, call)
        torch.cuda.synchronize()
        check_close(out, r, fp8, "%s call %d vs pa_decode" % (label, call))
        check_close(out, oref, fp8, "%s call %d vs oracle" % (label, call))
    assert pa.pa_device_errors(clear=True) == 0, label
    return need


def _to_dev(case):
    for name in ("q", "key_new", "value_new", "slot_mapping", "block_tables", "context_lens", "k_cache", "v_cache",
                 "fill_k_rows", "fill_v_rows", "fill_slots"):
        t = getattr(case, name)
        if t is not None:
            setattr(case, name, t.to(DEV))
    return case


def test_static_workspace_decode_matches_pa_decode_and_oracle(orc):
    # 1. a large call: 32 sequences of up to 4096 tokens in 512-token partitions (merged in the
    #    partition kernel), its partials filling the front of the array
    big = _check_static(orc, workloads.make_case("llama3_8b_b64", 21, B=32), 512, "bf16 P=512")
    # 2. more than 16 partitions per group (64-token partitions of ~2k-token contexts): the
    #    separate merge pass reads partials laid out with another stride over call 1's leftovers
    case = workloads.make_case("llama3_8b_b64", 23, B=6, ctx_range=(1800, 2300))
    assert -(-case.max_context_len // 64) > 16
    _check_static(orc, case, 64, "bf16 P=64 (separate merge)")
    # 3. no split: nothing goes to the array (pa_decode_workspace_size is 0)
    case = workloads.make_case("llama3_8b_b64", 24, B=5, ctx_range=(20, 700))
    assert pa.pa_decode_workspace_size(case.B, case.h_q, case.d, case.max_context_len, 0) == 0
    _check_static(orc, case, 0, "bf16 P=0")
    # 4. PA_PARTITION_AUTO (the balanced schedule with its own partial layout; 16 query heads keep
    #    the largest AUTO workspace inside the array)
    _check_static(orc, workloads.make_case("llama3_8b_b64", 25, B=12, h_q=16), pa.PA_PARTITION_AUTO, "bf16 AUTO")
    # 5. a one-byte-code cache (INT8, per-tensor scales) on the tensor-core q8 kernel
    _check_static(orc, workloads.make_case("int8_mha_b32_bs16", 26, B=4, ctx_fixed=1500), 512, "int8 P=512")
    assert big > 0


def test_static_workspace_rejects_requests_beyond_its_size():
    case = workloads.make_case("llama3_8b_b64", 22, device=DEV, B=4)
    out = torch.empty((case.B, case.h_q, case.d), dtype=torch.bfloat16, device=DEV)
    # 4 sequences declared as 131072 tokens long with 16-token partitions: far beyond the array
    huge = pa.pa_decode_workspace_size(case.B, case.h_q, case.d, 131072, 16)
    assert huge > pa.PA_STATIC_WS_BYTES
    rc = pa.lib().pa_decode_static_ws(
        out.data_ptr(), case.q.data_ptr(), case.k_cache.data_ptr(), case.v_cache.data_ptr(),
        case.block_tables.data_ptr(), case.block_tables.shape[1], case.context_lens.data_ptr(), case.B, 131072,
        case.h_q, case.h_kv, case.d, case.bs, case.num_blocks, ctypes.c_float(case.scale), pa.PA_CACHE_BF16,
        ctypes.c_float(1.0), ctypes.c_float(1.0), 16, ctypes.c_void_p(0))
    assert rc == -3                                   # PA_ERR_WORKSPACE, nothing launched


def test_static_workspace_rejects_bad_arguments():
    """A call that fails pa_decode's argument checks returns their status (the checks run
    before the call queues its counter clear)."""
    case = workloads.make_case("llama3_8b_b64", 27, device=DEV, B=4)
    out = torch.empty((case.B, case.h_q, case.d), dtype=torch.bfloat16, device=DEV)

    def call(h_kv, head_dim, partition):
        return pa.lib().pa_decode_static_ws(
            out.data_ptr(), case.q.data_ptr(), case.k_cache.data_ptr(), case.v_cache.data_ptr(),
            case.block_tables.data_ptr(), case.block_tables.shape[1], case.context_lens.data_ptr(), case.B,
            case.max_context_len, case.h_q, h_kv, head_dim, case.bs, case.num_blocks, ctypes.c_float(case.scale),
            pa.PA_CACHE_BF16, ctypes.c_float(1.0), ctypes.c_float(1.0), partition, ctypes.c_void_p(0))
    assert call(5, case.d, 512) == -1                 # h_q % h_kv != 0: PA_ERR_INVALID_ARG
    assert call(case.h_kv, 96, 512) == -2             # head_dim 96: PA_ERR_UNSUPPORTED
    assert call(case.h_kv, case.d, 24) == -1          # partition not a multiple of the block size
    assert call(case.h_kv, case.d, -2) == -1          # below PA_PARTITION_AUTO
    torch.cuda.synchronize()
    assert pa.pa_device_errors(clear=True) == 0
