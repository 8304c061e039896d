"""B200-native paged-KV decode attention: Python binding of libpa.so (include/pa.h).

The binding only marshals arguments: it checks dtypes, shapes, devices and
contiguity of torch tensors, passes raw pointers and the current CUDA stream
to the C ABI, and raises :class:`PagedKVError` on a non-zero status.  Every
step of the computation runs in the library's CUDA kernels; there is no CPU
path.  Importing this package fails if libpa.so has not been built
(``python paged_kv_cache_428_b200/build.py``).

Functions keep the C names:

* :func:`pa_reshape_and_cache` -- write the step's new K/V rows into their slots
* :func:`pa_decode` -- split-context decode attention through the block table
  (= :func:`pa_decode_partitions` + :func:`pa_decode_merge`)
* :func:`pa_copy_blocks` -- copy-on-write block copy over all layers
* :class:`BlockAllocator` -- the host block allocator (free pool, refcounts,
  fork, copy-on-write decisions) that builds block tables and slot ids
"""
from __future__ import annotations

import ctypes
import math
from pathlib import Path
from typing import Optional, Sequence

import torch

_PKG = Path(__file__).resolve().parent
LIB_PATH = _PKG / "libpa.so"

PA_CACHE_BF16 = 0
PA_CACHE_E4M3 = 1
PA_CACHE_INT8 = 2
PA_PARTITION_AUTO = -1
PA_DEVERR_BAD_SLOT = 0x1
PA_DEVERR_BAD_BLOCK = 0x2
PA_DEVERR_BAD_PAIR = 0x4
PA_DEVERR_TIMEOUT = 0x8
PA_DEVERR_BAD_CHUNK = 0x10

STATUS = {0: "PA_OK", -1: "PA_ERR_INVALID_ARG", -2: "PA_ERR_UNSUPPORTED", -3: "PA_ERR_WORKSPACE",
          -4: "PA_ERR_OOM", -5: "PA_ERR_CUDA", -6: "PA_ERR_NOT_FOUND"}


class PagedKVError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__("%s: %s (%s)" % (what, STATUS.get(status, status), _lib.pa_status_str(status).decode()))


def _load() -> ctypes.CDLL:
    if not LIB_PATH.exists():
        raise ImportError("libpa.so is not built; run `python paged_kv_cache_428_b200/build.py` "
                          "(there is no fallback implementation)")
    L = ctypes.CDLL(str(LIB_PATH))
    vp, i32, i64, f32, sz, u64 = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float,
                                  ctypes.c_size_t, ctypes.c_uint64)
    P64 = ctypes.POINTER(ctypes.c_int64)
    P32 = ctypes.POINTER(ctypes.c_int32)
    PI = ctypes.POINTER(ctypes.c_int)
    sig = {
        "pa_status_str": (ctypes.c_char_p, [i32]),
        "pa_version": (i32, []),
        "pa_kv_bytes_per_token": (sz, [i32, i32, i32, i32]),
        "pa_kv_capacity_tokens": (sz, [sz, i32, i32, i32, i32]),
        "pa_reshape_and_cache": (i32, [vp, vp, i64, i64, vp, vp, vp, i32, i32, i32, i32, i32, i32, f32, f32, vp]),
        "pa_reshape_and_cache_head_scales": (i32, [vp, vp, i64, i64, vp, vp, vp, i32, i32, i32, i32, i32, i32, vp,
                                                   vp, vp]),
        "pa_decode_workspace_size": (sz, [i32, i32, i32, i32, i32]),
        "pa_decode": (i32, [vp, vp, vp, vp, vp, i32, vp, i32, i32, i32, i32, i32, i32, i32, f32, i32, f32, f32,
                            i32, vp, sz, vp]),
        "pa_decode_partitions": (i32, [vp, vp, vp, vp, vp, i32, vp, i32, i32, i32, i32, i32, i32, i32, f32, i32,
                                       f32, f32, i32, vp, sz, vp]),
        "pa_decode_merge": (i32, [vp, vp, i32, i32, i32, i32, i32, vp, sz, vp]),
        "pa_decode_head_scales": (i32, [vp, vp, vp, vp, vp, i32, vp, i32, i32, i32, i32, i32, i32, i32, f32, i32,
                                        vp, vp, i32, vp, sz, vp]),
        "pa_decode_static_ws": (i32, [vp, vp, vp, vp, vp, i32, vp, i32, i32, i32, i32, i32, i32, i32, f32, i32,
                                      f32, f32, i32, vp]),
        "pa_copy_blocks": (i32, [vp, vp, i32, vp, i32, sz, i32, vp]),
        "pa_decode_step": (i32, [vp, vp, i64, i64, vp, vp, vp, vp, vp, vp, i32, vp, i32, i32, i32, i32, i32, i32, i32,
                                 f32, i32, f32, f32, i32, vp, sz, vp]),
        "pa_prefill": (i32, [vp, vp, vp, vp, vp, i32, vp, vp, i32, i32, i32, i32, i32, i32, i32, f32, i32, vp]),
        "pa_prefill_workspace_size": (sz, []),
        "pa_prefill_ws": (i32, [vp, vp, vp, vp, vp, i32, vp, vp, i32, i32, i32, i32, i32, i32, i32, f32, i32, vp, sz,
                                vp]),
        "pa_device_errors": (i32, [ctypes.POINTER(ctypes.c_uint), i32]),
        "pa_validate_block_tables": (i32, [vp, i32, vp, i32, i32, i32]),
        "pa_validate_slots": (i32, [vp, i32, i32, i32]),
        "pa_alloc_create": (vp, [i32, i32, u64]),
        "pa_alloc_destroy": (None, [vp]),
        "pa_alloc_new_seq": (i32, [vp, P64]),
        "pa_alloc_append_slot": (i32, [vp, i64, P64, P64, P64]),
        "pa_alloc_append_n": (i32, [vp, i64, i32, vp, P64, P64]),
        "pa_alloc_append_batch": (i32, [vp, vp, i32, vp, vp, PI]),
        "pa_alloc_fork": (i32, [vp, i64, P64]),
        "pa_alloc_free_seq": (i32, [vp, i64]),
        "pa_alloc_block_table": (i32, [vp, vp, i32, vp, i32, vp]),
        "pa_alloc_seq_len": (i32, [vp, i64, P64]),
        "pa_alloc_stats": (i32, [vp, PI, PI, PI, P64]),
        "pa_alloc_refcount": (i32, [vp, i32]),
        "pa_alloc_new_seq_prefix": (i32, [vp, vp, i32, P64, vp, PI]),
        "pa_alloc_prefix_stats": (i32, [vp, P64, P64, PI, PI]),
        "pa_alloc_order_by_prefix": (i32, [vp, vp, i32, vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    return L


_lib = _load()


def lib() -> ctypes.CDLL:
    """The loaded libpa.so (ctypes handle)."""
    return _lib


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise PagedKVError(rc, what)


def _stream_ptr(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _need(t: torch.Tensor, name: str, dtypes, ndim: Optional[int] = None, cuda: bool = True) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a torch.Tensor" % name)
    if t.dtype not in dtypes:
        raise TypeError("%s: dtype %s, expected one of %s" % (name, t.dtype, dtypes))
    if ndim is not None and t.dim() != ndim:
        raise ValueError("%s: expected %d dims, got shape %s" % (name, ndim, tuple(t.shape)))
    if cuda and not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)


CACHE_DTYPES = (torch.bfloat16, torch.uint8, torch.float8_e4m3fn, torch.int8)


def cache_dtype_code(cache: torch.Tensor) -> int:
    """bf16 -> PA_CACHE_BF16; uint8 / float8_e4m3fn (E4M3 codes) -> PA_CACHE_E4M3;
    int8 (symmetric INT8 codes) -> PA_CACHE_INT8."""
    if cache.dtype == torch.bfloat16:
        return PA_CACHE_BF16
    if cache.dtype in (torch.uint8, torch.float8_e4m3fn):
        return PA_CACHE_E4M3
    if cache.dtype == torch.int8:
        return PA_CACHE_INT8
    raise TypeError("cache dtype must be bfloat16, uint8 / float8_e4m3fn (E4M3 codes) or int8, got %s"
                    % cache.dtype)


def _head_scales(k_scale, v_scale, h_kv: int):
    """(k_ptr, v_ptr) of per-KV-head scale tensors, or None for per-tensor float scales."""
    per_head = [isinstance(x, torch.Tensor) for x in (k_scale, v_scale)]
    if not any(per_head):
        return None
    if not all(per_head):
        raise TypeError("k_scale and v_scale must both be floats (per tensor) or both tensors (per KV head)")
    for t, n in ((k_scale, "k_scale"), (v_scale, "v_scale")):
        _need(t, n, (torch.float32,), 1)
        if t.shape[0] != h_kv:
            raise ValueError("%s: expected %d per-head scales, got %d" % (n, h_kv, t.shape[0]))
    return k_scale.data_ptr(), v_scale.data_ptr()


# ----------------------------------------------------------------------------------------------
def pa_kv_bytes_per_token(layers: int, h_kv: int, head_dim: int, elem_bytes: int) -> int:
    return int(_lib.pa_kv_bytes_per_token(layers, h_kv, head_dim, elem_bytes))


def pa_kv_capacity_tokens(budget_bytes: int, layers: int, h_kv: int, head_dim: int, elem_bytes: int) -> int:
    return int(_lib.pa_kv_capacity_tokens(budget_bytes, layers, h_kv, head_dim, elem_bytes))


def pa_version() -> int:
    return int(_lib.pa_version())


def pa_status_str(status: int) -> str:
    return _lib.pa_status_str(status).decode()


def pa_reshape_and_cache(key: torch.Tensor, value: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                         slot_mapping: torch.Tensor, k_scale=1.0, v_scale=1.0, stream=None) -> None:
    """key/value bf16 [T, h_kv, d] (rows may be strided in dim 0); caches [NB, h_kv, bs, d].
    Quantised caches take float scales (per tensor) or CUDA fp32 [h_kv] tensors (per KV head,
    pa_reshape_and_cache_head_scales)."""
    heads = _head_scales(k_scale, v_scale, key.shape[1])
    if heads is None:
        args = reshape_call_args(key, value, k_cache, v_cache, slot_mapping, k_scale, v_scale)
        _check(_lib.pa_reshape_and_cache(*args, _stream_ptr(stream)), "pa_reshape_and_cache")
    else:
        args = reshape_call_args(key, value, k_cache, v_cache, slot_mapping)[:-2]
        _check(_lib.pa_reshape_and_cache_head_scales(*args, *heads, _stream_ptr(stream)),
               "pa_reshape_and_cache_head_scales")


def pa_decode_workspace_size(num_seqs: int, h_q: int, head_dim: int, max_context_len: int,
                             partition_size: int) -> int:
    return int(_lib.pa_decode_workspace_size(num_seqs, h_q, head_dim, max_context_len, partition_size))


def make_workspace(num_seqs: int, h_q: int, head_dim: int, max_context_len: int, partition_size: int,
                   device="cuda") -> torch.Tensor:
    """A caller-owned, zero-filled workspace of the size pa_decode needs (uint8, possibly
    empty).  Reusable by consecutive calls that do not overlap on the GPU."""
    n = pa_decode_workspace_size(num_seqs, h_q, head_dim, max_context_len, partition_size)
    return torch.zeros(max(n, 16), dtype=torch.uint8, device=device)


def _decode_args(out, q, k_cache, v_cache, block_tables, context_lens, max_context_len, scale, partition_size,
                 k_scale, v_scale, workspace):
    _need(out, "out", (torch.bfloat16,), 3)
    _need(q, "q", (torch.bfloat16,), 3)
    _need(k_cache, "k_cache", CACHE_DTYPES, 4)
    _need(v_cache, "v_cache", (k_cache.dtype,), 4)
    _need(block_tables, "block_tables", (torch.int32,), 2)
    _need(context_lens, "context_lens", (torch.int32,), 1)
    B, h_q, d = q.shape
    NB, h_kv, bs, d2 = k_cache.shape
    if tuple(out.shape) != (B, h_q, d) or d2 != d or tuple(v_cache.shape) != tuple(k_cache.shape) \
            or block_tables.shape[0] != B or context_lens.shape[0] != B:
        raise ValueError("shape mismatch between out, q, caches, block_tables and context_lens")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    ws_ptr, ws_bytes = 0, 0
    if workspace is not None:
        _need(workspace, "workspace", (torch.uint8,), 1)
        ws_ptr, ws_bytes = workspace.data_ptr(), workspace.numel()
    return (out.data_ptr(), q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), block_tables.data_ptr(),
            block_tables.shape[1], context_lens.data_ptr(), B, int(max_context_len), h_q, h_kv, d, bs, NB,
            float(scale), cache_dtype_code(k_cache), _f(k_scale), _f(v_scale), int(partition_size),
            ws_ptr, ws_bytes)


def _f(x) -> float:
    return 1.0 if isinstance(x, torch.Tensor) else float(x)


def decode_call_args(out, q, k_cache, v_cache, block_tables, context_lens, max_context_len: int,
                     scale: float = None, partition_size: int = 512, k_scale: float = 1.0, v_scale: float = 1.0,
                     workspace: Optional[torch.Tensor] = None) -> tuple:
    """Checked raw arguments of pa_decode / pa_decode_partitions (all but the stream), for
    callers that issue the same call many times: ``lib().pa_decode(*args, stream)``."""
    return _decode_args(out, q, k_cache, v_cache, block_tables, context_lens, max_context_len, scale,
                        partition_size, k_scale, v_scale, workspace)


def merge_call_args(out, context_lens, max_context_len: int, partition_size: int,
                    workspace: Optional[torch.Tensor]) -> tuple:
    """Checked raw arguments of pa_decode_merge (all but the stream)."""
    _need(out, "out", (torch.bfloat16,), 3)
    _need(context_lens, "context_lens", (torch.int32,), 1)
    B, h_q, d = out.shape
    ws_ptr, ws_bytes = (workspace.data_ptr(), workspace.numel()) if workspace is not None else (0, 0)
    return (out.data_ptr(), context_lens.data_ptr(), B, int(max_context_len), h_q, d, int(partition_size), ws_ptr,
            ws_bytes)


def reshape_call_args(key, value, k_cache, v_cache, slot_mapping, k_scale: float = 1.0,
                      v_scale: float = 1.0) -> tuple:
    """Checked raw arguments of pa_reshape_and_cache (all but the stream)."""
    for t, n in ((key, "key"), (value, "value")):
        if t.dtype != torch.bfloat16 or not t.is_cuda or t.dim() != 3 or t.stride(2) != 1 or t.stride(1) != t.shape[2]:
            raise ValueError("%s must be a CUDA bf16 [T, h_kv, d] tensor with packed heads" % n)
    _need(k_cache, "k_cache", CACHE_DTYPES, 4)
    _need(v_cache, "v_cache", (k_cache.dtype,), 4)
    _need(slot_mapping, "slot_mapping", (torch.int64,), 1)
    T, h_kv, d = key.shape
    NB, h2, bs, d2 = k_cache.shape
    if h2 != h_kv or d2 != d or tuple(v_cache.shape) != tuple(k_cache.shape) or value.shape != key.shape \
            or slot_mapping.shape[0] != T:
        raise ValueError("shape mismatch between key/value, caches and slot_mapping")
    return (key.data_ptr(), value.data_ptr(), key.stride(0), value.stride(0), k_cache.data_ptr(), v_cache.data_ptr(),
            slot_mapping.data_ptr(), T, h_kv, d, bs, NB, cache_dtype_code(k_cache), float(k_scale), float(v_scale))


def pa_decode(out, q, k_cache, v_cache, block_tables, context_lens, max_context_len: int, scale: float = None,
              partition_size: int = 512, k_scale=1.0, v_scale=1.0,
              workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """out[s, h] = softmax(scale * q[s, h] . K^T) . V over the paged cache; returns out.
    Quantised caches take float scales (per tensor) or CUDA fp32 [h_kv] tensors (per KV head,
    pa_decode_head_scales)."""
    if workspace is None:
        workspace = make_workspace(q.shape[0], q.shape[1], q.shape[2], max_context_len, partition_size, q.device)
    args = _decode_args(out, q, k_cache, v_cache, block_tables, context_lens, max_context_len, scale,
                        partition_size, k_scale, v_scale, workspace)
    heads = _head_scales(k_scale, v_scale, k_cache.shape[1])
    if heads is None:
        _check(_lib.pa_decode(*args, _stream_ptr(stream)), "pa_decode")
    else:
        _check(_lib.pa_decode_head_scales(*args[:16], *heads, *args[18:], _stream_ptr(stream)),
               "pa_decode_head_scales")
    return out


def pa_decode_partitions(out, q, k_cache, v_cache, block_tables, context_lens, max_context_len: int,
                         scale: float = None, partition_size: int = 512, k_scale: float = 1.0,
                         v_scale: float = 1.0, workspace: Optional[torch.Tensor] = None, stream=None) -> None:
    if _head_scales(k_scale, v_scale, k_cache.shape[1]) is not None:
        raise TypeError("pa_decode_partitions takes per-tensor scales; use pa_decode for per-head scales")
    args = _decode_args(out, q, k_cache, v_cache, block_tables, context_lens, max_context_len, scale,
                        partition_size, k_scale, v_scale, workspace)
    _check(_lib.pa_decode_partitions(*args, _stream_ptr(stream)), "pa_decode_partitions")


def pa_decode_merge(out, context_lens, max_context_len: int, partition_size: int,
                    workspace: Optional[torch.Tensor], stream=None) -> None:
    _need(out, "out", (torch.bfloat16,), 3)
    _need(context_lens, "context_lens", (torch.int32,), 1)
    B, h_q, d = out.shape
    ws_ptr, ws_bytes = (workspace.data_ptr(), workspace.numel()) if workspace is not None else (0, 0)
    _check(_lib.pa_decode_merge(out.data_ptr(), context_lens.data_ptr(), B, int(max_context_len), h_q, d,
                                int(partition_size), ws_ptr, ws_bytes, _stream_ptr(stream)), "pa_decode_merge")


def step_call_args(key, value, slot_mapping, out, q, k_cache, v_cache, block_tables, context_lens,
                   max_context_len: int, scale: float = None, partition_size: int = 512, k_scale: float = 1.0,
                   v_scale: float = 1.0, workspace: Optional[torch.Tensor] = None) -> tuple:
    """Checked raw arguments of pa_decode_step (all but the stream)."""
    r = reshape_call_args(key, value, k_cache, v_cache, slot_mapping, k_scale, v_scale)
    d = _decode_args(out, q, k_cache, v_cache, block_tables, context_lens, max_context_len, scale, partition_size,
                     k_scale, v_scale, workspace)
    if key.shape[0] != q.shape[0]:
        raise ValueError("pa_decode_step appends one token per sequence: key has %d rows for %d sequences"
                         % (key.shape[0], q.shape[0]))
    # key, value, key_stride, value_stride, slot_mapping, then pa_decode's arguments
    return (r[0], r[1], r[2], r[3], r[6]) + d[:2] + (k_cache.data_ptr(), v_cache.data_ptr()) + d[4:]


def pa_decode_step(key, value, slot_mapping, out, q, k_cache, v_cache, block_tables, context_lens,
                   max_context_len: int, scale: float = None, partition_size: int = 512, k_scale: float = 1.0,
                   v_scale: float = 1.0, workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """One decode step: write each sequence's appended token (row s of key/value, slot_mapping[s]),
    then attend; the decode overlaps the write (programmatic dependent launch).  Returns out."""
    if workspace is None:
        workspace = make_workspace(q.shape[0], q.shape[1], q.shape[2], max_context_len, partition_size, q.device)
    args = step_call_args(key, value, slot_mapping, out, q, k_cache, v_cache, block_tables, context_lens,
                          max_context_len, scale, partition_size, k_scale, v_scale, workspace)
    _check(_lib.pa_decode_step(*args, _stream_ptr(stream)), "pa_decode_step")
    return out


PA_STATIC_WS_BYTES = 16 * 1024 * 1024


def pa_decode_static_ws(out, q, k_cache, v_cache, block_tables, context_lens, max_context_len: int,
                        scale: float = None, partition_size: int = 512, k_scale: float = 1.0, v_scale: float = 1.0,
                        stream=None) -> torch.Tensor:
    """pa_decode without a workspace argument and without any allocation: the partials go to
    the library's static per-device array (PA_STATIC_WS_BYTES).  For callers that may not
    allocate device memory where they run.  Calls that can overlap on the GPU race on that
    array; a request needing more scratch than the array raises PagedKVError (workspace)."""
    if _head_scales(k_scale, v_scale, k_cache.shape[1]) is not None:
        raise TypeError("pa_decode_static_ws takes per-tensor scales")
    args = _decode_args(out, q, k_cache, v_cache, block_tables, context_lens, max_context_len, scale,
                        partition_size, k_scale, v_scale, None)
    _check(_lib.pa_decode_static_ws(*args[:-2], _stream_ptr(stream)), "pa_decode_static_ws")
    return out


def prefill_call_args(out, q, k_cache, v_cache, block_tables, query_start, context_lens, max_query_len: int,
                      scale: float = None) -> tuple:
    """Checked raw arguments of pa_prefill (all but the stream)."""
    _need(out, "out", (torch.bfloat16,), 3)
    _need(q, "q", (torch.bfloat16,), 3)
    _need(k_cache, "k_cache", CACHE_DTYPES, 4)
    _need(v_cache, "v_cache", (k_cache.dtype,), 4)
    _need(block_tables, "block_tables", (torch.int32,), 2)
    _need(query_start, "query_start", (torch.int32,), 1)
    _need(context_lens, "context_lens", (torch.int32,), 1)
    T, h_q, d = q.shape
    NB, h_kv, bs, d2 = k_cache.shape
    B = context_lens.shape[0]
    if tuple(out.shape) != (T, h_q, d) or d2 != d or tuple(v_cache.shape) != tuple(k_cache.shape) \
            or block_tables.shape[0] != B or query_start.shape[0] != B + 1:
        raise ValueError("shape mismatch between out, q, caches, block_tables, query_start and context_lens")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    return (out.data_ptr(), q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), block_tables.data_ptr(),
            block_tables.shape[1], query_start.data_ptr(), context_lens.data_ptr(), B, int(max_query_len), h_q, h_kv,
            d, bs, NB, float(scale), cache_dtype_code(k_cache))


def pa_prefill(out, q, k_cache, v_cache, block_tables, query_start, context_lens, max_query_len: int,
               scale: float = None, stream=None) -> torch.Tensor:
    """Causal attention of each sequence's chunk of query rows over the paged cache; returns out."""
    args = prefill_call_args(out, q, k_cache, v_cache, block_tables, query_start, context_lens, max_query_len, scale)
    _check(_lib.pa_prefill(*args, _stream_ptr(stream)), "pa_prefill")
    return out


def pa_prefill_workspace_size() -> int:
    return int(_lib.pa_prefill_workspace_size())


def make_prefill_workspace(device="cuda") -> torch.Tensor:
    """A zero-filled workspace for pa_prefill_ws (each call leaves it zero again).  Calls that
    share one must not run at the same time."""
    return torch.zeros(pa_prefill_workspace_size(), dtype=torch.uint8, device=device)


def pa_prefill_ws(out, q, k_cache, v_cache, block_tables, query_start, context_lens, max_query_len: int,
                  workspace: torch.Tensor, scale: float = None, stream=None) -> torch.Tensor:
    """pa_prefill on the work-queue schedule (one CTA per SM claiming work items); returns out."""
    args = prefill_call_args(out, q, k_cache, v_cache, block_tables, query_start, context_lens, max_query_len, scale)
    _need(workspace, "workspace", (torch.uint8,), 1)
    _check(_lib.pa_prefill_ws(*args, workspace.data_ptr(), workspace.numel(), _stream_ptr(stream)), "pa_prefill_ws")
    return out


def pa_copy_blocks(k_caches: Sequence[torch.Tensor], v_caches: Sequence[torch.Tensor], block_pairs: torch.Tensor,
                   stream=None) -> None:
    """block_pairs int64 [n, 2] (src, dst) on the device; every layer's K and V block is copied."""
    if len(k_caches) != len(v_caches) or len(k_caches) == 0:
        raise ValueError("need the same, non-zero number of K and V caches")
    ref = k_caches[0]
    for t in list(k_caches) + list(v_caches):
        _need(t, "cache", (ref.dtype,), 4)
        if tuple(t.shape) != tuple(ref.shape):
            raise ValueError("all caches must have the same shape")
    _need(block_pairs, "block_pairs", (torch.int64,), 2)
    if block_pairs.shape[1] != 2:
        raise ValueError("block_pairs must be [n, 2]")
    L = len(k_caches)
    kp = (ctypes.c_void_p * L)(*[t.data_ptr() for t in k_caches])
    vp = (ctypes.c_void_p * L)(*[t.data_ptr() for t in v_caches])
    block_bytes = ref[0].numel() * ref.element_size()
    _check(_lib.pa_copy_blocks(ctypes.cast(kp, ctypes.c_void_p), ctypes.cast(vp, ctypes.c_void_p), L,
                               block_pairs.data_ptr(), block_pairs.shape[0], block_bytes, ref.shape[0],
                               _stream_ptr(stream)), "pa_copy_blocks")


def pa_device_errors(clear: bool = True) -> int:
    """Error bits the kernels recorded on the current device (synchronises the device)."""
    v = ctypes.c_uint(0)
    _check(_lib.pa_device_errors(ctypes.byref(v), int(clear)), "pa_device_errors")
    return int(v.value)


def pa_validate_block_tables(block_tables: torch.Tensor, context_lens: torch.Tensor, block_size: int,
                             num_blocks: int) -> int:
    """Host copies (CPU int32 tensors); returns the status code."""
    bt = block_tables.to("cpu", torch.int32).contiguous()
    cl = context_lens.to("cpu", torch.int32).contiguous()
    return int(_lib.pa_validate_block_tables(bt.data_ptr(), bt.shape[1], cl.data_ptr(), bt.shape[0], block_size,
                                             num_blocks))


def pa_validate_slots(slot_mapping: torch.Tensor, block_size: int, num_blocks: int) -> int:
    sm = slot_mapping.to("cpu", torch.int64).contiguous()
    return int(_lib.pa_validate_slots(sm.data_ptr(), sm.numel(), block_size, num_blocks))


# ----------------------------------------------------------------------------------------------
class BlockAllocator:
    """Host block allocator (pa_alloc_* in pa.h): global free pool, per-block refcounts,
    per-sequence block lists, fork, copy-on-write decisions, release."""

    def __init__(self, num_blocks: int, block_size: int, seed: int = 0):
        self._h = _lib.pa_alloc_create(num_blocks, block_size, seed)
        if not self._h:
            raise PagedKVError(-1, "pa_alloc_create")
        self.num_blocks = num_blocks
        self.block_size = block_size

    def close(self) -> None:
        if self._h:
            _lib.pa_alloc_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def new_seq(self) -> int:
        sid = ctypes.c_int64()
        _check(_lib.pa_alloc_new_seq(self._h, ctypes.byref(sid)), "pa_alloc_new_seq")
        return sid.value

    def append_slot(self, seq: int):
        """Returns (slot, (cow_src, cow_dst)); (-1, -1) when no copy is needed."""
        slot, s, d = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
        _check(_lib.pa_alloc_append_slot(self._h, seq, ctypes.byref(slot), ctypes.byref(s), ctypes.byref(d)),
               "pa_alloc_append_slot")
        return slot.value, (s.value, d.value)

    def append_n(self, seq: int, n: int):
        slots = (ctypes.c_int64 * max(n, 1))()
        s, d = ctypes.c_int64(), ctypes.c_int64()
        _check(_lib.pa_alloc_append_n(self._h, seq, n, ctypes.cast(slots, ctypes.c_void_p), ctypes.byref(s),
                                      ctypes.byref(d)), "pa_alloc_append_n")
        return list(slots)[:n], (s.value, d.value)

    def append_batch(self, seqs: Sequence[int]):
        """One token for each sequence (a decode step): (slots, [(src, dst), ...])."""
        n = len(seqs)
        sq = (ctypes.c_int64 * max(n, 1))(*seqs)
        slots = (ctypes.c_int64 * max(n, 1))()
        pairs = (ctypes.c_int64 * max(2 * n, 2))()
        ncow = ctypes.c_int()
        _check(_lib.pa_alloc_append_batch(self._h, ctypes.cast(sq, ctypes.c_void_p), n,
                                          ctypes.cast(slots, ctypes.c_void_p), ctypes.cast(pairs, ctypes.c_void_p),
                                          ctypes.byref(ncow)), "pa_alloc_append_batch")
        return list(slots)[:n], [(pairs[2 * i], pairs[2 * i + 1]) for i in range(ncow.value)]

    def fork(self, parent: int) -> int:
        c = ctypes.c_int64()
        _check(_lib.pa_alloc_fork(self._h, parent, ctypes.byref(c)), "pa_alloc_fork")
        return c.value

    def free_seq(self, seq: int) -> None:
        _check(_lib.pa_alloc_free_seq(self._h, seq), "pa_alloc_free_seq")

    def block_table(self, seqs: Sequence[int], max_blocks: int):
        """(table int32 [n, max_blocks] with -1 padding, context_lens int32 [n]) as CPU tensors."""
        n = len(seqs)
        sq = torch.tensor(list(seqs), dtype=torch.int64)
        table = torch.empty((n, max_blocks), dtype=torch.int32)
        lens = torch.empty((n,), dtype=torch.int32)
        _check(_lib.pa_alloc_block_table(self._h, sq.data_ptr(), n, table.data_ptr(), max_blocks, lens.data_ptr()),
               "pa_alloc_block_table")
        return table, lens

    def seq_len(self, seq: int) -> int:
        n = ctypes.c_int64()
        _check(_lib.pa_alloc_seq_len(self._h, seq, ctypes.byref(n)), "pa_alloc_seq_len")
        return n.value

    def stats(self) -> dict:
        f, u, s = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
        fr = ctypes.c_int64()
        _check(_lib.pa_alloc_stats(self._h, ctypes.byref(f), ctypes.byref(u), ctypes.byref(s), ctypes.byref(fr)),
               "pa_alloc_stats")
        return {"free": f.value, "used": u.value, "shared": s.value, "frag_tokens": fr.value}

    def new_seq_prefix(self, tokens: Sequence[int]):
        """A sequence holding the prompt `tokens`, sharing cached full blocks of an identical
        prefix: returns (seq_id, slots, cached_tokens); write K/V only for tokens[cached:]."""
        n = len(tokens)
        tk = (ctypes.c_int32 * max(n, 1))(*tokens)
        slots = (ctypes.c_int64 * max(n, 1))()
        sid, cached = ctypes.c_int64(), ctypes.c_int()
        _check(_lib.pa_alloc_new_seq_prefix(self._h, ctypes.cast(tk, ctypes.c_void_p), n, ctypes.byref(sid),
                                            ctypes.cast(slots, ctypes.c_void_p), ctypes.byref(cached)),
               "pa_alloc_new_seq_prefix")
        return sid.value, list(slots)[:n], cached.value

    def prefix_stats(self) -> dict:
        h, m = ctypes.c_int64(), ctypes.c_int64()
        c, e = ctypes.c_int(), ctypes.c_int()
        _check(_lib.pa_alloc_prefix_stats(self._h, ctypes.byref(h), ctypes.byref(m), ctypes.byref(c),
                                          ctypes.byref(e)), "pa_alloc_prefix_stats")
        return {"hit_tokens": h.value, "miss_tokens": m.value, "cached_blocks": c.value, "evictable": e.value}

    def order_by_prefix(self, seqs: Sequence[int]) -> list:
        n = len(seqs)
        sq = (ctypes.c_int64 * max(n, 1))(*seqs)
        order = (ctypes.c_int32 * max(n, 1))()
        _check(_lib.pa_alloc_order_by_prefix(self._h, ctypes.cast(sq, ctypes.c_void_p), n,
                                             ctypes.cast(order, ctypes.c_void_p)), "pa_alloc_order_by_prefix")
        return list(order)[:n]

    def refcount(self, block: int) -> int:
        rc = _lib.pa_alloc_refcount(self._h, block)
        if rc < 0:
            raise PagedKVError(rc, "pa_alloc_refcount")
        return rc
