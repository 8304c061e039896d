"""CPU oracle for paged KV-cache decode -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The
product library (``paged_kv_cache_428_b200``) never imports it and shares no
code with it; the two meet only through the seeded input generator
(``workloads.py``), which holds no attention, codec or cache arithmetic.

The arithmetic lives in ``oracle.c`` (plain C, fp64, single-threaded); this
module compiles it with gcc on first use (or via :func:`build`) and marshals
numpy arrays into it.  ``alloc_model.py`` holds the reference model of the
block allocator.

Status of the pins (see tests/test_oracle_pins.py): every function here is
pinned against something other than itself (the pages' closed forms and
worked block-table example, torch's bf16 / float8_e4m3fn casts, fp64 SDPA on
gathered contiguous rows, brute-force loops, special cases).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "oracle.c"
_LIB = _HERE / "liboracle.so"

_c_double_p = ctypes.POINTER(ctypes.c_double)


_LIB_OMP = _HERE / "liboracle_omp.so"


def build(src: Path = _SRC, out: Path = _LIB, openmp: bool = False) -> Path:
    """Compile the oracle with gcc (IEEE semantics: no fast-math, no FP contraction).  With
    `openmp`, the same source built with -fopenmp: the decode's independent rows run on all host
    threads (the multi-core CPU baseline); the arithmetic of each row is unchanged."""
    cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
           *(["-fopenmp"] if openmp else []), "-o", str(out), str(src), "-lm"]
    subprocess.run(cmd, check=True)
    return out


def build_all() -> None:
    """Both libraries: the single-threaded oracle and its OpenMP build."""
    build()
    build(out=_LIB_OMP, openmp=True)


def _stale(src: Path, out: Path) -> bool:
    return (not out.exists()) or out.stat().st_mtime < src.stat().st_mtime


_cache: dict[str, "Oracle"] = {}

CACHE_CODES = {"bf16": 0, "e4m3": 1, "int8": 2}


def _cache_code(cache: str | None, fp8: bool) -> int:
    if cache is None:
        cache = "e4m3" if fp8 else "bf16"
    if cache not in CACHE_CODES:
        raise ValueError("unknown cache type %r" % (cache,))
    return CACHE_CODES[cache]


def _head_scales(scale, h_kv: int) -> np.ndarray:
    """fp32 [h_kv]: a scalar is the per-tensor case (the same scale for every KV head)."""
    a = np.asarray(scale, dtype=np.float32).reshape(-1)
    if a.size == 1:
        a = np.full(h_kv, a[0], dtype=np.float32)
    if a.size != h_kv:
        raise ValueError("expected one scale or %d per-head scales, got %d" % (h_kv, a.size))
    return np.ascontiguousarray(a)


class Oracle:
    """ctypes façade over one compiled copy of oracle.c (the tests may load a
    mutated copy to show the pins catch planted mistakes)."""

    def __init__(self, lib_path: Path):
        self.path = Path(lib_path)
        L = ctypes.CDLL(str(self.path))
        self._L = L
        vp, i32, i64, f32, f64, u64 = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64,
                                       ctypes.c_float, ctypes.c_double, ctypes.c_uint64)
        L.or_bf16_decode.restype = f64; L.or_bf16_decode.argtypes = [ctypes.c_uint16]
        L.or_bf16_encode_rne.restype = ctypes.c_uint16; L.or_bf16_encode_rne.argtypes = [f32]
        L.or_e4m3_decode.restype = f64; L.or_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.or_e4m3_encode_satfinite.restype = ctypes.c_uint8; L.or_e4m3_encode_satfinite.argtypes = [f32]
        L.or_div_f32.restype = f32; L.or_div_f32.argtypes = [f32, f32]
        L.or_int8_encode_sat.restype = ctypes.c_int8; L.or_int8_encode_sat.argtypes = [f32]
        L.or_int8_decode.restype = f64; L.or_int8_decode.argtypes = [ctypes.c_int8]
        for name in ("or_bf16_decode_n", "or_bf16_encode_rne_n", "or_e4m3_decode_n",
                     "or_e4m3_encode_satfinite_n", "or_int8_encode_sat_n", "or_int8_decode_n"):
            getattr(L, name).restype = None
            getattr(L, name).argtypes = [vp, vp, i64]
        L.or_div_f32_n.restype = None; L.or_div_f32_n.argtypes = [vp, f32, vp, i64]
        L.or_kv_bytes_per_token.restype = u64; L.or_kv_bytes_per_token.argtypes = [i32] * 4
        L.or_kv_bytes_sequence.restype = u64
        L.or_kv_bytes_sequence.argtypes = [i32, u64, i32, i32, i32]
        L.or_reshape_and_cache.restype = i32
        L.or_reshape_and_cache.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, vp, vp]
        L.or_copy_blocks.restype = i32
        L.or_copy_blocks.argtypes = [vp, vp, i32, vp, i32, u64, i32]
        L.or_paged_decode.restype = i32
        L.or_paged_decode.argtypes = [vp, vp, vp, vp, vp, i32, vp, i32, i32, i32, i32, i32, i32,
                                      f64, i32, vp, vp]
        L.or_paged_prefill_rows.restype = i32
        L.or_paged_prefill_rows.argtypes = [vp, vp, i32, vp, vp, vp, vp, i32, vp, vp, i32, i32, i32, i32, i32, i32,
                                            f64, i32, vp, vp]
        L.or_paged_decode_rows.restype = i32
        L.or_paged_decode_rows.argtypes = [vp, vp, i32, vp, vp, vp, vp, i32, vp, i32, i32, i32, i32,
                                           i32, f64, i32, vp, vp]

    # -- number formats ---------------------------------------------------
    def bf16_decode(self, bits) -> np.ndarray:
        b = np.ascontiguousarray(bits, dtype=np.uint16)
        out = np.empty(b.shape, dtype=np.float64)
        self._L.or_bf16_decode_n(b.ctypes.data, out.ctypes.data, b.size)
        return out

    def bf16_encode_rne(self, x) -> np.ndarray:
        a = np.ascontiguousarray(x, dtype=np.float32)
        out = np.empty(a.shape, dtype=np.uint16)
        self._L.or_bf16_encode_rne_n(a.ctypes.data, out.ctypes.data, a.size)
        return out

    def e4m3_decode(self, codes) -> np.ndarray:
        c = np.ascontiguousarray(codes, dtype=np.uint8)
        out = np.empty(c.shape, dtype=np.float64)
        self._L.or_e4m3_decode_n(c.ctypes.data, out.ctypes.data, c.size)
        return out

    def e4m3_encode_satfinite(self, x) -> np.ndarray:
        a = np.ascontiguousarray(x, dtype=np.float32)
        out = np.empty(a.shape, dtype=np.uint8)
        self._L.or_e4m3_encode_satfinite_n(a.ctypes.data, out.ctypes.data, a.size)
        return out

    def int8_encode_sat(self, x) -> np.ndarray:
        a = np.ascontiguousarray(x, dtype=np.float32)
        out = np.empty(a.shape, dtype=np.int8)
        self._L.or_int8_encode_sat_n(a.ctypes.data, out.ctypes.data, a.size)
        return out

    def int8_decode(self, codes) -> np.ndarray:
        c = np.ascontiguousarray(codes, dtype=np.int8)
        out = np.empty(c.shape, dtype=np.float64)
        self._L.or_int8_decode_n(c.ctypes.data, out.ctypes.data, c.size)
        return out

    def div_f32(self, x, s: float) -> np.ndarray:
        a = np.ascontiguousarray(x, dtype=np.float32)
        out = np.empty(a.shape, dtype=np.float32)
        self._L.or_div_f32_n(a.ctypes.data, ctypes.c_float(s), out.ctypes.data, a.size)
        return out

    # -- closed forms ------------------------------------------------------
    def kv_bytes_per_token(self, layers: int, h_kv: int, head_dim: int, elem_bytes: int) -> int:
        return int(self._L.or_kv_bytes_per_token(layers, h_kv, head_dim, elem_bytes))

    def kv_bytes_sequence(self, layers: int, tokens: int, h_kv: int, head_dim: int,
                          elem_bytes: int) -> int:
        return int(self._L.or_kv_bytes_sequence(layers, tokens, h_kv, head_dim, elem_bytes))

    # -- cache operations (in place on numpy arrays) -----------------------
    def reshape_and_cache(self, key_bits, value_bits, k_cache, v_cache, slot_mapping, *,
                          h_kv: int, d: int, bs: int, num_blocks: int, cache: str | None = None,
                          fp8: bool = False, k_scale=1.0, v_scale=1.0) -> None:
        """``cache`` is "bf16", "e4m3" or "int8" (``fp8=True`` means "e4m3"); ``k_scale`` /
        ``v_scale`` are one float (per tensor) or ``h_kv`` floats (per KV head)."""
        dt = _cache_code(cache, fp8)
        key = np.ascontiguousarray(key_bits, dtype=np.uint16)
        val = np.ascontiguousarray(value_bits, dtype=np.uint16)
        slots = np.ascontiguousarray(slot_mapping, dtype=np.int64)
        want = (np.uint16, np.uint8, np.int8)[dt]
        for c in (k_cache, v_cache):
            if c.dtype != want or not c.flags["C_CONTIGUOUS"]:
                raise TypeError("cache must be a C-contiguous %s array" % np.dtype(want).name)
        ks, vs = _head_scales(k_scale, h_kv), _head_scales(v_scale, h_kv)
        rc = self._L.or_reshape_and_cache(key.ctypes.data, val.ctypes.data, k_cache.ctypes.data,
                                          v_cache.ctypes.data, slots.ctypes.data, slots.size,
                                          h_kv, d, bs, num_blocks, dt, ks.ctypes.data, vs.ctypes.data)
        if rc:
            raise ValueError("oracle reshape_and_cache failed with code %d" % rc)

    def copy_blocks(self, k_caches, v_caches, pairs, *, block_bytes: int, num_blocks: int) -> None:
        n_layers = len(k_caches)
        kp = (ctypes.c_void_p * n_layers)(*[c.ctypes.data for c in k_caches])
        vp_ = (ctypes.c_void_p * n_layers)(*[c.ctypes.data for c in v_caches])
        pr = np.ascontiguousarray(pairs, dtype=np.int64).reshape(-1, 2)
        rc = self._L.or_copy_blocks(ctypes.cast(kp, ctypes.c_void_p), ctypes.cast(vp_, ctypes.c_void_p),
                                    n_layers, pr.ctypes.data, pr.shape[0], block_bytes, num_blocks)
        if rc:
            raise ValueError("oracle copy_blocks: block id outside the pool")

    # -- decode attention --------------------------------------------------
    def paged_decode(self, q_bits, k_cache, v_cache, block_tables, context_lens, *, h_kv: int,
                     bs: int, scale: float, cache: str | None = None, fp8: bool = False, k_scale=1.0,
                     v_scale=1.0) -> np.ndarray:
        dt = _cache_code(cache, fp8)
        q = np.ascontiguousarray(q_bits, dtype=np.uint16)
        B, h_q, d = q.shape
        tab = np.ascontiguousarray(block_tables, dtype=np.int32)
        ctx = np.ascontiguousarray(context_lens, dtype=np.int32)
        num_blocks = k_cache.shape[0]
        ks, vs = _head_scales(k_scale, h_kv), _head_scales(v_scale, h_kv)
        out = np.empty((B, h_q, d), dtype=np.float64)
        rc = self._L.or_paged_decode(out.ctypes.data, q.ctypes.data, k_cache.ctypes.data,
                                     v_cache.ctypes.data, tab.ctypes.data, tab.shape[1], ctx.ctypes.data,
                                     B, h_q, h_kv, d, bs, num_blocks, scale, dt, ks.ctypes.data, vs.ctypes.data)
        if rc:
            raise ValueError("oracle paged_decode failed with code %d" % rc)
        return out

    def paged_decode_rows(self, rows, q_bits, k_cache, v_cache, block_tables, context_lens, *,
                          h_kv: int, bs: int, scale: float, cache: str | None = None, fp8: bool = False,
                          k_scale=1.0, v_scale=1.0) -> np.ndarray:
        """Outputs for the listed (sequence, query head) rows only: [len(rows), d]."""
        dt = _cache_code(cache, fp8)
        q = np.ascontiguousarray(q_bits, dtype=np.uint16)
        _, h_q, d = q.shape
        pr = np.ascontiguousarray(rows, dtype=np.int32).reshape(-1, 2)
        tab = np.ascontiguousarray(block_tables, dtype=np.int32)
        ctx = np.ascontiguousarray(context_lens, dtype=np.int32)
        ks, vs = _head_scales(k_scale, h_kv), _head_scales(v_scale, h_kv)
        out = np.empty((pr.shape[0], d), dtype=np.float64)
        rc = self._L.or_paged_decode_rows(out.ctypes.data, pr.ctypes.data, pr.shape[0], q.ctypes.data,
                                          k_cache.ctypes.data, v_cache.ctypes.data, tab.ctypes.data,
                                          tab.shape[1], ctx.ctypes.data, h_q, h_kv, d, bs,
                                          k_cache.shape[0], scale, dt, ks.ctypes.data, vs.ctypes.data)
        if rc:
            raise ValueError("oracle paged_decode_rows failed with code %d" % rc)
        return out

    # -- prefill (chunked) attention -----------------------------------------
    def paged_prefill(self, q_bits, k_cache, v_cache, block_tables, query_start, context_lens, *, h_kv: int,
                      bs: int, scale: float, rows=None, cache: str | None = None, k_scale=1.0,
                      v_scale=1.0) -> np.ndarray:
        """Causal attention of every chunk row over its sequence's paged cache.  q [T, h_q, d];
        query_start [B+1]; context_lens [B] (including the chunk).  rows: (query row, head)
        pairs -> [len(rows), d]; None -> all rows, [T, h_q, d]."""
        dt = _cache_code(cache, False)
        q = np.ascontiguousarray(q_bits, dtype=np.uint16)
        T, h_q, d = q.shape
        qs = np.ascontiguousarray(query_start, dtype=np.int32)
        ctx = np.ascontiguousarray(context_lens, dtype=np.int32)
        tab = np.ascontiguousarray(block_tables, dtype=np.int32)
        full = rows is None
        if full:
            rows = [(t, h) for t in range(T) for h in range(h_q)]
        pr = np.ascontiguousarray(rows, dtype=np.int32).reshape(-1, 2)
        ks, vs = _head_scales(k_scale, h_kv), _head_scales(v_scale, h_kv)
        out = np.empty((pr.shape[0], d), dtype=np.float64)
        rc = self._L.or_paged_prefill_rows(out.ctypes.data, pr.ctypes.data, pr.shape[0], q.ctypes.data,
                                           k_cache.ctypes.data, v_cache.ctypes.data, tab.ctypes.data, tab.shape[1],
                                           qs.ctypes.data, ctx.ctypes.data, ctx.shape[0], h_q, h_kv, d, bs,
                                           k_cache.shape[0], scale, dt, ks.ctypes.data, vs.ctypes.data)
        if rc:
            raise ValueError("oracle paged_prefill failed with code %d" % rc)
        return out.reshape(T, h_q, d) if full else out


def load(lib_path: os.PathLike | None = None, openmp: bool = False) -> Oracle:
    """The oracle compiled from oracle.c (built on demand), or a given library.  `openmp`
    selects the OpenMP build of the same source (multi-core baseline timing only)."""
    if lib_path is None:
        if openmp:
            if _stale(_SRC, _LIB_OMP):
                build(out=_LIB_OMP, openmp=True)
            lib_path = _LIB_OMP
        else:
            if _stale(_SRC, _LIB):
                build()
            lib_path = _LIB
    key = str(lib_path)
    if key not in _cache:
        _cache[key] = Oracle(Path(lib_path))
    return _cache[key]
