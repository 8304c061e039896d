// pa_lib.cu -- C-ABI entry points of the device calls (argument checks, dispatch, launch).
// All device code of the library is in this one translation unit.
#include <algorithm>
#include <climits>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <type_traits>
#include <utility>

#include "common.cuh"
#include "cache_ops.cuh"
#include "decode.cuh"
#include "decode_mma.cuh"
#include "decode_q8.cuh"
#include "prefill.cuh"
#include "prefill_tc.cuh"
#include "decode_balanced.cuh"
#include "decode_allheads.cuh"

using namespace pa;

namespace {

constexpr float kLog2e = 1.4426950408889634f;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// pa_prefill_ws: the claim counter and the finished-CTA counter, padded
constexpr size_t kPrefillWorkspaceBytes = 256;

int launch_status()
{
    return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

// Launch `kernel`; with `pdl`, as a programmatic dependent of the grid before it on the stream
// (it may start while that grid runs; the kernel waits for it where it reads its results).
template <typename... KArgs, typename... Args>
int launch_ex(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, bool pdl,
              Args &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = pdl ? attr : nullptr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...) == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

bool supported_head_dim(int d) { return d == 64 || d == 128; }
bool supported_block_size(int bs) { return bs == 16 || bs == 32 || bs == 64; }
bool supported_group(int g) { return g == 1 || g == 2 || g == 4 || g == 8; }

bool valid_cache_dtype(int t) { return t == PA_CACHE_BF16 || t == PA_CACHE_E4M3 || t == PA_CACHE_INT8; }

// Scales of a quantised cache: per tensor (k_scales == v_scales == null; both floats finite
// and > 0) or per KV head (both device arrays given; their values are the caller's to check).
bool valid_scales(int cache_dtype, float k_scale, float v_scale, const float *k_scales, const float *v_scales)
{
    if (!valid_cache_dtype(cache_dtype)) return false;
    if (cache_dtype == PA_CACHE_BF16) return k_scales == nullptr && v_scales == nullptr;
    if (k_scales != nullptr || v_scales != nullptr) return k_scales != nullptr && v_scales != nullptr;
    return std::isfinite(k_scale) && std::isfinite(v_scale) && k_scale > 0.f && v_scale > 0.f;
}

int grid_partitions(int max_context_len, int partition_size)
{
    if (partition_size <= 0) return 1;
    const long long n = ((long long)max_context_len + partition_size - 1) / partition_size;
    return n < 1 ? 1 : static_cast<int>(n);
}

size_t round256(size_t b) { return (b + 255) / 256 * 256; }

// Workspace of the split-context decode: [group counters][m, l partials][o partials].
// The counters (one int per sequence x query head, an upper bound of the KV heads) must be
// zero before the first launch; every launch leaves them zero again.
struct WsLayout {
    size_t ml = 0, o = 0, total = 0, counters_bytes = 0;
};

WsLayout ws_layout(int num_seqs, int h_q, int head_dim, int p_max)
{
    WsLayout L;
    L.counters_bytes = round256((size_t)num_seqs * h_q * sizeof(int));
    L.ml = L.counters_bytes;
    L.o = L.ml + round256((size_t)num_seqs * h_q * p_max * 2 * sizeof(float));
    L.total = L.o + (size_t)num_seqs * h_q * p_max * head_dim * sizeof(float);
    return L;
}

// ---------------------------------------------------------------------------------------
template <int D, int BS, int G, bool FP8>
int launch_partition(const DecodeParams &prm, int num_seqs, cudaStream_t st)
{
    using C = DecodeConfig<D, BS, G, FP8>;
    static std::atomic<unsigned long long> smem_set{0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return PA_ERR_CUDA;
    const unsigned long long bit = 1ull << (dev & 63);
    if (!(smem_set.load(std::memory_order_acquire) & bit)) {
        if (cudaFuncSetAttribute(paged_decode_partition_kernel<D, BS, G, FP8>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess)
            return PA_ERR_CUDA;
        smem_set.fetch_or(bit, std::memory_order_release);
    }
    const dim3 grid(prm.p_max, prm.h_kv, num_seqs);
    return launch_ex(paged_decode_partition_kernel<D, BS, G, FP8>, grid, dim3(C::THREADS), C::SMEM, st,
                     prm.pdl_wait_last != 0, prm);
}

// ---- tensor maps of the bf16 caches (2-D: rows of head_dim elements, 128B swizzle) -----
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled()
{
    static EncodeTiledFn fn = []() -> EncodeTiledFn {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<EncodeTiledFn>(ptr);
    }();
    return fn;
}

// The cache viewed as [num_blocks * h_kv * block_size rows][head_dim] elements.  bf16: a box is
// 64 elements (128 bytes) by block_size rows, swizzled in 128-byte atoms (two boxes per row at
// head_dim 128).  One-byte codes: a box is a whole row (head_dim bytes) by block_size rows,
// 128-byte swizzle for 128-byte rows, 64-byte swizzle for 64-byte rows.
// box_rows: rows of one box (block_size for one KV head's tile; h_kv * block_size for a whole block).
int make_cache_map(CUtensorMap *map, const void *cache, int num_blocks, int h_kv, int block_size, int head_dim,
                   int elem_bytes, int box_rows)
{
    EncodeTiledFn enc = encode_tiled();
    if (!enc) return PA_ERR_CUDA;
    const cuuint64_t dims[2] = {(cuuint64_t)head_dim, (cuuint64_t)num_blocks * h_kv * block_size};
    const cuuint64_t strides[1] = {(cuuint64_t)head_dim * elem_bytes};
    const cuuint32_t box[2] = {elem_bytes == 2 ? 64u : (cuuint32_t)head_dim, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUtensorMapDataType dt = elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
    const CUtensorMapSwizzle sw = (elem_bytes == 1 && head_dim == 64) ? CU_TENSOR_MAP_SWIZZLE_64B
                                                                       : CU_TENSOR_MAP_SWIZZLE_128B;
    const CUresult r = enc(map, dt, 2, const_cast<void *>(cache), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? PA_OK : PA_ERR_CUDA;
}

// The prefill queries q [tokens][h_q][head_dim] as a 3-D map (head_dim, h_q, tokens) whose box is
// one query tile: 64 elements (128 bytes, 128-byte swizzle) x g heads x 128 / g tokens, landing as
// the swizzled Q tile the S products read.  `tokens` only bounds the coordinates: the kernel loads
// only tiles that lie inside their sequence's chunk.  q must be 16-byte aligned with 16-byte
// strides, else the encoding fails and the kernel copies every tile itself.
int make_q_map(CUtensorMap *map, const void *q, int h_q, int head_dim, int g, long long tokens)
{
    EncodeTiledFn enc = encode_tiled();
    if (!enc || tokens <= 0 || 128 % g != 0) return PA_ERR_CUDA;
    const cuuint64_t dims[3] = {(cuuint64_t)head_dim, (cuuint64_t)h_q, (cuuint64_t)tokens};
    const cuuint64_t strides[2] = {(cuuint64_t)head_dim * 2, (cuuint64_t)h_q * head_dim * 2};
    const cuuint32_t box[3] = {64u, (cuuint32_t)g, (cuuint32_t)(128 / g)};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(q), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? PA_OK : PA_ERR_CUDA;
}

// Encoded maps of recently used caches (per host thread): a decode step reuses the same
// cache tensors call after call, and encoding costs host time on every launch otherwise.
struct CachedMap {
    const void *base = nullptr;
    int num_blocks = 0, h_kv = 0, block_size = 0, head_dim = 0, elem_bytes = 0, box_rows = 0;
    CUtensorMap map;
};

int cached_cache_map(CUtensorMap *map, const void *cache, int num_blocks, int h_kv, int block_size, int head_dim,
                     int elem_bytes = 2, int box_rows = 0)
{
    constexpr int kSlots = 8;
    static thread_local CachedMap slots[kSlots];
    static thread_local int next = 0;
    if (box_rows <= 0) box_rows = block_size;
    for (const CachedMap &c : slots) {
        if (c.base == cache && c.num_blocks == num_blocks && c.h_kv == h_kv && c.block_size == block_size &&
            c.head_dim == head_dim && c.elem_bytes == elem_bytes && c.box_rows == box_rows) {
            *map = c.map;
            return PA_OK;
        }
    }
    CachedMap &c = slots[next];
    next = (next + 1) % kSlots;
    const int rc = make_cache_map(&c.map, cache, num_blocks, h_kv, block_size, head_dim, elem_bytes, box_rows);
    if (rc != PA_OK) {
        c.base = nullptr;
        return rc;
    }
    c.base = cache;
    c.num_blocks = num_blocks;
    c.h_kv = h_kv;
    c.block_size = block_size;
    c.head_dim = head_dim;
    c.elem_bytes = elem_bytes;
    c.box_rows = box_rows;
    *map = c.map;
    return PA_OK;
}

template <int D, int BS, int G>
int launch_partition_mma(const DecodeParams &prm, int num_seqs, cudaStream_t st)
{
    using C = MmaDecodeConfig<D, BS, G>;
    static std::atomic<unsigned long long> smem_set{0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return PA_ERR_CUDA;
    const unsigned long long bit = 1ull << (dev & 63);
    if (!(smem_set.load(std::memory_order_acquire) & bit)) {
        if (cudaFuncSetAttribute(paged_decode_partition_mma_kernel<D, BS, G>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess)
            return PA_ERR_CUDA;
        smem_set.fetch_or(bit, std::memory_order_release);
    }
    CUtensorMap mk, mv;
    int rc = cached_cache_map(&mk, prm.k_cache, prm.num_blocks, prm.h_kv, BS, D);
    if (rc == PA_OK) rc = cached_cache_map(&mv, prm.v_cache, prm.num_blocks, prm.h_kv, BS, D);
    if (rc != PA_OK) return rc;
    const dim3 grid(prm.p_max, prm.h_kv, num_seqs);
    return launch_ex(paged_decode_partition_mma_kernel<D, BS, G>, grid, dim3(C::THREADS), C::SMEM, st,
                     prm.pdl_wait_last != 0, prm, mk, mv);
}

// Consumer warps and ring bytes of the one-byte-code kernel: 2 warps and a 32 KB ring (6 CTAs
// per SM) measured best at every block size (against 1, 3 and 4 warps, 16 to 64 KB rings).
template <int BS>
struct Q8Tuning {
    static constexpr int NW = 2;
    static constexpr int RING = 32768;
};

template <int D, int BS, int G, int QT>
int launch_partition_q8(const DecodeParams &prm, int num_seqs, cudaStream_t st)
{
    constexpr int NW = Q8Tuning<BS>::NW, RING = Q8Tuning<BS>::RING;
    using C = MmaQ8Config<D, BS, G, NW, RING>;
    static std::atomic<unsigned long long> smem_set{0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return PA_ERR_CUDA;
    const unsigned long long bit = 1ull << (dev & 63);
    if (!(smem_set.load(std::memory_order_acquire) & bit)) {
        if (cudaFuncSetAttribute(paged_decode_partition_q8_kernel<D, BS, G, QT, NW, RING>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess)
            return PA_ERR_CUDA;
        smem_set.fetch_or(bit, std::memory_order_release);
    }
    CUtensorMap mk, mv;
    int rc = cached_cache_map(&mk, prm.k_cache, prm.num_blocks, prm.h_kv, BS, D, 1);
    if (rc == PA_OK) rc = cached_cache_map(&mv, prm.v_cache, prm.num_blocks, prm.h_kv, BS, D, 1);
    if (rc != PA_OK) return rc;
    const dim3 grid(prm.p_max, prm.h_kv, num_seqs);
    return launch_ex(paged_decode_partition_q8_kernel<D, BS, G, QT, NW, RING>, grid, dim3(C::THREADS), C::SMEM, st,
                     prm.pdl_wait_last != 0, prm, mk, mv);
}

bool env_flag(const char *name)
{
    const char *e = std::getenv(name);
    return e != nullptr && std::strcmp(e, "1") == 0;
}

// Both cache types run on the tensor cores; PA_DECODE_BF16_CUDA_CORES=1 and
// PA_DECODE_E4M3_CUDA_CORES=1 select the CUDA-core kernel instead (kept for A/B
// measurements; each read once per process).
bool bf16_on_cuda_cores()
{
    static const bool v = env_flag("PA_DECODE_BF16_CUDA_CORES");
    return v;
}

bool e4m3_on_cuda_cores()
{
    static const bool v = env_flag("PA_DECODE_E4M3_CUDA_CORES");
    return v;
}

// Cache element types of the kernels: 0 = bf16, 1 = E4M3, 2 = INT8 (the pa_cache_dtype values).
template <class F>
int switch_group(int g, F &&f)
{
    switch (g) {
    case 1: return f(std::integral_constant<int, 1>{});
    case 2: return f(std::integral_constant<int, 2>{});
    case 4: return f(std::integral_constant<int, 4>{});
    case 8: return f(std::integral_constant<int, 8>{});
    default: return PA_ERR_UNSUPPORTED;
    }
}

template <int D, int BS, int QT>
int dispatch_group(int g, const DecodeParams &prm, int n, cudaStream_t st)
{
    return switch_group(g, [&](auto gc) {
        constexpr int G = decltype(gc)::value;
        if constexpr (QT == PA_CACHE_BF16) {
            if (!bf16_on_cuda_cores()) return launch_partition_mma<D, BS, G>(prm, n, st);
            return launch_partition<D, BS, G, false>(prm, n, st);
        } else if constexpr (QT == PA_CACHE_E4M3) {
            if (!e4m3_on_cuda_cores()) return launch_partition_q8<D, BS, G, QT>(prm, n, st);
            return launch_partition<D, BS, G, true>(prm, n, st);
        } else {
            return launch_partition_q8<D, BS, G, QT>(prm, n, st);
        }
    });
}

template <int D, int QT>
int dispatch_block(int bs, int g, const DecodeParams &prm, int n, cudaStream_t st)
{
    switch (bs) {
    case 16: return dispatch_group<D, 16, QT>(g, prm, n, st);
    case 32: return dispatch_group<D, 32, QT>(g, prm, n, st);
    case 64: return dispatch_group<D, 64, QT>(g, prm, n, st);
    default: return PA_ERR_UNSUPPORTED;
    }
}

template <int D>
int dispatch_type(int qt, int bs, int g, const DecodeParams &prm, int n, cudaStream_t st)
{
    switch (qt) {
    case PA_CACHE_BF16: return dispatch_block<D, PA_CACHE_BF16>(bs, g, prm, n, st);
    case PA_CACHE_E4M3: return dispatch_block<D, PA_CACHE_E4M3>(bs, g, prm, n, st);
    case PA_CACHE_INT8: return dispatch_block<D, PA_CACHE_INT8>(bs, g, prm, n, st);
    default: return PA_ERR_INVALID_ARG;
    }
}

int dispatch_partition(int d, int bs, int g, int qt, const DecodeParams &prm, int n, cudaStream_t st)
{
    if (d == 64) return dispatch_type<64>(qt, bs, g, prm, n, st);
    if (d == 128) return dispatch_type<128>(qt, bs, g, prm, n, st);
    return PA_ERR_UNSUPPORTED;
}

// ---- balanced schedule (PA_PARTITION_AUTO) ------------------------------------------------
// Workspace: [group counters][partial (m, l): kBalancedMaxCtas x 2 x Gmax x 2][partial o].
// Gmax = min(8, h_q) bounds the query heads per KV head (h_kv is not an argument of
// pa_decode_workspace_size).  The same workspace also serves the 512-token fallback.
// Partitions of the AUTO fallback: at least 512 tokens, and never more than
// kFusedMergeMaxPartitions per sequence (a multiple of 64 tokens, so of every block size),
// so that every group is merged inside the partition kernel.
int auto_fallback_partition(int max_context_len)
{
    const long long need = ((long long)max_context_len + kFusedMergeMaxPartitions - 1) / kFusedMergeMaxPartitions;
    const long long p = (need + 63) / 64 * 64;
    return (int)(p > 512 ? p : 512);
}

struct BalLayout {
    size_t ml = 0, o = 0, total = 0, counters_bytes = 0;
};

BalLayout bal_layout(int num_seqs, int h_q, int head_dim)
{
    const size_t gmax = (size_t)(h_q < kBalancedMaxGroup ? h_q : kBalancedMaxGroup);
    BalLayout L;
    L.counters_bytes = round256((size_t)num_seqs * h_q * sizeof(int));
    L.ml = L.counters_bytes;
    L.o = L.ml + round256((size_t)kBalancedMaxCtas * 2 * gmax * 2 * sizeof(float));
    L.total = L.o + (size_t)kBalancedMaxCtas * 2 * gmax * head_dim * sizeof(float);
    return L;
}

bool balanced_applies(int num_seqs, int h_q, int h_kv, int cache_dtype)
{
    return cache_dtype == PA_CACHE_BF16 && !bf16_on_cuda_cores() && num_seqs <= kBalancedMaxSeqs &&
           h_q / h_kv <= kBalancedMaxGroup;
}

struct SmCount {
    int dev = -1, count = 0;
};

int sm_count()
{
    static thread_local SmCount cache;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    if (cache.dev != dev) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
        cache.dev = dev;
        cache.count = n;
    }
    return cache.count;
}

template <int D, int BS, int G>
int launch_balanced(const DecodeParams &prm, int num_seqs, const BalLayout &lay, void *workspace, cudaStream_t st)
{
    using BC = BalancedConfig<D, BS, G>;
    static std::atomic<unsigned long long> smem_set{0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return PA_ERR_CUDA;
    const unsigned long long bit = 1ull << (dev & 63);
    if (!(smem_set.load(std::memory_order_acquire) & bit)) {
        if (cudaFuncSetAttribute(paged_decode_balanced_kernel<D, BS, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 BC::smem_bytes(kBalancedMaxSeqs)) != cudaSuccess)
            return PA_ERR_CUDA;
        smem_set.fetch_or(bit, std::memory_order_release);
    }
    const int smem = BC::smem_bytes(num_seqs);
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, paged_decode_balanced_kernel<D, BS, G>, BC::THREADS,
                                                      smem) != cudaSuccess || per_sm < 1)
        return PA_ERR_CUDA;
    const int sms = sm_count();
    if (sms < 1) return PA_ERR_CUDA;
    int ctas = per_sm * sms;
    if (ctas > kBalancedMaxCtas) ctas = kBalancedMaxCtas;
    CUtensorMap mk, mv;
    int rc = cached_cache_map(&mk, prm.k_cache, prm.num_blocks, prm.h_kv, BS, D);
    if (rc == PA_OK) rc = cached_cache_map(&mv, prm.v_cache, prm.num_blocks, prm.h_kv, BS, D);
    if (rc != PA_OK) return rc;
    BalancedParams bp{};
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    bp.out = prm.out;
    bp.q = prm.q;
    bp.block_tables = prm.block_tables;
    bp.context_lens = prm.context_lens;
    bp.counters = reinterpret_cast<int *>(ws);
    bp.part_ml = reinterpret_cast<float *>(ws + lay.ml);
    bp.part_o = reinterpret_cast<float *>(ws + lay.o);
    bp.max_blocks_per_seq = prm.max_blocks_per_seq;
    bp.num_seqs = num_seqs;
    bp.h_q = prm.h_q;
    bp.h_kv = prm.h_kv;
    bp.num_blocks = prm.num_blocks;
    bp.num_ctas = ctas;
    bp.qk_scale = prm.qk_scale;
    bp.pdl_wait = prm.pdl_wait_last;
    return launch_ex(paged_decode_balanced_kernel<D, BS, G>, dim3(ctas), dim3(BC::THREADS), (size_t)smem, st,
                     prm.pdl_wait_last != 0, bp, mk, mv);
}

template <int D, int BS>
int dispatch_balanced_group(int g, const DecodeParams &prm, int n, const BalLayout &lay, void *ws, cudaStream_t st)
{
    switch (g) {
    case 1: return launch_balanced<D, BS, 1>(prm, n, lay, ws, st);
    case 2: return launch_balanced<D, BS, 2>(prm, n, lay, ws, st);
    case 4: return launch_balanced<D, BS, 4>(prm, n, lay, ws, st);
    case 8: return launch_balanced<D, BS, 8>(prm, n, lay, ws, st);
    default: return PA_ERR_UNSUPPORTED;
    }
}

int dispatch_balanced(int d, int bs, int g, const DecodeParams &prm, int n, const BalLayout &lay, void *ws,
                      cudaStream_t st)
{
    if (d == 64) {
        if (bs == 16) return dispatch_balanced_group<64, 16>(g, prm, n, lay, ws, st);
        if (bs == 32) return dispatch_balanced_group<64, 32>(g, prm, n, lay, ws, st);
        if (bs == 64) return dispatch_balanced_group<64, 64>(g, prm, n, lay, ws, st);
    } else if (d == 128) {
        if (bs == 16) return dispatch_balanced_group<128, 16>(g, prm, n, lay, ws, st);
        if (bs == 32) return dispatch_balanced_group<128, 32>(g, prm, n, lay, ws, st);
        if (bs == 64) return dispatch_balanced_group<128, 64>(g, prm, n, lay, ws, st);
    }
    return PA_ERR_UNSUPPORTED;
}

// ---- whole-block schedule (PA_PARTITION_AUTO, 8 KV heads) ------------------------------------
// Workspace: [chunk pool: 16 ints][block prefix sums: num_seqs + 1 ints] (counters_bytes, zero
// before the first launch; every launch leaves the pool zero) [partial (m, l): kAllHeadsSlots x
// h_q x 2 floats][partial o: kAllHeadsSlots x h_q x head_dim floats].
struct AllHeadsLayout {
    size_t prefix = 0, ml = 0, o = 0, total = 0, counters_bytes = 0;
};

AllHeadsLayout allheads_layout(int num_seqs, int h_q, int head_dim)
{
    AllHeadsLayout L;
    L.prefix = 16 * sizeof(int);
    L.counters_bytes = round256(L.prefix + ((size_t)num_seqs + 1) * sizeof(int));
    L.ml = L.counters_bytes;
    L.o = L.ml + round256((size_t)kAllHeadsSlots * h_q * 2 * sizeof(float));
    L.total = L.o + (size_t)kAllHeadsSlots * h_q * head_dim * sizeof(float);
    return L;
}

// PA_DECODE_AUTO_WHOLE_BLOCK=1 runs PA_PARTITION_AUTO at 8 KV heads on the whole-block kernel
// instead of the per-KV-head balanced kernel (A/B runs: measured slower on the 64-sequence
// workload, 114.6 against 108.7 us, the streaming rate being the same and its merge a second launch).
bool auto_whole_block()
{
    static const bool v = env_flag("PA_DECODE_AUTO_WHOLE_BLOCK");
    return v;
}

bool allheads_applies(int num_seqs, int h_kv, int head_dim, int block_size, int cache_dtype)
{
    return cache_dtype == PA_CACHE_BF16 && !bf16_on_cuda_cores() && auto_whole_block() && h_kv == kAllHeadsHkv &&
           num_seqs <= kAllHeadsMaxSeqs && (block_size == 16 || block_size == 32) &&
           (head_dim == 64 || head_dim == 128);
}

template <int D, int BS, int G>
int launch_allheads(const DecodeParams &prm, int num_seqs, void *workspace, cudaStream_t st)
{
    constexpr int HKV = kAllHeadsHkv;
    using AC = AllHeadsConfig<D, BS, G, HKV>;
    static std::atomic<unsigned long long> smem_set{0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return PA_ERR_CUDA;
    const unsigned long long bit = 1ull << (dev & 63);
    if (!(smem_set.load(std::memory_order_acquire) & bit)) {
        if (cudaFuncSetAttribute(paged_decode_allheads_kernel<D, BS, G, HKV>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, AC::smem_bytes(kAllHeadsMaxSeqs)) !=
            cudaSuccess)
            return PA_ERR_CUDA;
        smem_set.fetch_or(bit, std::memory_order_release);
    }
    const int sms = sm_count();
    if (sms < 1) return PA_ERR_CUDA;
    const int ctas = sms < kAllHeadsMaxCtas ? sms : kAllHeadsMaxCtas;
    CUtensorMap mk, mv;
    int rc = cached_cache_map(&mk, prm.k_cache, prm.num_blocks, HKV, BS, D, 2, HKV * BS);
    if (rc == PA_OK) rc = cached_cache_map(&mv, prm.v_cache, prm.num_blocks, HKV, BS, D, 2, HKV * BS);
    if (rc != PA_OK) return rc;
    const AllHeadsLayout lay = allheads_layout(num_seqs, prm.h_q, D);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    AllHeadsParams ap{};
    ap.out = prm.out;
    ap.q = prm.q;
    ap.block_tables = prm.block_tables;
    ap.context_lens = prm.context_lens;
    ap.pool = reinterpret_cast<int *>(ws);
    ap.prefix_out = reinterpret_cast<int *>(ws + lay.prefix);
    ap.part_ml = reinterpret_cast<float *>(ws + lay.ml);
    ap.part_o = reinterpret_cast<float *>(ws + lay.o);
    ap.max_blocks_per_seq = prm.max_blocks_per_seq;
    ap.num_seqs = num_seqs;
    ap.num_blocks = prm.num_blocks;
    ap.num_ctas = ctas;
    ap.qk_scale = prm.qk_scale;
    ap.pdl_wait_last = prm.pdl_wait_last;
    rc = launch_ex(paged_decode_allheads_kernel<D, BS, G, HKV>, dim3(ctas), dim3(AC::THREADS),
                   (size_t)AC::smem_bytes(num_seqs), st, prm.pdl_wait_last != 0, ap, mk, mv);
    if (rc != PA_OK) return rc;
    // the split sequences' pieces, combined by a second launch that may start while the first
    // one finishes (it waits for it before reading anything)
    AllHeadsMergeParams mp{};
    mp.out = prm.out;
    mp.prefix = ap.prefix_out;
    mp.part_ml = ap.part_ml;
    mp.part_o = ap.part_o;
    mp.num_seqs = num_seqs;
    mp.h_q = prm.h_q;
    mp.num_ctas = ctas;
    return launch_ex(paged_decode_allheads_merge_kernel<D>, dim3(prm.h_q, num_seqs), dim3(kAllHeadsMergeWarps * 32), 0,
                     st, true, mp);
}

template <int D, int BS>
int dispatch_allheads_group(int g, const DecodeParams &prm, int n, void *ws, cudaStream_t st)
{
    return switch_group(g, [&](auto gc) {
        constexpr int G = decltype(gc)::value;
        return launch_allheads<D, BS, G>(prm, n, ws, st);
    });
}

int dispatch_allheads(int d, int bs, int g, const DecodeParams &prm, int n, void *ws, cudaStream_t st)
{
    if (d == 64) {
        if (bs == 16) return dispatch_allheads_group<64, 16>(g, prm, n, ws, st);
        if (bs == 32) return dispatch_allheads_group<64, 32>(g, prm, n, ws, st);
    } else if (d == 128) {
        if (bs == 16) return dispatch_allheads_group<128, 16>(g, prm, n, ws, st);
        if (bs == 32) return dispatch_allheads_group<128, 32>(g, prm, n, ws, st);
    }
    return PA_ERR_UNSUPPORTED;
}

// Shared argument checks of the decode calls.  Returns PA_OK and fills `prm`.
int prepare_decode(DecodeParams &prm, void *out, const void *q, const void *k_cache, const void *v_cache,
                   const int32_t *block_tables, int max_blocks_per_seq, const int32_t *context_lens,
                   int num_seqs, int max_context_len, int h_q, int h_kv, int head_dim, int block_size,
                   int num_blocks, float scale, int cache_dtype, float k_scale, float v_scale,
                   const float *k_scales, const float *v_scales, int partition_size, void *workspace,
                   size_t workspace_bytes)
{
    if (num_seqs < 0 || max_context_len < 0 || h_q <= 0 || h_kv <= 0 || num_blocks <= 0 ||
        max_blocks_per_seq <= 0 || partition_size < PA_PARTITION_AUTO)
        return PA_ERR_INVALID_ARG;
    if (h_q % h_kv != 0) return PA_ERR_INVALID_ARG;
    if (!std::isfinite(scale)) return PA_ERR_INVALID_ARG;
    if (!valid_scales(cache_dtype, k_scale, v_scale, k_scales, v_scales)) return PA_ERR_INVALID_ARG;
    if (!supported_head_dim(head_dim) || !supported_block_size(block_size) || !supported_group(h_q / h_kv))
        return PA_ERR_UNSUPPORTED;
    if (partition_size > 0 && partition_size % block_size != 0) return PA_ERR_INVALID_ARG;
    if (partition_size == PA_PARTITION_AUTO) {
        // the balanced kernel (set up by the caller) or, where it does not apply, 512-token partitions
        if (pa_decode_workspace_size(num_seqs, h_q, head_dim, max_context_len, PA_PARTITION_AUTO) > 0 &&
            (workspace == nullptr || workspace_bytes < pa_decode_workspace_size(num_seqs, h_q, head_dim,
                                                                                max_context_len, PA_PARTITION_AUTO) ||
             !aligned16(workspace)))
            return PA_ERR_WORKSPACE;
        partition_size = auto_fallback_partition(max_context_len);
    }
    if (h_kv > 65535 || num_seqs > 65535) return PA_ERR_UNSUPPORTED;
    if (num_seqs > 0) {
        if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens) return PA_ERR_INVALID_ARG;
        if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache))
            return PA_ERR_INVALID_ARG;
    }
    const int p_max = grid_partitions(max_context_len, partition_size);
    const size_t need = pa_decode_workspace_size(num_seqs, h_q, head_dim, max_context_len, partition_size);
    if (need > 0 && (workspace == nullptr || workspace_bytes < need || !aligned16(workspace)))
        return PA_ERR_WORKSPACE;

    prm.out = static_cast<__nv_bfloat16 *>(out);
    prm.q = static_cast<const __nv_bfloat16 *>(q);
    prm.k_cache = static_cast<const uint8_t *>(k_cache);
    prm.v_cache = static_cast<const uint8_t *>(v_cache);
    prm.block_tables = block_tables;
    prm.context_lens = context_lens;
    const WsLayout lay = ws_layout(num_seqs, h_q, head_dim, p_max);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    prm.counters = need > 0 ? reinterpret_cast<int *>(ws) : nullptr;
    prm.ws_ml = need > 0 ? reinterpret_cast<float *>(ws + lay.ml) : nullptr;
    prm.ws_o = need > 0 ? reinterpret_cast<float *>(ws + lay.o) : nullptr;
    prm.max_blocks_per_seq = max_blocks_per_seq;
    prm.h_q = h_q;
    prm.h_kv = h_kv;
    prm.num_blocks = num_blocks;
    prm.partition_size = need > 0 ? partition_size : 0;
    prm.p_max = need > 0 ? p_max : 1;
    const bool per_tensor = cache_dtype != PA_CACHE_BF16 && k_scales == nullptr;
    prm.qk_scale = scale * kLog2e * (per_tensor ? k_scale : 1.f);
    prm.v_scale = per_tensor ? v_scale : 1.f;
    prm.k_scales = cache_dtype != PA_CACHE_BF16 ? k_scales : nullptr;
    prm.v_scales = cache_dtype != PA_CACHE_BF16 ? v_scales : nullptr;
    return PA_OK;
}

// Decode first pass for both scale forms (per tensor: k_scales == v_scales == null).
int decode_partitions_impl(void *out, const void *q, const void *k_cache, const void *v_cache,
                           const int32_t *block_tables, int max_blocks_per_seq, const int32_t *context_lens,
                           int num_seqs, int max_context_len, int h_q, int h_kv, int head_dim, int block_size,
                           int num_blocks, float scale, int cache_dtype, float k_scale, float v_scale,
                           const float *k_scales, const float *v_scales, int partition_size, void *workspace,
                           size_t workspace_bytes, void *stream, bool after_append = false)
{
    DecodeParams prm{};
    int rc = prepare_decode(prm, out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                            num_seqs, max_context_len, h_q, h_kv, head_dim, block_size, num_blocks, scale,
                            cache_dtype, k_scale, v_scale, k_scales, v_scales, partition_size, workspace,
                            workspace_bytes);
    if (rc != PA_OK || num_seqs == 0) return rc;
    prm.pdl_wait_last = after_append ? 1 : 0;
    if (partition_size == PA_PARTITION_AUTO && allheads_applies(num_seqs, h_kv, head_dim, block_size, cache_dtype))
        return dispatch_allheads(head_dim, block_size, h_q / h_kv, prm, num_seqs, workspace,
                                 static_cast<cudaStream_t>(stream));
    if (partition_size == PA_PARTITION_AUTO && balanced_applies(num_seqs, h_q, h_kv, cache_dtype))
        return dispatch_balanced(head_dim, block_size, h_q / h_kv, prm, num_seqs, bal_layout(num_seqs, h_q, head_dim),
                                 workspace, static_cast<cudaStream_t>(stream));
    return dispatch_partition(head_dim, block_size, h_q / h_kv, cache_dtype, prm, num_seqs,
                              static_cast<cudaStream_t>(stream));
}

template <int D>
void launch_reshape(int cache_dtype, unsigned blocks, const CacheWriteParams &p, cudaStream_t st)
{
    if (cache_dtype == PA_CACHE_E4M3) reshape_and_cache_quant_kernel<D, 1><<<blocks, 256, 0, st>>>(p);
    else if (cache_dtype == PA_CACHE_INT8) reshape_and_cache_quant_kernel<D, 2><<<blocks, 256, 0, st>>>(p);
    else reshape_and_cache_bf16_kernel<D><<<blocks, 256, 0, st>>>(p);
}

int reshape_impl(const void *key, const void *value, int64_t key_stride, int64_t value_stride, void *k_cache,
                 void *v_cache, const int64_t *slot_mapping, int num_tokens, int h_kv, int head_dim, int block_size,
                 int num_blocks, int cache_dtype, float k_scale, float v_scale, const float *k_scales,
                 const float *v_scales, void *stream)
{
    if (num_tokens < 0 || h_kv <= 0 || num_blocks <= 0) return PA_ERR_INVALID_ARG;
    if (!valid_scales(cache_dtype, k_scale, v_scale, k_scales, v_scales)) return PA_ERR_INVALID_ARG;
    if (!supported_head_dim(head_dim) || !supported_block_size(block_size)) return PA_ERR_UNSUPPORTED;
    const int64_t row = (int64_t)h_kv * head_dim;
    if (key_stride == 0) key_stride = row;
    if (value_stride == 0) value_stride = row;
    if (key_stride < row || value_stride < row || key_stride % 8 != 0 || value_stride % 8 != 0)
        return PA_ERR_INVALID_ARG;
    if (num_tokens == 0) return PA_OK;
    if (!key || !value || !k_cache || !v_cache || !slot_mapping) return PA_ERR_INVALID_ARG;
    if (!aligned16(key) || !aligned16(value) || !aligned16(k_cache) || !aligned16(v_cache))
        return PA_ERR_INVALID_ARG;

    CacheWriteParams p{};
    p.key = static_cast<const __nv_bfloat16 *>(key);
    p.value = static_cast<const __nv_bfloat16 *>(value);
    p.key_stride = key_stride;
    p.value_stride = value_stride;
    p.k_cache = static_cast<uint8_t *>(k_cache);
    p.v_cache = static_cast<uint8_t *>(v_cache);
    p.slot_mapping = slot_mapping;
    p.num_tokens = num_tokens;
    p.h_kv = h_kv;
    p.block_size = block_size;
    p.num_slots = (long long)num_blocks * block_size;
    p.k_scale = k_scale;
    p.v_scale = v_scale;
    p.k_scales = k_scales;
    p.v_scales = v_scales;
    const long long threads = (long long)num_tokens * h_kv * 2 * (head_dim / 8);
    const long long blocks = (threads + 255) / 256;
    if (blocks > 0x7fffffffLL) return PA_ERR_UNSUPPORTED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (head_dim == 64) launch_reshape<64>(cache_dtype, (unsigned)blocks, p, st);
    else launch_reshape<128>(cache_dtype, (unsigned)blocks, p, st);
    return launch_status();
}

// ---- chunked prefill ------------------------------------------------------------------------
template <int D, int BS, int G>
int launch_prefill(const PrefillParams &pp, int num_seqs, int max_query_len, cudaStream_t st)
{
    using C = PrefillConfig<D, BS, G>;
    static std::atomic<unsigned long long> smem_set{0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return PA_ERR_CUDA;
    const unsigned long long bit = 1ull << (dev & 63);
    if (!(smem_set.load(std::memory_order_acquire) & bit)) {
        if (cudaFuncSetAttribute(paged_prefill_kernel<D, BS, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 C::SMEM) != cudaSuccess)
            return PA_ERR_CUDA;
        smem_set.fetch_or(bit, std::memory_order_release);
    }
    CUtensorMap mk, mv;
    int rc = cached_cache_map(&mk, pp.k_cache, pp.num_blocks, pp.h_kv, BS, D);
    if (rc == PA_OK) rc = cached_cache_map(&mv, pp.v_cache, pp.num_blocks, pp.h_kv, BS, D);
    if (rc != PA_OK) return rc;
    const dim3 grid(prefill_tiles<C::TQ>(max_query_len), pp.h_kv, num_seqs);
    paged_prefill_kernel<D, BS, G><<<grid, C::THREADS, C::SMEM, st>>>(pp, mk, mv);
    return launch_status();
}

template <int D, int BS, int G>
int launch_prefill_tc(const PrefillParams &pp, int num_seqs, int max_query_len, int *counters, cudaStream_t st)
{
    using C = PrefillTcConfig<D, BS, G>;
    static std::atomic<unsigned long long> smem_set{0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return PA_ERR_CUDA;
    const unsigned long long bit = 1ull << (dev & 63);
    if (!(smem_set.load(std::memory_order_acquire) & bit)) {
        if (cudaFuncSetAttribute(paged_prefill_tc_kernel<D, BS, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 C::SMEM) != cudaSuccess)
            return PA_ERR_CUDA;
        smem_set.fetch_or(bit, std::memory_order_release);
    }
    CUtensorMap mk, mv;
    int rc = cached_cache_map(&mk, pp.k_cache, pp.num_blocks, pp.h_kv, BS, D);
    if (rc == PA_OK) rc = cached_cache_map(&mv, pp.v_cache, pp.num_blocks, pp.h_kv, BS, D);
    if (rc != PA_OK) return rc;
    const int pairs = (prefill_tiles<C::TQ>(max_query_len) + C::NQ - 1) / C::NQ;
    const long long items = (long long)pairs * pp.h_kv * num_seqs;
    if (items > INT_MAX) return PA_ERR_UNSUPPORTED;
    PrefillSched sc{};
    sc.counters = counters;
    sc.num_seqs = num_seqs;
    sc.pairs_max = pairs;
    sc.total_items = (int)items;
    CUtensorMap mq;
    sc.q_tma = make_q_map(&mq, pp.q, pp.h_q, D, G, (long long)num_seqs * max_query_len) == PA_OK;
    if (!sc.q_tma) std::memset(&mq, 0, sizeof(mq));
    dim3 grid(pairs, pp.h_kv, num_seqs);                      // one CTA per item
    if (counters) {
        const int sms = sm_count();                              // one CTA per SM, claiming items
        if (sms <= 0) return PA_ERR_CUDA;
        grid = dim3((unsigned)std::min<long long>(sms, items));
    }
    paged_prefill_tc_kernel<D, BS, G><<<grid, C::THREADS, C::SMEM, st>>>(pp, sc, mk, mv, mq);
    return launch_status();
}

// The tcgen05 kernel by default; PA_PREFILL_MMA_SYNC=1 selects the mma.sync kernel (A/B runs).
bool prefill_on_mma_sync()
{
    static const bool v = env_flag("PA_PREFILL_MMA_SYNC");
    return v;
}

template <int D, int BS>
int dispatch_prefill_group(int g, const PrefillParams &pp, int n, int mql, int *counters, cudaStream_t st)
{
    return switch_group(g, [&](auto gc) {
        constexpr int G = decltype(gc)::value;
        if (prefill_on_mma_sync()) return launch_prefill<D, BS, G>(pp, n, mql, st);
        return launch_prefill_tc<D, BS, G>(pp, n, mql, counters, st);
    });
}

int dispatch_prefill(int d, int bs, int g, const PrefillParams &pp, int n, int mql, int *counters, cudaStream_t st)
{
    if (d == 64) {
        if (bs == 16) return dispatch_prefill_group<64, 16>(g, pp, n, mql, counters, st);
        if (bs == 32) return dispatch_prefill_group<64, 32>(g, pp, n, mql, counters, st);
        if (bs == 64) return dispatch_prefill_group<64, 64>(g, pp, n, mql, counters, st);
    } else if (d == 128) {
        if (bs == 16) return dispatch_prefill_group<128, 16>(g, pp, n, mql, counters, st);
        if (bs == 32) return dispatch_prefill_group<128, 32>(g, pp, n, mql, counters, st);
        if (bs == 64) return dispatch_prefill_group<128, 64>(g, pp, n, mql, counters, st);
    }
    return PA_ERR_UNSUPPORTED;
}

}  // namespace

// Scratch of pa_decode_static_ws: one array per device in global memory (no allocation).
// Host code must not use this symbol as an address: its device address comes from
// cudaGetSymbolAddress, looked up once per device with that device current.
static __device__ __align__(256) unsigned char g_pa_static_ws[PA_STATIC_WS_BYTES];

namespace {

constexpr int kMaxDevices = 64;

// The array's device address belongs to the CUDA context that was current when it was looked
// up (the device's primary context).  After cudaDeviceReset the module is loaded again, in a
// new context, possibly at another address; so the cache entry carries the context's id and
// is looked up again when the current context's id differs.
struct StaticWsEntry {
    std::atomic<void *> addr{nullptr};
    std::atomic<unsigned long long> ctx_id{0};
};
StaticWsEntry g_static_ws[kMaxDevices];

using CtxGetCurrentFn = CUresult (*)(CUcontext *);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long *);

template <class Fn>
Fn driver_fn(const char *name)
{
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint(name, &ptr, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess)
        return nullptr;
    return reinterpret_cast<Fn>(ptr);
}

// Id of the CUDA context current on this thread (0 when none is current or it is unknown).
unsigned long long current_ctx_id()
{
    static const CtxGetCurrentFn get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
    static const CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
    if (!get_current || !get_id) return 0;
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

// Device address of g_pa_static_ws on the current device, looked up on the first call on a
// device (and again after the device's context was replaced).
int static_ws_address(void **addr)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return PA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return PA_ERR_UNSUPPORTED;
    StaticWsEntry &e = g_static_ws[dev];
    void *p = e.addr.load(std::memory_order_acquire);
    const unsigned long long id = current_ctx_id();
    if (p == nullptr || id == 0 || id != e.ctx_id.load(std::memory_order_acquire)) {
        p = nullptr;
        if (cudaGetSymbolAddress(&p, g_pa_static_ws) != cudaSuccess || p == nullptr) return PA_ERR_CUDA;
        e.ctx_id.store(current_ctx_id(), std::memory_order_release);   // the lookup made a context current
        e.addr.store(p, std::memory_order_release);
    }
    *addr = p;
    return PA_OK;
}

}  // namespace

extern "C" {

int pa_decode_static_ws(void *out, const void *q, const void *k_cache, const void *v_cache,
                        const int32_t *block_tables, int max_blocks_per_seq, const int32_t *context_lens,
                        int num_seqs, int max_context_len, int h_q, int h_kv, int head_dim, int block_size,
                        int num_blocks, float scale, int cache_dtype, float k_scale, float v_scale,
                        int partition_size, void *stream)
{
    if (num_seqs < 0 || h_q <= 0 || head_dim <= 0 || max_context_len < 0 || partition_size < PA_PARTITION_AUTO)
        return PA_ERR_INVALID_ARG;
    const size_t need = pa_decode_workspace_size(num_seqs, h_q, head_dim, max_context_len, partition_size);
    if (need > PA_STATIC_WS_BYTES) return PA_ERR_WORKSPACE;           // beyond the static array
    void *ws = nullptr;
    if (need > 0) {
        const int rc = static_ws_address(&ws);
        if (rc != PA_OK) return rc;
    }
    const size_t ws_bytes = need > 0 ? (size_t)PA_STATIC_WS_BYTES : 0;
    // every argument check of pa_decode first, so that a rejected call queues nothing
    DecodeParams chk{};
    int rc = prepare_decode(chk, out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                            num_seqs, max_context_len, h_q, h_kv, head_dim, block_size, num_blocks, scale,
                            cache_dtype, k_scale, v_scale, nullptr, nullptr, partition_size, ws, ws_bytes);
    if (rc != PA_OK || num_seqs == 0) return rc;
    if (need > 0) {
        // the counters at the front of the scratch must start at zero (a launch that stopped
        // early could have left counts behind): the largest counter area of the workspace
        // layouts (fixed partitions, the PA_PARTITION_AUTO schedules), which every layout's
        // size covers
        const size_t counters = std::max(round256((size_t)num_seqs * h_q * sizeof(int)),
                                         allheads_layout(num_seqs, h_q, head_dim).counters_bytes);
        if (cudaMemsetAsync(ws, 0, counters, static_cast<cudaStream_t>(stream)) != cudaSuccess) return PA_ERR_CUDA;
    }
    return pa_decode(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens, num_seqs,
                     max_context_len, h_q, h_kv, head_dim, block_size, num_blocks, scale, cache_dtype, k_scale,
                     v_scale, partition_size, ws, ws_bytes, stream);
}

size_t pa_decode_workspace_size(int num_seqs, int h_q, int head_dim, int max_context_len, int partition_size)
{
    if (num_seqs <= 0 || h_q <= 0 || head_dim <= 0) return 0;
    if (partition_size == PA_PARTITION_AUTO) {
        // the largest of the schedules AUTO can pick (h_kv is not an argument here)
        size_t need = bal_layout(num_seqs, h_q, head_dim).total;
        const size_t all = allheads_layout(num_seqs, h_q, head_dim).total;
        const size_t grid = pa_decode_workspace_size(num_seqs, h_q, head_dim, max_context_len,
                                                     auto_fallback_partition(max_context_len));
        if (all > need) need = all;
        return grid > need ? grid : need;
    }
    if (partition_size <= 0) return 0;
    const int p_max = grid_partitions(max_context_len, partition_size);
    if (p_max <= 1) return 0;
    return ws_layout(num_seqs, h_q, head_dim, p_max).total;
}

int pa_decode_partitions(void *out, const void *q, const void *k_cache, const void *v_cache,
                         const int32_t *block_tables, int max_blocks_per_seq, const int32_t *context_lens,
                         int num_seqs, int max_context_len, int h_q, int h_kv, int head_dim, int block_size,
                         int num_blocks, float scale, int cache_dtype, float k_scale, float v_scale,
                         int partition_size, void *workspace, size_t workspace_bytes, void *stream)
{
    return decode_partitions_impl(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                                  num_seqs, max_context_len, h_q, h_kv, head_dim, block_size, num_blocks, scale,
                                  cache_dtype, k_scale, v_scale, nullptr, nullptr, partition_size, workspace,
                                  workspace_bytes, stream);
}

int pa_decode_merge(void *out, const int32_t *context_lens, int num_seqs, int max_context_len, int h_q,
                    int head_dim, int partition_size, const void *workspace, size_t workspace_bytes,
                    void *stream)
{
    if (num_seqs < 0 || h_q <= 0 || max_context_len < 0 || partition_size < PA_PARTITION_AUTO)
        return PA_ERR_INVALID_ARG;
    if (!supported_head_dim(head_dim)) return PA_ERR_UNSUPPORTED;
    if (partition_size == PA_PARTITION_AUTO) return PA_OK;       // merged inside the first pass
    if (num_seqs > 65535 || h_q > 65535) return PA_ERR_UNSUPPORTED;
    const size_t need = pa_decode_workspace_size(num_seqs, h_q, head_dim, max_context_len, partition_size);
    if (need == 0 || num_seqs == 0) return PA_OK;                 // single partition: nothing to merge
    if (!out || !context_lens) return PA_ERR_INVALID_ARG;
    if (workspace == nullptr || workspace_bytes < need || !aligned16(workspace)) return PA_ERR_WORKSPACE;
    const int p_max = grid_partitions(max_context_len, partition_size);
    if (p_max <= kFusedMergeMaxPartitions) return PA_OK;         // every group merged by pass 1
    const WsLayout lay = ws_layout(num_seqs, h_q, head_dim, p_max);
    MergeParams mp{};
    mp.out = static_cast<__nv_bfloat16 *>(out);
    mp.context_lens = context_lens;
    mp.ws_ml = reinterpret_cast<const float *>(static_cast<const uint8_t *>(workspace) + lay.ml);
    mp.ws_o = reinterpret_cast<const float *>(static_cast<const uint8_t *>(workspace) + lay.o);
    mp.h_q = h_q;
    mp.partition_size = partition_size;
    mp.p_max = p_max;
    const dim3 grid(h_q, num_seqs);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (head_dim == 64)
        paged_decode_merge_kernel<64><<<grid, 512, 0, st>>>(mp);
    else
        paged_decode_merge_kernel<128><<<grid, 512, 0, st>>>(mp);
    return launch_status();
}

int pa_decode(void *out, const void *q, const void *k_cache, const void *v_cache, const int32_t *block_tables,
              int max_blocks_per_seq, const int32_t *context_lens, int num_seqs, int max_context_len, int h_q,
              int h_kv, int head_dim, int block_size, int num_blocks, float scale, int cache_dtype,
              float k_scale, float v_scale, int partition_size, void *workspace, size_t workspace_bytes,
              void *stream)
{
    int rc = pa_decode_partitions(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                                  num_seqs, max_context_len, h_q, h_kv, head_dim, block_size, num_blocks, scale,
                                  cache_dtype, k_scale, v_scale, partition_size, workspace, workspace_bytes,
                                  stream);
    if (rc != PA_OK) return rc;
    return pa_decode_merge(out, context_lens, num_seqs, max_context_len, h_q, head_dim, partition_size,
                           workspace, workspace_bytes, stream);
}

int pa_decode_head_scales(void *out, const void *q, const void *k_cache, const void *v_cache,
                          const int32_t *block_tables, int max_blocks_per_seq, const int32_t *context_lens,
                          int num_seqs, int max_context_len, int h_q, int h_kv, int head_dim, int block_size,
                          int num_blocks, float scale, int cache_dtype, const float *k_scales,
                          const float *v_scales, int partition_size, void *workspace, size_t workspace_bytes,
                          void *stream)
{
    if (cache_dtype == PA_CACHE_BF16 || k_scales == nullptr || v_scales == nullptr) return PA_ERR_INVALID_ARG;
    int rc = decode_partitions_impl(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                                    num_seqs, max_context_len, h_q, h_kv, head_dim, block_size, num_blocks, scale,
                                    cache_dtype, 1.f, 1.f, k_scales, v_scales, partition_size, workspace,
                                    workspace_bytes, stream);
    if (rc != PA_OK) return rc;
    return pa_decode_merge(out, context_lens, num_seqs, max_context_len, h_q, head_dim, partition_size,
                           workspace, workspace_bytes, stream);
}

int pa_decode_step(const void *key, const void *value, int64_t key_stride, int64_t value_stride,
                   const int64_t *slot_mapping, void *out, const void *q, void *k_cache, void *v_cache,
                   const int32_t *block_tables, int max_blocks_per_seq, const int32_t *context_lens, int num_seqs,
                   int max_context_len, int h_q, int h_kv, int head_dim, int block_size, int num_blocks, float scale,
                   int cache_dtype, float k_scale, float v_scale, int partition_size, void *workspace,
                   size_t workspace_bytes, void *stream)
{
    if (num_seqs < 0) return PA_ERR_INVALID_ARG;
    if (num_seqs == 0) return PA_OK;
    // the decode's argument checks first, so that nothing is launched on a bad call
    DecodeParams chk{};
    int rc = prepare_decode(chk, out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens, num_seqs,
                            max_context_len, h_q, h_kv, head_dim, block_size, num_blocks, scale, cache_dtype,
                            k_scale, v_scale, nullptr, nullptr, partition_size, workspace, workspace_bytes);
    if (rc != PA_OK) return rc;
    rc = reshape_impl(key, value, key_stride, value_stride, k_cache, v_cache, slot_mapping, num_seqs, h_kv, head_dim,
                      block_size, num_blocks, cache_dtype, k_scale, v_scale, nullptr, nullptr, stream);
    if (rc != PA_OK) return rc;
    rc = decode_partitions_impl(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens, num_seqs,
                                max_context_len, h_q, h_kv, head_dim, block_size, num_blocks, scale, cache_dtype,
                                k_scale, v_scale, nullptr, nullptr, partition_size, workspace, workspace_bytes, stream,
                                true);
    if (rc != PA_OK) return rc;
    return pa_decode_merge(out, context_lens, num_seqs, max_context_len, h_q, head_dim, partition_size, workspace,
                           workspace_bytes, stream);
}

int pa_reshape_and_cache(const void *key, const void *value, int64_t key_stride, int64_t value_stride,
                         void *k_cache, void *v_cache, const int64_t *slot_mapping, int num_tokens, int h_kv,
                         int head_dim, int block_size, int num_blocks, int cache_dtype, float k_scale,
                         float v_scale, void *stream)
{
    return reshape_impl(key, value, key_stride, value_stride, k_cache, v_cache, slot_mapping, num_tokens, h_kv,
                        head_dim, block_size, num_blocks, cache_dtype, k_scale, v_scale, nullptr, nullptr, stream);
}

int pa_reshape_and_cache_head_scales(const void *key, const void *value, int64_t key_stride, int64_t value_stride,
                                     void *k_cache, void *v_cache, const int64_t *slot_mapping, int num_tokens,
                                     int h_kv, int head_dim, int block_size, int num_blocks, int cache_dtype,
                                     const float *k_scales, const float *v_scales, void *stream)
{
    if (cache_dtype == PA_CACHE_BF16 || k_scales == nullptr || v_scales == nullptr) return PA_ERR_INVALID_ARG;
    return reshape_impl(key, value, key_stride, value_stride, k_cache, v_cache, slot_mapping, num_tokens, h_kv,
                        head_dim, block_size, num_blocks, cache_dtype, 1.f, 1.f, k_scales, v_scales, stream);
}

namespace {
int prefill_impl(void *out, const void *q, const void *k_cache, const void *v_cache, const int32_t *block_tables,
                 int max_blocks_per_seq, const int32_t *query_start, const int32_t *context_lens, int num_seqs,
                 int max_query_len, int h_q, int h_kv, int head_dim, int block_size, int num_blocks, float scale,
                 int cache_dtype, int *counters, void *stream)
{
    if (num_seqs < 0 || max_query_len < 0 || h_q <= 0 || h_kv <= 0 || num_blocks <= 0 || max_blocks_per_seq <= 0)
        return PA_ERR_INVALID_ARG;
    // scale >= 0: the kernel takes the row max of the raw scores and scales it afterwards
    if (h_q % h_kv != 0 || !std::isfinite(scale) || scale < 0.f || !valid_cache_dtype(cache_dtype))
        return PA_ERR_INVALID_ARG;
    if (cache_dtype != PA_CACHE_BF16) return PA_ERR_UNSUPPORTED;
    if (!supported_head_dim(head_dim) || !supported_block_size(block_size) || !supported_group(h_q / h_kv))
        return PA_ERR_UNSUPPORTED;
    if (h_kv > 65535 || num_seqs > 65535) return PA_ERR_UNSUPPORTED;
    if (num_seqs == 0 || max_query_len == 0) return PA_OK;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !query_start || !context_lens)
        return PA_ERR_INVALID_ARG;
    if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache)) return PA_ERR_INVALID_ARG;
    PrefillParams pp{};
    pp.out = static_cast<__nv_bfloat16 *>(out);
    pp.q = static_cast<const __nv_bfloat16 *>(q);
    pp.k_cache = static_cast<const uint8_t *>(k_cache);
    pp.v_cache = static_cast<const uint8_t *>(v_cache);
    pp.block_tables = block_tables;
    pp.query_start = query_start;
    pp.context_lens = context_lens;
    pp.max_blocks_per_seq = max_blocks_per_seq;
    pp.h_q = h_q;
    pp.h_kv = h_kv;
    pp.num_blocks = num_blocks;
    pp.qk_scale = scale * kLog2e;
    return dispatch_prefill(head_dim, block_size, h_q / h_kv, pp, num_seqs, max_query_len, counters,
                            static_cast<cudaStream_t>(stream));
}
}  // namespace

int pa_prefill(void *out, const void *q, const void *k_cache, const void *v_cache, const int32_t *block_tables,
               int max_blocks_per_seq, const int32_t *query_start, const int32_t *context_lens, int num_seqs,
               int max_query_len, int h_q, int h_kv, int head_dim, int block_size, int num_blocks, float scale,
               int cache_dtype, void *stream)
{
    return prefill_impl(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, query_start, context_lens,
                        num_seqs, max_query_len, h_q, h_kv, head_dim, block_size, num_blocks, scale, cache_dtype,
                        nullptr, stream);
}

size_t pa_prefill_workspace_size(void) { return kPrefillWorkspaceBytes; }

int pa_prefill_ws(void *out, const void *q, const void *k_cache, const void *v_cache, const int32_t *block_tables,
                  int max_blocks_per_seq, const int32_t *query_start, const int32_t *context_lens, int num_seqs,
                  int max_query_len, int h_q, int h_kv, int head_dim, int block_size, int num_blocks, float scale,
                  int cache_dtype, void *workspace, size_t workspace_bytes, void *stream)
{
    if (workspace == nullptr || workspace_bytes < kPrefillWorkspaceBytes || !aligned16(workspace))
        return PA_ERR_WORKSPACE;
    return prefill_impl(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, query_start, context_lens,
                        num_seqs, max_query_len, h_q, h_kv, head_dim, block_size, num_blocks, scale, cache_dtype,
                        static_cast<int *>(workspace), stream);
}


int pa_copy_blocks(void *const *k_caches, void *const *v_caches, int num_layers, const int64_t *block_pairs,
                   int num_pairs, size_t block_bytes, int num_blocks, void *stream)
{
    if (num_layers < 0 || num_pairs < 0 || num_blocks <= 0) return PA_ERR_INVALID_ARG;
    if (block_bytes == 0 || block_bytes % 16 != 0) return PA_ERR_INVALID_ARG;
    if (num_layers == 0 || num_pairs == 0) return PA_OK;
    if (!k_caches || !v_caches || !block_pairs) return PA_ERR_INVALID_ARG;
    for (int l = 0; l < num_layers; ++l)
        if (!k_caches[l] || !v_caches[l] || !aligned16(k_caches[l]) || !aligned16(v_caches[l]))
            return PA_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    for (int l0 = 0; l0 < num_layers; l0 += kMaxLayersPerLaunch) {
        const int nl = num_layers - l0 < kMaxLayersPerLaunch ? num_layers - l0 : kMaxLayersPerLaunch;
        CopyBlocksParams p{};
        for (int l = 0; l < nl; ++l) {
            p.k[l] = static_cast<uint8_t *>(k_caches[l0 + l]);
            p.v[l] = static_cast<uint8_t *>(v_caches[l0 + l]);
        }
        p.pairs = block_pairs;
        p.block_bytes = static_cast<long long>(block_bytes);
        p.num_blocks = num_blocks;
        copy_blocks_kernel<<<dim3(num_pairs, nl, 2), 256, 0, st>>>(p);
        const int rc = launch_status();
        if (rc != PA_OK) return rc;
    }
    return PA_OK;
}

int pa_device_errors(unsigned int *flags, int clear)
{
    if (!flags) return PA_ERR_INVALID_ARG;
    if (cudaDeviceSynchronize() != cudaSuccess) return PA_ERR_CUDA;
    unsigned int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_errors, sizeof(v)) != cudaSuccess) return PA_ERR_CUDA;
    *flags = v;
    if (clear) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbol(g_device_errors, &zero, sizeof(zero)) != cudaSuccess) return PA_ERR_CUDA;
    }
    return PA_OK;
}

}  // extern "C"
