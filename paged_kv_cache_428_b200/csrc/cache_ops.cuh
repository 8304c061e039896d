// cache_ops.cuh -- cache write (reshape_and_cache) and copy-on-write block copy.
//
// Both are pure data movement (plus the E4M3 / INT8 quantisation of the write), bound by
// latency at decode-step sizes.  Every thread moves one 16-byte chunk, so a warp
// touches 512 contiguous bytes of a row or block: fully coalesced on both sides.
#pragma once

#include "common.cuh"

namespace pa {

// ---- reshape_and_cache -----------------------------------------------------------------
// Store the step's new K/V rows: cache[slot/bs][h][slot%bs][:] = row[t][h][:].
// ("现代 AI 的“推理加速之谜”…" section 1: only the new token's K and V are computed each
// step and kept; "vLLM 推理原理…" section "KV Cache 缓存的究竟是什么".)
struct CacheWriteParams {
    const __nv_bfloat16 *key;
    const __nv_bfloat16 *value;
    int64_t key_stride;      // elements between consecutive tokens
    int64_t value_stride;
    uint8_t *k_cache;
    uint8_t *v_cache;
    const int64_t *slot_mapping;
    int num_tokens;
    int h_kv;
    int block_size;
    long long num_slots;     // num_blocks * block_size
    float k_scale;
    float v_scale;
    const float *k_scales;   // per-KV-head scales [h_kv] (device), or null: k_scale for all
    const float *v_scales;
};

__device__ __forceinline__ float head_scale(const float *per_head, float per_tensor, int h)
{
    return per_head ? __ldg(per_head + h) : per_tensor;
}

// bf16 cache: bits copied unchanged.  Thread -> (token, head, K|V, 16-byte chunk).
template <int D>
__global__ void __launch_bounds__(256) reshape_and_cache_bf16_kernel(CacheWriteParams p)
{
    pdl_launch_dependents();                           // a decode launched after this may start
    constexpr int CHUNKS = D * 2 / 16;                 // 16-byte chunks per row
    const long long tid = blockIdx.x * (long long)blockDim.x + threadIdx.x;
    const long long per_token = (long long)p.h_kv * 2 * CHUNKS;
    if (tid >= per_token * p.num_tokens) return;
    const int t = static_cast<int>(tid / per_token);
    int r = static_cast<int>(tid % per_token);
    const int h = r / (2 * CHUNKS);
    r %= 2 * CHUNKS;
    const bool is_v = r >= CHUNKS;
    const int chunk = is_v ? r - CHUNKS : r;

    const long long slot = p.slot_mapping[t];
    if (slot < 0) return;                              // padding token
    if (slot >= p.num_slots) {
        if (h == 0 && r == 0) record_error(PA_DEVERR_BAD_SLOT);
        return;
    }
    const long long blk = slot / p.block_size;
    const int off = static_cast<int>(slot % p.block_size);
    const __nv_bfloat16 *src = (is_v ? p.value + t * p.value_stride : p.key + t * p.key_stride) + (size_t)h * D;
    uint8_t *cache = is_v ? p.v_cache : p.k_cache;
    const size_t dst = (((size_t)blk * p.h_kv + h) * p.block_size + off) * (size_t)D * 2;
    const uint4 v = reinterpret_cast<const uint4 *>(src)[chunk];
    reinterpret_cast<uint4 *>(cache + dst)[chunk] = v;
}

// Quantised caches, 8 elements per thread (reads 16 bytes, writes 8), x / scale an IEEE fp32
// division with the KV head's scale:
//   QT = 1 (E4M3): code = RNE-satfinite(x / scale)
//   QT = 2 (INT8): code = nearest integer of x / scale (ties to even) limited to [-127, 127]
// Thread -> (token, head, K|V, 8-element chunk).
template <int D, int QT>
__global__ void __launch_bounds__(256) reshape_and_cache_quant_kernel(CacheWriteParams p)
{
    pdl_launch_dependents();                           // a decode launched after this may start
    constexpr int CHUNKS = D / 8;
    const long long tid = blockIdx.x * (long long)blockDim.x + threadIdx.x;
    const long long per_token = (long long)p.h_kv * 2 * CHUNKS;
    if (tid >= per_token * p.num_tokens) return;
    const int t = static_cast<int>(tid / per_token);
    int r = static_cast<int>(tid % per_token);
    const int h = r / (2 * CHUNKS);
    r %= 2 * CHUNKS;
    const bool is_v = r >= CHUNKS;
    const int chunk = is_v ? r - CHUNKS : r;

    const long long slot = p.slot_mapping[t];
    if (slot < 0) return;
    if (slot >= p.num_slots) {
        if (h == 0 && r == 0) record_error(PA_DEVERR_BAD_SLOT);
        return;
    }
    const long long blk = slot / p.block_size;
    const int off = static_cast<int>(slot % p.block_size);
    const __nv_bfloat16 *src = (is_v ? p.value + t * p.value_stride : p.key + t * p.key_stride) + (size_t)h * D;
    const float scale = is_v ? head_scale(p.v_scales, p.v_scale, h) : head_scale(p.k_scales, p.k_scale, h);
    const uint4 raw = reinterpret_cast<const uint4 *>(src)[chunk];
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
    uint32_t out[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const float2 a = bf16x2_to_float2(w[2 * i]);
        const float2 b = bf16x2_to_float2(w[2 * i + 1]);
        const float x0 = __fdiv_rn(a.x, scale), x1 = __fdiv_rn(a.y, scale);
        const float x2 = __fdiv_rn(b.x, scale), x3 = __fdiv_rn(b.y, scale);
        if constexpr (QT == 1) {
            const uint16_t lo = float2_to_e4m3x2(x0, x1);
            const uint16_t hi = float2_to_e4m3x2(x2, x3);
            out[i] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
        } else {
            out[i] = (static_cast<uint32_t>(float_to_s8_sym(x0)) & 0xffu) |
                     ((static_cast<uint32_t>(float_to_s8_sym(x1)) & 0xffu) << 8) |
                     ((static_cast<uint32_t>(float_to_s8_sym(x2)) & 0xffu) << 16) |
                     (static_cast<uint32_t>(float_to_s8_sym(x3)) << 24);
        }
    }
    uint8_t *cache = is_v ? p.v_cache : p.k_cache;
    const size_t dst = (((size_t)blk * p.h_kv + h) * p.block_size + off) * (size_t)D;
    reinterpret_cast<uint2 *>(cache + dst)[chunk] = make_uint2(out[0], out[1]);
}

// ---- copy_blocks ---------------------------------------------------------------------------
// cache[dst] = cache[src] for every (src, dst) pair, layer, and K/V; byte for byte.
// ("深度解构…" section 2.3, copy-on-write; intelliparadigm section 3.1, copy then remap.)
constexpr int kMaxLayersPerLaunch = 128;

struct CopyBlocksParams {
    uint8_t *k[kMaxLayersPerLaunch];
    uint8_t *v[kMaxLayersPerLaunch];
    const int64_t *pairs;
    long long block_bytes;
    int num_blocks;
};

// grid (num_pairs, layers, 2): one CTA copies one block of one layer's K or V.
__global__ void __launch_bounds__(256) copy_blocks_kernel(CopyBlocksParams p)
{
    const int pair = blockIdx.x, layer = blockIdx.y, which = blockIdx.z;
    const long long src = p.pairs[2 * pair], dst = p.pairs[2 * pair + 1];
    if (src < 0 || dst < 0 || src >= p.num_blocks || dst >= p.num_blocks) {
        if (threadIdx.x == 0 && layer == 0 && which == 0) record_error(PA_DEVERR_BAD_PAIR);
        return;
    }
    uint8_t *base = which ? p.v[layer] : p.k[layer];
    const uint4 *s = reinterpret_cast<const uint4 *>(base + src * p.block_bytes);
    uint4 *d = reinterpret_cast<uint4 *>(base + dst * p.block_bytes);
    const long long n = p.block_bytes / 16;
    // each thread loads 8 chunks before it stores any, so the copy waits for one memory round
    // trip per 8 chunks (32 KB per CTA at 256 threads) instead of one per chunk
    constexpr int U = 8;
    for (long long i0 = threadIdx.x; i0 < n; i0 += (long long)blockDim.x * U) {
        uint4 v[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const long long i = i0 + (long long)u * blockDim.x;
            if (i < n) v[u] = s[i];
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const long long i = i0 + (long long)u * blockDim.x;
            if (i < n) d[i] = v[u];
        }
    }
}

}  // namespace pa
