// decode_q8.cuh -- paged decode partition pass over one-byte caches (E4M3, INT8) on the
// tensor cores, converting in registers.
//
// Same method, grid, pipeline and CTA merge as paged_decode_partition_mma_kernel
// (decode_mma.cuh): one CTA per (context partition, KV head, sequence), a producer warp
// streaming each physical block's K and V code tiles through an mbarrier ring, consumer warps
// folding whole blocks into their own online-softmax state with mma.sync m16n8k16 (fp16 in,
// fp32 accumulate).  Both code sets are exact in fp16.  INT8 K codes enter the scores as
// c + 1152 (one byte permute each, no subtraction); 1152 * sum(q) is taken off every score.
//
// The code tiles arrive by 2-D TMA exactly as stored (one byte per element, rows of D bytes,
// 128-byte swizzle for D = 128, 64-byte swizzle for D = 64) and are read with ldmatrix treating
// each pair of codes as one 16-bit element; the conversion to fp16 happens in registers, so
// shared memory carries each byte once in and once out, as for bf16 tiles.
//
//   S^T = K . Q^T   ldmatrix (no transpose) gives lane T four consecutive codes (dims 4(T%4) ..
//                   +3 of a 16-dim chunk) of token T/4.  The dot product does not depend on the
//                   order of its k terms, so the k-step's columns are taken in the order
//                   k 2t, 2t+1 <- dims 4t, 4t+1 and k 2t+8, 2t+9 <- dims 4t+2, 4t+3 (t = T%4);
//                   Q^T's B fragments are loaded in the same order.
//   O^T += V^T P^T  ldmatrix.trans gives lane T, for tokens 2(T%4) and 2(T%4)+1, the two codes
//                   of dims 2(T/4) and 2(T/4)+1 of a chunk.  One byte permute splits them into
//                   the fp16 pairs (dim 2(T/4); both tokens) and (dim 2(T/4)+1; both tokens),
//                   i.e. rows T/4 and T/4 + 8 of an A fragment whose 16 rows are the chunk's
//                   dims in the order 0, 2, .., 14, 1, 3, .., 15.  The accumulator rows follow
//                   that order; the epilogue writes them back to their dims.
// Tokens past the context: their scores are masked to -inf by select, and their V values are
// zeroed in registers (an E4M3 NaN code times a zero probability would poison the sum).
#pragma once

#include "decode_mma.cuh"

namespace pa {

template <int D, int BS, int G, int NW_ = 2, int RING_ = 32768>
struct MmaQ8Config {
    static constexpr int NW = NW_;                        // consumer warps
    static constexpr int THREADS = (NW + 1) * 32;         // + producer warp
    static constexpr int TILE = BS * D;                   // K (or V) code tile of one block: one TMA box
    static constexpr int STAGE_BYTES = 2 * TILE;
    // a multiple of NW (see MmaDecodeConfig::STAGES)
    static constexpr int STAGES = cmax(NW, cmin(32, RING_ / STAGE_BYTES) / NW * NW);
    static constexpr int KS = D / 16;                     // k-steps of q.K (one 16-byte chunk each)
    static constexpr int MT = D / 16;                     // m-tiles of O^T (one chunk of 16 dims each)
    static constexpr int NSUB = BS / 16;
    static constexpr int RING = STAGES * STAGE_BYTES;
    static constexpr int COMBINE_BYTES = NW * G * (D + 2) * 4;
    static constexpr int MERGE_BYTES = (2 * G * kFusedMergeMaxPartitions + 1) * 4;
    static constexpr int REGION0 = cmax(RING, COMBINE_BYTES + MERGE_BYTES);
    static constexpr int OFF_BARS = (REGION0 + 127) / 128 * 128;
    static constexpr int OFF_FLAGS = OFF_BARS + 2 * STAGES * 8;
    static constexpr int SMEM_USED = OFF_FLAGS + (STAGES + 4) * 4;
    static constexpr int SMEM = SMEM_USED + 1024;         // slack to align the ring to 1024 bytes
    static_assert(D == 64 || D == 128, "head dim");
    static_assert(BS % 16 == 0, "block size");
    static_assert(G <= 8, "group");
    static_assert(TILE % 1024 == 0, "tiles must keep the swizzle atoms aligned");
    static_assert(KS % 2 == 0 && MT % 2 == 0, "x4 loads cover two chunks");
    static_assert(STAGES % NW == 0, "stage ring must be a multiple of the consumer warps");
};

// Byte offset of 16-byte chunk `chunk` of token row `row` in a swizzled code tile: 128-byte
// rows with the 128-byte swizzle (chunk ^ row % 8), or 64-byte rows with the 64-byte swizzle
// (chunk ^ (row / 2) % 4).  Either way the 8 rows of one ldmatrix matrix hit 8 bank groups.
template <int D>
__device__ __forceinline__ uint32_t swz_q8(int row, int chunk)
{
    if constexpr (D == 128) return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
    else return static_cast<uint32_t>(row * 64 + ((chunk ^ ((row >> 1) & 3)) << 4));
}

// Four K codes (byte 0 first) -> fp16 pairs (codes 0, 1) and (codes 2, 3).  E4M3: the values.
// INT8: the values plus 1152 (the biased code c + 128 in the mantissa of 1024, exact), so the
// subtraction is left out here; q . (k + 1152) - 1152 * sum(q) is taken from the scores instead
// (q8_k_bias), one subtraction per score rather than two per four codes.
template <int QT>
__device__ __forceinline__ void q8_quad_to_f16(uint32_t w, uint32_t &lo, uint32_t &hi)
{
    if constexpr (QT == 1) {
        lo = e4m3x2_to_f16x2(w & 0xffffu);
        hi = e4m3x2_to_f16x2(w >> 16);
    } else {
        const uint32_t u = w ^ 0x80808080u;
        asm("prmt.b32 %0, %1, %2, 0x4140;" : "=r"(lo) : "r"(u), "r"(0x64646464u));
        asm("prmt.b32 %0, %1, %2, 0x4342;" : "=r"(hi) : "r"(u), "r"(0x64646464u));
    }
}

// For INT8 K codes: 1152 * sum over d of the (fp16) q of each of this lane's two heads 2t, 2t+1
// (t = lane % 4) -- what the scores of biased codes carry on top of q . k; 0 for E4M3.
template <class C, int QT>
__device__ __forceinline__ void q8_k_bias(const uint32_t (&qb)[C::KS][2], int lane, float (&bias)[2])
{
    bias[0] = bias[1] = 0.f;
    if constexpr (QT == 2) {
        float sum = 0.f;                              // this lane's dims of head lane / 4
#pragma unroll
        for (int ks = 0; ks < C::KS; ++ks) {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const __half2 h = *reinterpret_cast<const __half2 *>(&qb[ks][j]);
                const float2 f = __half22float2(h);
                sum += f.x + f.y;
            }
        }
        sum += __shfl_xor_sync(0xffffffffu, sum, 1);
        sum += __shfl_xor_sync(0xffffffffu, sum, 2);
        const int tq = lane & 3;
        bias[0] = 1152.f * __shfl_sync(0xffffffffu, sum, 4 * (2 * tq));
        bias[1] = 1152.f * __shfl_sync(0xffffffffu, sum, 4 * (2 * tq + 1));
    }
}

// Four codes (byte 0 first) -> fp16 pairs (codes 0, 2) and (codes 1, 3).
template <int QT>
__device__ __forceinline__ void q8_cross_to_f16(uint32_t w, uint32_t &even, uint32_t &odd)
{
    if constexpr (QT == 1) {
        uint32_t t;
        asm("prmt.b32 %0, %1, 0, 0x3120;" : "=r"(t) : "r"(w));
        even = e4m3x2_to_f16x2(t & 0xffffu);
        odd = e4m3x2_to_f16x2(t >> 16);
    } else {
        s8x4_to_f16x2x2_cross(w, even, odd);
    }
}

// Q^T fragments in fp16, k-steps in the permuted order above: qb[ks][0] = dims 16ks + 4t, +1
// and qb[ks][1] = dims 16ks + 4t + 2, +3 of query head T/4 of the group (zero for heads >= G).
// The whole group's q is scaled by 2^-e, e >= 0 the smallest exponent that brings max|q| to at
// most 2^14, so the conversion cannot overflow; returns 2^e, to be folded into the logit scale.
template <class C, int G, int D>
__device__ __forceinline__ float q8_load_q(uint32_t (&qb)[C::KS][2], const __nv_bfloat16 *qg, int lane)
{
    const int gq = lane >> 2, tq = lane & 3;
    const __nv_bfloat16 *qrow = qg + (size_t)(gq < G ? gq : 0) * D;
    uint2 raw[C::KS];
    float mx = 0.f;
#pragma unroll
    for (int ks = 0; ks < C::KS; ++ks) {
        raw[ks] = gq < G ? *reinterpret_cast<const uint2 *>(qrow + 16 * ks + 4 * tq) : make_uint2(0u, 0u);
        const float2 a = bf16x2_to_float2(raw[ks].x), b = bf16x2_to_float2(raw[ks].y);
        mx = fmaxf(mx, fmaxf(fmaxf(fabsf(a.x), fabsf(a.y)), fmaxf(fabsf(b.x), fabsf(b.y))));
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    int e = 0;
    while (e < 120 && mx > 16384.f) {
        mx *= 0.5f;
        ++e;
    }
    const float down = exp2f(-(float)e);
#pragma unroll
    for (int ks = 0; ks < C::KS; ++ks) {
        const float2 a = bf16x2_to_float2(raw[ks].x), b = bf16x2_to_float2(raw[ks].y);
        qb[ks][0] = pack_f16x2(a.x * down, a.y * down);
        qb[ks][1] = pack_f16x2(b.x * down, b.y * down);
    }
    return exp2f((float)e);
}

// O^T += V^T . P^T for one 16-token sub-block, two m-tiles (chunks) per x4 load.  MASKED:
// V values of tokens at or past `valid` are zeroed (this lane's tokens: u, u + 1, u + 8, u + 9).
template <class C, int D, int QT, bool MASKED>
__device__ __forceinline__ void q8_pv(uint32_t vbase, int tok, int mat, int u, int valid, uint32_t pb0, uint32_t pb1,
                                      float (&o)[C::MT][4])
{
    uint32_t keep_lo = 0xffffffffu, keep_hi = 0xffffffffu;
    if constexpr (MASKED) {
        keep_lo = (u < valid ? 0x0000ffffu : 0u) | (u + 1 < valid ? 0xffff0000u : 0u);
        keep_hi = (u + 8 < valid ? 0x0000ffffu : 0u) | (u + 9 < valid ? 0xffff0000u : 0u);
    }
#pragma unroll
    for (int mt = 0; mt < C::MT; mt += 2) {
        uint32_t w[4];
        ldmatrix_x4_trans(w, vbase + swz_q8<D>(tok, mt + (mat >> 1)));
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            uint32_t a0, a1, a2, a3;
            q8_cross_to_f16<QT>(w[2 * j], a0, a1);
            q8_cross_to_f16<QT>(w[2 * j + 1], a2, a3);
            if constexpr (MASKED) {
                a0 &= keep_lo;
                a1 &= keep_lo;
                a2 &= keep_hi;
                a3 &= keep_hi;
            }
            mma_f16_16816(o[mt + j], a0, a1, a2, a3, pb0, pb1);
        }
    }
}

// One physical block's code tiles (K at `ktile`, V right after it), already in shared memory,
// folded into a warp's online-softmax state; `valid` tokens of the block count.
// o[mt][0..1] are dim 16 mt + 2 (T/4), o[mt][2..3] dim 16 mt + 2 (T/4) + 1 (heads 2t, 2t+1).
template <class C, int D, int QT>
__device__ __forceinline__ void q8_consume_block(const uint8_t *ktile, int valid, const uint32_t (&qb)[C::KS][2],
                                                 const float (&kbias)[2], float qk_scale, float (&m_run)[2],
                                                 float (&l_run)[2], float (&o)[C::MT][4], int lane)
{
    constexpr unsigned FULL = 0xffffffffu;
    const uint32_t kbase = smem_addr(ktile);
    const uint32_t vbase = kbase + C::TILE;
    const int mrow = lane & 7, mat = lane >> 3;     // ldmatrix: row address this lane supplies
    const int r = lane >> 2, tq = lane & 3;
#pragma unroll 1
    for (int sub = 0; sub < C::NSUB; ++sub) {
        if (sub * 16 >= valid) break;
        // matrices of one x4 load: (tokens 0-7, chunk c), (tokens 8-15, chunk c), then chunk c + 1
        const int tok = sub * 16 + (mat & 1) * 8 + mrow;
        // ---- S^T = K . Q^T for 16 tokens (even and odd k-steps in two accumulators: two
        //      dependency chains of half the length) ----
        float sA[4] = {0.f, 0.f, 0.f, 0.f}, sB[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ks = 0; ks < C::KS; ks += 2) {
            uint32_t w[4];
            ldmatrix_x4(w, kbase + swz_q8<D>(tok, ks + (mat >> 1)));
            uint32_t a0, a1, a2, a3;
            q8_quad_to_f16<QT>(w[0], a0, a2);
            q8_quad_to_f16<QT>(w[1], a1, a3);
            mma_f16_16816(sA, a0, a1, a2, a3, qb[ks][0], qb[ks][1]);
            q8_quad_to_f16<QT>(w[2], a0, a2);
            q8_quad_to_f16<QT>(w[3], a1, a3);
            mma_f16_16816(sB, a0, a1, a2, a3, qb[ks + 1][0], qb[ks + 1][1]);
        }
        const float sT[4] = {sA[0] + sB[0] - kbias[0], sA[1] + sB[1] - kbias[1], sA[2] + sB[2] - kbias[0],
                             sA[3] + sB[3] - kbias[1]};
        // ---- online softmax: tokens r and r + 8, heads 2tq and 2tq + 1 ----
        const int t0 = sub * 16 + r;
        const float x0 = t0 < valid ? sT[0] * qk_scale : -INFINITY;
        const float x1 = t0 < valid ? sT[1] * qk_scale : -INFINITY;
        const float x2 = t0 + 8 < valid ? sT[2] * qk_scale : -INFINITY;
        const float x3 = t0 + 8 < valid ? sT[3] * qk_scale : -INFINITY;
        float mx0 = fmaxf(x0, x2), mx1 = fmaxf(x1, x3);
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(FULL, mx0, off));
            mx1 = fmaxf(mx1, __shfl_xor_sync(FULL, mx1, off));
        }
        const float mn0 = fmaxf(m_run[0], mx0), mn1 = fmaxf(m_run[1], mx1);
        const float al0 = exp2f(m_run[0] - mn0), al1 = exp2f(m_run[1] - mn1);
        m_run[0] = mn0;
        m_run[1] = mn1;
        const float p0 = exp2f(x0 - mn0), p1 = exp2f(x1 - mn1);
        const float p2 = exp2f(x2 - mn0), p3 = exp2f(x3 - mn1);
        l_run[0] = l_run[0] * al0 + (p0 + p2);
        l_run[1] = l_run[1] * al1 + (p1 + p3);
        const uint32_t pb0 = movmatrix_trans(pack_f16x2(p0, p1));
        const uint32_t pb1 = movmatrix_trans(pack_f16x2(p2, p3));
        // rescale the accumulators only when a running max moved (after the first few
        // sub-blocks it rarely does); the vote keeps the branch uniform over the warp
        if (__any_sync(FULL, (al0 != 1.f) | (al1 != 1.f))) {
#pragma unroll
            for (int mt = 0; mt < C::MT; ++mt) {
                o[mt][0] *= al0;
                o[mt][1] *= al1;
                o[mt][2] *= al0;
                o[mt][3] *= al1;
            }
        }
        if (valid < sub * 16 + 16)
            q8_pv<C, D, QT, true>(vbase, tok, mat, sub * 16 + 2 * tq, valid, pb0, pb1, o);
        else
            q8_pv<C, D, QT, false>(vbase, tok, mat, 0, 0, pb0, pb1, o);
    }
}

template <int D, int BS, int G, int QT, int NW_ = 2, int RING_ = 32768>
__global__ void __maxnreg__(96)
    paged_decode_partition_q8_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tmap_k,
                                     const __grid_constant__ CUtensorMap tmap_v)
{
    using C = MmaQ8Config<D, BS, G, NW_, RING_>;
    constexpr int NW = C::NW, STAGES = C::STAGES;
    constexpr unsigned FULL = 0xffffffffu;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *stages = smem;
    uint64_t *full_bar = reinterpret_cast<uint64_t *>(smem + C::OFF_BARS);
    uint64_t *empty_bar = full_bar + STAGES;
    volatile int *stage_bad = reinterpret_cast<volatile int *>(smem + C::OFF_FLAGS);
    volatile int *abort_flag = stage_bad + STAGES;
    volatile int *bad_flag = stage_bad + STAGES + 1;

    const int part = blockIdx.x, kvh = blockIdx.y, seq = blockIdx.z;
    const int ctx = p.context_lens[seq];
    const int n_part = decode_num_partitions(ctx, p.partition_size, p.p_max);
    if (part >= n_part) return;                                  // uniform over the CTA
    const int tok_begin = p.partition_size > 0 ? part * p.partition_size : 0;
    const int tok_end = (part == n_part - 1) ? ctx : tok_begin + p.partition_size;
    const int nblk = tok_end > tok_begin ? ceil_div(tok_end - tok_begin, BS) : 0;
    const int blk0 = tok_begin / BS;
    const int last_blk = ctx > 0 ? (ctx - 1) / BS : -1;    // holds the appended token
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(&full_bar[i], 1);
            mbar_init(&empty_bar[i], 1);
        }
        *abort_flag = 0;
        *bad_flag = 0;
        mbar_init_fence();
    }
    __syncthreads();

    const int tq = lane & 3;                 // this lane's heads: 2 tq and 2 tq + 1
    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
    float o[C::MT][4];
#pragma unroll
    for (int mt = 0; mt < C::MT; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;

    if (warp == NW) {
        // ------------------------------ producer ------------------------------
        if (lane == 0) {
            prefetch_tensormap(&tmap_k);
            prefetch_tensormap(&tmap_v);
        }
        const uint64_t pol = l2_policy_evict_first();
        const int32_t *trow = p.block_tables + (size_t)seq * p.max_blocks_per_seq;
        int issued = 0;
        bool ok = true;
        for (int i0 = 0; i0 < nblk && ok; i0 += 32) {
            const int i = i0 + lane;
            int phys = -1;
            if (i < nblk) {
                const int lb = blk0 + i;
                if (lb < p.max_blocks_per_seq) {
                    phys = trow[lb];
                    if (phys >= p.num_blocks) phys = -1;
                }
            }
            const int cnt = min(32, nblk - i0);
            for (int k = 0; k < cnt; ++k) {
                const int ph = __shfl_sync(FULL, phys, k);
                const int ii = i0 + k;
                const int st = ii % STAGES;
                if (lane == 0) {
                    if (ii >= STAGES) ok = mbar_wait_bounded(&empty_bar[st], ((ii / STAGES) - 1) & 1);
                    if (ok && *abort_flag) ok = false;
                    if (ok) {
                        if (p.pdl_wait_last && blk0 + ii == last_blk) pdl_wait();
                        if (ph >= 0) {
                            stage_bad[st] = 0;
                            mbar_arrive_expect_tx(&full_bar[st], C::STAGE_BYTES);
                            const int row = (ph * p.h_kv + kvh) * BS;
                            uint8_t *dst = stages + st * C::STAGE_BYTES;
                            tma_load_2d(dst, &tmap_k, 0, row, &full_bar[st], pol);
                            tma_load_2d(dst + C::TILE, &tmap_v, 0, row, &full_bar[st], pol);
                        } else {
                            stage_bad[st] = 1;
                            record_error(PA_DEVERR_BAD_BLOCK);
                            mbar_arrive(&full_bar[st]);
                        }
                        issued = ii + 1;
                    }
                }
                ok = __shfl_sync(FULL, ok, 0) != 0;
                if (!ok) break;
            }
        }
        if (lane == 0 && !ok) {
            if (!*abort_flag) record_error(PA_DEVERR_TIMEOUT);
            *abort_flag = 1;
            for (int ii = max(0, issued - STAGES); ii < issued; ++ii)
                mbar_wait_bounded(&full_bar[ii % STAGES], (ii / STAGES) & 1);
        }
    } else {
        // ------------------------------ consumers ------------------------------
        uint32_t qb[C::KS][2];
        const float qk_scale = p.qk_scale * head_k_factor(p, kvh) *
                               q8_load_q<C, G, D>(qb, p.q + ((size_t)seq * p.h_q + (size_t)kvh * G) * D, lane);
        float kbias[2];
        q8_k_bias<C, QT>(qb, lane, kbias);
        for (int i = warp; i < nblk; i += NW) {
            if (*abort_flag) break;
            const int st = i % STAGES;
            const bool ok = __all_sync(FULL, mbar_wait_bounded(&full_bar[st], (i / STAGES) & 1));
            if (!ok) {
                if (lane == 0) {
                    record_error(PA_DEVERR_TIMEOUT);
                    *abort_flag = 1;
                }
                break;
            }
            if (stage_bad[st]) {
                if (lane == 0) *bad_flag = 1;
            } else {
                q8_consume_block<C, D, QT>(stages + st * C::STAGE_BYTES, min(BS, tok_end - (tok_begin + i * BS)), qb,
                                           kbias, qk_scale, m_run, l_run, o, lane);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty_bar[st]);
        }
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
            l_run[0] += __shfl_xor_sync(FULL, l_run[0], off);
            l_run[1] += __shfl_xor_sync(FULL, l_run[1], off);
        }
    }

    __syncthreads();        // every stage consumed; the ring becomes the combine area
    float *cm = reinterpret_cast<float *>(smem);                 // [NW][G]
    float *cl = cm + NW * G;                                     // [NW][G]
    float *co = cl + NW * G;                                     // [NW][G][D]
    if (warp < NW) {
        const int r = lane >> 2;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int h = 2 * tq + j;
            if (h < G) {
                if (r == 0) {
                    cm[warp * G + h] = m_run[j];
                    cl[warp * G + h] = l_run[j];
                }
#pragma unroll
                for (int mt = 0; mt < C::MT; ++mt) {
                    co[(size_t)(warp * G + h) * D + 16 * mt + 2 * r] = o[mt][j];
                    co[(size_t)(warp * G + h) * D + 16 * mt + 2 * r + 1] = o[mt][2 + j];
                }
            }
        }
    }
    __syncthreads();
    cta_combine_and_write<NW, G, D>(p, cm, part, n_part, kvh, seq, (*abort_flag != 0) || (*bad_flag != 0),
                                    reinterpret_cast<float *>(smem + C::COMBINE_BYTES));
}

}  // namespace pa
