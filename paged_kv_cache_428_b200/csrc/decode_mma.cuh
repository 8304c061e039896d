// decode_mma.cuh -- bf16 paged decode partition pass on the tensor cores (mma.sync).
//
// Same method, grid and pipeline as paged_decode_partition_kernel (decode.cuh): one CTA per
// (context partition, KV head, sequence), a producer warp streaming each physical block's K
// and V tiles into an mbarrier-guarded shared-memory ring, consumer warps taking whole
// blocks with their own online-softmax state, and the same CTA combine.  What changes is
// how a consumer warp does the two products of a 16-token sub-block, both on mma.sync
// m16n8k16 (bf16 in, fp32 accumulate) with the tokens or head dims on the 16 M rows and the
// (up to 8) query heads of the group on the 8 N columns:
//
//   S^T = K . Q^T : A = the 16 x D K rows (ldmatrix), B = Q^T (registers, heads >= G zero),
//                   D/16 k-steps.  Lane T holds scores of tokens T/4 and T/4 + 8 for heads
//                   2(T%4) and 2(T%4)+1.
//   O^T += V^T . P^T : P^T (probabilities rounded to bf16) is the B operand; it comes out of
//                   the S^T accumulators with one movmatrix.trans per 8x8 tile.  A = V^T via
//                   ldmatrix.trans, D/16 m-tiles of 16 head dims.  A lane's output columns
//                   are the same two heads as its scores, so rescaling by the softmax
//                   correction needs no data exchange.
//
// ldmatrix reads 8 rows of one 16-byte column per matrix; with the cache's 256-byte rows
// those would all hit the same banks, so the tiles are brought in by 2-D TMA through tensor
// maps with 128-byte swizzle: a box is 64 elements (128 bytes) x BS rows, chunk c of row r
// lands at chunk c ^ (r % 8), and every ldmatrix phase touches 8 distinct bank groups.
// Rows of a partly filled last block past the context may hold anything: their scores are
// masked to -inf by select, and their V rows are zeroed in shared memory before P . V
// (a zero probability times a NaN would otherwise poison the accumulator).
#pragma once

#include "decode.cuh"

namespace pa {

// NW_ consumer warps; RING_ bytes of shared memory for the stage ring (at least NW_ stages).
template <int D, int BS, int G, int NW_ = 2, int RING_ = 32768>
struct MmaDecodeConfig {
    static constexpr int NW = NW_;                        // consumer warps
    static constexpr int THREADS = (NW + 1) * 32;         // + producer warp
    static constexpr int HALVES = D / 64;                 // 128-byte column halves of a row
    static constexpr int HALF_BYTES = BS * 128;           // one TMA box (1024-byte multiple)
    static constexpr int TILE = HALVES * HALF_BYTES;      // K (or V) tile of one block
    static constexpr int STAGE_BYTES = 2 * TILE;
    // A multiple of NW: consumer warp w takes blocks i = w (mod NW), and block i reuses the
    // stage of block i - STAGES.  Only when that earlier block belongs to the same warp is
    // the stage's full barrier guaranteed to have finished the previous phase before the
    // warp waits on it; otherwise a parity wait could pass one phase early.
    static constexpr int STAGES = cmax(NW, cmin(32, RING_ / STAGE_BYTES) / NW * NW);
    static constexpr int KS = D / 16;                     // k-steps of q.K
    static constexpr int MT = D / 16;                     // m-tiles of O^T (16 head dims each)
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
    static_assert(HALF_BYTES % 1024 == 0, "swizzle atoms");
    static_assert(STAGES % NW == 0, "stage ring must be a multiple of the consumer warps");
};

// Byte offset of 16-byte chunk `chunk` (0..7) of row `row` inside a 128B-swizzled box.
__device__ __forceinline__ uint32_t swz128(int row, int chunk)
{
    return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}

// B fragments of Q^T for one group: column n = query head T/4 of the group (zero when
// >= G); k-step ks covers dims [16 ks, 16 ks + 16): lo pair at 2 tq, hi pair at 8 + 2 tq.
// `qg` points at the group's first query head.
template <class C, int G, int D>
__device__ __forceinline__ void mma_load_q(uint32_t (&qb)[C::KS][2], const __nv_bfloat16 *qg, int lane)
{
    const int gq = lane >> 2, tq = lane & 3;
    const uint32_t *qrow = reinterpret_cast<const uint32_t *>(qg + (size_t)(gq < G ? gq : 0) * D);
#pragma unroll
    for (int ks = 0; ks < C::KS; ++ks) {
        qb[ks][0] = gq < G ? qrow[8 * ks + tq] : 0u;
        qb[ks][1] = gq < G ? qrow[8 * ks + 4 + tq] : 0u;
    }
}

// One physical block of one KV head, already in shared memory (K tile at `ktile`, V tile
// right after it, both as 128B-swizzled boxes), folded into a warp's online-softmax state:
// `valid` tokens of the block count; rows past them are masked and their V rows zeroed.
// State: m_run/l_run for heads 2tq, 2tq+1 (log2 domain), o = O^T fragments.
template <class C, int BS, int G>
__device__ __forceinline__ void mma_consume_block(uint8_t *ktile, int valid, const uint32_t (&qb)[C::KS][2],
                                                  float qk_scale, float (&m_run)[2], float (&l_run)[2],
                                                  float (&o)[C::MT][4], int lane)
{
    constexpr unsigned FULL = 0xffffffffu;
    uint8_t *vtile = ktile + C::TILE;
    if (valid < BS) {
        // zero the V rows past the context (both halves, whole 128-byte rows)
        const int n16 = (BS - valid) * 8 * C::HALVES;
        for (int e = lane; e < n16; e += 32) {
            const int hf = e / ((BS - valid) * 8);
            const int row = valid + (e / 8) % (BS - valid);
            reinterpret_cast<uint4 *>(vtile + hf * C::HALF_BYTES + row * 128)[e % 8] = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
        __syncwarp();
    }
    const uint32_t kbase = smem_addr(ktile);
    const uint32_t vbase = smem_addr(vtile);
    const int mrow = lane & 7, mat = lane >> 3;     // ldmatrix: row address this lane supplies
    const int r = lane >> 2;                        // token row of this lane's scores
#pragma unroll 1
    for (int sub = 0; sub < C::NSUB; ++sub) {
        if (sub * 16 >= valid) break;
        // ---- S^T = K . Q^T for 16 tokens ----
        float sT[4] = {0.f, 0.f, 0.f, 0.f};
        {
            const int tok = sub * 16 + (mat & 1) * 8 + mrow;
#pragma unroll
            for (int ks = 0; ks < C::KS; ++ks) {
                const int chunk = 2 * (ks & 3) + (mat >> 1);
                uint32_t a[4];
                ldmatrix_x4(a, kbase + (ks >> 2) * C::HALF_BYTES + swz128(tok, chunk));
                mma_bf16_16816(sT, a[0], a[1], a[2], a[3], qb[ks][0], qb[ks][1]);
            }
        }
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
        // P^T as the B operand: b0 = P[head T/4][tokens 2tq, 2tq+1], b1 = tokens + 8
        const uint32_t pb0 = movmatrix_trans(pack_bf16x2(p0, p1));
        const uint32_t pb1 = movmatrix_trans(pack_bf16x2(p2, p3));
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
        // ---- O^T += V^T . P^T (m-tiles of 16 head dims) ----
        const int tok = sub * 16 + (mat >> 1) * 8 + mrow;
#pragma unroll
        for (int mt = 0; mt < C::MT; ++mt) {
            const int chunk = ((2 * mt) & 7) + (mat & 1);
            uint32_t a[4];
            ldmatrix_x4_trans(a, vbase + (mt >> 2) * C::HALF_BYTES + swz128(tok, chunk));
            mma_bf16_16816(o[mt], a[0], a[1], a[2], a[3], pb0, pb1);
        }
    }
}

template <int D, int BS, int G, int NW_ = 2, int RING_ = 32768>
__global__ void __launch_bounds__(MmaDecodeConfig<D, BS, G, NW_, RING_>::THREADS)
    paged_decode_partition_mma_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tmap_k,
                                      const __grid_constant__ CUtensorMap tmap_v)
{
    using C = MmaDecodeConfig<D, BS, G, NW_, RING_>;
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
    float o[C::MT][4];                       // O^T: dims 16 mt + T/4 (+ 8) x heads 2tq, 2tq + 1
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
#pragma unroll
                            for (int hf = 0; hf < C::HALVES; ++hf) {
                                tma_load_2d(dst + hf * C::HALF_BYTES, &tmap_k, hf * 64, row, &full_bar[st], pol);
                                tma_load_2d(dst + C::TILE + hf * C::HALF_BYTES, &tmap_v, hf * 64, row, &full_bar[st],
                                            pol);
                            }
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
        mma_load_q<C, G, D>(qb, p.q + ((size_t)seq * p.h_q + (size_t)kvh * G) * D, lane);
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
                mma_consume_block<C, BS, G>(stages + st * C::STAGE_BYTES, min(BS, tok_end - (tok_begin + i * BS)),
                                            qb, p.qk_scale, m_run, l_run, o, lane);
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
                    co[(size_t)(warp * G + h) * D + 16 * mt + r] = o[mt][j];
                    co[(size_t)(warp * G + h) * D + 16 * mt + r + 8] = o[mt][2 + j];
                }
            }
        }
    }
    __syncthreads();
    cta_combine_and_write<NW, G, D>(p, cm, part, n_part, kvh, seq, (*abort_flag != 0) || (*bad_flag != 0),
                                    reinterpret_cast<float *>(smem + C::COMBINE_BYTES));
}

}  // namespace pa

