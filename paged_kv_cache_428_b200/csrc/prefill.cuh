// prefill.cuh -- chunked-prefill attention over the paged KV cache (bf16), on the tensor cores.
//
// For every sequence a chunk of new query rows ends at the sequence's last cached token: row i
// of a chunk of n rows sits at position p = ctx - n + i and attends causally to tokens 0..p,
// read through the block table ("vLLM 推理原理…" section 一次生成有两个阶段: prefill processes the
// input tokens and builds their KV, chunked prefill splits a long input into pieces; "现代
// AI…" section 1, attention formula; "深度解构…" section 2.1, block table).  The chunk's own K/V
// rows are in the cache already (pa_reshape_and_cache before this call).
//
// One CTA per (query tile, KV head, sequence).  A tile is 128 rows: TQ = 128 / G query tokens x
// the G query heads of the KV head (row r = token r / G, head r % G), so the K/V bytes the CTA
// reads serve G heads at once.  Eight consumer warps own 16 rows each (measured 1.3x faster than
// four: each K/V tile read from L2 serves twice the rows); a producer warp streams
// the KV range [0, last row's position] in tiles of 64 tokens through an mbarrier ring: per
// physical block, 2-D TMA boxes of 64 elements x BS rows with the 128-byte swizzle (the same
// tensor maps as decode), so the tile lands as [64 tokens][D] in 128-byte-swizzled halves.
// Per KV tile and warp (mma.sync m16n8k16, bf16 in, fp32 accumulate):
//   S = Q K^T   A = Q rows (registers, loaded once), B = K^T via ldmatrix of the K tile
//   online softmax over the row (log2 domain), causal / context mask by select
//   O += P V    A = P straight from the S accumulators (bf16), B = V via ldmatrix.trans
// V values of tokens past the context are zeroed in registers (a zero probability times an
// unwritten NaN slot would poison the sum); K values there only reach masked scores.
#pragma once

#include "decode.cuh"
#include "decode_mma.cuh"

namespace pa {

struct PrefillParams {
    __nv_bfloat16 *out;            // [T][h_q][D]
    const __nv_bfloat16 *q;        // [T][h_q][D]
    const uint8_t *k_cache;        // [NB][h_kv][bs][D] bf16
    const uint8_t *v_cache;
    const int32_t *block_tables;   // [B][max_blocks_per_seq]
    const int32_t *query_start;    // [B + 1]: chunk of sequence s = rows query_start[s] .. [s + 1] - 1
    const int32_t *context_lens;   // [B], each including its chunk
    int max_blocks_per_seq;
    int h_q;
    int h_kv;
    int num_blocks;
    float qk_scale;                // scale * log2(e)
};

template <int D, int BS, int G, int STAGES_ = 3, int NW_ = 8>
struct PrefillConfig {
    static constexpr int NW = NW_;                        // consumer warps, 16 rows each
    static constexpr int THREADS = (NW + 1) * 32;         // + producer warp
    static constexpr int BM = 16 * NW;                    // rows per CTA
    static constexpr int TQ = BM / G;                     // query tokens per CTA
    static constexpr int BN = 64;                         // KV tokens per tile
    static constexpr int HALVES = D / 64;
    static constexpr int HALF_BYTES = BN * 128;           // one 64-token half tile
    static constexpr int TILE = HALVES * HALF_BYTES;      // K (or V) tile
    static constexpr int STAGE_BYTES = 2 * TILE;
    static constexpr int STAGES = STAGES_;
    static constexpr int BLOCKS_PER_TILE = BN / BS;
    static constexpr int KS = D / 16;                     // k-steps of Q K^T
    static constexpr int NT = BN / 8;                     // n-tiles of S
    static constexpr int DT = D / 8;                      // n-tiles of O
    static constexpr int OFF_BARS = STAGES * STAGE_BYTES;
    static constexpr int OFF_FLAGS = OFF_BARS + 2 * STAGES * 8;
    static constexpr int SMEM = OFF_FLAGS + (STAGES + 4) * 4 + 1024;
    static_assert(D == 64 || D == 128, "head dim");
    static_assert(BS == 16 || BS == 32 || BS == 64, "block size");
    static_assert(BM % G == 0 && G <= 8, "group");
    static_assert((BS * 128) % 1024 == 0, "box destinations keep the swizzle atoms aligned");
};

// Number of query tiles of a chunk of n rows.
template <int TQ>
__host__ __device__ __forceinline__ int prefill_tiles(int n) { return (n + TQ - 1) / TQ; }

template <int D, int BS, int G, int STAGES_ = 3, int NW_ = 8>
__global__ void __launch_bounds__(PrefillConfig<D, BS, G, STAGES_, NW_>::THREADS)
    paged_prefill_kernel(const PrefillParams p, const __grid_constant__ CUtensorMap tmap_k,
                         const __grid_constant__ CUtensorMap tmap_v)
{
    using C = PrefillConfig<D, BS, G, STAGES_, NW_>;
    constexpr int STAGES = C::STAGES, BN = C::BN;
    constexpr unsigned FULL = 0xffffffffu;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full_bar = reinterpret_cast<uint64_t *>(smem + C::OFF_BARS);
    uint64_t *empty_bar = full_bar + STAGES;
    volatile int *stage_bad = reinterpret_cast<volatile int *>(smem + C::OFF_FLAGS);
    volatile int *abort_flag = stage_bad + STAGES;

    const int kvh = blockIdx.y, seq = blockIdx.z;
    const int q0 = p.query_start[seq], q1 = p.query_start[seq + 1];
    const int chunk = q1 - q0;
    const int ctx = p.context_lens[seq];
    const int ntiles = prefill_tiles<C::TQ>(chunk);
    const int tile = ntiles - 1 - (int)blockIdx.x;             // longest KV ranges first
    if (chunk > ctx) {                                         // rows left unwritten, flagged
        if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.y == 0) record_error(PA_DEVERR_BAD_CHUNK);
        return;
    }
    if (tile < 0 || chunk <= 0) return;                        // uniform over the CTA
    const int tok0 = tile * C::TQ;                             // first query token of the tile
    const int tok_end = min(chunk, tok0 + C::TQ);
    const int first_pos = ctx - chunk + tok0;                  // smallest position in the tile
    const int kv_len = ctx - chunk + tok_end;                  // KV tokens any row attends to
    const int nkv = ceil_div(kv_len, BN);
    const int nblk_seq = ceil_div(ctx, BS);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(&full_bar[i], 1);
            mbar_init(&empty_bar[i], C::NW);
        }
        *abort_flag = 0;
        mbar_init_fence();
    }
    __syncthreads();

    if (warp == C::NW) {
        // ------------------------------ producer ------------------------------
        if (lane == 0) {
            prefetch_tensormap(&tmap_k);
            prefetch_tensormap(&tmap_v);
            const uint64_t pol = l2_policy_evict_last();       // K/V tiles are re-read by other query tiles
            const int32_t *trow = p.block_tables + (size_t)seq * p.max_blocks_per_seq;
            int issued = 0;
            bool ok = true;
            for (int it = 0; it < nkv && ok; ++it) {
                const int st = it % STAGES;
                if (it >= STAGES) ok = mbar_wait_bounded(&empty_bar[st], ((it / STAGES) - 1) & 1);
                if (ok && *abort_flag) ok = false;
                if (!ok) break;
                // blocks of this tile that exist in the sequence
                const int b0 = it * C::BLOCKS_PER_TILE;
                const int nb = min(C::BLOCKS_PER_TILE, nblk_seq - b0);
                bool bad = false;
                int phys[C::BLOCKS_PER_TILE];
#pragma unroll
                for (int k = 0; k < C::BLOCKS_PER_TILE; ++k) {
                    phys[k] = -1;
                    if (k < nb) {
                        const int lb = b0 + k;
                        phys[k] = lb < p.max_blocks_per_seq ? trow[lb] : -1;
                        if (phys[k] < 0 || phys[k] >= p.num_blocks) bad = true;
                    }
                }
                if (bad) {
                    stage_bad[st] = 1;
                    record_error(PA_DEVERR_BAD_BLOCK);
                    mbar_arrive(&full_bar[st]);
                } else {
                    stage_bad[st] = 0;
                    mbar_arrive_expect_tx(&full_bar[st], (uint32_t)(nb * 2 * C::HALVES * BS * 128));
                    uint8_t *dst = smem + st * C::STAGE_BYTES;
                    for (int k = 0; k < nb; ++k) {
                        const int row = (phys[k] * p.h_kv + kvh) * BS;
#pragma unroll
                        for (int hf = 0; hf < C::HALVES; ++hf) {
                            uint8_t *kd = dst + hf * C::HALF_BYTES + k * BS * 128;
                            tma_load_2d(kd, &tmap_k, hf * 64, row, &full_bar[st], pol);
                            tma_load_2d(kd + C::TILE, &tmap_v, hf * 64, row, &full_bar[st], pol);
                        }
                    }
                }
                issued = it + 1;
            }
            if (!ok) {
                if (!*abort_flag) record_error(PA_DEVERR_TIMEOUT);
                *abort_flag = 1;
                for (int ii = max(0, issued - STAGES); ii < issued; ++ii)
                    mbar_wait_bounded(&full_bar[ii % STAGES], (ii / STAGES) & 1);
            }
        }
        return;
    }

    // ------------------------------ consumers ------------------------------
    const int gid = lane >> 2, tq = lane & 3;
    // the two rows of this lane: r = 16 warp + gid (+ 8)
    int pos[2];
    bool row_ok[2];
    const __nv_bfloat16 *qrow[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const int r = 16 * warp + gid + 8 * j;
        const int t = tok0 + r / G;
        row_ok[j] = t < tok_end;
        pos[j] = row_ok[j] ? ctx - chunk + t : 0;              // a padding row attends to token 0
        const int tt = row_ok[j] ? t : tok0;
        qrow[j] = p.q + ((size_t)(q0 + tt) * p.h_q + (size_t)kvh * G + r % G) * D;
    }
    // Q as A fragments: qa[ks] = {row gid dims 16ks+2tq.., row gid+8 .., row gid dims +8, row gid+8 +8}
    uint32_t qa[C::KS][4];
#pragma unroll
    for (int ks = 0; ks < C::KS; ++ks) {
        const uint32_t *q0p = reinterpret_cast<const uint32_t *>(qrow[0] + 16 * ks + 2 * tq);
        const uint32_t *q1p = reinterpret_cast<const uint32_t *>(qrow[1] + 16 * ks + 2 * tq);
        qa[ks][0] = row_ok[0] ? q0p[0] : 0u;
        qa[ks][1] = row_ok[1] ? q1p[0] : 0u;
        qa[ks][2] = row_ok[0] ? q0p[4] : 0u;
        qa[ks][3] = row_ok[1] ? q1p[4] : 0u;
    }
    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
    float o[C::DT][4];
#pragma unroll
    for (int i = 0; i < C::DT; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;

    const int mrow = lane & 7, mat = lane >> 3;
    bool failed = false;
    for (int it = 0; it < nkv; ++it) {
        if (*abort_flag) {
            failed = true;
            break;
        }
        const int st = it % STAGES;
        const bool ok = __all_sync(FULL, mbar_wait_bounded(&full_bar[st], (it / STAGES) & 1));
        if (!ok) {
            if (lane == 0) {
                record_error(PA_DEVERR_TIMEOUT);
                *abort_flag = 1;
            }
            failed = true;
            break;
        }
        if (stage_bad[st]) {
            failed = true;
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty_bar[st]);
            continue;
        }
        const uint32_t kbase = smem_addr(smem + st * C::STAGE_BYTES);
        const uint32_t vbase = kbase + C::TILE;
        const int kv0 = it * BN;
        // ---- S = Q K^T (16 rows x 64 tokens) ----
        float s[C::NT][4];
#pragma unroll
        for (int nt = 0; nt < C::NT; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
        for (int ks = 0; ks < C::KS; ++ks) {
#pragma unroll
            for (int nt = 0; nt < C::NT; nt += 2) {
                // matrices: (tokens 8nt.., dims 16ks..+7), (.., dims +8..), (tokens 8nt+8.., ..), (..)
                const int tok = 8 * nt + (mat >> 1) * 8 + mrow;
                const int chunk16 = 2 * (ks & 3) + (mat & 1);
                uint32_t b[4];
                ldmatrix_x4(b, kbase + (ks >> 2) * C::HALF_BYTES + swz128(tok, chunk16));
                mma_bf16_16816(s[nt], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], b[0], b[1]);
                mma_bf16_16816(s[nt + 1], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], b[2], b[3]);
            }
        }
        // ---- mask, online softmax ----
        const bool need_mask = kv0 + BN - 1 > first_pos;       // some token of the tile is past a row
        float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int nt = 0; nt < C::NT; ++nt) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int j = e >> 1;                          // row gid (0) or gid + 8 (1)
                const int t = kv0 + 8 * nt + 2 * tq + (e & 1);
                float x = s[nt][e] * p.qk_scale;
                if (need_mask && t > pos[j]) x = -INFINITY;
                s[nt][e] = x;
                mx[j] = fmaxf(mx[j], x);
            }
        }
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            mx[j] = fmaxf(mx[j], __shfl_xor_sync(FULL, mx[j], 1));
            mx[j] = fmaxf(mx[j], __shfl_xor_sync(FULL, mx[j], 2));
        }
        float al[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const float mn = fmaxf(m_run[j], mx[j]);
            al[j] = exp2f(m_run[j] - mn);
            m_run[j] = mn;
        }
        float rs[2] = {0.f, 0.f};
        uint32_t pa_[C::NT / 2][4];
#pragma unroll
        for (int nt = 0; nt < C::NT; ++nt) {
            const float p0 = exp2f(s[nt][0] - m_run[0]), p1 = exp2f(s[nt][1] - m_run[0]);
            const float p2 = exp2f(s[nt][2] - m_run[1]), p3 = exp2f(s[nt][3] - m_run[1]);
            rs[0] += p0 + p1;
            rs[1] += p2 + p3;
            // A fragment of P for k-step nt / 2: n-tile 2kk -> a0 (row gid), a1 (row gid+8);
            // n-tile 2kk+1 -> a2, a3
            pa_[nt >> 1][(nt & 1) * 2 + 0] = pack_bf16x2(p0, p1);
            pa_[nt >> 1][(nt & 1) * 2 + 1] = pack_bf16x2(p2, p3);
        }
        l_run[0] = l_run[0] * al[0] + rs[0];
        l_run[1] = l_run[1] * al[1] + rs[1];
        if (__any_sync(FULL, (al[0] != 1.f) | (al[1] != 1.f))) {
#pragma unroll
            for (int i = 0; i < C::DT; ++i) {
                o[i][0] *= al[0];
                o[i][1] *= al[0];
                o[i][2] *= al[1];
                o[i][3] *= al[1];
            }
        }
        // ---- O += P V ----
        const bool zero_v = kv0 + BN > ctx;                    // tokens past the context in this tile
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
            // tokens of this lane's B fragments: 16kk + 2tq (+1) and 16kk + 8 + 2tq (+1)
            uint32_t keep0 = 0xffffffffu, keep1 = 0xffffffffu;
            if (zero_v) {
                const int t = kv0 + 16 * kk + 2 * tq;
                keep0 = (t < ctx ? 0x0000ffffu : 0u) | (t + 1 < ctx ? 0xffff0000u : 0u);
                keep1 = (t + 8 < ctx ? 0x0000ffffu : 0u) | (t + 9 < ctx ? 0xffff0000u : 0u);
            }
            const int tok = 16 * kk + (mat & 1) * 8 + mrow;
#pragma unroll
            for (int dt = 0; dt < C::DT; dt += 2) {
                // matrices: (tokens 16kk..+7, dims 8dt..), (tokens +8.., dims 8dt..), (.., dims 8dt+8..), (..)
                const int chunk16 = (dt & 7) + (mat >> 1);
                uint32_t b[4];
                ldmatrix_x4_trans(b, vbase + (dt >> 3) * C::HALF_BYTES + swz128(tok, chunk16));
                mma_bf16_16816(o[dt], pa_[kk][0], pa_[kk][1], pa_[kk][2], pa_[kk][3], b[0] & keep0, b[1] & keep1);
                mma_bf16_16816(o[dt + 1], pa_[kk][0], pa_[kk][1], pa_[kk][2], pa_[kk][3], b[2] & keep0,
                               b[3] & keep1);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_bar[st]);
    }

    // ---- normalise and write ----
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        l_run[j] += __shfl_xor_sync(FULL, l_run[j], 1);
        l_run[j] += __shfl_xor_sync(FULL, l_run[j], 2);
    }
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        if (!row_ok[j]) continue;
        const float inv = (l_run[j] > 0.f && !failed) ? 1.f / l_run[j] : __int_as_float(0x7fc00000);
        const int r = 16 * warp + gid + 8 * j;
        __nv_bfloat16 *orow = p.out + ((size_t)(q0 + tok0 + r / G) * p.h_q + (size_t)kvh * G + r % G) * D;
#pragma unroll
        for (int dt = 0; dt < C::DT; ++dt)
            *reinterpret_cast<uint32_t *>(orow + 8 * dt + 2 * tq) =
                pack_bf16x2(o[dt][2 * j] * inv, o[dt][2 * j + 1] * inv);
    }
}

}  // namespace pa
