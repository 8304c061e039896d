// prefill_tc.cuh -- chunked-prefill attention over the paged bf16 KV cache on the
// 5th-generation tensor cores (tcgen05.mma, accumulators in tensor memory).
//
// Same computation and masking rules as paged_prefill_kernel (prefill.cuh).  One CTA per (pair
// of query tiles, KV head, sequence); a query tile is 128 rows = 128 / G tokens x the G heads of
// the KV head, and both tiles of a CTA share every K/V tile it streams.  Roles:
//   warps 0-7  two softmax warpgroups, one per query tile: thread t of a warpgroup owns row t of
//              its tile (= tensor-memory lane t of the tile's columns).  It reads its row of S
//              from tensor memory, applies the causal / context mask, keeps the running max
//              and sum (log2 domain), writes its row of P (bf16) into a 128-byte-swizzled
//              shared tile, rescales its row of O in tensor memory when its max moved, and
//              finally normalises O and writes the output row.
//   warp 8     tensor-memory allocation (all 512 columns: per tile two 64-column S buffers and
//              the O accumulator); lane 0 issues every tcgen05.mma: S = Q K_j^T (M 128, N 64,
//              K = D) for both tiles, then O += P V_{j-1} (M 128, N D, K 64) for both, with P
//              from shared memory and V read N-major, so one tile's S runs on the tensor core
//              while the other tile's softmax works; tcgen05.commit signals each step.
//   warp 9     lane 0 streams the 64-token K tiles, lane 1 the V tiles, per physical block with
//              2-D TMA (the decode tensor maps, 128-byte swizzle), so the tiles are the MMA
//              operands as they land.  K and V have separate rings: a K tile is free as soon as
//              the S products that read it finish, so K runs 4 tiles ahead; V (2 stages) is
//              needed only after the softmax.
// Q is copied into a swizzled shared tile once.  S_{j+1} is computed while the softmax works on
// S_j (two S buffers per query tile); P is double-buffered.  V rows past the context are zeroed in shared memory
// before the P V step (an unwritten NaN slot times a zero probability would poison O).  Every
// wait is bounded; on a timeout or a bad block the CTA records the error, stops, drains its
// MMAs and frees its tensor memory; its rows come out NaN.
#pragma once

#include "prefill.cuh"
#include "tc.cuh"

namespace pa {

// 2^x with the MUFU instruction (flush-to-zero; x <= 0 here, -inf gives 0).
__device__ __forceinline__ float ex2_approx(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

template <int D, int BS, int G, int NQ_ = 2, int KST_ = 4, int VST_ = 2>
struct PrefillTcConfig {
    static constexpr int NQ = NQ_;                        // 128-row query tiles per CTA
    static constexpr int THREADS = 128 * NQ + 64;         // softmax warpgroups, MMA warp, TMA warp
    static constexpr int MMA_WARP = 4 * NQ, TMA_WARP = 4 * NQ + 1;
    static constexpr int BM = 128;                        // rows per query tile = tensor-memory lanes
    static constexpr int TQ = BM / G;                     // query tokens per query tile
    static constexpr int BN = 64;                         // KV tokens per tile
    static constexpr int HALVES = D / 64;
    static constexpr int KV_HALF = BN * 128;              // [64 tokens][64 elements]
    static constexpr int KV_TILE = HALVES * KV_HALF;      // K (or V) tile
    static constexpr int KST = KST_;                      // K ring: freed as soon as S is computed
    static constexpr int VST = VST_;                      // V ring: freed after P V
    static constexpr int BLOCKS_PER_TILE = BN / BS;
    static constexpr int Q_HALF = BM * 128;               // [128 rows][64 elements]
    static constexpr int Q_BYTES = HALVES * Q_HALF;
    static constexpr int P_BYTES = BM * 128;              // [128 rows][64 tokens] bf16
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = NQ * Q_BYTES;
    static constexpr int OFF_V = OFF_K + KST * KV_TILE;
    static constexpr int OFF_P = OFF_V + VST * KV_TILE;
    static constexpr int OFF_BARS = OFF_P + NQ * 2 * P_BYTES;
    static constexpr int NBARS = 2 * KST + 2 * VST + NQ * 8 + 1; // k, v full/empty; per tile s full/free, p full, o done; drain
    static constexpr int OFF_MISC = OFF_BARS + NBARS * 8; // tensor-memory base, abort flag
    static constexpr int SMEM = OFF_MISC + 16 + 1024;
    static constexpr int TMEM_PER_Q = 256;                // S0 [0,64), S1 [64,128), O [128, 128 + D)
    static constexpr int TMEM_COLS = NQ * TMEM_PER_Q;
    static constexpr int COL_O = 128;
    static constexpr uint32_t IDESC_S = umma_idesc_bf16(BM, BN, false);
    static constexpr uint32_t IDESC_O = umma_idesc_bf16(BM, D, true);
    static_assert(D == 64 || D == 128, "head dim");
    static_assert(BS == 16 || BS == 32 || BS == 64, "block size");
    static_assert(BM % G == 0 && G <= 8, "group");
    static_assert(NQ == 1 || NQ == 2, "query tiles");
    static_assert(SMEM <= 227 * 1024, "shared memory");
};

template <int D, int BS, int G, int NQ_ = 2, int KST_ = 4, int VST_ = 2>
__global__ void __launch_bounds__(PrefillTcConfig<D, BS, G, NQ_, KST_, VST_>::THREADS, 1)
    paged_prefill_tc_kernel(const PrefillParams p, const __grid_constant__ CUtensorMap tmap_k,
                            const __grid_constant__ CUtensorMap tmap_v)
{
    using C = PrefillTcConfig<D, BS, G, NQ_, KST_, VST_>;
    constexpr int KST = C::KST, VST = C::VST, BN = C::BN, NQ = C::NQ;
    constexpr unsigned FULL = 0xffffffffu;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BARS);
    uint64_t *k_full = bars, *k_empty = bars + KST, *v_full = bars + 2 * KST, *v_empty = v_full + VST;
    // per query tile q and buffer b: index 2 q + b
    uint64_t *s_full = bars + 2 * KST + 2 * VST, *s_free = s_full + 2 * NQ, *p_full = s_free + 2 * NQ, *o_done = p_full + 2 * NQ;
    uint64_t *drain = o_done + 2 * NQ;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);

    const int kvh = blockIdx.y, seq = blockIdx.z;
    const int q0 = p.query_start[seq], q1 = p.query_start[seq + 1];
    const int chunk = q1 - q0;
    const int ctx = p.context_lens[seq];
    const int ntiles = prefill_tiles<C::TQ>(chunk);
    const int npairs = (ntiles + NQ - 1) / NQ;
    const int pair = npairs - 1 - (int)blockIdx.x;             // longest KV ranges first
    if (chunk > ctx) {                                         // rows left unwritten, flagged
        if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.y == 0) record_error(PA_DEVERR_BAD_CHUNK);
        return;
    }
    if (pair < 0 || chunk <= 0) return;                        // uniform over the CTA
    // query tile q of this CTA: tokens [tok0(q), tok_end(q)); it reads KV tiles 0 .. nkv(q) - 1
    auto tok0_of = [&](int q) { return (pair * NQ + q) * C::TQ; };
    auto nkv_of = [&](int q) {
        const int t0 = tok0_of(q);
        if (t0 >= chunk) return 0;
        return ceil_div(ctx - chunk + min(chunk, t0 + C::TQ), BN);
    };
    int nkv = 0;
#pragma unroll
    for (int q = 0; q < NQ; ++q) nkv = max(nkv, nkv_of(q));
    const int nblk_seq = ceil_div(ctx, BS);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < KST; ++i) {
            mbar_init(&k_full[i], 1);
            mbar_init(&k_empty[i], 1);
        }
        for (int i = 0; i < VST; ++i) {
            mbar_init(&v_full[i], 1);
            mbar_init(&v_empty[i], 1);
        }
        for (int b = 0; b < 2 * NQ; ++b) {
            mbar_init(&s_full[b], 1);
            mbar_init(&s_free[b], 4);
            mbar_init(&p_full[b], 4);
            mbar_init(&o_done[b], 1);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        mbar_init_fence();
    }
    if (warp == C::MMA_WARP) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    if (warp < 4 * NQ) {
        // Q rows of query tile q into its swizzled shared tile (row t = token t / G, head t % G)
        const int q = warp >> 2, t = threadIdx.x & 127;
        const int tok = tok0_of(q) + t / G;
        const bool ok = tok < chunk;
        const uint4 *src = reinterpret_cast<const uint4 *>(
            p.q + ((size_t)(q0 + (ok ? tok : 0)) * p.h_q + (size_t)kvh * G + t % G) * D);
#pragma unroll
        for (int c = 0; c < D / 8; ++c) {
            const uint4 v = ok ? src[c] : make_uint4(0u, 0u, 0u, 0u);
            *reinterpret_cast<uint4 *>(smem + C::OFF_Q + q * C::Q_BYTES + (c >> 3) * C::Q_HALF + swz128(t, c & 7)) = v;
        }
        fence_proxy_async_smem();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == C::TMA_WARP) {
        // ------------------------------ TMA producers ------------------------------
        // lane 0 streams the K tiles (ring of KST, freed once S is computed), lane 1 the V tiles
        // (ring of VST, freed after P V); each checks the block-table entries of its tiles.
        if (lane < 2) {
            const bool is_v = lane == 1;
            const int nst = is_v ? VST : KST;
            uint64_t *full = is_v ? v_full : k_full;
            uint64_t *empty = is_v ? v_empty : k_empty;
            const CUtensorMap *map = is_v ? &tmap_v : &tmap_k;
            prefetch_tensormap(map);
            const uint64_t pol = l2_policy_evict_last();
            const int32_t *trow = p.block_tables + (size_t)seq * p.max_blocks_per_seq;
            for (int it = 0; it < nkv; ++it) {
                const int st = it % nst;
                if (it >= nst && !mbar_wait_bounded(&empty[st], ((it / nst) - 1) & 1)) {
                    if (!*abort_flag) record_error(PA_DEVERR_TIMEOUT);
                    *abort_flag = 1;
                    break;
                }
                if (*abort_flag) break;
                const int b0 = it * C::BLOCKS_PER_TILE;
                const int nb = min(C::BLOCKS_PER_TILE, nblk_seq - b0);
                int phys[C::BLOCKS_PER_TILE];
                bool bad = false;
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
                    record_error(PA_DEVERR_BAD_BLOCK);
                    *abort_flag = 1;
                    mbar_arrive(&full[st]);                    // wake the MMA thread
                    break;
                }
                mbar_arrive_expect_tx(&full[st], (uint32_t)(nb * C::HALVES * BS * 128));
                uint8_t *dst = smem + (is_v ? C::OFF_V : C::OFF_K) + st * C::KV_TILE;
                for (int k = 0; k < nb; ++k) {
                    const int row = (phys[k] * p.h_kv + kvh) * BS;
#pragma unroll
                    for (int hf = 0; hf < C::HALVES; ++hf)
                        tma_load_2d(dst + hf * C::KV_HALF + k * BS * 128, map, hf * 64, row, &full[st], pol);
                }
            }
        }
    } else if (warp == C::MMA_WARP) {
        // ------------------------------ MMA issue ------------------------------
        if (lane == 0) {
            int nkvq[NQ];
#pragma unroll
            for (int q = 0; q < NQ; ++q) nkvq[q] = nkv_of(q);
            auto pv = [&](int q, int i) -> bool {
                if (!mbar_wait_bounded(&p_full[2 * q + (i & 1)], (i >> 1) & 1) || *abort_flag) return false;
                tc_fence_after_sync();
                const uint32_t vbase = smem_addr(smem + C::OFF_V + (i % VST) * C::KV_TILE);
                const uint32_t pbase = smem_addr(smem + C::OFF_P + (2 * q + (i & 1)) * C::P_BYTES);
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk)
                    umma_bf16_ss(tmem + q * C::TMEM_PER_Q + C::COL_O, umma_desc_sw128(pbase + kk * 32, 16, 1024),
                                 umma_desc_sw128(vbase + kk * 2048, C::KV_HALF, 1024), C::IDESC_O, i > 0 || kk > 0);
                umma_commit(&o_done[2 * q + (i & 1)]);
                return true;
            };
            // S_q,j for tile q into S buffer j % 2 (K tile j must have landed); the last tile to
            // read K tile j releases it
            auto s_mma = [&](int q, int j) -> bool {
                const int st = j % KST;
                if (!mbar_wait_bounded(&k_full[st], (j / KST) & 1) || *abort_flag) return false;
                if (j >= 2 && (!mbar_wait_bounded(&s_free[2 * q + (j & 1)], ((j - 2) >> 1) & 1) || *abort_flag))
                    return false;
                tc_fence_after_sync();
                const uint32_t kbase = smem_addr(smem + C::OFF_K + st * C::KV_TILE);
                const uint32_t qbase = smem_addr(smem + C::OFF_Q + q * C::Q_BYTES);
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks)
                    umma_bf16_ss(tmem + q * C::TMEM_PER_Q + (uint32_t)((j & 1) * 64),
                                 umma_desc_sw128(qbase + (ks >> 2) * C::Q_HALF + (ks & 3) * 32, 16, 1024),
                                 umma_desc_sw128(kbase + (ks >> 2) * C::KV_HALF + (ks & 3) * 32, 16, 1024),
                                 C::IDESC_S, ks > 0);
                umma_commit(&s_full[2 * q + (j & 1)]);
                bool last_reader = true;
#pragma unroll
                for (int r = q + 1; r < NQ; ++r)
                    if (j < nkvq[r]) last_reader = false;
                if (last_reader) umma_commit(&k_empty[st]);
                return true;
            };
            // Schedule: S for the first two KV tiles of every query tile, then per KV tile j and
            // query tile q: O += P V_j as soon as that tile's softmax has produced P_j, then
            // S_q,j+2 into the S buffer P_j's softmax has just released.  Each query tile keeps
            // one S product in flight while its softmax works on the other.
            bool ok = true;
            for (int j = 0; j < 2 && ok; ++j)
#pragma unroll
                for (int q = 0; q < NQ; ++q)
                    if (ok && j < nkvq[q]) ok = s_mma(q, j);
            for (int j = 0; j < nkv && ok; ++j) {
                ok = mbar_wait_bounded(&v_full[j % VST], (j / VST) & 1) && !*abort_flag;
#pragma unroll
                for (int q = 0; q < NQ; ++q) {
                    if (!ok || j >= nkvq[q]) continue;
                    ok = pv(q, j);
                    if (ok && j + 2 < nkvq[q]) ok = s_mma(q, j + 2);
                }
                if (ok) umma_commit(&v_empty[j % VST]);
            }
            if (!ok) {
                if (!*abort_flag) record_error(PA_DEVERR_TIMEOUT);
                *abort_flag = 1;
            }
            umma_commit(drain);                                 // every MMA issued so far has finished
            mbar_wait_bounded(drain, 0);
        }
        __syncwarp();
    } else {
        // ------------------------------ softmax warpgroups ------------------------------
        const int q = warp >> 2, t = threadIdx.x & 127;
        const int tok0 = tok0_of(q), nkv_q = nkv_of(q);
        const int tok = tok0 + t / G;
        const bool row_ok = tok < chunk;
        const int pos = row_ok ? ctx - chunk + tok : 0;
        const int first_pos = ctx - chunk + tok0;
        const uint32_t lane_tm = tmem + q * C::TMEM_PER_Q + ((uint32_t)(32 * (warp & 3)) << 16);
        uint64_t *my_s_full = s_full + 2 * q, *my_s_free = s_free + 2 * q;
        uint64_t *my_p_full = p_full + 2 * q, *my_o_done = o_done + 2 * q;
        float m_run = -INFINITY, l_run = 0.f;
        bool failed = false;
        for (int j = 0; j < nkv_q; ++j) {
            bool ok = __all_sync(FULL, mbar_wait_bounded(&my_s_full[j & 1], (j >> 1) & 1));
            if (!ok || *abort_flag) {
                failed = true;
                break;
            }
            tc_fence_after_sync();
            uint32_t sr[2][32];
            tmem_ld32(lane_tm + (uint32_t)((j & 1) * 64), sr[0]);
            tmem_ld32(lane_tm + (uint32_t)((j & 1) * 64 + 32), sr[1]);
            tmem_wait_ld();
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&my_s_free[j & 1]);

            // raw scores s; the log2-domain logit is s * qk_scale (qk_scale > 0, so the max of
            // the logits is the scaled max of the scores), p = 2^(s * qk_scale - m) by one FMA
            const int kv0 = j * BN;
            if (kv0 + BN - 1 > first_pos) {
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int c = 0; c < 32; ++c)
                        if (kv0 + 32 * h + c > pos) sr[h][c] = 0xff800000u;        // -inf
            }
            float mx = -INFINITY;
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int c = 0; c < 32; ++c) mx = fmaxf(mx, __uint_as_float(sr[h][c]));
            // m_run is the reference the exponentials are taken against.  It moves (and O and
            // l are rescaled) only when the tile's max exceeds it by more than 8, so p <= 2^8;
            // O / l does not depend on the reference, and rescaling becomes rare, which keeps
            // the softmax from waiting for the previous P V.
            const float m_tile = mx * p.qk_scale;
            float alpha = 1.f;
            bool moved = false;
            if (j == 0) {
                m_run = m_tile;
            } else if (m_tile > m_run + 8.f) {
                alpha = ex2_approx(m_run - m_tile);
                m_run = m_tile;
                moved = true;
            }
            const float mn = m_run;
            float rs = 0.f;
            uint32_t pk[32];
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int c = 0; c < 32; c += 2) {
                    const float a = ex2_approx(fmaf(__uint_as_float(sr[h][c]), p.qk_scale, -mn));
                    const float b = ex2_approx(fmaf(__uint_as_float(sr[h][c + 1]), p.qk_scale, -mn));
                    rs += a + b;
                    pk[16 * h + c / 2] = pack_bf16x2(a, b);
                }
            l_run = l_run * alpha + rs;
            // rescale this warp's rows of O when any of their maxima moved (PV_{j-1} must be done)
            if (__any_sync(FULL, moved)) {
                ok = __all_sync(FULL, mbar_wait_bounded(&my_o_done[(j - 1) & 1], ((j - 1) >> 1) & 1));
                if (!ok || *abort_flag) {
                    failed = true;
                    break;
                }
                tc_fence_after_sync();
#pragma unroll
                for (int cb = 0; cb < D / 32; ++cb) {
                    uint32_t o[32];
                    tmem_ld32(lane_tm + C::COL_O + 32 * cb, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
                    tmem_st32(lane_tm + C::COL_O + 32 * cb, o);
                }
                tmem_wait_st();
            }
            // V rows past the context (last tile): zero them before the P V step reads the tile
            if (kv0 + BN > ctx) {
                ok = __all_sync(FULL, mbar_wait_bounded(&v_full[j % VST], (j / VST) & 1));
                if (!ok) {
                    failed = true;
                    break;
                }
                const int r0 = max(0, ctx - kv0);
                uint8_t *vt = smem + C::OFF_V + (j % VST) * C::KV_TILE;
                const int per_half = (BN - r0) * 8;
                for (int idx = t; idx < C::HALVES * per_half; idx += 128) {
                    const int hf = idx / per_half, rem = idx % per_half;
                    *reinterpret_cast<uint4 *>(vt + hf * C::KV_HALF + (r0 + rem / 8) * 128 + (rem % 8) * 16) =
                        make_uint4(0u, 0u, 0u, 0u);
                }
            }
            // P buffer j % 2 is free once P V_{j-2} has finished
            if (j >= 2) {
                ok = __all_sync(FULL, mbar_wait_bounded(&my_o_done[j & 1], ((j - 2) >> 1) & 1));
                if (!ok || *abort_flag) {
                    failed = true;
                    break;
                }
            }
            uint8_t *prow = smem + C::OFF_P + (2 * q + (j & 1)) * C::P_BYTES;
#pragma unroll
            for (int c = 0; c < 8; ++c)
                *reinterpret_cast<uint4 *>(prow + swz128(t, c)) =
                    make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
            fence_proxy_async_smem();
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&my_p_full[j & 1]);
        }
        if (!failed && nkv_q > 0) {
            const bool ok = __all_sync(FULL, mbar_wait_bounded(&my_o_done[(nkv_q - 1) & 1], ((nkv_q - 1) >> 1) & 1));
            failed = !ok || *abort_flag;
        }
        if (nkv_q > 0) {
            if (!failed) tc_fence_after_sync();
            // normalise and write this row
            const float inv = (!failed && l_run > 0.f) ? 1.f / l_run : __int_as_float(0x7fc00000);
            __nv_bfloat16 *orow = p.out + ((size_t)(q0 + (row_ok ? tok : 0)) * p.h_q + (size_t)kvh * G + t % G) * D;
#pragma unroll
            for (int cb = 0; cb < D / 32; ++cb) {
                uint32_t o[32];
                if (!failed) {
                    tmem_ld32(lane_tm + C::COL_O + 32 * cb, o);
                    tmem_wait_ld();
                }
                if (row_ok) {
                    uint32_t w[16];
#pragma unroll
                    for (int c = 0; c < 16; ++c)
                        w[c] = failed ? 0x7fc07fc0u
                                      : pack_bf16x2(__uint_as_float(o[2 * c]) * inv, __uint_as_float(o[2 * c + 1]) * inv);
#pragma unroll
                    for (int v = 0; v < 4; ++v)
                        reinterpret_cast<uint4 *>(orow + 32 * cb)[v] =
                            make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
                }
            }
        }
        tc_fence_before_sync();
    }
    __syncthreads();
    if (warp == C::MMA_WARP) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace pa
