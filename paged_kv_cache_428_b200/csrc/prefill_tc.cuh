// prefill_tc.cuh -- chunked-prefill attention over the paged bf16 KV cache on the
// 5th-generation tensor cores (tcgen05.mma, accumulators in tensor memory).
//
// Same computation and masking rules as paged_prefill_kernel (prefill.cuh).  One CTA per (pair
// of query tiles, KV head, sequence); a query tile is 128 rows = 128 / G tokens x the G heads of
// the KV head, and both tiles of a CTA share every K/V tile it streams.  Tensor memory per query
// tile (256 of the 512 columns): S [0,64) fp32, P0 / P1 [64,128) bf16 pairs, O [128,128+D) fp32.
// Roles:
//   warps 0-7  two softmax warpgroups, one per query tile: thread t of a warpgroup owns row t of
//              its tile (= tensor-memory lane t).  It loads its row of S_j from tensor memory
//              (which frees S for S_{j+1}), applies the causal / context mask, keeps the running
//              max and sum (log2 domain; a quarter of the exponentials by a polynomial on
//              the FMA pipe, beside the MUFU unit), stores its row of P_j (bf16) into tensor memory,
//              rescales its row of O when its max moved, and finally normalises O and writes the
//              output row.
//   warps 8-9  one MMA warp per query tile: lane 0 issues S_{j+1} = Q K_{j+1}^T (M 128, N 64,
//              K = D, both operands in shared memory) as soon as the softmax has loaded S_j, and
//              O += P_j V_j (M 128, N = D, K 64) with P read from tensor memory and V read N-major
//              from shared memory; tcgen05.commit signals each step.  With one issuing thread per
//              tile, one tile's barrier waits overlap the other tile's MMAs on the tensor core.
//              Warp 8 also allocates the 512 tensor-memory columns.
//   warps 10-11 K and V producers: 2-D TMA copies per physical block (the decode tensor maps,
//              128-byte swizzle), so the tiles are the MMA operands as they land.  Each warp
//              reads the block table 32 entries at a time, the next 32 in flight meanwhile, and
//              its lanes issue the copies of one tile.  K and V have rings of their own; a slot
//              is free when both query tiles have released it (their MMAs that read it finished,
//              or the tile's KV range ended before it).
// Q is copied into a swizzled shared tile once.  V rows past the context are zeroed in shared
// memory before the P V step (an unwritten NaN slot times a zero probability would poison O).
// Every wait is bounded and also ends when another role has stopped the CTA; on a timeout or a
// bad block the CTA records the error, stops, waits for its copies and MMAs in flight and frees
// its tensor memory; its rows come out NaN.
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

// Coefficients of the cubic that interpolates 2^f at the four Chebyshev nodes of [-1/2, 1/2]
// (relative error below 1.0e-4 there, i.e. under 2^-13, against the 2^-9 rounding of P to bf16).
#define PA_EX2_C0 0.999924541f
#define PA_EX2_C1 0.693136752f
#define PA_EX2_C2 0.242639482f
#define PA_EX2_C3 0.0558382832f

// 2^x for a pair, on the FMA pipe instead of the MUFU unit: Cody-Waite style range reduction
// x = n + f with n = round(x) (adding 1.5 * 2^23 leaves n in the low mantissa bits), f in
// [-1/2, 1/2]; 2^f by the cubic above; 2^n added to the exponent field.  x is clamped to -125
// first, so results below 2^-125 come out as about 2^-125 instead of 0 (x <= 8 here).
__device__ __forceinline__ float2 ex2_poly2(float2 x)
{
    constexpr float R = 12582912.f;                       // 1.5 * 2^23
    x.x = fmaxf(x.x, -125.f);
    x.y = fmaxf(x.y, -125.f);
    const float2 t = __fadd2_rn(x, make_float2(R, R));
    const float2 n = __fadd2_rn(t, make_float2(-R, -R));
    const float2 f = __ffma2_rn(n, make_float2(-1.f, -1.f), x);
    float2 c = __ffma2_rn(make_float2(PA_EX2_C3, PA_EX2_C3), f, make_float2(PA_EX2_C2, PA_EX2_C2));
    c = __ffma2_rn(c, f, make_float2(PA_EX2_C1, PA_EX2_C1));
    c = __ffma2_rn(c, f, make_float2(PA_EX2_C0, PA_EX2_C0));
    return make_float2(__int_as_float(__float_as_int(c.x) + (__float_as_int(t.x) << 23)),
                       __int_as_float(__float_as_int(c.y) + (__float_as_int(t.y) << 23)));
}

// As mbar_wait_bounded, but also gives up (false) as soon as *abort reads non-zero, so once one
// role of the CTA has stopped the others do not sit out the full limit in each of their waits.
__device__ __forceinline__ bool mbar_wait_or_abort(uint64_t *bar, uint32_t parity, const volatile int *abort)
{
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (*abort) return false;
        if (global_timer_ns() - t0 > kWaitLimitNs) return false;
    }
    return true;
}

// max(a, b, c) in one instruction
__device__ __forceinline__ float max3f(float a, float b, float c)
{
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

template <int D, int BS, int G, int NQ_ = 2, int KST_ = 4, int VST_ = 4>
struct PrefillTcConfig {
    static constexpr int NQ = NQ_;                        // 128-row query tiles per CTA
    static constexpr int THREADS = 128 * NQ + 32 * NQ + 64; // softmax warpgroups, one MMA warp per query tile, K and V TMA warps
    static constexpr int MMA_WARP = 4 * NQ, TMA_WARP = 5 * NQ;
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
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = NQ * Q_BYTES;
    static constexpr int OFF_V = OFF_K + KST * KV_TILE;
    static constexpr int OFF_BARS = OFF_V + VST * KV_TILE;
    static constexpr int NBARS = 2 * KST + 2 * VST + NQ * 8; // k, v full/empty; per tile s full, s free, p full x2, o done x2, drain, q full
    static constexpr int OFF_MISC = OFF_BARS + NBARS * 8; // tensor-memory base, abort flag
    static constexpr int SMEM = OFF_MISC + 16 + 1024;
    static constexpr int TMEM_PER_Q = 256;                // S [0,64), P0 [64,96), P1 [96,128), O [128, 128 + D)
    static constexpr int COL_P = 64;
    static constexpr int POLY_PAIRS = 2;                  // of every 8 pairs of P, on the FMA pipe
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

template <int D, int BS, int G, int NQ_ = 2, int KST_ = 4, int VST_ = 4>
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
    uint64_t *s_full = bars + 2 * KST + 2 * VST, *s_free = s_full + NQ, *p_full = s_free + NQ, *o_done = p_full + 2 * NQ;
    uint64_t *drain = o_done + 2 * NQ;                          // one per query tile
    uint64_t *q_full = drain + NQ;                              // one per query tile: Q in shared memory
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
            mbar_init(&k_empty[i], NQ);
        }
        for (int i = 0; i < VST; ++i) {
            mbar_init(&v_full[i], 1);
            mbar_init(&v_empty[i], NQ);
        }
        for (int q = 0; q < NQ; ++q) {
            mbar_init(&s_full[q], 1);
            mbar_init(&s_free[q], 4);
        }
        for (int b = 0; b < 2 * NQ; ++b) {
            mbar_init(&p_full[b], 4);
            mbar_init(&o_done[b], 1);
        }
        for (int q = 0; q < NQ; ++q) mbar_init(&drain[q], 1);
        for (int q = 0; q < NQ; ++q) mbar_init(&q_full[q], 128);
        *abort_flag = 0;
        mbar_init_fence();
    }
    if (warp == C::MMA_WARP) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == C::TMA_WARP || warp == C::TMA_WARP + 1) {
        // ------------------------------ TMA producers ------------------------------
        // one warp per operand: the warp reads the block table 32 entries at a time (the next
        // 32 are in flight meanwhile), lane 0 waits for the ring slot, and lane l issues the copy
        // of block l / HALVES, half l % HALVES of the tile
        const bool is_v = warp != C::TMA_WARP;
        const int nst = is_v ? VST : KST;
        uint64_t *full = is_v ? v_full : k_full;
        uint64_t *empty = is_v ? v_empty : k_empty;
        const CUtensorMap *map = is_v ? &tmap_v : &tmap_k;
        if (lane == 0) prefetch_tensormap(map);
        const uint64_t pol = l2_policy_evict_last();
        const int32_t *trow = p.block_tables + (size_t)seq * p.max_blocks_per_seq;
        constexpr int BPT = C::BLOCKS_PER_TILE, TPB = 32 / BPT;
        auto entry = [&](int lb) -> int {
            return (lb < nblk_seq && lb < p.max_blocks_per_seq) ? __ldg(trow + lb) : -1;
        };
        int cur = entry(lane), nxt = entry(32 + lane);
        const int k = lane / C::HALVES, hf = lane % C::HALVES;
        int issued = 0;                                        // tiles whose copies were issued
        for (int it = 0; it < nkv; ++it) {
            if (it > 0 && it % TPB == 0) {
                cur = nxt;
                nxt = entry((it / TPB + 1) * 32 + lane);
            }
            const int st = it % nst;
            int go = 1;
            if (lane == 0) {
                if (it >= nst && !mbar_wait_or_abort(&empty[st], ((it / nst) - 1) & 1, abort_flag)) {
                    if (!*abort_flag) record_error(PA_DEVERR_TIMEOUT);
                    *abort_flag = 1;
                }
                go = *abort_flag ? 0 : 1;
            }
            if (!__shfl_sync(FULL, go, 0)) break;
            const int nb = min(BPT, nblk_seq - it * BPT);
            const int phys = __shfl_sync(FULL, cur, (it % TPB) * BPT + min(k, BPT - 1));
            const bool mine = lane < nb * C::HALVES;
            if (__any_sync(FULL, mine && (phys < 0 || phys >= p.num_blocks))) {
                if (lane == 0) {
                    record_error(PA_DEVERR_BAD_BLOCK);
                    *abort_flag = 1;                           // the MMA warps' waits see it
                }
                break;
            }
            if (lane == 0) mbar_arrive_expect_tx(&full[st], (uint32_t)(nb * C::HALVES * BS * 128));
            __syncwarp();
            if (mine)
                tma_load_2d(smem + (is_v ? C::OFF_V : C::OFF_K) + st * C::KV_TILE + hf * C::KV_HALF + k * BS * 128, map,
                            hf * 64, (phys * p.h_kv + kvh) * BS, &full[st], pol);
            ++issued;
        }
        // Every copy this warp issued has landed before the CTA can exit, also when it stopped
        // early and nobody consumed the last tiles: wait (bounded) for each of the last nst
        // tiles.  The tile nst before each was consumed before the slot was refilled, so each
        // wait's phase is unambiguous; on the normal path these waits return at once.
        if (lane == 0)
            for (int i = max(0, issued - nst); i < issued; ++i) mbar_wait_bounded(&full[i % nst], (i / nst) & 1);
        __syncwarp();
    } else if (warp >= C::MMA_WARP && warp < C::MMA_WARP + NQ) {
        // ------------------------------ MMA issue, one warp per query tile ------------------------------
        // Lane 0 issues S_j = Q K_j^T and O += P_j V_j for its tile.  Every query tile releases
        // every K and V slot once per KV tile: a tile that reads the slot commits after its MMAs,
        // a tile whose range ended arrives as soon as the slot's data has landed (so the
        // arrival falls into that tile's phase of the empty barrier).
        const int q = warp - C::MMA_WARP;
        if (lane == 0) {
            const int nkq = nkv_of(q);
            const uint32_t d_s = tmem + q * C::TMEM_PER_Q, d_o = d_s + C::COL_O, d_p = d_s + C::COL_P;
            const uint64_t qdesc = umma_desc_sw128(smem_addr(smem + C::OFF_Q + q * C::Q_BYTES), 16, 1024);
            const uint64_t kdesc = umma_desc_sw128(smem_addr(smem + C::OFF_K), 16, 1024);
            const uint64_t vdesc = umma_desc_sw128(smem_addr(smem + C::OFF_V), C::KV_HALF, 1024);
            auto s_mma = [&](int j) -> bool {
                const int st = j % KST;
                if (!mbar_wait_or_abort(&k_full[st], (j / KST) & 1, abort_flag) || *abort_flag) return false;
                if (j >= 1 && (!mbar_wait_or_abort(&s_free[q], (j - 1) & 1, abort_flag) || *abort_flag)) return false;
                tc_fence_after_sync();
                const uint64_t kd = kdesc + (uint64_t)((st * C::KV_TILE) >> 4);
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks)
                    umma_bf16_ss(d_s, qdesc + (uint64_t)(((ks >> 2) * C::Q_HALF + (ks & 3) * 32) >> 4),
                                 kd + (uint64_t)(((ks >> 2) * C::KV_HALF + (ks & 3) * 32) >> 4), C::IDESC_S, ks > 0);
                umma_commit(&s_full[q]);
                umma_commit(&k_empty[st]);
                return true;
            };
            auto pv = [&](int i) -> bool {
                if (!mbar_wait_or_abort(&v_full[i % VST], (i / VST) & 1, abort_flag) || *abort_flag) return false;
                if (!mbar_wait_or_abort(&p_full[2 * q + (i & 1)], (i >> 1) & 1, abort_flag) || *abort_flag) return false;
                tc_fence_after_sync();
                const uint64_t vd = vdesc + (uint64_t)(((i % VST) * C::KV_TILE) >> 4);
                const uint32_t pt = d_p + 32 * (i & 1);
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk)
                    umma_bf16_ts(d_o, pt + 8 * kk, vd + (uint64_t)((kk * 2048) >> 4), C::IDESC_O, i > 0 || kk > 0);
                umma_commit(&o_done[2 * q + (i & 1)]);
                umma_commit(&v_empty[i % VST]);
                return true;
            };
            bool ok = true;
            if (nkq > 0) {
                // the tile's Q rows, written by its softmax warpgroup after the CTA barrier
                ok = mbar_wait_or_abort(&q_full[q], 0, abort_flag) && !*abort_flag;
                if (ok) ok = s_mma(0);
            }
            for (int j = 0; j < nkq && ok; ++j) {
                if (j + 1 < nkq) ok = s_mma(j + 1);
                if (ok) ok = pv(j);
            }
            // the KV tiles past this query tile's range: release their slots as they land
            for (int j = nkq; j < nkv && ok; ++j) {
                ok = mbar_wait_or_abort(&k_full[j % KST], (j / KST) & 1, abort_flag) && !*abort_flag;
                if (ok) mbar_arrive(&k_empty[j % KST]);
                ok = ok && mbar_wait_or_abort(&v_full[j % VST], (j / VST) & 1, abort_flag) && !*abort_flag;
                if (ok) mbar_arrive(&v_empty[j % VST]);
            }
            if (!ok) {
                if (!*abort_flag) record_error(PA_DEVERR_TIMEOUT);
                *abort_flag = 1;
            }
            umma_commit(&drain[q]);                             // every MMA this thread issued has finished
            mbar_wait_bounded(&drain[q], 0);
        }
        __syncwarp();
    } else {
        // ------------------------------ softmax warpgroups ------------------------------
        const int q = warp >> 2, t = threadIdx.x & 127;
        const int tok0 = tok0_of(q), nkv_q = nkv_of(q);
        const int tok = tok0 + t / G;
        const bool row_ok = tok < chunk;
        {
            // this thread's Q row into the tile's swizzled shared tile (row t = token t / G, head
            // t % G), after the CTA barrier so that the loads overlap the producers' first K/V
            // copies; the MMA warp waits for all 128 rows on q_full before the tile's first S
            const uint4 *src = reinterpret_cast<const uint4 *>(
                p.q + ((size_t)(q0 + (row_ok ? tok : 0)) * p.h_q + (size_t)kvh * G + t % G) * D);
            uint4 v[D / 8];
#pragma unroll
            for (int c = 0; c < D / 8; ++c) v[c] = row_ok ? src[c] : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int c = 0; c < D / 8; ++c)
                *reinterpret_cast<uint4 *>(smem + C::OFF_Q + q * C::Q_BYTES + (c >> 3) * C::Q_HALF + swz128(t, c & 7)) =
                    v[c];
            fence_proxy_async_smem();
            mbar_arrive(&q_full[q]);
        }
        const int pos = row_ok ? ctx - chunk + tok : 0;
        const int first_pos = ctx - chunk + tok0;
        const uint32_t lane_tm = tmem + q * C::TMEM_PER_Q + ((uint32_t)(32 * (warp & 3)) << 16);
        uint64_t *my_s_full = s_full + q, *my_s_free = s_free + q;
        uint64_t *my_p_full = p_full + 2 * q, *my_o_done = o_done + 2 * q;
        float m_run = -INFINITY, l_run = 0.f;
        bool failed = false;
        for (int j = 0; j < nkv_q; ++j) {
            bool ok = __all_sync(FULL, mbar_wait_or_abort(my_s_full, j & 1, abort_flag));
            if (!ok || *abort_flag) {
                failed = true;
                break;
            }
            tc_fence_after_sync();
            uint32_t sr[2][32];
            tmem_ld32(lane_tm, sr[0]);
            tmem_ld32(lane_tm + 32u, sr[1]);
            tmem_wait_ld();
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(my_s_free);

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
            // pair i of the row tile = columns 2i, 2i + 1
            auto pair_of = [&](int i) {
                return make_float2(__uint_as_float(sr[i >> 4][2 * (i & 15)]), __uint_as_float(sr[i >> 4][2 * (i & 15) + 1]));
            };
            float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const float2 s2 = pair_of(i);
                m4[i & 3] = max3f(m4[i & 3], s2.x, s2.y);
            }
            const float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
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
            // p = 2^(s * qk_scale - m) in pairs: one packed FMA, then the MUFU unit for most pairs
            // and the FMA-pipe polynomial for POLY_PAIRS of every 8 (the two units run side by
            // side); the row sum in two packed partial sums
            uint32_t pk[32];
            const float2 sc2 = make_float2(p.qk_scale, p.qk_scale), nm2 = make_float2(-mn, -mn);
            float2 rsa = make_float2(0.f, 0.f), rsb = make_float2(0.f, 0.f);
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const float2 x2 = __ffma2_rn(pair_of(i), sc2, nm2);
                const float2 e2 = (i & 7) < C::POLY_PAIRS ? ex2_poly2(x2) : make_float2(ex2_approx(x2.x), ex2_approx(x2.y));
                if (i & 1) rsb = __fadd2_rn(rsb, e2);
                else rsa = __fadd2_rn(rsa, e2);
                pk[i] = pack_bf16x2(e2.x, e2.y);
            }
            const float rs = (rsa.x + rsb.x) + (rsa.y + rsb.y);
            l_run = l_run * alpha + rs;
            // rescale this warp's rows of O when any of their maxima moved (PV_{j-1} must be done)
            if (__any_sync(FULL, moved)) {
                ok = __all_sync(FULL, mbar_wait_or_abort(&my_o_done[(j - 1) & 1], ((j - 1) >> 1) & 1, abort_flag));
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
                ok = __all_sync(FULL, mbar_wait_or_abort(&v_full[j % VST], (j / VST) & 1, abort_flag));
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
                fence_proxy_async_smem();
            }
            // P buffer j % 2 is free once P V_{j-2} has finished
            if (j >= 2) {
                ok = __all_sync(FULL, mbar_wait_or_abort(&my_o_done[j & 1], ((j - 2) >> 1) & 1, abort_flag));
                if (!ok || *abort_flag) {
                    failed = true;
                    break;
                }
            }
            tmem_st32(lane_tm + (uint32_t)(C::COL_P + 32 * (j & 1)), pk);
            tmem_wait_st();
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&my_p_full[j & 1]);
        }
        if (!failed && nkv_q > 0) {
            const bool ok = __all_sync(FULL, mbar_wait_or_abort(&my_o_done[(nkv_q - 1) & 1], ((nkv_q - 1) >> 1) & 1, abort_flag));
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
