// prefill_tc.cuh -- chunked-prefill attention over the paged bf16 KV cache on the
// 5th-generation tensor cores (tcgen05.mma, accumulators in tensor memory).
//
// Same computation and masking rules as paged_prefill_kernel (prefill.cuh).  A work item is
// (pair of query tiles, KV head, sequence); a query tile is 128 rows = 128 / G tokens x the G
// heads of the KV head, and both tiles of an item share every K/V tile it streams.  Tensor
// memory per query tile (256 of the 512 columns): S [0,64) fp32, P [64,96) bf16 pairs, Q dims
// 0-63 [96,128) bf16 pairs, O [128,128+D) fp32.
//
// Scheduling.  With a claim counter (pa_prefill_ws) the grid is one CTA per SM and every CTA
// claims items one after another from a global atomic counter, sequences in order of context
// length, longest first, and within a sequence pair by pair (longest KV range first), each pair
// for every KV head: the items of a sequence run at about the same time, so they share their
// K/V tiles through L2, and the last items claimed are the shortest.  Without one (pa_prefill) the
// grid has one CTA per item.  In both cases the next item is known before the current one ends:
// the producers start its block-table reads and K/V copies while the current item's last tiles
// are in use, and the softmax warps start copying its Q rows once the current item's P V products
// are done, so an item costs its KV tiles plus an epilogue instead of a chain of dependent loads.
//
// Roles:
//   warps 0-7  two softmax warpgroups, one per query tile: thread t of a warpgroup owns row t of
//              its tile (= tensor-memory lane t).  It loads its row of S_j from tensor memory
//              (which frees S for S_{j+1}), applies the causal / context mask, keeps the running
//              max and sum (log2 domain; the exponentials on the MUFU unit, with a polynomial on
//              the FMA pipe for POLY_PAIRS of every 8 pairs, 0 as measured best), stores its row
//              of P_j (bf16) into tensor memory,
//              rescales its row of O when its max moved, and at the end of the item normalises O
//              and writes the output row.  A query tile wholly inside its chunk arrives in the
//              swizzled Q tile by one TMA load from the K producer; otherwise each thread copies
//              its Q row (cp.async, zero-filled past the chunk), starting before the epilogue
//              when the next item is published already.  Either way the thread then puts the
//              row's first 64 dims into tensor memory and arrives on the tile's q_full.  P has one
//              buffer: P_j is stored once P V_{j-1} has finished (seen on o_done).
//   warps 8-9  one MMA warp per query tile: lane 0 issues S_{j+1} = Q K_{j+1}^T (M 128, N 64,
//              K = D; K from shared memory, Q dims 0-63 from tensor memory and the rest from
//              shared memory, which leaves the N = 64 products less bound by shared-memory
//              operand reads) as soon as the softmax has loaded S_j, and
//              O += P_j V_j (M 128, N = D, K 64) with P read from tensor memory and V read N-major
//              from shared memory; tcgen05.commit signals each step.  With one issuing thread per
//              tile, one tile's barrier waits overlap the other tile's MMAs on the tensor core.
//              Warp 8 also allocates the 512 tensor-memory columns, once per CTA.
//   warps 10-11 K and V producers: 2-D TMA copies per physical block (the decode tensor maps,
//              128-byte swizzle), so the tiles are the MMA operands as they land.  Each warp
//              reads the block table 32 entries at a time, the next 32 in flight meanwhile, and
//              its lanes issue the copies of one tile.  K and V have rings of their own, indexed
//              across items; a slot is free when both query tiles have released it (their MMAs
//              that read it finished, or the tile's KV range ended before it).  V rows past the
//              context in an item's last tile are zeroed by the V producer once the copy has
//              landed and before the tile is marked full (an unwritten NaN slot times a zero
//              probability would poison O).  The K warp also claims the work items and
//              publishes each through a two-entry ring in shared memory that every other warp
//              reads; it claims the next item once the current one's last K tile is issued.  At
//              the start of an item it loads the item's whole query tiles (3-D TMA of q, one box
//              per tile) once both tiles have released the previous item's last K tile, i.e. once
//              every S product that read the Q tiles has finished.
// Every wait on the data path is bounded and also ends when another role has stopped the CTA; on
// a timeout or a bad block the CTA records the error, stops claiming, writes NaN into the rows
// of the items it holds, waits for its copies and MMAs in flight and frees its tensor memory.
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


// 16-byte cp.async into shared memory; zero-fill instead of reading when !ok.
__device__ __forceinline__ void cp_async_16_zfill(void *dst, const void *src, bool ok)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_addr(dst)), "l"(src), "r"(ok ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// 3-D tiled TMA load global -> shared (no multicast), completing on an mbarrier.
__device__ __forceinline__ void tma_load_3d(void *dst, const void *tmap, int x, int y, int z, uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(z), "r"(smem_addr(bar))
        : "memory");
}

// Non-blocking test of an mbarrier phase (test_wait never suspends the thread).
__device__ __forceinline__ bool mbar_test_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

// Sequence tables (query_start, context_lens) and the claim order are kept in shared memory for
// up to this many sequences; beyond it the K producer reads them from global memory and claims in
// sequence order.
constexpr int kPrefillSeqsInSmem = 1024;

// Work distribution of one launch.
struct PrefillSched {
    int *counters;      // device [2]: next item to claim, CTAs finished (zero between launches);
                        // nullptr: one CTA per item, item = blockIdx
    int num_seqs;
    int pairs_max;      // query-tile pairs of the longest chunk = items per (sequence, KV head)
    int total_items;    // num_seqs * h_kv * pairs_max
    int q_tma;          // the Q tensor map is valid: query tiles inside their chunk come by TMA
};

template <int D, int BS, int G, int NQ_ = 2, int KST_ = 4, int VST_ = 4>
struct PrefillTcConfig {
    static constexpr int NQ = NQ_;                        // 128-row query tiles per item
    // softmax warpgroups, one MMA warp per query tile, K and V TMA warps (the K warp also claims
    // and publishes the work items)
    static constexpr int THREADS = 128 * NQ + 32 * NQ + 64;
    static constexpr int MMA_WARP = 4 * NQ, TMA_WARP = 5 * NQ;
    static constexpr int ITEM_READERS = 4 * NQ + NQ + 1;  // warps that read each published item
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
    // k, v full/empty; per tile: s full, s free, p full x2, o done x2, drain, q full; item ring
    // full x2 / empty x2; the V tail copy; per tile: Q landed (TMA)
    static constexpr int NBARS = 2 * KST + 2 * VST + NQ * 9 + 5;
    static constexpr int OFF_ITEMS = OFF_BARS + NBARS * 8;   // item ring: 2 x 8 ints
    static constexpr int OFF_MISC = OFF_ITEMS + 64;       // tensor-memory base, abort flag
    static constexpr int OFF_SEQ = OFF_MISC + 16;         // query_start, context_lens, claim order
    static constexpr int SMEM = OFF_SEQ + (3 * kPrefillSeqsInSmem + 1) * 4 + 1024;
    static constexpr int TMEM_PER_Q = 256;                // S [0,64), P [64,96), Q dims 0-63 [96,128), O [128, 128 + D)
    static constexpr int COL_P = 64;
    static constexpr int COL_QT = 96;
    static constexpr int POLY_PAIRS = 0;                  // of every 8 pairs of P, on the FMA pipe
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

// Item layout in the ring: seq (< 0: no more items), KV head, pair, first query row, chunk
// length, context length, KV tiles of query tile 0 and of query tile 1.
enum { IT_SEQ, IT_KVH, IT_PAIR, IT_Q0, IT_CHUNK, IT_CTX, IT_NKV0, IT_NKV1, IT_N };

template <int D, int BS, int G, int NQ_ = 2, int KST_ = 4, int VST_ = 4>
__global__ void __launch_bounds__(PrefillTcConfig<D, BS, G, NQ_, KST_, VST_>::THREADS, 1)
    paged_prefill_tc_kernel(const PrefillParams p, const PrefillSched sc, const __grid_constant__ CUtensorMap tmap_k,
                            const __grid_constant__ CUtensorMap tmap_v, const __grid_constant__ CUtensorMap tmap_q)
{
    using C = PrefillTcConfig<D, BS, G, NQ_, KST_, VST_>;
    constexpr int KST = C::KST, VST = C::VST, BN = C::BN, NQ = C::NQ;
    constexpr unsigned FULL = 0xffffffffu;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BARS);
    uint64_t *k_full = bars, *k_empty = bars + KST, *v_full = bars + 2 * KST, *v_empty = v_full + VST;
    // p_full / o_done: two per query tile q, used by alternate steps g (index 2 q + g % 2), so a
    // parity wait never meets a barrier more than one phase ahead
    uint64_t *s_full = bars + 2 * KST + 2 * VST, *s_free = s_full + NQ, *p_full = s_free + NQ, *o_done = p_full + 2 * NQ;
    uint64_t *drain = o_done + 2 * NQ;                          // one per query tile
    uint64_t *q_full = drain + NQ;                              // one per query tile: Q copied
    uint64_t *item_full = q_full + NQ, *item_empty = item_full + 2, *v_tail = item_empty + 2;
    uint64_t *q_land = v_tail + 1;                               // one per query tile: its Q tile landed (TMA)
    volatile int *items = reinterpret_cast<volatile int *>(smem + C::OFF_ITEMS);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);
    int *seq_qs = reinterpret_cast<int *>(smem + C::OFF_SEQ);
    int *seq_ctx = seq_qs + kPrefillSeqsInSmem + 1, *seq_order = seq_ctx + kPrefillSeqsInSmem;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bool claiming = sc.counters != nullptr;
    const bool tables = claiming && sc.num_seqs <= kPrefillSeqsInSmem;

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
            mbar_init(&drain[q], 1);
            mbar_init(&q_full[q], 4);
        }
        for (int b = 0; b < 2 * NQ; ++b) {
            mbar_init(&p_full[b], 4);
            mbar_init(&o_done[b], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&item_full[s], 1);
            mbar_init(&item_empty[s], C::ITEM_READERS);
        }
        mbar_init(v_tail, 1);
        for (int q = 0; q < NQ; ++q) mbar_init(&q_land[q], 1);
        *abort_flag = 0;
        mbar_init_fence();
    }
    if (warp == C::MMA_WARP) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    if (tables)
        for (int i = threadIdx.x; i <= sc.num_seqs; i += C::THREADS) {
            seq_qs[i] = __ldg(p.query_start + i);
            if (i < sc.num_seqs) seq_ctx[i] = __ldg(p.context_lens + i);
        }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    if (tables) {
        // claim order: sequences by context length, longest first (ties by index)
        for (int s = threadIdx.x; s < sc.num_seqs; s += C::THREADS) {
            const int c = seq_ctx[s];
            int r = 0;
            for (int u = 0; u < sc.num_seqs; ++u) {
                const int cu = seq_ctx[u];
                r += (cu > c) || (cu == c && u < s);
            }
            seq_order[r] = s;
        }
        __syncthreads();
    }

    // the n-th published item of this CTA, read by a whole warp; every reading warp arrives once
    auto read_item = [&](int n, int (&it)[IT_N]) {
        const int slot = n & 1;
        const bool ok = mbar_wait_bounded(&item_full[slot], (n >> 1) & 1);
#pragma unroll
        for (int i = 0; i < IT_N; ++i) it[i] = items[slot * IT_N + i];
        if (!ok) {
            it[IT_SEQ] = -1;                                   // no item came: stop
            if (lane == 0) {
                record_error(PA_DEVERR_TIMEOUT);
                *abort_flag = 1;
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&item_empty[slot]);
    };
    // query tile q of a pair lies wholly inside the chunk: its Q tile comes by one TMA load
    auto q_by_tma = [&](int pair, int chunk, int q) { return sc.q_tma && (pair * NQ + q + 1) * C::TQ <= chunk; };
    auto nkv_tile = [&](int chunk, int ctx, int pair, int q) {
        const int t0 = (pair * NQ + q) * C::TQ;
        return t0 >= chunk ? 0 : ceil_div(ctx - chunk + min(chunk, t0 + C::TQ), BN);
    };


    if (warp == C::TMA_WARP || warp == C::TMA_WARP + 1) {
        // ------------------------------ TMA producers ------------------------------
        // one warp per operand: the warp reads the block table 32 entries at a time (the next
        // 32 are in flight meanwhile), lane 0 waits for the ring slot, and lane l issues the copy
        // of block l / HALVES, half l % HALVES of the tile.  The K warp also claims the work
        // items and publishes them through the two-entry ring; it claims the next item once it
        // has issued the current item's last K tile: the ring then still holds about KST tiles
        // of the current item, which hides the claim and the next item's first table reads, and
        // a CTA deep in a long item does not hold on to an item that an idle CTA could run.
        const bool is_v = warp != C::TMA_WARP;
        const int nst = is_v ? VST : KST;
        uint64_t *full = is_v ? v_full : k_full;
        uint64_t *empty = is_v ? v_empty : k_empty;
        const CUtensorMap *map = is_v ? &tmap_v : &tmap_k;
        if (lane == 0) prefetch_tensormap(map);
        const uint64_t pol = l2_policy_evict_last();
        constexpr int BPT = C::BLOCKS_PER_TILE, TPB = 32 / BPT;
        const int k = lane / C::HALVES, hf = lane % C::HALVES;
        int issued = 0, ntail = 0;                             // tiles whose copies were issued (all items)

        // ---- claiming and publishing (K warp) ----
        int published = 0;
        bool more = true;                                      // lane 0: claims may continue
        auto seq_q0 = [&](int s) { return tables ? seq_qs[s] : __ldg(p.query_start + s); };
        auto seq_cx = [&](int s) { return tables ? seq_ctx[s] : __ldg(p.context_lens + s); };
        // the next item with work, or the end (lane 0 claims, the warp gets it)
        auto claim = [&](int (&it)[IT_N]) {
#pragma unroll
            for (int i = 0; i < IT_N; ++i) it[i] = -1;
            if (lane == 0) {
                while (more) {
                    int x, kvh, zi;
                    if (claiming) {
                        if (*abort_flag) {
                            more = false;
                            break;
                        }
                        const int kk = atomicAdd(sc.counters, 1);
                        if (kk >= sc.total_items) {
                            more = false;
                            break;
                        }
                        // within a sequence pair-major (every KV head's pair x, then pair x + 1):
                        // the last items claimed are the shortest pairs of all heads
                        kvh = kk % p.h_kv;
                        x = (kk / p.h_kv) % sc.pairs_max;
                        zi = kk / (p.h_kv * sc.pairs_max);
                    } else {
                        x = blockIdx.x;
                        kvh = blockIdx.y;
                        zi = blockIdx.z;
                        more = false;                          // one item per CTA
                    }
                    const int seq = tables ? seq_order[zi] : zi;
                    const int q0 = seq_q0(seq), chunk = seq_q0(seq + 1) - q0, ctx = seq_cx(seq);
                    if (chunk > ctx) {                         // rows left unwritten, flagged
                        if (x == 0 && kvh == 0) record_error(PA_DEVERR_BAD_CHUNK);
                        continue;
                    }
                    const int pair = ceil_div(prefill_tiles<C::TQ>(chunk), NQ) - 1 - x;   // x = 0: longest KV range
                    if (pair < 0 || chunk <= 0) continue;
                    it[IT_SEQ] = seq;
                    it[IT_KVH] = kvh;
                    it[IT_PAIR] = pair;
                    it[IT_Q0] = q0;
                    it[IT_CHUNK] = chunk;
                    it[IT_CTX] = ctx;
                    it[IT_NKV0] = nkv_tile(chunk, ctx, pair, 0);
                    it[IT_NKV1] = NQ > 1 ? nkv_tile(chunk, ctx, pair, 1) : 0;
                    break;
                }
            }
#pragma unroll
            for (int i = 0; i < IT_N; ++i) it[i] = __shfl_sync(FULL, it[i], 0);
        };
        auto publish = [&](const int (&it)[IT_N]) {
            const int slot = published & 1;
            if (lane == 0) {
                // the slot's previous item has been read by every reader (bounded; on a timeout
                // the CTA is stopped and the item is written all the same, so readers see the end)
                if (published >= 2 && !mbar_wait_bounded(&item_empty[slot], ((published >> 1) - 1) & 1)) {
                    record_error(PA_DEVERR_TIMEOUT);
                    *abort_flag = 1;
                }
#pragma unroll
                for (int i = 0; i < IT_N; ++i) items[slot * IT_N + i] = it[i];
                mbar_arrive(&item_full[slot]);
            }
            __syncwarp();
            ++published;
        };

        int cur[IT_N], nxt[IT_N];
        if (!is_v) {
            claim(cur);
            publish(cur);
        } else {
            read_item(0, cur);
        }
        int q_tma_n[NQ];                                       // K warp, lane 0: Q tiles loaded by TMA
#pragma unroll
        for (int qq = 0; qq < NQ; ++qq) q_tma_n[qq] = 0;
        for (int n = 0; cur[IT_SEQ] >= 0; ++n) {
            const int ctx = cur[IT_CTX], nkv = max(cur[IT_NKV0], cur[IT_NKV1]);
            const int nblk_seq = ceil_div(ctx, BS);
            if (!is_v && sc.q_tma && lane == 0) {
                // the item's query tiles that lie inside the chunk: one TMA load each into the Q
                // tile, once every S product of the previous item has finished (the release of its
                // last K tile by both query tiles says so)
                if (issued > 0 && !*abort_flag) {
                    const int gl = issued - 1;
                    if (!mbar_wait_or_abort(&empty[gl % nst], (gl / nst) & 1, abort_flag)) {
                        if (!*abort_flag) record_error(PA_DEVERR_TIMEOUT);
                        *abort_flag = 1;
                    }
                }
#pragma unroll
                for (int qq = 0; qq < NQ; ++qq) {
                    if ((qq == 0 ? cur[IT_NKV0] : cur[IT_NKV1]) > 0 && q_by_tma(cur[IT_PAIR], cur[IT_CHUNK], qq) &&
                        !*abort_flag) {
                        uint8_t *dst = smem + C::OFF_Q + qq * C::Q_BYTES;
                        mbar_arrive_expect_tx(&q_land[qq], (uint32_t)C::Q_BYTES);
#pragma unroll
                        for (int h = 0; h < C::HALVES; ++h)
                            tma_load_3d(dst + h * C::Q_HALF, &tmap_q, 64 * h, cur[IT_KVH] * G,
                                        cur[IT_Q0] + (cur[IT_PAIR] * NQ + qq) * C::TQ, &q_land[qq]);
                        ++q_tma_n[qq];
                    }
                }
            }
            __syncwarp();
            const int32_t *trow = p.block_tables + (size_t)cur[IT_SEQ] * p.max_blocks_per_seq;
            auto entry = [&](int lb) -> int {
                return (lb < nblk_seq && lb < p.max_blocks_per_seq) ? __ldg(trow + lb) : -1;
            };
            int ecur = entry(lane), enxt = entry(32 + lane);
            const int row_kvh = cur[IT_KVH];
            bool next_known = is_v;                            // K warp: next item claimed and published
            for (int t = 0; t < nkv; ++t) {
                if (t > 0 && t % TPB == 0) {
                    ecur = enxt;
                    enxt = entry((t / TPB + 1) * 32 + lane);
                }
                const int st = issued % nst;
                int go = 1;
                if (lane == 0) {
                    if (issued >= nst && !mbar_wait_or_abort(&empty[st], ((issued / nst) - 1) & 1, abort_flag)) {
                        if (!*abort_flag) record_error(PA_DEVERR_TIMEOUT);
                        *abort_flag = 1;
                    }
                    go = *abort_flag ? 0 : 1;
                }
                if (!__shfl_sync(FULL, go, 0)) break;
                const int nb = min(BPT, nblk_seq - t * BPT);
                const int phys = __shfl_sync(FULL, ecur, (t % TPB) * BPT + min(k, BPT - 1));
                const bool mine = lane < nb * C::HALVES;
                if (__any_sync(FULL, mine && (phys < 0 || phys >= p.num_blocks))) {
                    if (lane == 0) {
                        record_error(PA_DEVERR_BAD_BLOCK);
                        *abort_flag = 1;                       // the other roles' waits see it
                    }
                    break;
                }
                // V tile holding rows past the context: the copy lands on v_tail, the rows past
                // the context are zeroed, and only then is the tile marked full
                const bool tail = is_v && (t + 1) * BN > ctx;
                uint64_t *bar = tail ? v_tail : &full[st];
                uint8_t *dst = smem + (is_v ? C::OFF_V : C::OFF_K) + st * C::KV_TILE;
                if (lane == 0) mbar_arrive_expect_tx(bar, (uint32_t)(nb * C::HALVES * BS * 128));
                __syncwarp();
                if (mine)
                    tma_load_2d(dst + hf * C::KV_HALF + k * BS * 128, map, hf * 64, (phys * p.h_kv + row_kvh) * BS, bar, pol);
                ++issued;
                if (tail) {
                    // our own copy: wait for it whatever the abort flag says (bounded)
                    const int landed = __shfl_sync(FULL, lane == 0 ? (int)mbar_wait_bounded(v_tail, ntail & 1) : 0, 0);
                    ++ntail;
                    if (landed) {
                        const int r0 = ctx - t * BN, per_half = (BN - r0) * 8;
                        for (int idx = lane; idx < C::HALVES * per_half; idx += 32) {
                            const int h = idx / per_half, rem = idx % per_half;
                            *reinterpret_cast<uint4 *>(dst + h * C::KV_HALF + (r0 + rem / 8) * 128 + (rem % 8) * 16) =
                                make_uint4(0u, 0u, 0u, 0u);
                        }
                        fence_proxy_async_smem();
                    } else if (lane == 0) {
                        record_error(PA_DEVERR_TIMEOUT);
                        *abort_flag = 1;
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&full[st]);     // completes the phase (no bytes expected)
                }
                if (!next_known && t == nkv - 1) {
                    claim(nxt);
                    publish(nxt);
                    next_known = true;
                }
            }
            if (!next_known) {                                 // stopped early: publish the end
                claim(nxt);
                publish(nxt);
            }
            if (is_v) read_item(n + 1, nxt);
#pragma unroll
            for (int i = 0; i < IT_N; ++i) cur[i] = nxt[i];
        }
        // Every copy this warp issued has landed before the CTA can exit, also when it stopped
        // early and nobody consumed the last tiles: wait (bounded) for each of the last nst
        // tiles.  The tile nst before each was consumed before the slot was refilled, so each
        // wait's phase is unambiguous; on the normal path these waits return at once.
        if (lane == 0) {
            for (int i = max(0, issued - nst); i < issued; ++i) mbar_wait_bounded(&full[i % nst], (i / nst) & 1);
#pragma unroll
            for (int qq = 0; qq < NQ; ++qq)                        // and every Q tile it loaded
                if (!is_v && q_tma_n[qq] > 0) mbar_wait_bounded(&q_land[qq], (q_tma_n[qq] - 1) & 1);
        }
        __syncwarp();
    } else if (warp >= C::MMA_WARP && warp < C::MMA_WARP + NQ) {
        // ------------------------------ MMA issue, one warp per query tile ------------------------------
        // Lane 0 issues S_j = Q K_j^T and O += P_j V_j for its tile.  Every query tile releases
        // every K and V slot once per KV tile: a tile that reads the slot commits after its MMAs,
        // a tile whose range ended arrives as soon as the slot's data has landed (so the
        // arrival falls into that tile's phase of the empty barrier).  Ring slots and the S / P
        // / O barriers are counted across items (gk: KV tiles so far, gs: this tile's steps so far).
        const int q = warp - C::MMA_WARP;
        const uint32_t d_s = tmem + q * C::TMEM_PER_Q, d_o = d_s + C::COL_O, d_p = d_s + C::COL_P,
                       d_qt = d_s + C::COL_QT;
        const uint64_t qdesc = umma_desc_sw128(smem_addr(smem + C::OFF_Q + q * C::Q_BYTES), 16, 1024);
        const uint64_t kdesc = umma_desc_sw128(smem_addr(smem + C::OFF_K), 16, 1024);
        const uint64_t vdesc = umma_desc_sw128(smem_addr(smem + C::OFF_V), C::KV_HALF, 1024);
        int gk = 0, gs = 0, nq = 0;                            // nq: items with work for this tile so far
        bool ok = true;
        for (int n = 0;; ++n) {
            int it[IT_N];
            read_item(n, it);
            if (it[IT_SEQ] < 0) break;
            if (lane == 0) {
                const int nkq = (q == 0 ? it[IT_NKV0] : it[IT_NKV1]), nkv = max(it[IT_NKV0], it[IT_NKV1]);
                auto s_mma = [&](int j) -> bool {
                    const int gt = gk + j, st = gt % KST, gj = gs + j;
                    if (!mbar_wait_or_abort(&k_full[st], (gt / KST) & 1, abort_flag) || *abort_flag) return false;
                    if (gj >= 1 && (!mbar_wait_or_abort(&s_free[q], (gj - 1) & 1, abort_flag) || *abort_flag)) return false;
                    tc_fence_after_sync();
                    const uint64_t kd = kdesc + (uint64_t)((st * C::KV_TILE) >> 4);
#pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks) {
                        const uint64_t kb = kd + (uint64_t)(((ks >> 2) * C::KV_HALF + (ks & 3) * 32) >> 4);
                        if (ks < 4)         // dims 0-63 of Q from tensor memory: only K is read from shared memory
                            umma_bf16_ts(d_s, d_qt + 8 * ks, kb, C::IDESC_S, ks > 0);
                        else
                            umma_bf16_ss(d_s, qdesc + (uint64_t)(((ks >> 2) * C::Q_HALF + (ks & 3) * 32) >> 4), kb,
                                         C::IDESC_S, ks > 0);
                    }
                    umma_commit(&s_full[q]);
                    umma_commit(&k_empty[st]);
                    return true;
                };
                auto pv = [&](int i) -> bool {
                    const int gt = gk + i, gi = gs + i;
                    if (!mbar_wait_or_abort(&v_full[gt % VST], (gt / VST) & 1, abort_flag) || *abort_flag) return false;
                    if (!mbar_wait_or_abort(&p_full[2 * q + (gi & 1)], (gi >> 1) & 1, abort_flag) || *abort_flag) return false;
                    tc_fence_after_sync();
                    const uint64_t vd = vdesc + (uint64_t)(((gt % VST) * C::KV_TILE) >> 4);
                    const uint32_t pt = d_p;
#pragma unroll
                    for (int kk = 0; kk < BN / 16; ++kk)
                        umma_bf16_ts(d_o, pt + 8 * kk, vd + (uint64_t)((kk * 2048) >> 4), C::IDESC_O, i > 0 || kk > 0);
                    umma_commit(&o_done[2 * q + (gi & 1)]);
                    umma_commit(&v_empty[gt % VST]);
                    return true;
                };
                // the item's Q tile, copied by the tile's softmax warps.  Only items with work for
                // the tile use the barrier, on both sides: the softmax cannot finish such an item
                // before its S products, so it never runs a phase ahead of this wait
                if (nkq > 0) {
                    if (ok) ok = mbar_wait_or_abort(&q_full[q], nq & 1, abort_flag) && !*abort_flag;
                    ++nq;
                    if (ok) ok = s_mma(0);
                }
                for (int j = 0; j < nkq && ok; ++j) {
                    if (j + 1 < nkq) ok = s_mma(j + 1);
                    if (ok) ok = pv(j);
                }
                // the KV tiles past this query tile's range: release their slots as they land
                for (int j = nkq; j < nkv && ok; ++j) {
                    const int gt = gk + j;
                    ok = mbar_wait_or_abort(&k_full[gt % KST], (gt / KST) & 1, abort_flag) && !*abort_flag;
                    if (ok) mbar_arrive(&k_empty[gt % KST]);
                    ok = ok && mbar_wait_or_abort(&v_full[gt % VST], (gt / VST) & 1, abort_flag) && !*abort_flag;
                    if (ok) mbar_arrive(&v_empty[gt % VST]);
                }
                if (!ok) {
                    if (!*abort_flag) record_error(PA_DEVERR_TIMEOUT);
                    *abort_flag = 1;
                }
                gk += nkv;
                gs += nkq;
            }
            __syncwarp();
        }
        if (lane == 0) {
            umma_commit(&drain[q]);                             // every MMA this thread issued has finished
            mbar_wait_bounded(&drain[q], 0);
        }
        __syncwarp();
    } else {
        // ------------------------------ softmax warpgroups ------------------------------
        const int q = warp >> 2, t = threadIdx.x & 127;
        const uint32_t lane_tm = tmem + q * C::TMEM_PER_Q + ((uint32_t)(32 * (warp & 3)) << 16);
        uint64_t *my_s_full = s_full + q, *my_s_free = s_free + q;
        uint64_t *my_p_full = p_full + 2 * q, *my_o_done = o_done + 2 * q;
        // this thread's Q row of the tile into its swizzled shared tile (row t = token t / G, head
        // t % G), zero-filled past the chunk; cp.async, completed by q_ready
        auto copy_q = [&](int pair, int q0, int chunk, int kvh) {
            const int tq = (pair * NQ + q) * C::TQ + t / G;
            const bool ok = tq < chunk;
            const __nv_bfloat16 *src = p.q + ((size_t)(q0 + (ok ? tq : 0)) * p.h_q + (size_t)kvh * G + t % G) * D;
            uint8_t *qt = smem + C::OFF_Q + q * C::Q_BYTES;
#pragma unroll
            for (int c = 0; c < D / 8; ++c) cp_async_16_zfill(qt + (c >> 3) * C::Q_HALF + swz128(t, c & 7), src + 8 * c, ok);
        };
        int nqt = 0;                                           // Q tiles of this query tile that came by TMA
        // the row's first 64 dims into tensor memory, then q_full: once all four warps arrive the
        // MMA warp may read the tile
        auto q_to_tmem = [&]() {
            {
                // dims 0-63 of this row also into tensor memory (lane t, two dims per column), the
                // A operand of the first four k-steps of S
                const uint8_t *qt = smem + C::OFF_Q + q * C::Q_BYTES;
#pragma unroll 1
                for (int c = 0; c < 8; c += 2) {
                    const uint4 a = *reinterpret_cast<const uint4 *>(qt + swz128(t, c));
                    const uint4 b = *reinterpret_cast<const uint4 *>(qt + swz128(t, c + 1));
                    const uint32_t r[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
                    tmem_st8(lane_tm + (uint32_t)(C::COL_QT + 4 * c), r);
                }
                tmem_wait_st();
            }
            fence_proxy_async_smem();
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&q_full[q]);
        };
        // this thread's copies landed
        auto q_ready = [&]() {
            cp_async_wait_all();
            q_to_tmem();
        };
        // the tile's TMA load landed (bounded; a stopped CTA goes on with NaN rows)
        auto q_ready_tma = [&]() {
            if (!__all_sync(FULL, mbar_wait_or_abort(&q_land[q], nqt & 1, abort_flag)) && lane == 0) {
                if (!*abort_flag) record_error(PA_DEVERR_TIMEOUT);
                *abort_flag = 1;
            }
            ++nqt;
            q_to_tmem();
        };
        int gs = 0;                                            // this tile's steps so far (all items)
        bool q_copying = false;                                // the next item's Q copy is in flight
        bool q_announced = false;                              // ... and already announced on q_full
        for (int n = 0;; ++n) {
            int it[IT_N];
            read_item(n, it);
            if (it[IT_SEQ] < 0) break;
            const int chunk = it[IT_CHUNK], ctx = it[IT_CTX], nkv_q = (q == 0 ? it[IT_NKV0] : it[IT_NKV1]);
            if (nkv_q > 0 && !q_announced) {                   // only items with work use q_full
                if (q_by_tma(it[IT_PAIR], chunk, q)) {
                    q_ready_tma();
                } else {
                    if (!q_copying && !*abort_flag) copy_q(it[IT_PAIR], it[IT_Q0], chunk, it[IT_KVH]);
                    q_ready();
                }
            }
            q_copying = false;
            q_announced = false;
            const int tok0 = (it[IT_PAIR] * NQ + q) * C::TQ;
            const int tok = tok0 + t / G;
            const bool row_ok = tok < chunk;
            const int pos = row_ok ? ctx - chunk + tok : 0;
            const int first_pos = ctx - chunk + tok0;
            float m_run = -INFINITY, l_run = 0.f;
            bool failed = *abort_flag != 0;                    // a stopped CTA writes NaN rows
            for (int j = 0; j < nkv_q && !failed; ++j) {
                const int gj = gs + j;
                bool ok = __all_sync(FULL, mbar_wait_or_abort(my_s_full, gj & 1, abort_flag));
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
                // rescale this warp's rows of O when any of their maxima moved (P V_{j-1} must be done)
                if (__any_sync(FULL, moved)) {
                    ok = __all_sync(FULL, mbar_wait_or_abort(&my_o_done[(gj - 1) & 1], ((gj - 1) >> 1) & 1, abort_flag));
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
                // the P columns are free once P V_{gj-1} has finished
                if (gj >= 1) {
                    ok = __all_sync(FULL, mbar_wait_or_abort(&my_o_done[(gj - 1) & 1], ((gj - 1) >> 1) & 1, abort_flag));
                    if (!ok || *abort_flag) {
                        failed = true;
                        break;
                    }
                }
                tmem_st32(lane_tm + (uint32_t)C::COL_P, pk);
                tmem_wait_st();
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&my_p_full[gj & 1]);
            }
            if (!failed && nkv_q > 0) {
                // every S product of the item is done, so the tile's Q rows are no longer read:
                // start copying the next item's rows (if it is published already) before the
                // epilogue, which then overlaps the copy
                const int ns = (n + 1) & 1;
                if (mbar_test_wait(&item_full[ns], ((n + 1) >> 1) & 1)) {
                    const volatile int *nx = items + ns * IT_N;
                    if (nx[IT_SEQ] >= 0 && (q == 0 ? nx[IT_NKV0] : nx[IT_NKV1]) > 0 &&
                        !q_by_tma(nx[IT_PAIR], nx[IT_CHUNK], q) && !*abort_flag) {
                        copy_q(nx[IT_PAIR], nx[IT_Q0], nx[IT_CHUNK], nx[IT_KVH]);
                        q_copying = true;
                    }
                }
            }
            if (!failed && nkv_q > 0) {
                const int gl = gs + nkv_q - 1;
                const bool ok = __all_sync(FULL, mbar_wait_or_abort(&my_o_done[gl & 1], (gl >> 1) & 1, abort_flag));
                failed = !ok || *abort_flag;
            }
            if (q_copying) {
                // the next item's Q rows have had the last P V to land: announce them now, so
                // its first S product runs during this item's epilogue
                q_ready();
                q_announced = true;
            } else if (sc.q_tma && !failed && nkv_q > 0) {
                // likewise for a next-item tile that came by TMA, if it has landed already
                int go = 0;
                if (lane == 0) {
                    const int ns = (n + 1) & 1;
                    if (mbar_test_wait(&item_full[ns], ((n + 1) >> 1) & 1)) {
                        const volatile int *nx = items + ns * IT_N;
                        go = nx[IT_SEQ] >= 0 && (q == 0 ? nx[IT_NKV0] : nx[IT_NKV1]) > 0 &&
                             q_by_tma(nx[IT_PAIR], nx[IT_CHUNK], q) && mbar_test_wait(&q_land[q], nqt & 1);
                    }
                }
                if (__shfl_sync(FULL, go, 0)) {
                    q_ready_tma();
                    q_announced = true;
                }
            }
            if (nkv_q > 0) {
                if (!failed) tc_fence_after_sync();
                // normalise and write this row
                const float inv = (!failed && l_run > 0.f) ? 1.f / l_run : __int_as_float(0x7fc00000);
                __nv_bfloat16 *orow =
                    p.out + ((size_t)(it[IT_Q0] + (row_ok ? tok : 0)) * p.h_q + (size_t)it[IT_KVH] * G + t % G) * D;
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
                // the O reads are complete (tcgen05.wait::ld) before this warp arrives on the
                // next item's first p_full, which lets the next item's first P V overwrite O
                tc_fence_before_sync();
            }
            gs += nkv_q;
        }
        cp_async_wait_all();                                   // no copy in flight at exit
        tc_fence_before_sync();
    }
    __syncthreads();
    if (warp == C::MMA_WARP) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
    if (claiming && threadIdx.x == 0) {
        // the last CTA to finish leaves the counters at zero for the next launch
        __threadfence();
        if (atomicAdd(sc.counters + 1, 1) == (int)gridDim.x - 1) {
            atomicExch(sc.counters, 0);
            atomicExch(sc.counters + 1, 0);
        }
    }
}

}  // namespace pa
