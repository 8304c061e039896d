// decode_allheads.cuh -- bf16 paged decode streaming whole physical blocks (every KV head), with
// a static-then-dynamic schedule.
//
// Same attention as the partition kernels (decode.cuh, decode_mma.cuh):
//   out[s][h] = softmax(scale * q[s][h] . K_s^T) . V_s
// with token t of sequence s in physical block block_tables[s][t / bs] at offset t % bs and
// query head h reading KV head h / G ("现代 AI 的“推理加速之谜”…" section 1, attention;
// "深度解构 LLM 推理优化…" section 2.1, block table; section 3.A of the first page, GQA).
//
// Unit of streaming.  In the [NB][h_kv][bs][d] cache layout the K (or V) of one physical block
// for every KV head is one contiguous span (32 KB at 8 heads, bs 16, d 128).  One CTA fetches it
// with two TMA boxes (64 elements x h_kv*bs rows each) and its h_kv consumer warps -- warp w
// serves KV head w and its G query heads -- read their rows of it.  A unit is one block of one
// sequence, all heads; the step's units are numbered sequence by sequence, x = prefix[s] + lb.
//
// Schedule.  A persistent grid of one CTA per SM (the ring takes most of the shared memory).
// CTA c owns the range [c*T/C, (c+1)*T/C) of the T units.  Equal byte counts do not make equal
// times: SMs stream at different rates (by their place on the chip; about +-10 % here), so a
// purely static split ends with part of the GPU idle.  Each range is therefore cut into a
// static segment (its first ~85 %) and NCH tail chunks of U units each.  A CTA streams its
// static segment, then claims tail chunks -- its own or any other CTA's -- from one global
// counter until none is left; SMs that run ahead take more chunks.
// Pieces.  A piece is the part of one sequence inside one segment (static segment or chunk).
// A piece that is its whole sequence is finished at once (bf16 rows).  Otherwise the warp writes
// a partial (m, l, o) for its G query heads into the segment's slot 0 (the piece starts the
// segment) or slot 1 (it ends it) -- plain stores, nothing waits on them -- and the merge
// kernel, launched after this one as its programmatic dependent, combines each split sequence's
// pieces (out = sum 2^(m_i - M) o_i / sum 2^(m_i - M) l_i); it finds them from the same segment
// arithmetic.  No CTA waits on another.  The last CTA to finish resets the chunk counter.
//
// Ring: NST stages of one block's K or V (every head).  Stream position k (one unit) uses stage
// (2k) % NST for K and (2k+1) % NST for V; a warp releases the K stage as soon as its scores are
// computed and the V stage after P.V, so most of the ring is in flight.  Every consumer warp
// consumes every stage in order (empty barrier count = h_kv), so a parity wait can never see a
// phase other than the one it means.  The producer publishes each position's unit and segment
// in a small shared table (the unit -1 ends the stream); consumers read it after the K stage's
// full barrier, and peek one position ahead to load the next sequence's q early.
// Per 16-token sub-block a warp computes S^T = K . Q^T and O^T += V^T . P^T with mma.sync
// m16n8k16 (bf16 in, fp32 accumulate), as in decode_mma.cuh; the whole block's scores are
// taken before its softmax, so a block costs one max / rescale step.  P is rounded to bf16
// for the second product; the normaliser sums the fp32 probabilities.
#pragma once

#include "decode_balanced.cuh"

namespace pa {

constexpr int kAllHeadsMaxCtas = 160;     // CTAs of a launch (one per SM; B200 has 148)
constexpr int kAllHeadsMaxSeqs = 2048;    // sequences per launch (prefix sums in shared memory)
constexpr int kAllHeadsHkv = 8;           // KV heads the kernel is built for (one warp each)
constexpr int kTailChunks = 4;            // NCH: dynamic chunks cut from the end of every range
constexpr int kTailPercent = 15;          // of each range, rounded up to whole chunks
constexpr int kAllHeadsSlots = 2 * kAllHeadsMaxCtas * (1 + kTailChunks);   // partial slots
constexpr int kMetaRing = 64;             // stream positions in the shared unit table
constexpr int kClaimAhead = 4;            // units left in a segment when the next chunk is claimed

struct AllHeadsParams {
    __nv_bfloat16 *out;            // [B][h_q][D]
    const __nv_bfloat16 *q;        // [B][h_q][D]
    const int32_t *block_tables;   // [B][max_blocks_per_seq]
    const int32_t *context_lens;   // [B]
    int *pool;                     // [0] chunks claimed, [1] CTAs finished; zero between launches
    int *prefix_out;               // [B + 1] the block prefix sums, for the merge kernel
    float *part_ml;                // [kAllHeadsSlots][h_q][2]  (m, l), log2 domain
    float *part_o;                 // [kAllHeadsSlots][h_q][D]  unnormalised
    int max_blocks_per_seq;
    int num_seqs;
    int num_blocks;
    int num_ctas;                  // gridDim.x (<= kAllHeadsMaxCtas)
    float qk_scale;                // scale * log2(e)
    int pdl_wait_last;             // launched right after the cache write of each sequence's
                                   // appended token: wait for it before loading a sequence's last block
};

template <int D, int BS, int G, int HKV>
struct AllHeadsConfig {
    static constexpr int NW = HKV;                        // consumer warps, one per KV head
    static constexpr int THREADS = (NW + 1) * 32;         // + producer warp
    static constexpr int HQ = HKV * G;
    static constexpr int HALVES = D / 64;                 // 128-byte column halves of a row
    static constexpr int HEAD_BYTES = BS * 128;           // one head's rows of one half
    static constexpr int HALF_BYTES = HKV * HEAD_BYTES;   // one TMA box: 64 elements x HKV*BS rows
    static constexpr int STAGE_BYTES = HALVES * HALF_BYTES;   // K (or V) of one block, every head
    static constexpr int RING_MAX = 196608;               // 192 KB of stages
    static constexpr int NST = RING_MAX / STAGE_BYTES;    // stages
    static constexpr int KS = D / 16;                     // k-steps of q.K
    static constexpr int MT = D / 16;                     // m-tiles of O^T
    static constexpr int NSUB = BS / 16;
    static constexpr int RING = NST * STAGE_BYTES;
    static constexpr int OFF_BARS = RING;
    static constexpr int OFF_FLAGS = OFF_BARS + 2 * NST * 8;
    static constexpr int OFF_META = OFF_FLAGS + (NST + 4) * 4;          // unit, segment per position
    static constexpr int OFF_SCAN = OFF_META + 2 * kMetaRing * 4;
    static constexpr int OFF_PREFIX = OFF_SCAN + 32 * 4;
    // dynamic shared memory for num_seqs sequences (+1024 to align the ring)
    __host__ __device__ static constexpr int smem_bytes(int num_seqs) { return OFF_PREFIX + (num_seqs + 1) * 4 + 1024; }
    static_assert(D == 64 || D == 128, "head dim");
    static_assert(BS == 16 || BS == 32, "block size");
    static_assert(G <= 8, "group");
    static_assert(HKV * BS <= 256, "a TMA box holds at most 256 rows");
    static_assert(HEAD_BYTES % 1024 == 0, "each head's rows start on a swizzle atom");
    static_assert(NST >= 3 && NST / 2 + 2 < kMetaRing, "ring");
};

// Unit x of the flat block space (sequence by sequence): sequence s, block lb within it and
// the sequence's block count nb (> 0).
struct UnitPos {
    int s, lb, nb;
};

__device__ __forceinline__ UnitPos locate_unit(const int *prefix, int num_seqs, int x)
{
    int lo = 0, hi = num_seqs - 1;               // last s with prefix[s] <= x
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (prefix[mid] <= x) lo = mid;
        else hi = mid - 1;
    }
    UnitPos u;
    u.s = lo;
    u.nb = prefix[lo + 1] - prefix[lo];
    u.lb = x - prefix[lo];
    return u;
}

// The segments of one launch (the same in every CTA).  Range c = [a(c), b(c)); its static
// segment [a, ts) and its chunks j = 0..NCH-1 of U units taken from the end:
// chunk j = [max(ts, b - (NCH - j) U), max(that, b - (NCH - 1 - j) U)).  Segment id
// g = c (1 + NCH) + k, k = 0 static, k = 1 + j chunk j; ids increase with position.
struct AllHeadsSegs {
    int T, Ce, U;
    // T units over C CTAs: Ce = min(C, T) ranges, U units per chunk (NCH chunks make ~15 % of a range)
    __host__ __device__ static AllHeadsSegs make(int T, int C)
    {
        AllHeadsSegs sg;
        sg.T = T;
        sg.Ce = T < C ? T : C;
        const int per = sg.Ce > 0 ? T / sg.Ce : 0;
        const int tail = (per * kTailPercent + 99) / 100;
        sg.U = cmax(1, (tail + kTailChunks - 1) / kTailChunks);
        return sg;
    }
    // c * T and (x + 1) * Ce stay below 2^32 (T < 2^24 units, Ce <= kAllHeadsMaxCtas)
    __host__ __device__ __forceinline__ int a(int c) const { return (int)((unsigned)c * (unsigned)T / (unsigned)Ce); }
    __host__ __device__ __forceinline__ int b(int c) const { return a(c + 1); }
    __host__ __device__ __forceinline__ int cta_of(int x) const
    {
        return (int)(((unsigned)x * (unsigned)Ce + (unsigned)Ce - 1u) / (unsigned)T);
    }
    __host__ __device__ __forceinline__ int ts(int c) const { return cmax(a(c), b(c) - kTailChunks * U); }
    __host__ __device__ __forceinline__ void bounds(int g, int &lo, int &hi) const
    {
        const int c = g / (1 + kTailChunks), k = g % (1 + kTailChunks);
        const int ac = a(c), bc = b(c), t = cmax(ac, bc - kTailChunks * U);
        if (k == 0) {
            lo = ac;
            hi = t;
        } else {
            const int j = k - 1;
            lo = cmax(t, bc - (kTailChunks - j) * U);
            hi = cmax(lo, bc - (kTailChunks - 1 - j) * U);
        }
    }
    __host__ __device__ __forceinline__ int seg_of(int x) const
    {
        const int c = cta_of(x);
        const int bc = b(c);
        if (x < cmax(a(c), bc - kTailChunks * U)) return c * (1 + kTailChunks);
        return c * (1 + kTailChunks) + kTailChunks - (bc - 1 - x) / U;
    }
};

struct AllHeadsMergeParams {
    __nv_bfloat16 *out;            // [B][h_q][D]
    const int *prefix;             // [B + 1] block prefix sums written by the decode kernel
    const float *part_ml;          // [kAllHeadsSlots][h_q][2]
    const float *part_o;           // [kAllHeadsSlots][h_q][D]
    int num_seqs;
    int h_q;
    int num_ctas;                  // the decode launch's gridDim.x
};

constexpr int kAllHeadsMergeWarps = 8;

// The pieces of each split sequence, combined: CTA (query head qh, sequence s).  The sequence's
// units are [gs, ge); its pieces are the non-empty segments g0..g1 it overlaps, segment g's
// piece holding its partial in slot 2 g + (gs <= lo_g ? 0 : 1).  M = max of the pieces' m; warp
// w sums the pieces w, w + 8, ... (lanes own D/32 dims); the CTA adds the warps' sums.
// Launched as the decode kernel's programmatic dependent: griddepcontrol.wait orders every read
// after the decode grid's writes.
template <int D>
__global__ void __launch_bounds__(kAllHeadsMergeWarps * 32) paged_decode_allheads_merge_kernel(const AllHeadsMergeParams p)
{
    constexpr int NWM = kAllHeadsMergeWarps, DPL = D / 32;
    pdl_wait();
    const int qh = blockIdx.x, s = blockIdx.y;
    const int gs = p.prefix[s], ge = p.prefix[s + 1];
    if (gs == ge) return;                                        // no context: rows written by the decode
    const AllHeadsSegs sg = AllHeadsSegs::make(p.prefix[p.num_seqs], p.num_ctas);
    const int g0 = sg.seg_of(gs), g1 = sg.seg_of(ge - 1);
    if (g0 == g1) return;                                        // one piece: finished by the decode
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __shared__ float red[NWM];
    __shared__ float lsum[NWM];
    __shared__ float acc_s[NWM][D];
    auto slot_of = [&](int g) -> int {
        int lo, hi;
        sg.bounds(g, lo, hi);
        return lo < hi ? 2 * g + (gs <= lo ? 0 : 1) : -1;
    };
    float m = -INFINITY;
    for (int g = g0 + (int)threadIdx.x; g <= g1; g += blockDim.x) {
        const int sl = slot_of(g);
        if (sl >= 0) m = fmaxf(m, __ldcg(p.part_ml + ((size_t)sl * p.h_q + qh) * 2));
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    if (lane == 0) red[warp] = m;
    __syncthreads();
    float M = red[0];
#pragma unroll
    for (int w = 1; w < NWM; ++w) M = fmaxf(M, red[w]);
    float L = 0.f, acc[DPL];
#pragma unroll
    for (int e = 0; e < DPL; ++e) acc[e] = 0.f;
    for (int g = g0 + warp; g <= g1; g += NWM) {
        const int sl = slot_of(g);
        if (sl < 0) continue;
        const size_t row = (size_t)sl * p.h_q + qh;
        const float2 ml = __ldcg(reinterpret_cast<const float2 *>(p.part_ml + row * 2));
        const float w = exp2f(ml.x - M);
        L += w * ml.y;
        const float *po = p.part_o + row * D + lane * DPL;
        if constexpr (DPL == 4) {
            const float4 v = __ldcg(reinterpret_cast<const float4 *>(po));
            acc[0] += w * v.x; acc[1] += w * v.y; acc[2] += w * v.z; acc[3] += w * v.w;
        } else {
            const float2 v = __ldcg(reinterpret_cast<const float2 *>(po));
            acc[0] += w * v.x; acc[1] += w * v.y;
        }
    }
    if (lane == 0) lsum[warp] = L;
#pragma unroll
    for (int e = 0; e < DPL; ++e) acc_s[warp][lane * DPL + e] = acc[e];
    __syncthreads();
    if (threadIdx.x < D) {
        float Lt = 0.f, o = 0.f;
#pragma unroll
        for (int w = 0; w < NWM; ++w) {
            Lt += lsum[w];
            o += acc_s[w][threadIdx.x];
        }
        p.out[((size_t)s * p.h_q + qh) * D + threadIdx.x] = __float2bfloat16_rn(o / Lt);
    }
}

template <int D, int BS, int G, int HKV>
__global__ void __launch_bounds__(AllHeadsConfig<D, BS, G, HKV>::THREADS, 1)
    paged_decode_allheads_kernel(const AllHeadsParams p, const __grid_constant__ CUtensorMap tmap_k,
                                 const __grid_constant__ CUtensorMap tmap_v)
{
    using C = AllHeadsConfig<D, BS, G, HKV>;
    constexpr int NW = C::NW, NST = C::NST, HQ = C::HQ;
    constexpr unsigned FULL = 0xffffffffu;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *ring = smem;
    uint64_t *full_bar = reinterpret_cast<uint64_t *>(smem + C::OFF_BARS);
    uint64_t *empty_bar = full_bar + NST;
    volatile int *stage_bad = reinterpret_cast<volatile int *>(smem + C::OFF_FLAGS);
    volatile int *abort_flag = stage_bad + NST;
    volatile int *published = stage_bad + NST + 1;          // stream positions whose unit is in the table
    volatile int *meta_x = reinterpret_cast<volatile int *>(smem + C::OFF_META);   // [kMetaRing] unit, -1 = end
    volatile int *meta_g = meta_x + kMetaRing;                                     // [kMetaRing] segment
    int *scan = reinterpret_cast<int *>(smem + C::OFF_SCAN);
    int *prefix = reinterpret_cast<int *>(smem + C::OFF_PREFIX);

    const int B = p.num_seqs, Cn = p.num_ctas, c = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    block_prefix<C::THREADS>(prefix, scan, p.context_lens, B, BS);
    if (threadIdx.x == 0) {
        for (int i = 0; i < NST; ++i) {
            mbar_init(&full_bar[i], 1);
            mbar_init(&empty_bar[i], NW);
        }
        *abort_flag = 0;
        *published = 0;
        mbar_init_fence();
    }
    // sequences with no context get zero rows (one writer per sequence)
    for (int s = c; s < B; s += Cn) {
        if (prefix[s + 1] == prefix[s]) {
            __nv_bfloat16 *row = p.out + (size_t)s * HQ * D;
            for (int i = threadIdx.x; i < HQ * D; i += C::THREADS) row[i] = __float2bfloat16_rn(0.f);
        }
    }
    __syncthreads();

    // ranges over Ce = min(C, T) CTAs: every range that exists is non-empty
    const AllHeadsSegs sg = AllHeadsSegs::make(prefix[B], Cn);
    if (c == 0)
        for (int i = threadIdx.x; i <= B; i += C::THREADS) p.prefix_out[i] = prefix[i];
    pdl_launch_dependents();                                // the merge kernel may start its prologue
    const int n_chunks = sg.Ce * kTailChunks;

    if (warp == NW) {
        // ------------------------------ producer ------------------------------
        if (lane == 0) {
            prefetch_tensormap(&tmap_k);
            prefetch_tensormap(&tmap_v);
        }
        const uint64_t pol = l2_policy_evict_first();
        int pos = 0;                                        // stream positions issued
        int issued = 0;                                     // stage uses issued (lane 0)
        bool ok = true;
        // the next tail chunk is claimed while the last few units of the current segment are
        // still being issued, so that the claim's round trip overlaps them
        int claim_val = 0;                                  // lane 0: the claim in flight
        bool pending = false;
        auto claim = [&]() {
            if (!pending) {
                if (lane == 0) claim_val = atomicAdd(p.pool, 1);
                pending = true;
            }
        };
        // stream the units [lo, hi) of segment g: table entries 32 at a time, one lane each
        auto stream_segment = [&](int g, int lo, int hi) {
            for (int x0 = lo; x0 < hi && ok; x0 += 32) {
                const int x = x0 + lane;
                int row = -1;                               // TMA row of the block's first head, -1 = bad
                bool last = false;
                if (x < hi) {
                    const UnitPos u = locate_unit(prefix, B, x);
                    if (u.lb < p.max_blocks_per_seq) {
                        const int phys = p.block_tables[(size_t)u.s * p.max_blocks_per_seq + u.lb];
                        if (phys >= 0 && phys < p.num_blocks) row = phys * HKV * BS;
                    }
                    last = (u.lb == u.nb - 1);
                }
                const int cnt = min(32, hi - x0);
                for (int jj = 0; jj < cnt; ++jj) {
                    if (hi - (x0 + jj) <= kClaimAhead) claim();
                    const int rw = __shfl_sync(FULL, row, jj);
                    const bool lst = __shfl_sync(FULL, last, jj) != 0;
                    if (lane == 0) {
                        if (p.pdl_wait_last && lst) pdl_wait();   // the block holding the appended token
#pragma unroll
                        for (int kv = 0; kv < 2; ++kv) {
                            const int j = 2 * pos + kv, st = j % NST;
                            if (ok && j >= NST) ok = mbar_wait_bounded(&empty_bar[st], ((j / NST) - 1) & 1);
                            if (ok && *abort_flag) ok = false;
                            if (ok) {
                                if (kv == 0) {
                                    meta_x[pos % kMetaRing] = x0 + jj;
                                    meta_g[pos % kMetaRing] = g;
                                    __threadfence_block();
                                    *published = pos + 1;
                                }
                                if (rw >= 0) {
                                    stage_bad[st] = 0;
                                    mbar_arrive_expect_tx(&full_bar[st], C::STAGE_BYTES);
                                    uint8_t *dst = ring + st * C::STAGE_BYTES;
#pragma unroll
                                    for (int hf = 0; hf < C::HALVES; ++hf)
                                        tma_load_2d(dst + hf * C::HALF_BYTES, kv ? &tmap_v : &tmap_k, hf * 64, rw,
                                                    &full_bar[st], pol);
                                } else {
                                    stage_bad[st] = 1;
                                    if (kv == 0) record_error(PA_DEVERR_BAD_BLOCK);
                                    mbar_arrive(&full_bar[st]);
                                }
                                issued = j + 1;
                            }
                        }
                    }
                    ok = __shfl_sync(FULL, ok, 0) != 0;
                    if (!ok) break;
                    ++pos;
                }
            }
        };
        if (c < sg.Ce) stream_segment(c * (1 + kTailChunks), sg.a(c), sg.ts(c));
        // then tail chunks from the global counter until none is left
        while (ok) {
            claim();
            const int q = __shfl_sync(FULL, claim_val, 0);
            pending = false;
            if (q >= n_chunks) break;
            const int g = (q / kTailChunks) * (1 + kTailChunks) + 1 + q % kTailChunks;
            int lo, hi;
            sg.bounds(g, lo, hi);
            stream_segment(g, lo, hi);
        }
        // the end of the stream: position pos holds unit -1 (its K stage's full barrier completes
        // without data)
        if (lane == 0 && ok) {
            const int j = 2 * pos, st = j % NST;
            if (j >= NST) ok = mbar_wait_bounded(&empty_bar[st], ((j / NST) - 1) & 1);
            if (ok) {
                meta_x[pos % kMetaRing] = -1;
                meta_g[pos % kMetaRing] = -1;
                __threadfence_block();
                *published = pos + 1;
                stage_bad[st] = 0;
                mbar_arrive(&full_bar[st]);
            }
        }
        ok = __shfl_sync(FULL, ok, 0) != 0;
        if (lane == 0 && !ok) {
            if (!*abort_flag) record_error(PA_DEVERR_TIMEOUT);
            *abort_flag = 1;
            // wait (bounded) for the copies still in flight: the last NST stage uses issued
            for (int j = max(0, issued - NST); j < issued; ++j)
                mbar_wait_bounded(&full_bar[j % NST], (j / NST) & 1);
        }
    } else {
        // ------------------------------ consumers ------------------------------
        const int kvh = warp;
        const int tq = lane & 3, r = lane >> 2;
        const int mrow = lane & 7, mat = lane >> 3;         // ldmatrix: row address this lane supplies
        const uint32_t ring_s = smem_addr(ring);
        float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
        float o[C::MT][4];
#pragma unroll
        for (int mt = 0; mt < C::MT; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
        uint32_t qb[C::KS][2], qn[C::KS][2];
        int qn_seq = -1;                                    // sequence whose q sits in qn
        int cur_s = -1, cur_g = -1, gs = 0, ge = 0, ctx_cur = 0;
        bool bad = false;

        // finish the current piece: final rows, or its partial (plain stores; the merge kernel reads them)
        auto close_piece = [&]() {
#pragma unroll
            for (int off = 4; off < 32; off <<= 1) {
                l_run[0] += __shfl_xor_sync(FULL, l_run[0], off);
                l_run[1] += __shfl_xor_sync(FULL, l_run[1], off);
            }
            const bool failed = bad || (*abort_flag != 0);
            const int g0 = sg.seg_of(gs), g1 = sg.seg_of(ge - 1);
            const size_t row0 = (size_t)cur_s * HQ + (size_t)kvh * G;
            if (g0 == g1) {                                 // the whole sequence is this piece
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int h = 2 * tq + j;
                    if (h < G) {
                        __nv_bfloat16 *dst = p.out + (row0 + h) * D;
#pragma unroll
                        for (int mt = 0; mt < C::MT; ++mt) {
                            const float v0 = failed ? __int_as_float(0x7fc00000) : o[mt][j] / l_run[j];
                            const float v1 = failed ? __int_as_float(0x7fc00000) : o[mt][2 + j] / l_run[j];
                            dst[16 * mt + r] = __float2bfloat16_rn(v0);
                            dst[16 * mt + r + 8] = __float2bfloat16_rn(v1);
                        }
                    }
                }
                return;
            }
            int lo, hi;
            sg.bounds(cur_g, lo, hi);
            const int slot = 2 * cur_g + (gs <= lo ? 0 : 1);
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int h = 2 * tq + j;
                if (h < G) {
                    const size_t row = (size_t)slot * HQ + (size_t)kvh * G + h;
                    float *po = p.part_o + row * D;
#pragma unroll
                    for (int mt = 0; mt < C::MT; ++mt) {
                        po[16 * mt + r] = failed ? __int_as_float(0x7fc00000) : o[mt][j];
                        po[16 * mt + r + 8] = failed ? __int_as_float(0x7fc00000) : o[mt][2 + j];
                    }
                    if (r == 0) {
                        p.part_ml[row * 2] = failed ? 0.f : m_run[j];
                        p.part_ml[row * 2 + 1] = failed ? __int_as_float(0x7fc00000) : l_run[j];
                    }
                }
            }
        };

        for (int k = 0;; ++k) {
            if (*abort_flag) break;
            const int jk = 2 * k, stk = jk % NST, jv = jk + 1, stv = jv % NST;
            if (!__all_sync(FULL, mbar_wait_bounded(&full_bar[stk], (jk / NST) & 1))) {
                if (lane == 0) {
                    record_error(PA_DEVERR_TIMEOUT);
                    *abort_flag = 1;
                }
                break;
            }
            const int x = meta_x[k % kMetaRing], g = meta_g[k % kMetaRing];
            if (x < 0) break;                               // end of the stream
            if (x < gs || x >= ge || g != cur_g) {
                // a new piece: close the current one, take the new sequence's q and context
                if (cur_s >= 0) close_piece();
                const UnitPos u = locate_unit(prefix, B, x);
                if (u.s != cur_s) {
                    if (qn_seq == u.s) {
#pragma unroll
                        for (int ks = 0; ks < C::KS; ++ks) {
                            qb[ks][0] = qn[ks][0];
                            qb[ks][1] = qn[ks][1];
                        }
                    } else {
                        mma_load_q<C, G, D>(qb, p.q + ((size_t)u.s * HQ + (size_t)kvh * G) * D, lane);
                    }
                    ctx_cur = p.context_lens[u.s];
                }
                cur_s = u.s;
                cur_g = g;
                gs = prefix[u.s];
                ge = prefix[u.s + 1];
                m_run[0] = m_run[1] = -INFINITY;
                l_run[0] = l_run[1] = 0.f;
#pragma unroll
                for (int mt = 0; mt < C::MT; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
                bad = false;
            }
            // peek at the next position: a new sequence there gets its q loaded now
            if (*published > k + 1) {
                __threadfence_block();                      // the table entry after its count
                const int x1 = meta_x[(k + 1) % kMetaRing];
                if (x1 >= 0 && (x1 < gs || x1 >= ge)) {
                    const int s1 = locate_unit(prefix, B, x1).s;
                    if (s1 != qn_seq) {
                        mma_load_q<C, G, D>(qn, p.q + ((size_t)s1 * HQ + (size_t)kvh * G) * D, lane);
                        qn_seq = s1;
                    }
                }
            }
            const int lb = x - gs;
            const int valid = min(BS, ctx_cur - lb * BS);
            // ---- K stage: S^T = K . Q^T for every 16-token sub-block of the block ----
            const bool kbad = stage_bad[stk] != 0;
            float sT[C::NSUB][4];
#pragma unroll
            for (int sub = 0; sub < C::NSUB; ++sub) sT[sub][0] = sT[sub][1] = sT[sub][2] = sT[sub][3] = 0.f;
            if (!kbad) {
                const uint32_t kbase = ring_s + stk * C::STAGE_BYTES + kvh * C::HEAD_BYTES;
#pragma unroll
                for (int sub = 0; sub < C::NSUB; ++sub) {
                    float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
                    if (sub * 16 < valid) {
                        const int tok = sub * 16 + (mat & 1) * 8 + mrow;
#pragma unroll
                        for (int ks = 0; ks < C::KS; ++ks) {
                            const int chunk = 2 * (ks & 3) + (mat >> 1);
                            uint32_t af[4];
                            ldmatrix_x4(af, kbase + (ks >> 2) * C::HALF_BYTES + swz128(tok, chunk));
                            if (ks & 1) mma_bf16_16816(s1, af[0], af[1], af[2], af[3], qb[ks][0], qb[ks][1]);
                            else mma_bf16_16816(s0, af[0], af[1], af[2], af[3], qb[ks][0], qb[ks][1]);
                        }
                    }
#pragma unroll
                    for (int i = 0; i < 4; ++i) sT[sub][i] = s0[i] + s1[i];
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty_bar[stk]);     // K stage read
            // ---- online softmax over the block: tokens sub*16 + r (+ 8), heads 2tq, 2tq + 1 ----
            float pr[C::NSUB][4];
            float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
            for (int sub = 0; sub < C::NSUB; ++sub) {
                const int t0 = sub * 16 + r;
                pr[sub][0] = t0 < valid ? sT[sub][0] * p.qk_scale : -INFINITY;
                pr[sub][1] = t0 < valid ? sT[sub][1] * p.qk_scale : -INFINITY;
                pr[sub][2] = t0 + 8 < valid ? sT[sub][2] * p.qk_scale : -INFINITY;
                pr[sub][3] = t0 + 8 < valid ? sT[sub][3] * p.qk_scale : -INFINITY;
                mx0 = fmaxf(mx0, fmaxf(pr[sub][0], pr[sub][2]));
                mx1 = fmaxf(mx1, fmaxf(pr[sub][1], pr[sub][3]));
            }
#pragma unroll
            for (int off = 4; off < 32; off <<= 1) {
                mx0 = fmaxf(mx0, __shfl_xor_sync(FULL, mx0, off));
                mx1 = fmaxf(mx1, __shfl_xor_sync(FULL, mx1, off));
            }
            const float mn0 = fmaxf(m_run[0], mx0), mn1 = fmaxf(m_run[1], mx1);
            const float al0 = exp2f(m_run[0] - mn0), al1 = exp2f(m_run[1] - mn1);
            m_run[0] = mn0;
            m_run[1] = mn1;
            float ps0 = 0.f, ps1 = 0.f;
            uint32_t pb[C::NSUB][2];
#pragma unroll
            for (int sub = 0; sub < C::NSUB; ++sub) {
                const float p0 = exp2f(pr[sub][0] - mn0), p1 = exp2f(pr[sub][1] - mn1);
                const float p2 = exp2f(pr[sub][2] - mn0), p3 = exp2f(pr[sub][3] - mn1);
                ps0 += p0 + p2;
                ps1 += p1 + p3;
                // P^T as the B operand: b0 = P[head T/4][tokens 2tq, 2tq+1], b1 = tokens + 8
                pb[sub][0] = movmatrix_trans(pack_bf16x2(p0, p1));
                pb[sub][1] = movmatrix_trans(pack_bf16x2(p2, p3));
            }
            l_run[0] = l_run[0] * al0 + ps0;
            l_run[1] = l_run[1] * al1 + ps1;
            if (__any_sync(FULL, (al0 != 1.f) | (al1 != 1.f))) {
#pragma unroll
                for (int mt = 0; mt < C::MT; ++mt) {
                    o[mt][0] *= al0;
                    o[mt][1] *= al1;
                    o[mt][2] *= al0;
                    o[mt][3] *= al1;
                }
            }
            // ---- V stage: O^T += V^T . P^T ----
            if (!__all_sync(FULL, mbar_wait_bounded(&full_bar[stv], (jv / NST) & 1))) {
                if (lane == 0) {
                    record_error(PA_DEVERR_TIMEOUT);
                    *abort_flag = 1;
                }
                break;
            }
            if (kbad || stage_bad[stv]) {
                bad = true;
            } else {
                uint8_t *vhead = ring + stv * C::STAGE_BYTES + kvh * C::HEAD_BYTES;
                if (valid < BS) {
                    // zero this head's V rows past the context (whole 128-byte rows of each half):
                    // a zero probability times a NaN slot would poison the accumulator
                    const int nrow = BS - valid;
                    for (int e = lane; e < nrow * 8 * C::HALVES; e += 32) {
                        const int hf = e / (nrow * 8);
                        const int rr = valid + (e / 8) % nrow;
                        reinterpret_cast<uint4 *>(vhead + hf * C::HALF_BYTES + rr * 128)[e % 8] = make_uint4(0, 0, 0, 0);
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                }
                const uint32_t vbase = smem_addr(vhead);
#pragma unroll
                for (int sub = 0; sub < C::NSUB; ++sub) {
                    if (sub * 16 < valid) {
                        const int tok = sub * 16 + (mat >> 1) * 8 + mrow;
#pragma unroll
                        for (int mt = 0; mt < C::MT; ++mt) {
                            const int chunk = ((2 * mt) & 7) + (mat & 1);
                            uint32_t af[4];
                            ldmatrix_x4_trans(af, vbase + (mt >> 2) * C::HALF_BYTES + swz128(tok, chunk));
                            mma_bf16_16816(o[mt], af[0], af[1], af[2], af[3], pb[sub][0], pb[sub][1]);
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty_bar[stv]);     // V stage read
        }
        if (cur_s >= 0) close_piece();
    }
    __syncthreads();
    // the CTA is done (every claim made): count it; the last one resets the chunk counter
    if (threadIdx.x == 0) {
        __threadfence();
        const int done = atomicAdd(p.pool + 1, 1);
        if (done == Cn - 1) {
            p.pool[0] = 0;
            p.pool[1] = 0;
        }
    }
}

}  // namespace pa
