// decode_allheads.cuh -- bf16 paged decode streaming whole physical blocks (every KV head).
//
// Same attention as the partition kernels (decode.cuh, decode_mma.cuh):
//   out[s][h] = softmax(scale * q[s][h] . K_s^T) . V_s
// with token t of sequence s in physical block block_tables[s][t / bs] at offset t % bs and
// query head h reading KV head h / G ("现代 AI 的“推理加速之谜”…" section 1, attention;
// "深度解构 LLM 推理优化…" section 2.1, block table; section 3.A of the first page, GQA).
//
// What differs is the unit of streaming.  In the [NB][h_kv][bs][d] cache layout the K (or V)
// of one physical block for every KV head is one contiguous span (32 KB at 8 heads, bs 16,
// d 128).  The other kernels fetch it as h_kv separate 4 KB tiles from h_kv different CTAs;
// here one CTA fetches the whole span with two TMA boxes (64 elements x h_kv*bs rows each) and
// its h_kv consumer warps -- warp w serves KV head w and its G query heads -- read their rows
// of it.  HBM sees long contiguous reads at scattered block addresses instead of short ones.
//
// Schedule: a persistent grid of one CTA per SM (the ring takes most of the shared memory).
// The step's blocks are laid out sequence by sequence, x = prefix[s] + lb, and CTA c takes
// [c*T/C, (c+1)*T/C), so every CTA moves the same number of bytes.  A sequence whose blocks
// lie in one CTA's range is finished there; otherwise each CTA holding part of it writes a
// partial (m, l, o) per query head -- into slot 0 when it is the first sequence of the
// range, slot 1 when the last -- and counts itself on the (sequence, KV head) counter; the
// warp that completes the count merges the partials (out = sum_c 2^(m_c - M) o_c /
// sum_c 2^(m_c - M) l_c) and resets the counter.  No CTA waits on another.
//
// Ring: NST stages of one block's K or V (every head).  Unit k (one block) uses stage
// (2k) % NST for K and (2k+1) % NST for V; a warp releases the K stage as soon as its scores
// are computed and the V stage after P.V, so most of the ring is in flight.  Every consumer
// warp consumes every stage in order (empty barrier count = h_kv), so a parity wait can never
// see a phase other than the one it means.
// Per 16-token sub-block a warp computes S^T = K . Q^T and O^T += V^T . P^T with mma.sync
// m16n8k16 (bf16 in, fp32 accumulate), as in decode_mma.cuh; the whole block's scores are
// taken before its softmax, so a block costs one max / rescale step.  P is rounded to bf16
// for the second product; the normaliser sums the fp32 probabilities.
#pragma once

#include "decode_balanced.cuh"

namespace pa {

constexpr int kAllHeadsMaxCtas = 256;     // partial slots in the workspace (one CTA per SM)
constexpr int kAllHeadsMaxSeqs = 2048;    // sequences per launch (prefix sums in shared memory)
constexpr int kAllHeadsHkv = 8;           // KV heads the kernel is built for (one warp each)

struct AllHeadsParams {
    __nv_bfloat16 *out;            // [B][h_q][D]
    const __nv_bfloat16 *q;        // [B][h_q][D]
    const int32_t *block_tables;   // [B][max_blocks_per_seq]
    const int32_t *context_lens;   // [B]
    int *counters;                 // [B][h_kv] contributing CTAs counted; zero between launches
    float *part_ml;                // [num_ctas][2][h_q][2]  (m, l), log2 domain
    float *part_o;                 // [num_ctas][2][h_q][D]  unnormalised
    int max_blocks_per_seq;
    int num_seqs;
    int num_blocks;
    int num_ctas;                  // gridDim.x
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
    static constexpr int OFF_SCAN = OFF_FLAGS + (NST + 4) * 4;
    static constexpr int OFF_PREFIX = OFF_SCAN + 32 * 4;
    // dynamic shared memory for num_seqs sequences (+1024 to align the ring)
    __host__ __device__ static constexpr int smem_bytes(int num_seqs) { return OFF_PREFIX + (num_seqs + 1) * 4 + 1024; }
    static_assert(D == 64 || D == 128, "head dim");
    static_assert(BS == 16 || BS == 32, "block size");
    static_assert(G <= 8, "group");
    static_assert(HKV * BS <= 256, "a TMA box holds at most 256 rows");
    static_assert(HEAD_BYTES % 1024 == 0, "each head's rows start on a swizzle atom");
    static_assert(NST >= 3, "ring");
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

// (m, l) <- the online-softmax combination of (m, l) and (m2, l2); m = -inf marks "nothing yet"
// (a written partial always has a finite m: a failed one carries m = 0 and l = NaN, which the
// combination passes on).
__device__ __forceinline__ void ml_combine(float &m, float &l, float m2, float l2)
{
    if (m2 == -INFINITY) return;
    if (m == -INFINITY) {
        m = m2;
        l = l2;
        return;
    }
    const float mx = fmaxf(m, m2);
    l = l * exp2f(m - mx) + l2 * exp2f(m2 - mx);
    m = mx;
}

// The merge of one (sequence, KV head) split over CTAs c0..c1, by the warp that completed its
// count: out = sum_c 2^(m_c - M) o_c / sum_c 2^(m_c - M) l_c for the G query heads.  Loads are
// issued together rather than one after another: the (m, l) pairs one per lane (lane % G is the
// head), combined across the lanes of each head; then the o rows, 8/G partials per round,
// each lane owning D/32 dims of every head.
template <int D, int G, int HQ>
__device__ __forceinline__ void allheads_merge(const AllHeadsParams &p, int s, int kvh, int c0, int c1, int gstart,
                                               int T, int Ce, int lane)
{
    constexpr unsigned FULL = 0xffffffffu;
    constexpr int DPL = D / 32;
    const int n = c1 - c0 + 1;
    // CTA cc > c0 holds its partial in slot 0; c0 in slot 0 when the sequence starts its range,
    // else in slot 1
    const int slot0 = (gstart == (int)((long long)c0 * T / Ce)) ? 0 : 1;
    auto prow = [&](int i, int h) -> size_t {
        const int cc = c0 + i;
        return ((size_t)cc * 2 + (i == 0 ? slot0 : 0)) * HQ + (size_t)kvh * G + h;
    };
    const int hl = lane % G;
    float mm = -INFINITY, ll = 0.f;
    for (int i = lane / G; i < n; i += 32 / G) {
        const float2 ml = __ldcg(reinterpret_cast<const float2 *>(p.part_ml + prow(i, hl) * 2));
        ml_combine(mm, ll, ml.x, ml.y);
    }
#pragma unroll
    for (int off = 16; off >= G; off >>= 1) {
        const float m2 = __shfl_xor_sync(FULL, mm, off), l2 = __shfl_xor_sync(FULL, ll, off);
        ml_combine(mm, ll, m2, l2);
    }
    float Mx[G], invL[G], acc[G][DPL];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        Mx[h] = __shfl_sync(FULL, mm, h);                   // lane h holds head h
        invL[h] = 1.f / __shfl_sync(FULL, ll, h);
#pragma unroll
        for (int e = 0; e < DPL; ++e) acc[h][e] = 0.f;
    }
    constexpr int UNR = cmax(1, 8 / G);                     // partials per round: 8 (head, partial) rows
    for (int i0 = 0; i0 < n; i0 += UNR) {
        float mv[UNR][G];
        float ov[UNR][G][DPL];
#pragma unroll
        for (int u = 0; u < UNR; ++u) {
            const int i = i0 + u < n ? i0 + u : n - 1;      // past the end: re-read the last one, weight 0
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const size_t ps = prow(i, h);
                mv[u][h] = __ldcg(p.part_ml + ps * 2);
                const float *po = p.part_o + ps * D + DPL * lane;
                if constexpr (DPL == 4) {
                    const float4 v = __ldcg(reinterpret_cast<const float4 *>(po));
                    ov[u][h][0] = v.x; ov[u][h][1] = v.y; ov[u][h][2] = v.z; ov[u][h][3] = v.w;
                } else {
                    const float2 v = __ldcg(reinterpret_cast<const float2 *>(po));
                    ov[u][h][0] = v.x; ov[u][h][1] = v.y;
                }
            }
        }
#pragma unroll
        for (int u = 0; u < UNR; ++u) {
            if (i0 + u < n) {
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    const float w = exp2f(mv[u][h] - Mx[h]) * invL[h];
#pragma unroll
                    for (int e = 0; e < DPL; ++e) acc[h][e] += w * ov[u][h][e];
                }
            }
        }
    }
#pragma unroll
    for (int h = 0; h < G; ++h) {
        __nv_bfloat16 *dst = p.out + ((size_t)s * HQ + (size_t)kvh * G + h) * D + DPL * lane;
        if constexpr (DPL == 4)
            *reinterpret_cast<uint2 *>(dst) = make_uint2(pack_bf16x2(acc[h][0], acc[h][1]), pack_bf16x2(acc[h][2], acc[h][3]));
        else
            *reinterpret_cast<uint32_t *>(dst) = pack_bf16x2(acc[h][0], acc[h][1]);
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

    // ranges over Ce = min(C, T) CTAs: every range that exists is non-empty, and the CTAs
    // holding a sequence's blocks are exactly cta_of_block(first) .. cta_of_block(last)
    const int T = prefix[B];
    const int Ce = T < Cn ? T : Cn;
    const int a = c < Ce ? (int)((long long)c * T / Ce) : 0;
    const int b = c < Ce ? (int)((long long)(c + 1) * T / Ce) : 0;
    const int n_units = b - a;

    if (warp == NW) {
        // ------------------------------ producer ------------------------------
        if (lane == 0) {
            prefetch_tensormap(&tmap_k);
            prefetch_tensormap(&tmap_v);
        }
        const uint64_t pol = l2_policy_evict_first();
        int issued = 0;                                     // stage uses issued (K and V count one each)
        bool ok = true;
        for (int k0 = 0; k0 < n_units && ok; k0 += 32) {
            const int k = k0 + lane;
            int row = -1;                                   // TMA row of the block's first head, -1 = bad
            bool last = false;
            if (k < n_units) {
                const UnitPos u = locate_unit(prefix, B, a + k);
                if (u.lb < p.max_blocks_per_seq) {
                    const int phys = p.block_tables[(size_t)u.s * p.max_blocks_per_seq + u.lb];
                    if (phys >= 0 && phys < p.num_blocks) row = phys * HKV * BS;
                }
                last = (u.lb == u.nb - 1);
            }
            const int cnt = min(32, n_units - k0);
            for (int jj = 0; jj < cnt; ++jj) {
                const int rw = __shfl_sync(FULL, row, jj);
                const bool lst = __shfl_sync(FULL, last, jj) != 0;
                if (lane == 0) {
                    if (p.pdl_wait_last && lst) pdl_wait();   // the block holding the appended token
#pragma unroll
                    for (int kv = 0; kv < 2; ++kv) {
                        const int j = 2 * (k0 + jj) + kv, st = j % NST;
                        if (ok && j >= NST) ok = mbar_wait_bounded(&empty_bar[st], ((j / NST) - 1) & 1);
                        if (ok && *abort_flag) ok = false;
                        if (ok) {
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
            }
        }
        if (lane == 0 && !ok) {
            if (!*abort_flag) record_error(PA_DEVERR_TIMEOUT);
            *abort_flag = 1;
            for (int j = max(0, issued - NST); j < issued; ++j)
                mbar_wait_bounded(&full_bar[j % NST], (j / NST) & 1);
        }
    } else if (n_units > 0) {
        // ------------------------------ consumers ------------------------------
        const int kvh = warp;
        const int tq = lane & 3, r = lane >> 2;
        const int mrow = lane & 7, mat = lane >> 3;         // ldmatrix: row address this lane supplies
        const uint32_t ring_s = smem_addr(ring);
        float m_run[2], l_run[2];
        float o[C::MT][4];
        uint32_t qb[C::KS][2], qn[C::KS][2];
        int x = a;
        int k = 0;                                          // unit index within the range
        UnitPos cur = locate_unit(prefix, B, x);
        mma_load_q<C, G, D>(qb, p.q + ((size_t)cur.s * HQ + (size_t)kvh * G) * D, lane);
        int ctx_cur = p.context_lens[cur.s];
        while (x < b) {
            const int gstart = x - cur.lb, gend = gstart + cur.nb;
            const int seg_end = gend < b ? gend : b;
            const int n = seg_end - x;
            // the next sequence's q and context length load while this one runs
            const bool has_next = seg_end < b;
            UnitPos nxt = cur;
            int ctx_next = 0;
            if (has_next) {
                nxt = locate_unit(prefix, B, seg_end);
                mma_load_q<C, G, D>(qn, p.q + ((size_t)nxt.s * HQ + (size_t)kvh * G) * D, lane);
                ctx_next = p.context_lens[nxt.s];
            }
            m_run[0] = m_run[1] = -INFINITY;
            l_run[0] = l_run[1] = 0.f;
#pragma unroll
            for (int mt = 0; mt < C::MT; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
            bool bad = false;

            for (int u = 0; u < n; ++u, ++k) {
                if (*abort_flag) continue;                  // keep walking the sequences, skip the work
                const int jk = 2 * k, stk = jk % NST, jv = jk + 1, stv = jv % NST;
                const int valid = min(BS, ctx_cur - (cur.lb + u) * BS);
                // ---- K stage: S^T = K . Q^T for every 16-token sub-block of the block ----
                if (!__all_sync(FULL, mbar_wait_bounded(&full_bar[stk], (jk / NST) & 1))) {
                    if (lane == 0) {
                        record_error(PA_DEVERR_TIMEOUT);
                        *abort_flag = 1;
                    }
                    continue;
                }
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
                    continue;
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
                            reinterpret_cast<uint4 *>(vhead + hf * C::HALF_BYTES + rr * 128)[e % 8] =
                                make_uint4(0, 0, 0, 0);
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
#pragma unroll
            for (int off = 4; off < 32; off <<= 1) {
                l_run[0] += __shfl_xor_sync(FULL, l_run[0], off);
                l_run[1] += __shfl_xor_sync(FULL, l_run[1], off);
            }

            // ---- this warp's (sequence, KV head): final rows or a partial ----
            const bool failed = bad || (*abort_flag != 0);
            const bool whole = (x == gstart) && (seg_end == gend);
            const size_t row0 = (size_t)cur.s * HQ + (size_t)kvh * G;
            if (whole) {
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
            } else {
                const int slot = (x == a) ? 0 : 1;          // first sequence of the range, else the last
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int h = 2 * tq + j;
                    if (h < G) {
                        const size_t ps = ((size_t)c * 2 + slot) * HQ + (size_t)kvh * G + h;
                        float *po = p.part_o + ps * D;
#pragma unroll
                        for (int mt = 0; mt < C::MT; ++mt) {
                            po[16 * mt + r] = failed ? __int_as_float(0x7fc00000) : o[mt][j];
                            po[16 * mt + r + 8] = failed ? __int_as_float(0x7fc00000) : o[mt][2 + j];
                        }
                        if (r == 0) {
                            p.part_ml[ps * 2] = failed ? 0.f : m_run[j];
                            p.part_ml[ps * 2 + 1] = failed ? __int_as_float(0x7fc00000) : l_run[j];
                        }
                    }
                }
                // publish: the warp's writes, then one device-scope fence and the counter
                // update by lane 0 (release); the warp that completes the count fences again
                // before reading the other CTAs' partials (acquire)
                __syncwarp();
                const int c0 = cta_of_block(gstart, T, Ce), c1 = cta_of_block(gend - 1, T, Ce);
                int last = 0;
                if (lane == 0) {
                    int *cnt = p.counters + (size_t)cur.s * HKV + kvh;
                    __threadfence();
                    const int prev = atomicAdd(cnt, 1);
                    last = (prev == c1 - c0);
                    if (last) {
                        *cnt = 0;                           // every contributing CTA has counted
                        __threadfence();
                    }
                }
                last = __shfl_sync(FULL, last, 0);
                if (last) allheads_merge<D, G, HQ>(p, cur.s, kvh, c0, c1, gstart, T, Ce, lane);
            }
            // ---- next sequence ----
            x = seg_end;
            if (has_next) {
                cur = nxt;
                ctx_cur = ctx_next;
#pragma unroll
                for (int ks = 0; ks < C::KS; ++ks) {
                    qb[ks][0] = qn[ks][0];
                    qb[ks][1] = qn[ks][1];
                }
            }
        }
    }
    __syncthreads();
}

}  // namespace pa
