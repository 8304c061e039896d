// decode_balanced.cuh -- bf16 paged decode with a block-balanced persistent schedule.
//
// Same attention as the partition kernels (decode.cuh / decode_mma.cuh), scheduled
// differently.  Fixed-size context partitions give every CTA a whole number of ~equal
// items; with a few hundred resident CTAs and a few thousand items the last wave leaves
// SMs idle (about 1/8 of the kernel for 64 sequences of 512..4096 tokens).  Here the
// launch has exactly as many CTAs as fit on the GPU at once, and CTA c takes the blocks
// [c*T/C, (c+1)*T/C) of the whole step, T being the number of (KV head, sequence, block)
// triples (see locate_block for the order).  Every CTA therefore moves the same number of
// blocks and they finish together.
//
// Inside a CTA the producer warp streams the range's blocks through the stage ring
// without a pause at group boundaries (a group = one (sequence, KV head)); consumer warps
// take blocks k = w (mod NW) as before, finish a group together (named barrier), merge
// their states, and write:
//   * the final bf16 rows, when the whole group lies inside this CTA's range;
//   * otherwise a partial (m, l, o) in one of the CTA's two partial slots (slot 0 for the
//     first group of the range, slot 1 for the last).  The CTA that completes the group's
//     count of contributing CTAs merges the partials and resets the counter.  No CTA ever
//     waits for another.
// The per-sequence block prefix sums that define the ranges are computed by every CTA
// from context_lens (at most kBalancedMaxSeqs sequences, kept in shared memory).
#pragma once

#include "decode_mma.cuh"

namespace pa {

constexpr int kBalancedMaxSeqs = 4096;   // sequences per launch (prefix sums in shared memory)
constexpr int kBalancedMaxCtas = 1024;   // the workspace holds partial slots for this many CTAs
constexpr int kBalancedMaxGroup = 8;     // partial slots are sized for up to 8 query heads per KV head

struct BalancedParams {
    __nv_bfloat16 *out;            // [B][h_q][D]
    const __nv_bfloat16 *q;        // [B][h_q][D]
    const int32_t *block_tables;   // [B][max_blocks_per_seq]
    const int32_t *context_lens;   // [B]
    int *counters;                 // [B][h_kv] contributing CTAs seen; zero between launches
    float *part_ml;                // [num_ctas][2][G][2]  (m, l), log2 domain
    float *part_o;                 // [num_ctas][2][G][D]  unnormalised
    int max_blocks_per_seq;
    int num_seqs;
    int h_q;
    int h_kv;
    int num_blocks;
    int num_ctas;                  // C: gridDim.x
    float qk_scale;                // scale * log2(e)
    int pdl_wait;                  // launched right after the cache write: wait for it before loading
};

// NW_ consumer warps, RING_ bytes of stage ring, MINB_ = CTAs per SM the register budget
// must allow (0: no bound).
template <int D, int BS, int G, int NW_ = 2, int RING_ = 32768, int MINB_ = 0>
struct BalancedConfig {
    using M = MmaDecodeConfig<D, BS, G, NW_, RING_>;
    static constexpr int NW = NW_;
    static constexpr int THREADS = (NW + 1) * 32;
    static constexpr int CONS = NW * 32;                        // consumer threads
    static constexpr int OFF_BARS = M::RING;                    // after the 1024-aligned ring
    static constexpr int OFF_FLAGS = OFF_BARS + 2 * M::STAGES * 8;
    static constexpr int N_FLAGS = M::STAGES + 8 + 8;           // stage flags, state flags, scan scratch
    static constexpr int OFF_COMB = (OFF_FLAGS + N_FLAGS * 4 + 15) / 16 * 16;
    static constexpr int COMB_FLOATS = NW * G * (D + 2);        // o [NW][G][D], m [NW][G], l [NW][G]
    static constexpr int OFF_SCR = OFF_COMB + COMB_FLOATS * 4;  // merge scratch: M[G], 1/L[G]
    static constexpr int OFF_PREFIX = OFF_SCR + 2 * G * 4;
    // dynamic shared memory for num_seqs sequences (+1024 to align the ring)
    __host__ __device__ static constexpr int smem_bytes(int num_seqs) { return OFF_PREFIX + (num_seqs + 1) * 4 + 1024; }
    static_assert(G <= kBalancedMaxGroup, "group");
};

__device__ __forceinline__ void named_barrier_sync(int id, int threads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// prefix[s] = sum over s' < s of ceil(ctx[s'] / bs) (negative contexts count as 0),
// prefix[n] = the total.  All threads of the CTA take part; `scan` holds 32 ints.
template <int THREADS>
__device__ __forceinline__ void block_prefix(int *prefix, int *scan, const int32_t *ctx, int n, int bs)
{
    const int per = (n + THREADS - 1) / THREADS;
    const int lo = min(n, (int)threadIdx.x * per), hi = min(n, lo + per);
    int sum = 0;
    for (int i = lo; i < hi; ++i) {
        const int c = ctx[i];
        const int nb = c > 0 ? (c + bs - 1) / bs : 0;
        prefix[i] = nb;
        sum += nb;
    }
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
    }
    if (lane == 31) scan[warp] = incl;
    __syncthreads();
    int base = 0;
    for (int w = 0; w < warp; ++w) base += scan[w];
    int off = base + incl - sum;
    for (int i = lo; i < hi; ++i) {
        const int nb = prefix[i];
        prefix[i] = off;
        off += nb;
    }
    if (threadIdx.x == THREADS - 1) {
        int total = 0;
        for (int w = 0; w < THREADS / 32; ++w) total += scan[w];
        prefix[n] = total;
    }
    __syncthreads();
}

// The flat block space is laid out KV head by KV head, sequence by sequence within a head:
// x = kvh * S + prefix[s] + lb with S = prefix[num_seqs].  With C a multiple of h_kv, CTAs
// c and c + C/h_kv then sit at the same offset of their heads' slices, so the CTAs reading
// the h_kv tiles of one physical block (adjacent in memory) do so at about the same time.
// Returns the group of x: sequence s, KV head kvh, block lb within the sequence, and the
// sequence's block count nb (> 0).
struct FlatPos {
    int s, kvh, lb, nb;
};

__device__ __forceinline__ FlatPos locate_block(const int *prefix, int num_seqs, int h_kv, long long x)
{
    const int S = prefix[num_seqs];
    FlatPos f;
    f.kvh = (int)(x / S);
    const int r = (int)(x - (long long)f.kvh * S);
    int lo = 0, hi = num_seqs - 1;               // last s with prefix[s] <= r
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (prefix[mid] <= r) lo = mid;
        else hi = mid - 1;
    }
    f.s = lo;
    f.nb = prefix[lo + 1] - prefix[lo];
    f.lb = r - prefix[lo];
    return f;
}

// CTA whose range holds flat block x: the largest c with floor(c T / C) <= x (C <= T).
__host__ __device__ __forceinline__ int cta_of_block(long long x, long long total, int num_ctas)
{
    return (int)(((x + 1) * num_ctas - 1) / total);
}

template <int D, int BS, int G, int NW_ = 2, int RING_ = 32768, int MINB_ = 0>
__global__ void __launch_bounds__(BalancedConfig<D, BS, G, NW_, RING_, MINB_>::THREADS, MINB_)
    paged_decode_balanced_kernel(const BalancedParams p, const __grid_constant__ CUtensorMap tmap_k,
                                 const __grid_constant__ CUtensorMap tmap_v)
{
    using BC = BalancedConfig<D, BS, G, NW_, RING_, MINB_>;
    using M = typename BC::M;
    constexpr int NW = NW_, STAGES = M::STAGES, CONS = BC::CONS;
    constexpr unsigned FULL = 0xffffffffu;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *ring = smem;
    uint64_t *full_bar = reinterpret_cast<uint64_t *>(smem + BC::OFF_BARS);
    uint64_t *empty_bar = full_bar + STAGES;
    volatile int *stage_bad = reinterpret_cast<volatile int *>(smem + BC::OFF_FLAGS);
    volatile int *abort_flag = stage_bad + STAGES;
    volatile int *grp_bad = stage_bad + STAGES + 1;      // [2]: by group parity
    volatile int *last_flag = stage_bad + STAGES + 3;
    int *scan = const_cast<int *>(stage_bad + STAGES + 8);
    float *comb = reinterpret_cast<float *>(smem + BC::OFF_COMB);
    float *scr = reinterpret_cast<float *>(smem + BC::OFF_SCR);
    int *prefix = reinterpret_cast<int *>(smem + BC::OFF_PREFIX);

    const int B = p.num_seqs, HKV = p.h_kv, Cn = p.num_ctas, c = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    block_prefix<BC::THREADS>(prefix, scan, p.context_lens, B, BS);
    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(&full_bar[i], 1);
            mbar_init(&empty_bar[i], 1);
        }
        *abort_flag = 0;
        grp_bad[0] = grp_bad[1] = 0;
        mbar_init_fence();
    }
    // groups of empty sequences get zero rows (one writer per group)
    for (int g = c; g < B * HKV; g += Cn) {
        const int s = g / HKV;
        if (prefix[s + 1] == prefix[s]) {
            __nv_bfloat16 *row = p.out + ((size_t)s * p.h_q + (size_t)(g % HKV) * G) * D;
            for (int i = threadIdx.x; i < G * D; i += blockDim.x) row[i] = __float2bfloat16_rn(0.f);
        }
    }
    __syncthreads();

    // ranges over Ce = min(C, T) CTAs, so that every range that exists is non-empty and the
    // CTAs holding a group's blocks are exactly cta_of_block(first) .. cta_of_block(last)
    const long long T = (long long)HKV * prefix[B];
    const int Ce = (int)(T < Cn ? T : Cn);
    const long long a = c < Ce ? (long long)c * T / Ce : 0, b = c < Ce ? (long long)(c + 1) * T / Ce : 0;
    const int n_blk = (int)(b - a);

    if (warp == NW) {
        // ------------------------------ producer ------------------------------
        if (lane == 0) {
            prefetch_tensormap(&tmap_k);
            prefetch_tensormap(&tmap_v);
            if (p.pdl_wait) pdl_wait();
        }
        const uint64_t pol = l2_policy_evict_first();
        int issued = 0;
        bool ok = true;
        for (int k0 = 0; k0 < n_blk && ok; k0 += 32) {
            const int k = k0 + lane;
            int row = -1;                                   // TMA row of the block's tile, -1 = bad
            if (k < n_blk) {
                const FlatPos f = locate_block(prefix, B, HKV, a + k);
                if (f.lb < p.max_blocks_per_seq) {
                    const int phys = p.block_tables[(size_t)f.s * p.max_blocks_per_seq + f.lb];
                    if (phys >= 0 && phys < p.num_blocks) row = (phys * HKV + f.kvh) * BS;
                }
            }
            const int cnt = min(32, n_blk - k0);
            for (int j = 0; j < cnt; ++j) {
                const int rw = __shfl_sync(FULL, row, j);
                const int kk = k0 + j;
                const int st = kk % STAGES;
                if (lane == 0) {
                    if (kk >= STAGES) ok = mbar_wait_bounded(&empty_bar[st], ((kk / STAGES) - 1) & 1);
                    if (ok && *abort_flag) ok = false;
                    if (ok) {
                        if (rw >= 0) {
                            stage_bad[st] = 0;
                            mbar_arrive_expect_tx(&full_bar[st], M::STAGE_BYTES);
                            uint8_t *dst = ring + st * M::STAGE_BYTES;
#pragma unroll
                            for (int hf = 0; hf < M::HALVES; ++hf) {
                                tma_load_2d(dst + hf * M::HALF_BYTES, &tmap_k, hf * 64, rw, &full_bar[st], pol);
                                tma_load_2d(dst + M::TILE + hf * M::HALF_BYTES, &tmap_v, hf * 64, rw, &full_bar[st], pol);
                            }
                        } else {
                            stage_bad[st] = 1;
                            record_error(PA_DEVERR_BAD_BLOCK);
                            mbar_arrive(&full_bar[st]);
                        }
                        issued = kk + 1;
                    }
                }
                ok = __shfl_sync(FULL, ok, 0) != 0;
                if (!ok) break;
            }
        }
        if (lane == 0 && !ok) {
            if (!*abort_flag) record_error(PA_DEVERR_TIMEOUT);
            *abort_flag = 1;
            for (int kk = max(0, issued - STAGES); kk < issued; ++kk)
                mbar_wait_bounded(&full_bar[kk % STAGES], (kk / STAGES) & 1);
        }
    } else if (n_blk > 0) {
        // ------------------------------ consumers ------------------------------
        const int ctid = threadIdx.x;                       // 0 .. CONS-1
        const int tq = lane & 3, r = lane >> 2;
        float m_run[2], l_run[2];
        float o[M::MT][4];
        uint32_t qb[M::KS][2], qn[M::KS][2];
        long long x = a;
        int kbase = 0;
        FlatPos cur = locate_block(prefix, B, HKV, x);
        mma_load_q<M, G, D>(qb, p.q + ((size_t)cur.s * p.h_q + (size_t)cur.kvh * G) * D, lane);
        int ctx_cur = p.context_lens[cur.s];
        int gi = 0;                                         // group number within the range
        while (x < b) {
            const long long gstart = x - cur.lb, gend = gstart + cur.nb;
            const long long seg_end = gend < b ? gend : b;
            const int n = (int)(seg_end - x);
            // prefetch the next group's q and context length while this one runs
            const bool has_next = seg_end < b;
            FlatPos nxt = cur;
            int ctx_next = 0;
            if (has_next) {
                nxt = locate_block(prefix, B, HKV, seg_end);
                mma_load_q<M, G, D>(qn, p.q + ((size_t)nxt.s * p.h_q + (size_t)nxt.kvh * G) * D, lane);
                ctx_next = p.context_lens[nxt.s];
            }
            m_run[0] = m_run[1] = -INFINITY;
            l_run[0] = l_run[1] = 0.f;
#pragma unroll
            for (int mt = 0; mt < M::MT; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;

            for (int k = kbase + (((warp - kbase) % NW) + NW) % NW; k < kbase + n; k += NW) {
                if (*abort_flag) continue;                  // keep walking the groups, skip the work
                const int st = k % STAGES;
                const bool ok = __all_sync(FULL, mbar_wait_bounded(&full_bar[st], (k / STAGES) & 1));
                if (!ok) {
                    if (lane == 0) {
                        record_error(PA_DEVERR_TIMEOUT);
                        *abort_flag = 1;
                    }
                    continue;
                }
                if (stage_bad[st]) {
                    if (lane == 0) grp_bad[gi & 1] = 1;
                } else {
                    const int lb = cur.lb + (k - kbase);
                    mma_consume_block<M, BS, G>(ring + st * M::STAGE_BYTES, min(BS, ctx_cur - lb * BS), qb,
                                                p.qk_scale, m_run, l_run, o, lane);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty_bar[st]);
            }
#pragma unroll
            for (int off = 4; off < 32; off <<= 1) {
                l_run[0] += __shfl_xor_sync(FULL, l_run[0], off);
                l_run[1] += __shfl_xor_sync(FULL, l_run[1], off);
            }
            // ---- deposit this warp's state: o [NW][G][D], m [NW][G], l [NW][G] ----
            float *cm = comb + NW * G * D;
            float *cl = cm + NW * G;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int h = 2 * tq + j;
                if (h < G) {
                    if (r == 0) {
                        cm[warp * G + h] = m_run[j];
                        cl[warp * G + h] = l_run[j];
                    }
#pragma unroll
                    for (int mt = 0; mt < M::MT; ++mt) {
                        comb[(warp * G + h) * D + 16 * mt + r] = o[mt][j];
                        comb[(warp * G + h) * D + 16 * mt + r + 8] = o[mt][2 + j];
                    }
                }
            }
            named_barrier_sync(1, CONS);
            const bool failed = (*abort_flag != 0) || (grp_bad[gi & 1] != 0);
            const bool whole = (cur.lb == 0) && (seg_end == gend);
            const int slot = (x == a) ? 0 : 1;              // first group of the range, else the last
            const size_t qrow0 = (size_t)cur.s * p.h_q + (size_t)cur.kvh * G;
            for (int idx = ctid; idx < G * D; idx += CONS) {
                const int h = idx / D, dd = idx % D;
                float Mx = -INFINITY;
#pragma unroll
                for (int w = 0; w < NW; ++w) Mx = fmaxf(Mx, cm[w * G + h]);
                float L = 0.f, O = 0.f;
#pragma unroll
                for (int w = 0; w < NW; ++w) {
                    const float sc = cm[w * G + h] == -INFINITY ? 0.f : exp2f(cm[w * G + h] - Mx);
                    L += cl[w * G + h] * sc;
                    O += comb[(w * G + h) * D + dd] * sc;
                }
                if (whole) {
                    const float res = failed ? __int_as_float(0x7fc00000) : O / L;
                    p.out[(qrow0 + h) * D + dd] = __float2bfloat16_rn(res);
                } else {
                    const size_t ps = ((size_t)c * 2 + slot) * G + h;
                    p.part_o[ps * D + dd] = failed ? __int_as_float(0x7fc00000) : O;
                    if (dd == 0) {
                        p.part_ml[ps * 2] = Mx;
                        p.part_ml[ps * 2 + 1] = failed ? __int_as_float(0x7fc00000) : L;
                    }
                }
            }
            if (ctid == 0) grp_bad[(gi + 1) & 1] = 0;       // no warp is in the next group yet
            named_barrier_sync(1, CONS);                    // combine area free; partial written
            if (!whole) {
                const int g = cur.s * HKV + cur.kvh;
                const int c0 = cta_of_block(gstart, T, Ce), c1 = cta_of_block(gend - 1, T, Ce);
                if (ctid == 0) {
                    __threadfence();                        // this CTA's partial, device-wide
                    const int prev = atomicAdd(p.counters + g, 1);
                    const int last = (prev == c1 - c0);
                    if (last) p.counters[g] = 0;
                    *last_flag = last;
                    if (last) __threadfence();              // the others' partials before our reads
                }
                named_barrier_sync(1, CONS);
                if (*last_flag) {
                    // merge the contributing CTAs' partials: CTA c > c0 holds it in slot 0;
                    // c0 in slot 0 when the group starts its range, else in slot 1
                    const long long a0 = (long long)c0 * T / Ce;
                    const int slot0 = (gstart == a0) ? 0 : 1;
                    if (ctid < G) {
                        const int h = ctid;
                        float Mx = -INFINITY;
                        for (int cc = c0; cc <= c1; ++cc) {
                            const size_t ps = ((size_t)cc * 2 + (cc == c0 ? slot0 : 0)) * G + h;
                            Mx = fmaxf(Mx, __ldcg(p.part_ml + ps * 2));
                        }
                        float L = 0.f;
                        for (int cc = c0; cc <= c1; ++cc) {
                            const size_t ps = ((size_t)cc * 2 + (cc == c0 ? slot0 : 0)) * G + h;
                            L += exp2f(__ldcg(p.part_ml + ps * 2) - Mx) * __ldcg(p.part_ml + ps * 2 + 1);
                        }
                        scr[h] = Mx;
                        scr[G + h] = 1.f / L;
                    }
                    named_barrier_sync(1, CONS);
                    for (int idx = ctid; idx < G * D / 4; idx += CONS) {
                        const int h = idx / (D / 4), d4 = idx % (D / 4);
                        const float Mx = scr[h], invL = scr[G + h];
                        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
                        for (int cc = c0; cc <= c1; ++cc) {
                            const size_t ps = ((size_t)cc * 2 + (cc == c0 ? slot0 : 0)) * G + h;
                            const float w = exp2f(__ldcg(p.part_ml + ps * 2) - Mx) * invL;
                            const float4 v = __ldcg(reinterpret_cast<const float4 *>(p.part_o + ps * D + 4 * d4));
                            acc.x += w * v.x; acc.y += w * v.y; acc.z += w * v.z; acc.w += w * v.w;
                        }
                        *reinterpret_cast<uint2 *>(p.out + (qrow0 + h) * D + 4 * d4) =
                            make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
                    }
                    named_barrier_sync(1, CONS);            // scratch reusable
                }
            }
            // ---- next group ----
            x = seg_end;
            kbase += n;
            ++gi;
            if (has_next) {
                cur = nxt;
                ctx_cur = ctx_next;
#pragma unroll
                for (int ks = 0; ks < M::KS; ++ks) {
                    qb[ks][0] = qn[ks][0];
                    qb[ks][1] = qn[ks][1];
                }
            }
        }
    }
    __syncthreads();
}

}  // namespace pa
