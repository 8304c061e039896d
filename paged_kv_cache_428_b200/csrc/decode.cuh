// decode.cuh -- single-query (decode-step) attention over a paged KV cache.
//
//   out[s][h] = softmax(scale * q[s][h] . K_s^T) . V_s              (fp32 accumulation)
// with K_s / V_s the first ctx[s] tokens of sequence s, token t in physical block
// block_tables[s][t / bs] at offset t % bs, and query head h reading KV head h / G.
// ("现代 AI 的“推理加速之谜”…" section 1, attention formula and KV caching;
//  "深度解构 LLM 推理优化…" section 2.1, block table; "vLLM 推理原理…" section
//  "PagedAttention 怎样整理这些缓存", logical -> physical blocks, partly filled last block;
//  section 3.A of the first page and section 1.1 of the second: GQA head groups.)
//
// Pass 1 (partition kernel): one CTA per (context partition, KV head, sequence) serves
// the whole query-head group G of that KV head, so every K/V byte is read from HBM once
// per step.  Warp NW (the producer) reads the partition's block-table entries and issues,
// per physical block, two 1-D bulk copies (TMA engine, no tensor map, no multicast): the
// block's K tile and V tile, each one contiguous span of bs*d elements in the
// [NB][H_kv][bs][d] layout.  They land in a ring of STAGES shared-memory stages guarded
// by full/empty mbarriers.  Consumer warps 0..NW-1 take whole blocks in turn and keep
// their own online-softmax state (running max m, running sum l, unnormalised o), working
// in the log2 domain (scores pre-multiplied by log2 e).  The CTA then merges its warps.
// A sequence that fits one partition is finished here (bf16 out); otherwise the CTA
// writes its partial (m, l, o) to the workspace.
// Pass 2 (merge kernel): per (sequence, query head) combine the partials:
//   M = max_p m_p,  out = sum_p 2^(m_p - M) o_p / sum_p 2^(m_p - M) l_p.
//
// Consumer warp work split for one 16-token sub-block (all index maps are compile-time):
//   q.K   : LPT lanes per token, each owning CPL 16-byte chunks of the row (fp32 FMAs,
//           packed two-wide with __ffma2_rn); the G*PS partial dot products of a lane are
//           summed across its LPT lanes with a transposed butterfly (each step halves the
//           values a lane keeps), so shuffles are shared between heads and passes.
//   softmax: per-head max by butterflies over the lanes holding other tokens of the head.
//   p.V   : lane owns D/32 output dims for all G heads; p and the rescale factors go
//           through a per-warp shared-memory slice and are read as broadcasts.
#pragma once

#include "common.cuh"

namespace pa {

struct DecodeParams {
    __nv_bfloat16 *out;            // [B][h_q][D]
    const __nv_bfloat16 *q;        // [B][h_q][D]
    const uint8_t *k_cache;        // [NB][h_kv][bs][D] elements
    const uint8_t *v_cache;
    const int32_t *block_tables;   // [B][max_blocks_per_seq]
    const int32_t *context_lens;   // [B]
    float *ws_ml;                  // [B][h_q][p_max][2]  (m, l), log2 domain
    float *ws_o;                   // [B][h_q][p_max][D]  unnormalised, v_scale applied
    int *counters;                 // [B][h_kv] partitions finished; zero between launches
    int max_blocks_per_seq;
    int h_q;
    int h_kv;
    int num_blocks;
    int partition_size;            // tokens per partition, 0 = whole context
    int p_max;                     // partitions per sequence in the grid
    float qk_scale;                // scale * log2(e) (* the per-tensor k_scale of a quantised cache)
    float v_scale;                 // per-tensor V scale (1 for bf16)
    const float *k_scales;         // per-KV-head scales [h_kv] of a quantised cache, or null
    const float *v_scales;         //   (then qk_scale holds no K scale and v_scale is unused)
    int pdl_wait_last;             // launched right after the cache write of each sequence's
                                   // appended token: wait for it before loading a sequence's last block
};

// Factors of KV head kvh: the K scale folded into the logit scale and the V scale.
__device__ __forceinline__ float head_k_factor(const DecodeParams &p, int kvh)
{
    return p.k_scales ? __ldg(p.k_scales + kvh) : 1.f;
}
__device__ __forceinline__ float head_v_scale(const DecodeParams &p, int kvh)
{
    return p.v_scales ? __ldg(p.v_scales + kvh) : p.v_scale;
}

// Groups (sequence, KV head) with at most this many partitions are merged inside the
// partition kernel by the CTA that finishes last; larger groups go to the merge kernel,
// whose many CTAs keep more partial reads in flight than one CTA could.
constexpr int kFusedMergeMaxPartitions = 16;

__host__ __device__ __forceinline__ int decode_num_partitions(int ctx, int partition_size, int p_max)
{
    if (partition_size <= 0) return 1;
    int n = (ctx + partition_size - 1) / partition_size;
    if (n < 1) n = 1;
    return n < p_max ? n : p_max;
}

template <int D, int BS, int G, bool FP8>
struct DecodeShape {
    static constexpr int ELEM = FP8 ? 1 : 2;
    static constexpr int CHUNK = 16 / ELEM;        // elements per 16-byte chunk
    static constexpr int CPR = D / CHUNK;          // chunks per K row
    static constexpr int LPT = cmin(CPR, 8);       // lanes per token in q.K
    static constexpr int CPL = CPR / LPT;          // chunks per lane
    static constexpr int TPP = 32 / LPT;           // tokens per pass
    static constexpr int SUBT = 16;                // tokens per softmax sub-block
    static constexpr int NSUB = BS / SUBT;
    static constexpr int PS = SUBT / TPP;          // passes per sub-block
    static constexpr int DPL = D / 32;             // output dims per lane in p.V
    static constexpr int TILE = BS * D * ELEM;     // bytes of one (block, head) K tile
    static constexpr int ROW = D * ELEM;           // bytes of one token row
    static constexpr int QD = CPL * CHUNK;         // q dims per lane
    static constexpr int LOG_LPT = Log2<LPT>::value;
    static constexpr int LOG_G = Log2<G>::value;
    static constexpr int LOG_PS = Log2<PS>::value;
    static constexpr int U = G * PS;               // partial dots per lane, u = h*PS + pass
    static constexpr int UB = LOG_G + LOG_PS;
    static constexpr int HL = cmin(LOG_LPT, UB);   // butterfly levels that halve the values
    static constexpr int NF = 1 << (UB - HL);      // values a lane keeps after the reduction
    static constexpr int RPB = cmin(UB - HL, LOG_PS);   // pass bits kept in registers
    static constexpr int NH = 1 << (UB - HL - RPB);     // heads kept in registers
    static_assert(BS % SUBT == 0, "block size must be a multiple of 16");
    static_assert(CPR % LPT == 0, "row chunks must split evenly");
};

// Transposed butterfly: v[0..N) partial sums of N different outputs over the lanes
// whose lane index differs in bits OFF, OFF/2, ..., 1.  While N > 1 each level keeps the
// lower or upper half (by the lane bit) and adds the partner's copy of that half;
// afterwards plain butterflies finish.  On return v[0..max(1, N >> levels)) hold totals.
template <int N, int OFF>
__device__ __forceinline__ void transposed_reduce(float *v, int c)
{
    if constexpr (OFF >= 1) {
        if constexpr (N > 1) {
            const bool upper = (c & OFF) != 0;
#pragma unroll
            for (int f = 0; f < N / 2; ++f) {
                const float send = upper ? v[f] : v[f + N / 2];
                const float keep = upper ? v[f + N / 2] : v[f];
                v[f] = keep + __shfl_xor_sync(0xffffffffu, send, OFF);
            }
            transposed_reduce<N / 2, OFF / 2>(v, c);
        } else {
            v[0] += __shfl_xor_sync(0xffffffffu, v[0], OFF);
            transposed_reduce<1, OFF / 2>(v, c);
        }
    }
}

// Index (u) of the first value a lane keeps after transposed_reduce<N, OFF>.
template <int N, int OFF>
__device__ __forceinline__ int transposed_base(int c)
{
    if constexpr (OFF >= 1 && N > 1) {
        return ((c & OFF) ? N / 2 : 0) + transposed_base<N / 2, OFF / 2>(c);
    } else {
        return 0;
    }
}

template <int D, int BS, int G, bool FP8>
struct DecodeConfig {
    using S = DecodeShape<D, BS, G, FP8>;
    static constexpr int NW = 4;                                   // consumer warps
    static constexpr int THREADS = (NW + 1) * 32;                  // + producer warp
    // a multiple of NW (see MmaDecodeConfig: parity waits are safe only when block i and
    // block i - STAGES, which share a stage, belong to the same consumer warp)
    static constexpr int STAGES = cmax(NW, cmin(16, 98304 / (2 * S::TILE)) / NW * NW);
    static_assert(STAGES % NW == 0, "stage ring must be a multiple of the consumer warps");
    static constexpr int STAGE_BYTES = STAGES * 2 * S::TILE;
    static constexpr int PBUF_FLOATS = ((S::SUBT * G + G) + 3) / 4 * 4;   // per warp
    static constexpr int COMBINE_BYTES = NW * G * (D + 2) * 4;
    static constexpr int MERGE_BYTES = (2 * G * kFusedMergeMaxPartitions + 1) * 4;
    static constexpr int REGION0 = cmax(STAGE_BYTES, COMBINE_BYTES + MERGE_BYTES);  // stages, then combine + merge
    static constexpr int OFF_BARS = (REGION0 + 127) / 128 * 128;
    static constexpr int OFF_FLAGS = OFF_BARS + 2 * STAGES * 8;
    static constexpr int OFF_PBUF = (OFF_FLAGS + (STAGES + 4) * 4 + 15) / 16 * 16;
    static constexpr int SMEM = OFF_PBUF + NW * PBUF_FLOATS * 4;
};

// Merge the per-warp online-softmax states of one CTA and write the result: the final bf16
// row when the sequence has a single partition, else this partition's (m, l, o) partial.
// Shared memory holds cm[NW][G] (running max, log2 domain), cl[NW][G] (running sum) and
// co[NW][G][D] (unnormalised output); a warp that saw no token has m = -inf, l = 0, o = 0.
// For a group of at most kFusedMergeMaxPartitions partitions, the CTA then publishes its
// partial (fence, then one atomic increment of the group's counter); the CTA that makes the
// count complete merges all partials of the group (out = sum_p 2^(m_p - M) o_p /
// sum_p 2^(m_p - M) l_p) and resets the counter to zero.  No CTA waits on another.
// `scratch` is shared memory for 2 * G * kFusedMergeMaxPartitions + 1 floats, not
// overlapping cm/cl/co.
template <int NW, int G, int D>
__device__ __forceinline__ void cta_combine_and_write(const DecodeParams &p, const float *cm, int part, int n_part,
                                                      int kvh, int seq, bool failed, float *scratch)
{
    const float *cl = cm + NW * G;
    const float *co = cl + NW * G;
    const float v_scale = head_v_scale(p, kvh);
    for (int idx = threadIdx.x; idx < G * D; idx += blockDim.x) {
        const int h = idx / D, dd = idx % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < NW; ++w) M = fmaxf(M, cm[w * G + h]);
        float L = 0.f, O = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < NW; ++w) {
                const float sc = exp2f(cm[w * G + h] - M);
                L += cl[w * G + h] * sc;
                O += co[(w * G + h) * D + dd] * sc;
            }
        }
        const size_t qrow = (size_t)seq * p.h_q + (size_t)kvh * G + h;
        if (n_part == 1) {
            float r = L > 0.f ? (O / L) * v_scale : 0.f;
            if (failed) r = __int_as_float(0x7fc00000);
            p.out[qrow * D + dd] = __float2bfloat16_rn(r);
        } else {
            const size_t prow = qrow * p.p_max + part;
            p.ws_o[prow * D + dd] = failed ? __int_as_float(0x7fc00000) : O * v_scale;
            if (dd == 0) {
                p.ws_ml[prow * 2] = M;
                p.ws_ml[prow * 2 + 1] = failed ? __int_as_float(0x7fc00000) : L;
            }
        }
    }
    if (n_part == 1 || n_part > kFusedMergeMaxPartitions) return;

    // ---- publish this partial; the last CTA of the group merges ----
    // The CTA barrier orders every thread's partial writes before thread 0's device-scope
    // fence, which publishes them before the counter update (release); the CTA that sees
    // the count complete fences again before its threads read the other partials (acquire).
    int *last = reinterpret_cast<int *>(scratch + 2 * G * kFusedMergeMaxPartitions);
    __syncthreads();
    if (threadIdx.x == 0) {
        int *cnt = p.counters + (size_t)seq * p.h_kv + kvh;
        __threadfence();
        const int prev = atomicAdd(cnt, 1);
        const int is_last = (prev == n_part - 1);
        if (is_last) {
            *cnt = 0;                      // every partition of this launch has counted
            __threadfence();
        }
        *last = is_last;
    }
    __syncthreads();
    if (!*last) return;
    float *mw = scratch;                                         // [G][16] m_p, then weights
    float *lw = scratch + G * kFusedMergeMaxPartitions;          // [G][16] l_p
    const size_t row0 = (size_t)seq * p.h_q + (size_t)kvh * G;
    for (int idx = threadIdx.x; idx < G * n_part; idx += blockDim.x) {
        const int h = idx / n_part, q = idx % n_part;
        const float2 ml = __ldcg(reinterpret_cast<const float2 *>(p.ws_ml + ((row0 + h) * p.p_max + q) * 2));
        mw[h * kFusedMergeMaxPartitions + q] = ml.x;
        lw[h * kFusedMergeMaxPartitions + q] = ml.y;
    }
    __syncthreads();
    if (threadIdx.x < G) {
        const int h = threadIdx.x;
        float M = -INFINITY;
        for (int q = 0; q < n_part; ++q) M = fmaxf(M, mw[h * kFusedMergeMaxPartitions + q]);
        float L = 0.f;
        for (int q = 0; q < n_part; ++q) {
            const float w = exp2f(mw[h * kFusedMergeMaxPartitions + q] - M);
            mw[h * kFusedMergeMaxPartitions + q] = w;
            L += w * lw[h * kFusedMergeMaxPartitions + q];
        }
        const float inv = 1.f / L;
        for (int q = 0; q < n_part; ++q) mw[h * kFusedMergeMaxPartitions + q] *= inv;
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < G * D / 4; idx += blockDim.x) {
        const int h = idx / (D / 4), d4 = idx % (D / 4);
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        const float *po = p.ws_o + (row0 + h) * p.p_max * D + 4 * d4;
        // partials in rounds of four whose loads are issued together, summed in partition order
        constexpr int R = 4;
        for (int q0 = 0; q0 < n_part; q0 += R) {
            float4 x[R];
#pragma unroll
            for (int u = 0; u < R; ++u)
                if (q0 + u < n_part) x[u] = __ldcg(reinterpret_cast<const float4 *>(po + (size_t)(q0 + u) * D));
#pragma unroll
            for (int u = 0; u < R; ++u) {
                if (q0 + u < n_part) {
                    const float w = mw[h * kFusedMergeMaxPartitions + q0 + u];
                    acc.x += w * x[u].x; acc.y += w * x[u].y; acc.z += w * x[u].z; acc.w += w * x[u].w;
                }
            }
        }
        __nv_bfloat16 *dst = p.out + (row0 + h) * D + 4 * d4;
        *reinterpret_cast<uint2 *>(dst) = make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
    }
}

template <int D, int BS, int G, bool FP8>
__device__ __forceinline__ void load_row_chunk(const uint8_t *p, float2 (&out)[16 / (FP8 ? 1 : 2) / 2])
{
    const uint4 raw = *reinterpret_cast<const uint4 *>(p);
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
    if constexpr (FP8) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            out[2 * i] = e4m3x2_to_float2(w[i] & 0xffffu);
            out[2 * i + 1] = e4m3x2_to_float2(w[i] >> 16);
        }
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) out[i] = bf16x2_to_float2(w[i]);
    }
}

// DPL consecutive V elements of one token -> DPL/2 float2.
template <int DPL, bool FP8>
__device__ __forceinline__ void load_v_elems(const uint8_t *p, float2 (&out)[DPL / 2])
{
    if constexpr (!FP8) {
        if constexpr (DPL == 4) {
            const uint2 r = *reinterpret_cast<const uint2 *>(p);
            out[0] = bf16x2_to_float2(r.x);
            out[1] = bf16x2_to_float2(r.y);
        } else {
            out[0] = bf16x2_to_float2(*reinterpret_cast<const uint32_t *>(p));
        }
    } else {
        if constexpr (DPL == 4) {
            const uint32_t r = *reinterpret_cast<const uint32_t *>(p);
            out[0] = e4m3x2_to_float2(r & 0xffffu);
            out[1] = e4m3x2_to_float2(r >> 16);
        } else {
            out[0] = e4m3x2_to_float2(*reinterpret_cast<const uint16_t *>(p));
        }
    }
}

template <int D, int BS, int G, bool FP8>
__global__ void __launch_bounds__(DecodeConfig<D, BS, G, FP8>::THREADS)
    paged_decode_partition_kernel(const DecodeParams p)
{
    using S = DecodeShape<D, BS, G, FP8>;
    using C = DecodeConfig<D, BS, G, FP8>;
    constexpr int NW = C::NW, STAGES = C::STAGES;
    constexpr unsigned FULL = 0xffffffffu;

    extern __shared__ __align__(128) uint8_t smem[];
    uint8_t *stages = smem;
    uint64_t *full_bar = reinterpret_cast<uint64_t *>(smem + C::OFF_BARS);
    uint64_t *empty_bar = full_bar + STAGES;
    volatile int *stage_bad = reinterpret_cast<volatile int *>(smem + C::OFF_FLAGS);
    volatile int *abort_flag = stage_bad + STAGES;
    volatile int *bad_flag = stage_bad + STAGES + 1;
    float *pbuf_all = reinterpret_cast<float *>(smem + C::OFF_PBUF);

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

    // per-consumer-lane state (unused by the producer warp)
    float m_run[S::NH], l_run[S::NH];
    float2 o[G][S::DPL / 2];
#pragma unroll
    for (int hr = 0; hr < S::NH; ++hr) {
        m_run[hr] = -INFINITY;
        l_run[hr] = 0.f;
    }
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
        for (int e = 0; e < S::DPL / 2; ++e) o[h][e] = make_float2(0.f, 0.f);
    const int j = lane / S::LPT, c = lane % S::LPT;
    const int ubase = transposed_base<S::U, S::LPT / 2>(c);
    const int hbase = ubase >> S::LOG_PS;

    if (warp == NW) {
        // ------------------------------ producer ------------------------------
        const uint64_t pol = l2_policy_evict_first();
        const int32_t *trow = p.block_tables + (size_t)seq * p.max_blocks_per_seq;
        const size_t blk_stride = (size_t)p.h_kv * S::TILE;
        const uint8_t *kb = p.k_cache + (size_t)kvh * S::TILE;
        const uint8_t *vb = p.v_cache + (size_t)kvh * S::TILE;
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
                            mbar_arrive_expect_tx(&full_bar[st], 2 * S::TILE);
                            bulk_copy_g2s(stages + st * 2 * S::TILE, kb + (size_t)ph * blk_stride, S::TILE,
                                          &full_bar[st], pol);
                            bulk_copy_g2s(stages + st * 2 * S::TILE + S::TILE, vb + (size_t)ph * blk_stride,
                                          S::TILE, &full_bar[st], pol);
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
            // let copies already issued land before the CTA's shared memory goes away
            for (int ii = max(0, issued - STAGES); ii < issued; ++ii)
                mbar_wait_bounded(&full_bar[ii % STAGES], (ii / STAGES) & 1);
        }
    } else {
        // ------------------------------ consumers ------------------------------
        float *pw = pbuf_all + warp * C::PBUF_FLOATS;          // [16][G] probabilities, then [G] rescales
        // q for this lane's chunks, pre-scaled into the log2 domain
        float2 qf[G][S::QD / 2];
        {
            const __nv_bfloat16 *qrow = p.q + ((size_t)seq * p.h_q + (size_t)kvh * G) * D;
            const float qs = p.qk_scale * head_k_factor(p, kvh);
#pragma unroll
            for (int h = 0; h < G; ++h) {
#pragma unroll
                for (int k = 0; k < S::CPL; ++k) {
                    const int dim0 = (c + k * S::LPT) * S::CHUNK;
#pragma unroll
                    for (int w8 = 0; w8 < S::CHUNK / 8; ++w8) {
                        const uint4 raw = *reinterpret_cast<const uint4 *>(qrow + (size_t)h * D + dim0 + w8 * 8);
                        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 f = bf16x2_to_float2(w[e]);
                            qf[h][k * (S::CHUNK / 2) + w8 * 4 + e] = make_float2(f.x * qs, f.y * qs);
                        }
                    }
                }
            }
        }

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
                const uint8_t *ktile = stages + st * 2 * S::TILE;
                const uint8_t *vtile = ktile + S::TILE;
                const int valid = min(BS, tok_end - (tok_begin + i * BS));
#pragma unroll 1
                for (int sub = 0; sub < S::NSUB; ++sub) {
                    if (sub * S::SUBT >= valid) break;
                    // ---- q . K for 16 tokens: partial dots v[h*PS + pass] ----
                    float v[S::U];
#pragma unroll
                    for (int pass = 0; pass < S::PS; ++pass) {
                        const uint8_t *krow = ktile + (sub * S::SUBT + pass * S::TPP + j) * S::ROW;
                        float2 acc[G];
#pragma unroll
                        for (int h = 0; h < G; ++h) acc[h] = make_float2(0.f, 0.f);
#pragma unroll
                        for (int k = 0; k < S::CPL; ++k) {
                            float2 kf[S::CHUNK / 2];
                            load_row_chunk<D, BS, G, FP8>(krow + (c + k * S::LPT) * 16, kf);
#pragma unroll
                            for (int h = 0; h < G; ++h)
#pragma unroll
                                for (int e = 0; e < S::CHUNK / 2; ++e)
                                    acc[h] = __ffma2_rn(qf[h][k * (S::CHUNK / 2) + e], kf[e], acc[h]);
                        }
#pragma unroll
                        for (int h = 0; h < G; ++h) v[h * S::PS + pass] = acc[h].x + acc[h].y;
                    }
                    transposed_reduce<S::U, S::LPT / 2>(v, c);
                    // mask tokens past the context (their rows may hold anything)
#pragma unroll
                    for (int f = 0; f < S::NF; ++f) {
                        const int tok = sub * S::SUBT + ((ubase + f) & (S::PS - 1)) * S::TPP + j;
                        if (tok >= valid) v[f] = -INFINITY;
                    }
                    // ---- per-head max over the 16 tokens ----
                    float hm[S::NH];
#pragma unroll
                    for (int hr = 0; hr < S::NH; ++hr) {
                        hm[hr] = v[hr << S::RPB];
#pragma unroll
                        for (int pp = 1; pp < (1 << S::RPB); ++pp) hm[hr] = fmaxf(hm[hr], v[(hr << S::RPB) + pp]);
#pragma unroll
                        for (int b = S::UB - S::HL; b < S::LOG_PS; ++b)
                            hm[hr] = fmaxf(hm[hr], __shfl_xor_sync(FULL, hm[hr], S::LPT >> (S::UB - b)));
#pragma unroll
                        for (int off = S::LPT; off < 32; off <<= 1)
                            hm[hr] = fmaxf(hm[hr], __shfl_xor_sync(FULL, hm[hr], off));
                    }
                    // ---- online softmax update ----
                    float alpha[S::NH];
#pragma unroll
                    for (int hr = 0; hr < S::NH; ++hr) {
                        const float mnew = fmaxf(m_run[hr], hm[hr]);
                        alpha[hr] = exp2f(m_run[hr] - mnew);
                        m_run[hr] = mnew;
                        float ps = 0.f;
#pragma unroll
                        for (int pp = 0; pp < (1 << S::RPB); ++pp) {
                            const int f = (hr << S::RPB) + pp;
                            v[f] = exp2f(v[f] - mnew);
                            ps += v[f];
                        }
                        l_run[hr] = l_run[hr] * alpha[hr] + ps;
                    }
#pragma unroll
                    for (int f = 0; f < S::NF; ++f) {
                        const int u = ubase + f;
                        const int tok = (u & (S::PS - 1)) * S::TPP + j;
                        pw[tok * G + (u >> S::LOG_PS)] = v[f];
                    }
#pragma unroll
                    for (int hr = 0; hr < S::NH; ++hr) pw[S::SUBT * G + hbase + hr] = alpha[hr];
                    __syncwarp();
                    // ---- p . V ----
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        const float a = pw[S::SUBT * G + h];
#pragma unroll
                        for (int e = 0; e < S::DPL / 2; ++e) o[h][e] = __fmul2_rn(o[h][e], make_float2(a, a));
                    }
                    const uint8_t *vrow = vtile + sub * S::SUBT * S::ROW + lane * S::DPL * S::ELEM;
#pragma unroll
                    for (int t = 0; t < S::SUBT; ++t) {
                        if (sub * S::SUBT + t < valid) {
                            float2 vf[S::DPL / 2];
                            load_v_elems<S::DPL, FP8>(vrow + t * S::ROW, vf);
                            float pt[G];
                            if constexpr (G % 4 == 0) {
#pragma unroll
                                for (int h4 = 0; h4 < G / 4; ++h4) {
                                    const float4 x = *reinterpret_cast<const float4 *>(pw + t * G + 4 * h4);
                                    pt[4 * h4] = x.x; pt[4 * h4 + 1] = x.y; pt[4 * h4 + 2] = x.z; pt[4 * h4 + 3] = x.w;
                                }
                            } else if constexpr (G == 2) {
                                const float2 x = *reinterpret_cast<const float2 *>(pw + t * G);
                                pt[0] = x.x; pt[1] = x.y;
                            } else {
                                pt[0] = pw[t];
                            }
#pragma unroll
                            for (int h = 0; h < G; ++h)
#pragma unroll
                                for (int e = 0; e < S::DPL / 2; ++e)
                                    o[h][e] = __ffma2_rn(make_float2(pt[h], pt[h]), vf[e], o[h][e]);
                        }
                    }
                    __syncwarp();
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty_bar[st]);
        }
        // this warp's l: sum over lanes holding other tokens of the same heads
#pragma unroll
        for (int hr = 0; hr < S::NH; ++hr) {
#pragma unroll
            for (int b = S::UB - S::HL; b < S::LOG_PS; ++b)
                l_run[hr] += __shfl_xor_sync(FULL, l_run[hr], S::LPT >> (S::UB - b));
#pragma unroll
            for (int off = S::LPT; off < 32; off <<= 1) l_run[hr] += __shfl_xor_sync(FULL, l_run[hr], off);
        }
    }

    __syncthreads();        // every stage consumed; the stage area becomes the combine area
    float *cm = reinterpret_cast<float *>(smem);                 // [NW][G]
    float *cl = cm + NW * G;                                     // [NW][G]
    float *co = cl + NW * G;                                     // [NW][G][D]
    if (warp < NW) {
#pragma unroll
        for (int hr = 0; hr < S::NH; ++hr) {
            cm[warp * G + hbase + hr] = m_run[hr];
            cl[warp * G + hbase + hr] = l_run[hr];
        }
#pragma unroll
        for (int h = 0; h < G; ++h)
#pragma unroll
            for (int e = 0; e < S::DPL / 2; ++e)
                *reinterpret_cast<float2 *>(co + ((size_t)(warp * G + h) * D) + lane * S::DPL + 2 * e) = o[h][e];
    }
    __syncthreads();
    cta_combine_and_write<NW, G, D>(p, cm, part, n_part, kvh, seq, (*abort_flag != 0) || (*bad_flag != 0),
                                    reinterpret_cast<float *>(smem + C::COMBINE_BYTES));
}

// ---- pass 2: merge the partitions of each (sequence, query head) ------------------------
struct MergeParams {
    __nv_bfloat16 *out;
    const int32_t *context_lens;
    const float *ws_ml;
    const float *ws_o;
    int h_q;
    int partition_size;
    int p_max;
};

// One CTA of 16 warps per (sequence, query head): warp w takes partitions w, w+16, ... with
// two independent accumulators, so that many partial rows are in flight at once (a group
// can have hundreds of partitions: 256 for a 131072-token context at 512 tokens each).
template <int D>
__global__ void __launch_bounds__(512) paged_decode_merge_kernel(const MergeParams p)
{
    constexpr int NWM = 16, DPL = D / 32;
    const int qh = blockIdx.x, seq = blockIdx.y;
    const int ctx = p.context_lens[seq];
    const int n_part = decode_num_partitions(ctx, p.partition_size, p.p_max);
    if (n_part <= kFusedMergeMaxPartitions) return;              // finished by pass 1
    const size_t row = (size_t)seq * p.h_q + qh;
    const float *ml = p.ws_ml + row * p.p_max * 2;
    const float *po = p.ws_o + row * p.p_max * D;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __shared__ float red[NWM];
    __shared__ float lsum[NWM];
    __shared__ float acc_s[NWM][D];

    float m = -INFINITY;
    for (int i = threadIdx.x; i < n_part; i += blockDim.x) m = fmaxf(m, ml[2 * i]);
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    if (lane == 0) red[warp] = m;
    __syncthreads();
    float M = red[0];
#pragma unroll
    for (int w = 1; w < NWM; ++w) M = fmaxf(M, red[w]);

    float L0 = 0.f, L1 = 0.f;
    float a0[DPL], a1[DPL];
#pragma unroll
    for (int e = 0; e < DPL; ++e) a0[e] = a1[e] = 0.f;
    int i = warp;
    for (; i + NWM < n_part; i += 2 * NWM) {
        const float2 mi = *reinterpret_cast<const float2 *>(ml + 2 * i);
        const float2 mj = *reinterpret_cast<const float2 *>(ml + 2 * (i + NWM));
        const float *oi = po + (size_t)i * D + lane * DPL;
        const float *oj = po + (size_t)(i + NWM) * D + lane * DPL;
        float xi[DPL], xj[DPL];
#pragma unroll
        for (int e = 0; e < DPL; ++e) {
            xi[e] = oi[e];
            xj[e] = oj[e];
        }
        const float wi = exp2f(mi.x - M), wj = exp2f(mj.x - M);
        L0 += wi * mi.y;
        L1 += wj * mj.y;
#pragma unroll
        for (int e = 0; e < DPL; ++e) {
            a0[e] += wi * xi[e];
            a1[e] += wj * xj[e];
        }
    }
    if (i < n_part) {
        const float2 mi = *reinterpret_cast<const float2 *>(ml + 2 * i);
        const float wi = exp2f(mi.x - M);
        L0 += wi * mi.y;
        const float *oi = po + (size_t)i * D + lane * DPL;
#pragma unroll
        for (int e = 0; e < DPL; ++e) a0[e] += wi * oi[e];
    }
    if (lane == 0) lsum[warp] = L0 + L1;
#pragma unroll
    for (int e = 0; e < DPL; ++e) acc_s[warp][lane * DPL + e] = a0[e] + a1[e];
    __syncthreads();
    if (threadIdx.x < D) {
        float Lt = 0.f, Ot = 0.f;
#pragma unroll
        for (int w = 0; w < NWM; ++w) {
            Lt += lsum[w];
            Ot += acc_s[w][threadIdx.x];
        }
        p.out[row * D + threadIdx.x] = __float2bfloat16_rn(Ot / Lt);
    }
}

}  // namespace pa
