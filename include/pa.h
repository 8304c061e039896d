/*
 * pa.h -- C ABI of the B200 paged-KV decode library (libpa.so).
 *
 * Paged KV cache: the K and V of every sequence live in fixed-size physical
 * blocks of a shared pool; a per-sequence block table maps logical block i to
 * a physical block id, so a sequence's cache need not be contiguous.
 * Sources (web pages), cited by title and section:
 *   "深度解构 LLM 推理优化：从 KV Cache 冗余到 PagedAttention 内存分页映射"
 *       section 2.1 (block table), 2.2 (on-demand allocation from a global
 *       free pool), 2.3 (copy-on-write for shared prompts), 3.2 (FP8 KV)
 *   "现代 AI 的“推理加速之谜”：从 KV Cache 到 PagedAttention 的演进"
 *       section 1 (Attention(Q,K,V) = softmax(QK^T / sqrt(d_k)) V; only the
 *       new token's Q, K, V are computed each step), section 3.A (GQA)
 *   "KVCache技术背景与核心挑战 / PageAttention内存管理机制" (intelliparadigm)
 *       sections 2.1-2.2 (blocks with reference counts), 3.1 (copy-on-write)
 *   "vLLM 推理原理 从 KV Cache 到分页与连续批处理"
 *       section "PagedAttention 怎样整理这些缓存" (logical blocks -> physical
 *       blocks 2, 5, 1; the last block may be partly filled)
 *
 * Conventions for every call below
 *   - Device pointers are owned by the caller (e.g. allocated through
 *     PyTorch).  The library allocates no device memory: pa_decode takes a
 *     caller workspace sized by pa_decode_workspace_size.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Device calls only enqueue work; none synchronises.
 *   - Return value: PA_OK (0) or a negative PA_ERR_* code; nothing is
 *     launched when an argument check fails.  No exception crosses the ABI.
 *   - Cache layout: k_cache and v_cache are [num_blocks][h_kv][block_size]
 *     [head_dim], row-major; each (block, head) tile is one contiguous span
 *     of block_size*head_dim elements.  Elements are bf16 (PA_CACHE_BF16),
 *     OCP FP8 E4M3 bytes (PA_CACHE_E4M3) or symmetric INT8 codes
 *     (PA_CACHE_INT8, -127..127), a quantised element being worth code * scale
 *     with one fp32 scale per tensor (the calls below) or per KV head (the
 *     *_head_scales calls).
 *   - Supported shapes: head_dim in {64, 128}; block_size in {16, 32, 64};
 *     h_q / h_kv in {1, 2, 4, 8}.  Query head h reads KV head
 *     h / (h_q / h_kv) (contiguous groups).
 *   - Device-side guards: an out-of-range slot, block id or block pair is
 *     never dereferenced; the kernel skips it and records a bit in the
 *     device error word (pa_device_errors).  Every wait inside a kernel is
 *     bounded; a wait that runs out records PA_DEVERR_TIMEOUT.
 */
#ifndef PA_H
#define PA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------ */
#define PA_OK               0
#define PA_ERR_INVALID_ARG (-1)   /* null pointer, bad size, h_q % h_kv != 0, bad dtype ... */
#define PA_ERR_UNSUPPORTED (-2)   /* shape outside the supported set */
#define PA_ERR_WORKSPACE   (-3)   /* workspace missing or too small */
#define PA_ERR_OOM         (-4)   /* allocator: free pool cannot satisfy the request */
#define PA_ERR_CUDA        (-5)   /* a CUDA call or launch failed */
#define PA_ERR_NOT_FOUND   (-6)   /* allocator: unknown sequence id */

/* device error word bits (pa_device_errors) */
#define PA_DEVERR_BAD_SLOT  0x1u  /* a slot id outside the pool was skipped */
#define PA_DEVERR_BAD_BLOCK 0x2u  /* a block-table entry outside the pool (or row) was skipped */
#define PA_DEVERR_BAD_PAIR  0x4u  /* a copy pair outside the pool was skipped */
#define PA_DEVERR_TIMEOUT   0x8u  /* a bounded in-kernel wait ran out */
#define PA_DEVERR_BAD_CHUNK 0x10u /* a prefill chunk longer than its context was skipped */

typedef enum { PA_CACHE_BF16 = 0, PA_CACHE_E4M3 = 1, PA_CACHE_INT8 = 2 } pa_cache_dtype;

/* partition_size value of pa_decode: balanced split (see pa_decode) */
#define PA_PARTITION_AUTO (-1)

/* Human-readable text of a status code (static storage). */
const char *pa_status_str(int status);

/* Library version, major*10000 + minor*100 + patch. */
int pa_version(void);

/* KV bytes per cached token: 2 (K and V) x layers x h_kv x head_dim x
 * elem_bytes ("深度解构…" section 1.1, per-token memory equation; "vLLM 推理原理…"
 * M_KV estimate).  Host only. */
size_t pa_kv_bytes_per_token(int layers, int h_kv, int head_dim, int elem_bytes);

/* Whole tokens whose KV fits in budget_bytes: budget_bytes / pa_kv_bytes_per_token(...) (0
 * when the per-token size is 0).  "深度解构…" section 3.2: about 72k tokens of Llama-3-8B in
 * the ~9 GB a 24 GB card leaves after the weights, twice that with an FP8 cache.  Host only. */
size_t pa_kv_capacity_tokens(size_t budget_bytes, int layers, int h_kv, int head_dim, int elem_bytes);

/* ---- cache write --------------------------------------------------------
 * Store the step's new K and V rows in their physical slots: for token t and
 * KV head h, cache[slot/bs][h][slot%bs][:] = row[t][h][:]
 * ("现代 AI…" section 1: each step computes only the new token's K, V and
 * keeps them; "vLLM 推理原理…" section "KV Cache 缓存的究竟是什么").
 *   key, value     device bf16; row t, head h at key + t*key_stride + h*head_dim
 *                  (key_stride/value_stride in elements; 0 = packed h_kv*head_dim)
 *   k_cache/v_cache device, layout above, of cache_dtype
 *   slot_mapping   device int64 [num_tokens]; slot = block*block_size + offset;
 *                  a negative slot skips the token (padding); a slot past the
 *                  pool is skipped and flags PA_DEVERR_BAD_SLOT
 *   cache_dtype    PA_CACHE_BF16: bits are copied unchanged.
 *                  PA_CACHE_E4M3: code = RNE-satfinite(x / scale) with an IEEE
 *                  fp32 division ("深度解构…" section 3.2, FP8 KV cache)
 *                  PA_CACHE_INT8: code = the integer nearest to x / scale (ties
 *                  to even, IEEE fp32 division) limited to [-127, 127]; NaN
 *                  gives 0 ("深度解构…" section 4 item 1 and "现代 AI…" section
 *                  3.C: INT8 KV quantisation)
 *   k_scale/v_scale per-tensor fp32 scales (quantised caches only; must be > 0
 *                  and finite)
 * Bit-exact by construction: no arithmetic other than the quantisation. */
int pa_reshape_and_cache(const void *key, const void *value, int64_t key_stride, int64_t value_stride,
                         void *k_cache, void *v_cache, const int64_t *slot_mapping, int num_tokens,
                         int h_kv, int head_dim, int block_size, int num_blocks,
                         int cache_dtype, float k_scale, float v_scale, void *stream);

/* pa_reshape_and_cache with one scale per KV head: KV head h is quantised with
 * k_scales[h] (resp. v_scales[h]).  The pages name KV quantisation but fix no
 * scale granularity; this is the finer of the two readings (per tensor, per
 * head) and reduces to the per-tensor call when all scales are equal.
 *   cache_dtype    PA_CACHE_E4M3 or PA_CACHE_INT8 (bf16 -> PA_ERR_INVALID_ARG)
 *   k_scales/v_scales device fp32 [h_kv], each > 0 and finite (not checked on
 *                  the host: the values are never read there); owned by the
 *                  caller and read by the kernel, so they must stay valid until
 *                  the call has run on the stream. */
int pa_reshape_and_cache_head_scales(const void *key, const void *value, int64_t key_stride,
                                     int64_t value_stride, void *k_cache, void *v_cache,
                                     const int64_t *slot_mapping, int num_tokens, int h_kv, int head_dim,
                                     int block_size, int num_blocks, int cache_dtype, const float *k_scales,
                                     const float *v_scales, void *stream);

/* ---- decode attention ----------------------------------------------------
 * One decode step: for sequence s and query head h,
 *   out[s][h] = softmax(scale * q[s][h] . K_s^T) . V_s
 * over the first context_lens[s] tokens of sequence s, token t read from
 * physical block block_tables[s][t / bs] at offset t % bs
 * ("现代 AI…" section 1, attention formula; "深度解构…" section 2.1 and
 * "vLLM 推理原理…" section "PagedAttention 怎样整理这些缓存", block table).
 * context_lens[s] includes the token written this step; 0 gives a zero row.
 *
 * Long contexts are split into partitions of partition_size tokens; each
 * partition keeps its own running max, sum and unnormalised output and a
 * second pass merges them (split-context decode).  partition_size = 0 means
 * one partition per sequence; a positive value must be a multiple of
 * block_size.  PA_PARTITION_AUTO splits the step's blocks evenly over as many
 * CTAs as the GPU holds at once (each takes one contiguous range of
 * (sequence, KV head, block) triples, so all finish together), merging split
 * sequences in the same launch; it applies to bf16 caches with at most 4096
 * sequences and otherwise falls back to partitions of max(512, ~max_context_len
 * / 16) tokens; either way no separate merge pass is needed.
 *   out            device bf16 [num_seqs][h_q][head_dim] (RNE of the fp32 result)
 *   q              device bf16 [num_seqs][h_q][head_dim]
 *   block_tables   device int32 [num_seqs][max_blocks_per_seq]; entries past
 *                  ceil(ctx/bs) are never read
 *   context_lens   device int32 [num_seqs]
 *   max_context_len host-known upper bound of context_lens; it only sizes the
 *                  grid (no device->host read).  A longer context is still
 *                  computed correctly: its last partition grows.
 *   workspace      device, >= pa_decode_workspace_size(...) bytes, 16-byte
 *                  aligned; holds per-group counters and fp32 partials; may be
 *                  NULL when that size is 0.  It must be zero-filled before its
 *                  first use (e.g. one cudaMemset); every call leaves it ready
 *                  for the next one.  Calls sharing a workspace must not overlap
 *                  on the GPU.  After a call that recorded PA_DEVERR_TIMEOUT,
 *                  zero it again.
 * Groups (sequence, KV head) of at most 16 partitions are merged inside the
 * first pass by the CTA that finishes the group last; pa_decode launches the
 * merge pass only when a group can have more partitions. 
 * Quantised caches (E4M3, INT8) are converted to fp16 in shared memory (both
 * code sets are exact there) and attended on the tensor cores; the K scale is
 * folded into the logit scale and the V scale into the output.
 * Accuracy: fp32 accumulation; vs an fp64 evaluation of the same formula over
 * the cache contents, max|err| <= 2e-2 and <= 1e-2 * max|ref| for bf16 and INT8
 * caches, <= 6e-2 for E4M3. */
size_t pa_decode_workspace_size(int num_seqs, int h_q, int head_dim, int max_context_len,
                                int partition_size);

int pa_decode(void *out, const void *q, const void *k_cache, const void *v_cache,
              const int32_t *block_tables, int max_blocks_per_seq, const int32_t *context_lens,
              int num_seqs, int max_context_len, int h_q, int h_kv, int head_dim, int block_size,
              int num_blocks, float scale, int cache_dtype, float k_scale, float v_scale,
              int partition_size, void *workspace, size_t workspace_bytes, void *stream);

/* The two passes of pa_decode as separate launches (same arguments), so that
 * each can be timed on its own: pa_decode == pa_decode_partitions followed by
 * pa_decode_merge on the same stream.  Sequences that fit one partition are
 * finished by the first pass; the merge pass combines the others. */
int pa_decode_partitions(void *out, const void *q, const void *k_cache, const void *v_cache,
                         const int32_t *block_tables, int max_blocks_per_seq, const int32_t *context_lens,
                         int num_seqs, int max_context_len, int h_q, int h_kv, int head_dim,
                         int block_size, int num_blocks, float scale, int cache_dtype, float k_scale,
                         float v_scale, int partition_size, void *workspace, size_t workspace_bytes,
                         void *stream);

int pa_decode_merge(void *out, const int32_t *context_lens, int num_seqs, int max_context_len, int h_q,
                    int head_dim, int partition_size, const void *workspace, size_t workspace_bytes,
                    void *stream);

/* pa_decode over a quantised cache with one scale per KV head (the scales the
 * cache was written with by pa_reshape_and_cache_head_scales): KV head k's
 * elements are worth code * k_scales[k] (resp. v_scales[k]).  Same arguments
 * and result as pa_decode otherwise; cache_dtype must be PA_CACHE_E4M3 or
 * PA_CACHE_INT8.  k_scales/v_scales: device fp32 [h_kv], owned by the caller. */
int pa_decode_head_scales(void *out, const void *q, const void *k_cache, const void *v_cache,
                          const int32_t *block_tables, int max_blocks_per_seq, const int32_t *context_lens,
                          int num_seqs, int max_context_len, int h_q, int h_kv, int head_dim, int block_size,
                          int num_blocks, float scale, int cache_dtype, const float *k_scales,
                          const float *v_scales, int partition_size, void *workspace, size_t workspace_bytes,
                          void *stream);

/* ---- one decode step: append, then attend --------------------------------------------
 * pa_reshape_and_cache of one appended token per sequence followed by pa_decode, as one call:
 *   key, value     device bf16 rows of the appended tokens, row s = sequence s (strides as in
 *                  pa_reshape_and_cache; num_tokens = num_seqs)
 *   slot_mapping   device int64 [num_seqs]: the slot of sequence s's appended token, which
 *                  must be its position context_lens[s] - 1 (so it lies in the sequence's last
 *                  block); negative = nothing appended for that sequence
 *   everything else as pa_decode (per-tensor scales).
 * The decode grid is launched as a programmatic dependent of the cache write: it starts while
 * the write runs, and only the loads of each sequence's last block wait for the write to
 * finish, so the write's latency is hidden behind the decode.  Results are identical to the two
 * calls made separately.  All argument checks happen before anything is launched. */
int pa_decode_step(const void *key, const void *value, int64_t key_stride, int64_t value_stride,
                   const int64_t *slot_mapping, void *out, const void *q, void *k_cache, void *v_cache,
                   const int32_t *block_tables, int max_blocks_per_seq, const int32_t *context_lens, int num_seqs,
                   int max_context_len, int h_q, int h_kv, int head_dim, int block_size, int num_blocks, float scale,
                   int cache_dtype, float k_scale, float v_scale, int partition_size, void *workspace,
                   size_t workspace_bytes, void *stream);

/* ---- chunked-prefill attention ---------------------------------------------------
 * Causal attention of a chunk of new query rows per sequence over the paged cache
 * ("vLLM 推理原理…" section 一次生成有两个阶段: prefill processes the input tokens and builds
 * their KV; chunked prefill splits a long input into pieces).  The chunk of sequence s is query
 * rows query_start[s] .. query_start[s+1]-1 and ends at the sequence's last token: row i of a
 * chunk of n rows sits at position p = context_lens[s] - n + i and
 *   out[row][h] = softmax(scale * q[row][h] . K_s[0..p]^T) . V_s[0..p]
 * with token t of sequence s read from block block_tables[s][t / bs] at offset t % bs and
 * query head h reading KV head h / (h_q / h_kv).  The chunk's own K/V rows must be in the cache
 * (pa_reshape_and_cache of the chunk's tokens, e.g. with slots from pa_alloc_append_n).
 *   out, q         device bf16 [T][h_q][head_dim], T = query_start[num_seqs], 16-byte
 *                  aligned (else PA_ERR_INVALID_ARG); T <= num_seqs * max_query_len
 *   query_start    device int32 [num_seqs + 1], non-decreasing, query_start[0] = 0
 *   context_lens   device int32 [num_seqs], each including its chunk (>= the chunk length; a
 *                  longer chunk leaves its rows unwritten and flags PA_DEVERR_BAD_CHUNK)
 *   max_query_len  host-known upper bound of the chunk lengths (sizes the grid)
 *   scale          finite and >= 0 (else PA_ERR_INVALID_ARG)
 *   cache_dtype    PA_CACHE_BF16 (other types: PA_ERR_UNSUPPORTED)
 * A block-table entry outside the pool is never dereferenced: it flags PA_DEVERR_BAD_BLOCK
 * and turns the affected rows into NaN.  5th-generation tensor cores (tcgen05.mma, bf16 in,
 * fp32 accumulators in tensor memory; the environment variable PA_PREFILL_MMA_SYNC=1 selects
 * an mma.sync kernel instead); accuracy as pa_decode for bf16 caches (the softmax
 * exponentials by ex2.approx).  Allocates nothing; needs no
 * workspace.  One CTA per work item (a pair of 128-row query tiles of one sequence and KV
 * head); pa_prefill_ws computes the same result with fewer, longer-lived CTAs. */
int pa_prefill(void *out, const void *q, const void *k_cache, const void *v_cache, const int32_t *block_tables,
               int max_blocks_per_seq, const int32_t *query_start, const int32_t *context_lens, int num_seqs,
               int max_query_len, int h_q, int h_kv, int head_dim, int block_size, int num_blocks, float scale,
               int cache_dtype, void *stream);

/* Bytes of device workspace pa_prefill_ws needs (a constant: two int counters, padded). */
size_t pa_prefill_workspace_size(void);

/* pa_prefill with a work queue: the same arguments, result and errors, plus
 *   workspace        device memory of at least pa_prefill_workspace_size() bytes, 16-byte
 *                    aligned, all zero before the first call (e.g. cudaMemset once after
 *                    allocating it); every call leaves it zero again.  Calls that share a
 *                    workspace must not run at the same time (put them on one stream);
 *   workspace_bytes  its size; NULL, too small or misaligned: PA_ERR_WORKSPACE, checked
 *                    before anything else, nothing launched.
 * The grid is one CTA per SM; each CTA claims work items from the counter in the workspace,
 * sequences in order of context length, longest first (for up to 1024 sequences; beyond that
 * in sequence order), within a sequence the longest query-tile pairs first (each for every KV
 * head), and prepares the next item (block-table reads, K/V and Q copies) while it
 * finishes the current one.  The caller's memory is not allocated, freed or resized. With
 * PA_PREFILL_MMA_SYNC=1 the mma.sync kernel runs, which does not use the workspace. */
int pa_prefill_ws(void *out, const void *q, const void *k_cache, const void *v_cache, const int32_t *block_tables,
                  int max_blocks_per_seq, const int32_t *query_start, const int32_t *context_lens, int num_seqs,
                  int max_query_len, int h_q, int h_kv, int head_dim, int block_size, int num_blocks, float scale,
                  int cache_dtype, void *workspace, size_t workspace_bytes, void *stream);

/* ---- decode without any allocation (static scratch) ---------------------------
 * The pages have no counterpart for this call; it exists for callers that cannot
 * allocate device memory at the point where they run a decode step: code inside an
 * inference engine's enqueue callback (plugins must not call cudaMalloc there, because it
 * can synchronise the device and is not allowed while the engine records work), hosts with
 * a fixed memory budget, and runtimes whose allocator belongs to someone else.
 * Same arguments and result as pa_decode (PA_PARTITION_AUTO included), minus the
 * workspace: the split-context partials go to one library-owned array of
 * PA_STATIC_WS_BYTES in device global memory.  Every GPU on which the library's device code
 * is loaded holds that array until the process exits.
 *   - Returns PA_ERR_WORKSPACE, launching nothing, when pa_decode_workspace_size(...) for
 *     the arguments exceeds PA_STATIC_WS_BYTES (e.g. use a larger partition_size, or
 *     pa_decode with a caller workspace).  Every other argument error is also returned
 *     before anything is queued.
 *   - The first call on a device looks up the array's device address (cudaGetSymbolAddress,
 *     with that device current) and keeps it for that device's CUDA context; make that first
 *     call before any stream capture.  After cudaDeviceReset the next call sees a new context
 *     and looks the address up again, so it too should come before any capture.
 *   - All calls share the one array, and it keeps the previous call's contents.  The call
 *     itself clears what must start at zero (the per-group counters at the front of the
 *     array, one cudaMemsetAsync on `stream` before the decode); the caller clears nothing.
 *   - Calls that can overlap on the GPU -- on different streams without ordering between
 *     them -- race on the array (partials and counters) and must not be issued that way.
 *   - Calls no cudaMalloc, cudaFree or allocating library routine. */
#define PA_STATIC_WS_BYTES (16u * 1024u * 1024u)

int pa_decode_static_ws(void *out, const void *q, const void *k_cache, const void *v_cache,
                        const int32_t *block_tables, int max_blocks_per_seq, const int32_t *context_lens,
                        int num_seqs, int max_context_len, int h_q, int h_kv, int head_dim, int block_size,
                        int num_blocks, float scale, int cache_dtype, float k_scale, float v_scale,
                        int partition_size, void *stream);

/* ---- copy-on-write block copy ---------------------------------------------
 * For every pair (src, dst) and every layer: cache[dst] = cache[src], byte
 * for byte, for K and for V ("深度解构…" section 2.3; intelliparadigm section
 * 3.1: copy the shared block, then remap the writer's table).
 *   k_caches/v_caches host arrays of num_layers device pointers (<= 256)
 *   block_pairs     device int64 [num_pairs][2] = (src, dst); a pair outside
 *                   [0, num_blocks) is skipped and flags PA_DEVERR_BAD_PAIR
 *   block_bytes     bytes of one physical block of one layer
 *                   (h_kv*block_size*head_dim*elem); a multiple of 16 */
int pa_copy_blocks(void *const *k_caches, void *const *v_caches, int num_layers,
                   const int64_t *block_pairs, int num_pairs, size_t block_bytes, int num_blocks,
                   void *stream);

/* ---- device error word ------------------------------------------------------
 * Read (and optionally clear) the error bits the kernels recorded on the
 * current device.  SYNCHRONISES the device first.  Diagnostic use only. */
int pa_device_errors(unsigned int *flags, int clear);

/* ---- host-side validation (optional, before a launch) -------------------------
 * Host copies of the tables / slots: PA_OK or PA_ERR_INVALID_ARG. */
int pa_validate_block_tables(const int32_t *block_tables, int max_blocks_per_seq,
                             const int32_t *context_lens, int num_seqs, int block_size, int num_blocks);
int pa_validate_slots(const int64_t *slot_mapping, int num_tokens, int block_size, int num_blocks);

/* ---- host block allocator -----------------------------------------------------
 * A global free pool of num_blocks physical blocks with a reference count per
 * block; sequences own block lists ("深度解构…" sections 2.1-2.3;
 * intelliparadigm sections 2.1, 2.2, 3.1; "vLLM 推理原理…" generation flow:
 * release a finished request's blocks).  Policy: LIFO free pool, initial
 * order a Fisher-Yates shuffle by SplitMix64(seed) (seed 0 = identity); a
 * block is taken only when the previous one is full; fork shares all blocks
 * (refcount + 1); the first write into a partly filled block whose refcount
 * is > 1 takes a fresh block, reports (old, new) for pa_copy_blocks and
 * drops the old block's count (the last holder writes in place); freeing a
 * sequence returns blocks whose count reaches 0, last block first.
 * Failures leave the state unchanged.  Not thread-safe: one caller at a time. */
typedef struct pa_alloc pa_alloc;

pa_alloc *pa_alloc_create(int num_blocks, int block_size, uint64_t seed);   /* NULL on bad args */
void      pa_alloc_destroy(pa_alloc *a);
int  pa_alloc_new_seq(pa_alloc *a, int64_t *seq_id);
/* One token: its slot, and (cow_src, cow_dst) = (-1, -1) unless a copy is needed. */
int  pa_alloc_append_slot(pa_alloc *a, int64_t seq, int64_t *slot, int64_t *cow_src, int64_t *cow_dst);
/* n tokens (prefill-style growth); slots may be NULL, else n entries.  At most one
 * copy can be needed (the first, partly filled block). */
int  pa_alloc_append_n(pa_alloc *a, int64_t seq, int n, int64_t *slots, int64_t *cow_src, int64_t *cow_dst);
/* One token for each of n sequences, in order (a decode step).  slots: n entries;
 * cow_pairs: room for 2*n int64; *num_cow receives the number of pairs.  All or nothing. */
int  pa_alloc_append_batch(pa_alloc *a, const int64_t *seqs, int n, int64_t *slots,
                           int64_t *cow_pairs, int *num_cow);
int  pa_alloc_fork(pa_alloc *a, int64_t parent, int64_t *child);
int  pa_alloc_free_seq(pa_alloc *a, int64_t seq);
/* Host rows [num_seqs][max_blocks] (unused entries -1) and lengths. */
int  pa_alloc_block_table(const pa_alloc *a, const int64_t *seqs, int num_seqs, int32_t *table,
                          int max_blocks, int32_t *context_lens);
int  pa_alloc_seq_len(const pa_alloc *a, int64_t seq, int64_t *len);
/* free_blocks: blocks that can be handed out (free pool + evictable cached blocks);
 * used_blocks: count > 0; shared_blocks: count > 1; frag_tokens: sum over sequences of
 * allocated but unfilled slots. */
int  pa_alloc_stats(const pa_alloc *a, int *free_blocks, int *used_blocks, int *shared_blocks,
                    int64_t *frag_tokens);
/* Reference count of a block (>= 0), or PA_ERR_INVALID_ARG. */
int  pa_alloc_refcount(const pa_alloc *a, int block);

/* ---- prefix caching ------------------------------------------------------------
 * "vLLM 推理原理…" section 前缀缓存能省掉哪部分工作: requests that begin with the same text
 * reuse the KV of the common prefix, on an exact match only; the prefill of the cached part is
 * skipped, the rest (and decoding) still runs.
 * pa_alloc_new_seq_prefix creates a sequence holding the n prompt tokens `tokens` (host
 * int32 token ids).  Its full blocks are looked up in order: block k matches a cached block
 * registered with the same predecessor (the block this walk matched for k-1, or none for
 * k = 0) and the same bs token ids; every match is shared (count + 1, an evictable block
 * leaves the eviction list); the first miss ends the walk.  The remaining blocks are fresh,
 * and each fresh FULL block is registered for later prompts.  A partly filled last block is
 * never cached, so appends never write into a cached block.
 *   slots          NULL or n entries: slot of every prompt token (cached ones included)
 *   cached_tokens  tokens at the front whose KV is already in the cache (a multiple of
 *                  block_size); the caller writes K/V only for tokens [cached_tokens, n)
 * Cached blocks whose count drops to 0 stay cached and evictable; when the free pool is empty,
 * taking a block evicts the least recently released one (its registration is dropped and
 * entries naming it as predecessor can no longer match).  PA_ERR_OOM (state unchanged) when
 * free + evictable blocks, minus those the walk hit, cannot hold the fresh blocks. */
int  pa_alloc_new_seq_prefix(pa_alloc *a, const int32_t *tokens, int n, int64_t *seq_id, int64_t *slots,
                             int *cached_tokens);
/* Totals since creation: prompt tokens found cached / not cached by pa_alloc_new_seq_prefix;
 * blocks registered in the cache now, and those of them with count 0 (evictable). */
int  pa_alloc_prefix_stats(const pa_alloc *a, int64_t *hit_tokens, int64_t *miss_tokens, int *cached_blocks,
                           int *evictable_blocks);
/* An order of the batch `seqs` in which sequences that share physical blocks are adjacent:
 * order[i] = index into seqs, sorted by the sequences' block lists (lexicographically by
 * physical id; ties keep their input order).  Building the block tables in this order makes the
 * decode kernels of sharers run close together in time, so shared blocks are read from L2. */
int  pa_alloc_order_by_prefix(const pa_alloc *a, const int64_t *seqs, int n, int32_t *order);

#ifdef __cplusplus
}
#endif

#endif /* PA_H */
