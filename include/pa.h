/*
 * pa.h -- C ABI of the paged-KV-cache decode library (libpa.so, sm_100a).
 *
 * Three operations make one decode step of one attention layer:
 *
 *   pa_copy_blocks        copy-on-write block copies decided by the host
 *   pa_reshape_and_cache  write this step's new K/V rows into their slots
 *   pa_paged_decode       single-query attention over each sequence's
 *                         context, reached through its block table
 *
 * Declared below as well: pa_paged_decode_append (the cache write fused into
 * the decode launch), pa_paged_decode_no_alloc (library-owned scratch),
 * pa_paged_decode_shared_prefix (groups that share a stored prefix read it
 * once), the _fp8 and _int8 variants over one-byte K/V pools (one scale per
 * pool, or one per row with the _rowscale calls), pa_swap_blocks
 * (block copies between device and pinned host pools), and the size
 * queries.  The host block manager that hands out the block ids is declared
 * in pa_block_manager.h.
 *
 * Pages cited (title, then section):
 *   [VM-paging] "vLLM用虚拟内存分页思想管理KV Cache"
 *   [Practice]  "PagedAttention：大模型KV Cache分页管理优化实践"
 *   [Manager]   "深入解析 vLLM 的 KV Cache 管理器：从内存碎片到 PagedAttention 的完整技术剖析"
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Memory.  Every pointer argument is caller-owned DEVICE memory unless its
 *   comment says otherwise.  The library allocates nothing, keeps no state
 *   between calls, never synchronises the device and only enqueues work on
 *   `stream` (a cudaStream_t; NULL is the legacy default stream).  Calls
 *   return as soon as the work is enqueued.
 *
 * Element types.  query, key, value, k_cache, v_cache and out share one
 *   element type: IEEE binary16 (PA_DTYPE_F16) or bfloat16 (PA_DTYPE_BF16);
 *   the _fp8 / _int8 calls take one-byte K/V pools instead (see there).
 *   Attention accumulates in fp32 and rounds the output to nearest even.
 *
 * KV-cache layout (one layer; K and V in two pools of the same shape):
 *   k_cache, v_cache : [num_blocks][block_size][num_kv_heads][head_dim],
 *   row-major and contiguous.  A physical block holds block_size tokens of
 *   every kv head ([Practice §3.1 物理块分配器设计]).  The slot of a token is
 *   physical_block * block_size + offset_in_block, so the pools are also
 *   [num_blocks * block_size][num_kv_heads][head_dim] indexed by slot.
 *   Pool base addresses must be 16-byte aligned (256-byte alignment, which
 *   every CUDA allocation has, is what the pages recommend:
 *   [Practice §4.2 访存优化技术]).
 *
 * Synchronous errors (return value; nothing is enqueued when it is not
 *   PA_OK):
 *   PA_ERR_INVALID_ARG  null pointer, negative or zero size where a positive
 *                       one is needed, num_q_heads not a multiple of
 *                       num_kv_heads, partition_size not a multiple of
 *                       block_size, workspace too small, a pointer that is
 *                       not 16-byte aligned;
 *   PA_ERR_UNSUPPORTED  head_dim not 64 or 128, block_size not 8, 16 or 32,
 *                       num_q_heads / num_kv_heads not 1, 2, 4 or 8, an
 *                       unknown dtype;
 *   PA_ERR_CUDA         the launch failed (cudaGetLastError after launch).
 *
 * Asynchronous data errors (device status word).  `d_status` is an optional
 *   (may be NULL) device int32 that the kernels OR bits into; the caller
 *   clears it.  The offending token or block is skipped and the kernels
 *   finish normally (they never trap and every wait they make is bounded):
 *   PA_STATUS_BAD_BLOCK    a block id outside [0, num_blocks) -- in a block
 *                          table (that block's tokens are left out of the
 *                          softmax) or in a copy pair (the pair is skipped);
 *   PA_STATUS_BAD_SLOT     a slot at or beyond num_blocks * block_size (the
 *                          token is not written; negative slots are padding
 *                          and are skipped silently);
 *   PA_STATUS_BAD_CONTEXT  a context length that is negative, larger than
 *                          max_context_len or larger than
 *                          max_blocks_per_seq * block_size (the output row is
 *                          written as zeros);
 *   PA_STATUS_COPY_CONFLICT a copy destination that appears twice or is also
 *                          a source in the same call (those blocks' contents
 *                          are unspecified);
 *   PA_STATUS_TIMEOUT      a bounded wait for an asynchronous copy gave up
 *                          (should never happen; the output is unspecified).
 */
#ifndef PA_H_
#define PA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PA_API __attribute__((visibility("default")))
#else
#define PA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st* pa_stream_t;

typedef enum pa_status {
    PA_OK = 0,
    PA_ERR_INVALID_ARG = 1,
    PA_ERR_UNSUPPORTED = 2,
    PA_ERR_CUDA = 3
} pa_status;

typedef enum pa_dtype {
    PA_DTYPE_F16 = 0,
    PA_DTYPE_BF16 = 1,
    PA_DTYPE_FP8_E4M3 = 2,  /* cache pools only: block copies/swaps and the *_fp8 calls */
    PA_DTYPE_INT8 = 3,      /* cache pools only: block copies/swaps and the *_int8 calls */
    PA_DTYPE_F32 = 4        /* row-scale pools of the *_rowscale calls: block copies/swaps
                               only, with head_dim 1 */
} pa_dtype;

#define PA_STATUS_BAD_BLOCK 1
#define PA_STATUS_BAD_SLOT 2
#define PA_STATUS_BAD_CONTEXT 4
#define PA_STATUS_COPY_CONFLICT 8
#define PA_STATUS_TIMEOUT 16

/*
 * pa_reshape_and_cache -- write each new token's K and V rows into its slot.
 *
 * Defined by: [Practice §3.3 按需分配策略] step 4 (after the allocator has
 * found or created room in the sequence's last block, write the new token's
 * K/V vectors) and [Manager, 第一部分 KV Cache 的核心价值] (each decode step
 * stores the new token's K and V, then attends over the whole cache).
 *
 *   for t < num_tokens with slot = slot_mapping[t] >= 0:
 *     k_cache[slot][h][d] = key[t][h][d],  v_cache[slot][h][d] = value[t][h][d]
 *
 * A bit-exact copy.  Every other cache element is left untouched.
 *
 * key, value     [num_tokens][num_kv_heads][head_dim], contiguous, 16-byte aligned.
 * k_cache, v_cache  the pools (layout above); written in place.
 * slot_mapping   int64 [num_tokens]; negative = padding token, skipped.
 * num_tokens     >= 0 (0 enqueues nothing).
 * num_blocks     pool size in blocks (bounds check of the slots).
 * d_status       optional; PA_STATUS_BAD_SLOT.
 */
PA_API pa_status pa_reshape_and_cache(const void* key, const void* value, void* k_cache,
                               void* v_cache, const int64_t* slot_mapping,
                               int32_t num_tokens, int32_t num_kv_heads, int32_t head_dim,
                               int32_t block_size, int64_t num_blocks, pa_dtype dtype,
                               int32_t* d_status, pa_stream_t stream);

/*
 * pa_copy_blocks -- the data copy of copy-on-write.
 *
 * Defined by: [VM-paging, 写时复制与块共享机制] and [Practice §4.1 共享内存管理]
 * steps 1-4: a sequence that must modify a block shared with others (count
 * above 1) gets a new block holding a copy of the original's data, remaps
 * its table entry and drops one reference on the original.  The host decides
 * which blocks to copy and keeps the reference counts; this call performs
 * step 2 (copy the original data) for every pair at once.
 *
 *   for i < num_pairs: block block_mapping[i][1] of k_cache and v_cache
 *                      becomes a bit-exact copy of block block_mapping[i][0]
 *
 * block_mapping  int64 [num_pairs][2] of (src, dst) physical block ids.
 *                src == dst is a no-op.  Destinations must be distinct and
 *                must not be sources of other pairs (else
 *                PA_STATUS_COPY_CONFLICT).
 * num_pairs      >= 0 (0 enqueues nothing).
 * d_status       optional; PA_STATUS_BAD_BLOCK, PA_STATUS_COPY_CONFLICT.
 */
PA_API pa_status pa_copy_blocks(void* k_cache, void* v_cache, const int64_t* block_mapping,
                         int32_t num_pairs, int32_t num_kv_heads, int32_t head_dim,
                         int32_t block_size, int64_t num_blocks, pa_dtype dtype,
                         int32_t* d_status, pa_stream_t stream);

/*
 * pa_swap_blocks -- whole-block copies between two pools, one of which is
 * normally in pinned host memory: swap out (device -> host) when a waiting
 * request's blocks are evicted to make room, swap in (host -> device) when
 * it is scheduled again.
 *
 * Defined by: [VM-paging, 显存管理与调度策略设计] (eviction: under sustained
 * memory pressure the KV data of waiting requests moves to CPU memory and
 * comes back to the GPU when they are rescheduled) and [Manager, 第四部分]
 * (LRU block eviction and request preemption).  The host chooses the blocks
 * and keeps the tables; this call moves the data for every pair at once, in
 * one launch, with the GPU reading and writing the host pool directly.
 *
 *   for i < num_pairs: block block_mapping[i][1] of dst_k / dst_v becomes a
 *                      bit-exact copy of block block_mapping[i][0] of
 *                      src_k / src_v
 *
 * src_k, src_v   [src_num_blocks][block_size][num_kv_heads][head_dim]
 * dst_k, dst_v   [dst_num_blocks][...] of the same element type.  Each is
 *                device memory or pinned host memory that the device can
 *                address (cudaHostAlloc / cudaHostRegister with mapping; on a
 *                system with unified addressing the host pointer is the
 *                device pointer).  16-byte aligned.
 * block_mapping  int64 [num_pairs][2] of (src, dst) block ids, device or
 *                device-addressable host memory.  Destinations must be
 *                distinct (else PA_STATUS_COPY_CONFLICT); when the source
 *                and destination pools are the same memory this is
 *                pa_copy_blocks, with its conflict rule.
 * dtype          PA_DTYPE_F16, _BF16, _FP8_E4M3 or _INT8 (element size only).
 * d_status       optional; PA_STATUS_BAD_BLOCK (an id outside its pool;
 *                the pair is skipped), PA_STATUS_COPY_CONFLICT.
 * Errors: PA_ERR_INVALID_ARG for null or misaligned pointers, a pointer the
 * device cannot address (pageable host memory: checked with
 * cudaPointerGetAttributes before anything is enqueued), a negative count
 * or pool size; PA_ERR_UNSUPPORTED for shapes pa_copy_blocks refuses.
 */
PA_API pa_status pa_swap_blocks(const void* src_k, const void* src_v, void* dst_k, void* dst_v,
                                const int64_t* block_mapping, int32_t num_pairs,
                                int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                                int64_t src_num_blocks, int64_t dst_num_blocks, pa_dtype dtype,
                                int32_t* d_status, pa_stream_t stream);

/*
 * pa_paged_decode_partition_size -- the context partition length (tokens)
 * pa_paged_decode uses: `partition_size` itself when it is positive, else
 * the library's choice for this shape.  Host-only; returns 0 for arguments
 * pa_paged_decode would reject.
 */
PA_API int32_t pa_paged_decode_partition_size(int32_t num_seqs, int32_t num_q_heads,
                                       int32_t num_kv_heads, int32_t head_dim,
                                       int32_t block_size, int32_t max_context_len,
                                       int32_t partition_size);

/*
 * pa_paged_decode_workspace_size -- bytes of scratch pa_paged_decode needs
 * for these arguments (0 when every context fits in one partition).  The
 * workspace holds, per (sequence, query head, partition), the partition's
 * running max, exp-sum and normalised partial output in fp32.  Host-only.
 */
PA_API size_t pa_paged_decode_workspace_size(int32_t num_seqs, int32_t num_q_heads,
                                      int32_t num_kv_heads, int32_t head_dim,
                                      int32_t block_size, int32_t max_context_len,
                                      int32_t partition_size);

/*
 * pa_paged_decode -- single-query (decode) attention over a paged KV cache.
 *
 * Defined by: [VM-paging, PagedAttention的注意力计算流程] (for each request and
 * head: look up the physical blocks in the block table, score the query
 * against the Keys of every block, normalise with softmax, sum the Values
 * with those weights, all in one kernel launch); [Manager, 第二部分
 * PagedAttention 的核心思想] step 4 (the kernel reassembles K/V through the
 * block table at run time); [Practice §3.2 块表与地址转换] (logical block j ->
 * table[j] -> physical id -> base + offset); the softmax is taken blockwise
 * as [Practice §5.1 分块Softmax算法] lays out (per-block max, global max,
 * rescaled exp-sum, normalise), here in its single-pass running form, and
 * across context partitions by a second, reduction kernel.
 *
 * For sequence s, query head h, kv head g = h / (num_q_heads / num_kv_heads),
 * token t < context_lens[s] stored at
 *   k_cache[block_tables[s][t / block_size]][t % block_size][g][:]:
 *   x_t = scale * sum_d query[s][h][d] * K_t[d]
 *   out[s][h][:] = sum_t softmax(x)_t * V_t[:]
 * An empty context (context_lens[s] == 0) gives a zero row.
 *
 * out            [num_seqs][num_q_heads][head_dim], 16-byte aligned; written.
 * query          [num_seqs][num_q_heads][head_dim], 16-byte aligned.
 * block_tables   int32 [num_seqs][max_blocks_per_seq]; entries past a
 *                sequence's last block are never read.
 * context_lens   int32 [num_seqs]; includes the token appended this step.
 * max_context_len  host value: an upper bound of context_lens (it sizes the
 *                grid; the library never reads device data back).
 * scale          multiplier of q.k before the softmax (e.g. 1/sqrt(head_dim)).
 * partition_size 0 = library's choice; else a multiple of block_size.
 *                Contexts longer than one partition are split; the partial
 *                results go to `workspace` and a reduction kernel merges them.
 * workspace      device scratch of at least
 *                pa_paged_decode_workspace_size(...) bytes, 16-byte aligned
 *                (may be NULL when that size is 0).  Its contents on entry do
 *                not matter; calls that share it must not overlap.
 * d_status       optional; PA_STATUS_BAD_BLOCK, PA_STATUS_BAD_CONTEXT,
 *                PA_STATUS_TIMEOUT.
 *
 * Deterministic: the same inputs give bit-identical outputs, whatever the
 * physical placement of the blocks.
 */
PA_API pa_status pa_paged_decode(void* out, const void* query, const void* k_cache,
                          const void* v_cache, const int32_t* block_tables,
                          const int32_t* context_lens, int32_t num_seqs, int32_t num_q_heads,
                          int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                          int32_t max_blocks_per_seq, int64_t num_blocks,
                          int32_t max_context_len, float scale, int32_t partition_size,
                          void* workspace, size_t workspace_bytes, pa_dtype dtype,
                          int32_t* d_status, pa_stream_t stream);

/*
 * pa_paged_decode_append -- one decode step in one launch: each sequence's
 * new token is written into the cache and attended to, as
 * pa_reshape_and_cache followed by pa_paged_decode would do.
 *
 * Defined by: [Manager, 第一部分 KV Cache 的核心价值] (store the new token's K and
 * V, then attend over the whole cache) with the write of [Practice §3.3] step
 * 4 and the attention of pa_paged_decode.  For the usual decode batch in
 * which sequence s appends exactly one token, at position context_lens[s] - 1,
 * whose slot is given by its own block table:
 *   slot = block_tables[s][(ctx - 1) / block_size] * block_size + (ctx - 1) % block_size.
 * The CTA that owns a sequence's last context partition writes that token's
 * K/V row of each kv head it serves before loading the block that holds it,
 * so no separate cache-write kernel (and no launch dependency) is needed.
 *
 * key, value     [num_seqs][num_kv_heads][head_dim], 16-byte aligned: the new
 *                token of every sequence.  k_cache / v_cache are written.
 * Other arguments, results and errors as pa_paged_decode; a table entry
 * outside the pool for the new token sets PA_STATUS_BAD_SLOT and the token
 * is not written.  Sequences with context length 0 append nothing.
 */
PA_API pa_status pa_paged_decode_append(void* out, const void* query, const void* key,
                                        const void* value, void* k_cache, void* v_cache,
                                        const int32_t* block_tables, const int32_t* context_lens,
                                        int32_t num_seqs, int32_t num_q_heads,
                                        int32_t num_kv_heads, int32_t head_dim,
                                        int32_t block_size, int32_t max_blocks_per_seq,
                                        int64_t num_blocks, int32_t max_context_len, float scale,
                                        int32_t partition_size, void* workspace,
                                        size_t workspace_bytes, pa_dtype dtype,
                                        int32_t* d_status, pa_stream_t stream);

/*
 * FP8 KV cache -- pools of e4m3 codes (1 byte per element, OCP e4m3fn: no
 * infinities, largest finite 448) with one scale per pool: the cached value
 * of code c is decode(c) * k_scale (or v_scale).  Halves the bytes a decode
 * step moves.  Defined by: [Practice §7 演进方向与优化空间] (FP8/INT8 storage of
 * history blocks) and [VM-paging, PagedAttention的工程实践与局限] (low-precision
 * storage of the KV values in blocks); the scale-per-tensor form is this
 * library's reading.  Layout and slots as the 16-bit pools.  pa_copy_blocks
 * copies such pools with dtype PA_DTYPE_FP8_E4M3.
 *
 * pa_reshape_and_cache_fp8 -- the cache write, quantising:
 *   code = e4m3(fp32(x) * fp32(1 / scale)), round to nearest even,
 *   saturating at +-448 (NaN stays NaN).
 * key, value     [num_tokens][num_kv_heads][head_dim] of `dtype` (F16/BF16).
 * k_scale, v_scale  positive finite (else PA_ERR_INVALID_ARG).
 * Other arguments and errors as pa_reshape_and_cache.
 */
PA_API pa_status pa_reshape_and_cache_fp8(const void* key, const void* value, void* k_cache,
                                          void* v_cache, const int64_t* slot_mapping,
                                          int32_t num_tokens, int32_t num_kv_heads,
                                          int32_t head_dim, int32_t block_size,
                                          int64_t num_blocks, pa_dtype dtype, float k_scale,
                                          float v_scale, int32_t* d_status, pa_stream_t stream);

/*
 * pa_paged_decode_fp8 -- pa_paged_decode over FP8 pools.  query and out are
 * of `dtype` (F16/BF16); K and V are dequantised exactly (e4m3 values are
 * fp16 values) and the contractions run on fp16 tensor cores with fp32
 * accumulation, so a bf16 query is rounded to fp16 first (exact in its
 * normal range).  block_size 16 or 32 (else PA_ERR_UNSUPPORTED).  The
 * workspace is sized by pa_paged_decode_workspace_size.  Other arguments,
 * results and errors as pa_paged_decode.
 */
PA_API pa_status pa_paged_decode_fp8(void* out, const void* query, const void* k_cache,
                                     const void* v_cache, const int32_t* block_tables,
                                     const int32_t* context_lens, int32_t num_seqs,
                                     int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                     int32_t block_size, int32_t max_blocks_per_seq,
                                     int64_t num_blocks, int32_t max_context_len, float scale,
                                     float k_scale, float v_scale, int32_t partition_size,
                                     void* workspace, size_t workspace_bytes, pa_dtype dtype,
                                     int32_t* d_status, pa_stream_t stream);

/*
 * pa_paged_decode_fp8_append -- pa_paged_decode_append over FP8 pools: each
 * sequence's new token (key, value of `dtype`, [num_seqs][num_kv_heads]
 * [head_dim], 16-byte aligned) is quantised exactly as
 * pa_reshape_and_cache_fp8 does and written to its slot (the position
 * context_lens[s] - 1 of its own block table) inside the decode launch,
 * then attended to with the other tokens.  Arguments, results and errors as
 * pa_paged_decode_fp8 and pa_paged_decode_append; a table entry outside the
 * pool for the new token sets PA_STATUS_BAD_SLOT and the token is not
 * written.
 */
PA_API pa_status pa_paged_decode_fp8_append(
    void* out, const void* query, const void* key, const void* value, void* k_cache,
    void* v_cache, const int32_t* block_tables, const int32_t* context_lens, int32_t num_seqs,
    int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
    int32_t max_blocks_per_seq, int64_t num_blocks, int32_t max_context_len, float scale,
    float k_scale, float v_scale, int32_t partition_size, void* workspace, size_t workspace_bytes,
    pa_dtype dtype, int32_t* d_status, pa_stream_t stream);

/*
 * INT8 KV cache -- pools of two's-complement int8 codes (1 byte per element)
 * with one scale per pool: the cached value of code c is c * k_scale (or
 * v_scale).  Defined by the same passages as the FP8 pools above, which
 * name INT8 beside FP8; the scale-per-tensor form is this library's
 * reading.  Layout and slots as the 16-bit pools.  pa_copy_blocks and
 * pa_swap_blocks move such pools with dtype PA_DTYPE_INT8.
 *
 * pa_reshape_and_cache_int8 -- the cache write, quantising:
 *   code = fp32(x) * fp32(1 / scale), rounded to the nearest integer (ties
 *   to even) and saturated to [-128, 127]; NaN gives 0.
 * Other arguments and errors as pa_reshape_and_cache_fp8.
 *
 * pa_paged_decode_int8, pa_paged_decode_int8_append -- as the FP8 calls
 * above, over int8 pools (every code is an fp16 value, so K and V are again
 * dequantised exactly); the fused write quantises as
 * pa_reshape_and_cache_int8.  Arguments, results and errors as
 * pa_paged_decode_fp8 and pa_paged_decode_fp8_append.
 */
PA_API pa_status pa_reshape_and_cache_int8(const void* key, const void* value, void* k_cache,
                                           void* v_cache, const int64_t* slot_mapping,
                                           int32_t num_tokens, int32_t num_kv_heads,
                                           int32_t head_dim, int32_t block_size,
                                           int64_t num_blocks, pa_dtype dtype, float k_scale,
                                           float v_scale, int32_t* d_status, pa_stream_t stream);

PA_API pa_status pa_paged_decode_int8(void* out, const void* query, const void* k_cache,
                                      const void* v_cache, const int32_t* block_tables,
                                      const int32_t* context_lens, int32_t num_seqs,
                                      int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                      int32_t block_size, int32_t max_blocks_per_seq,
                                      int64_t num_blocks, int32_t max_context_len, float scale,
                                      float k_scale, float v_scale, int32_t partition_size,
                                      void* workspace, size_t workspace_bytes, pa_dtype dtype,
                                      int32_t* d_status, pa_stream_t stream);

PA_API pa_status pa_paged_decode_int8_append(
    void* out, const void* query, const void* key, const void* value, void* k_cache,
    void* v_cache, const int32_t* block_tables, const int32_t* context_lens, int32_t num_seqs,
    int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
    int32_t max_blocks_per_seq, int64_t num_blocks, int32_t max_context_len, float scale,
    float k_scale, float v_scale, int32_t partition_size, void* workspace, size_t workspace_bytes,
    pa_dtype dtype, int32_t* d_status, pa_stream_t stream);

/*
 * Row-scaled one-byte KV cache -- e4m3 or int8 code pools as above, but with
 * one fp32 scale per (token, kv head) row instead of one per pool, so heads
 * (and tokens) of very different magnitude each keep the full resolution of
 * the code.  Defined by the same passages as the FP8 pools ([Practice §7
 * 演进方向与优化空间], [VM-paging, PagedAttention的工程实践与局限]); the
 * per-row granularity is this library's reading: a row is quantised once,
 * when it is written, from its own values, and never rewritten.
 *
 * Scale pools (caller-owned, fp32, 16-byte aligned, one for K and one for V):
 *   k_scales, v_scales : [num_blocks][num_kv_heads][block_size]
 * The cached value of element d of the row of slot `slot`, kv head g, is
 *   decode(code) * scales[slot / block_size][g][slot % block_size].
 * A block's scales for one kv head are one contiguous run of block_size
 * floats.  Block copies and swaps move a scale pool with pa_copy_blocks /
 * pa_swap_blocks, dtype PA_DTYPE_F32, head_dim 1 (same block ids as the
 * code pools).  Extra HBM per token: 8 bytes per kv head (3% at D = 128).
 *
 * pa_reshape_and_cache_fp8_rowscale / _int8_rowscale -- the quantising
 * write: for each written (token, kv head) row x,
 *   s = fp32(max_d |x_d| / code_max)       (code_max 448 e4m3, 127 int8)
 *   code_d = encode(fp32(x_d * fp32(1 / s))), rounded and saturated as the
 *            per-pool write does (so the row's largest element takes the
 *            top code);
 * a row with s below the smallest normal fp32 (all zeros) stores s = 0 and
 * zero codes.  The codes go to the slot, s to the scale pools.  Arguments
 * and errors as pa_reshape_and_cache_fp8 without the two scales; block_size
 * 8, 16 or 32.
 *
 * pa_paged_decode_fp8_rowscale / _int8_rowscale -- pa_paged_decode_fp8 /
 * _int8 over row-scaled pools: the score of token t is multiplied by its K
 * row scale, and its V row by its V row scale.  block_size 16 or 32.  The
 * _append forms write each sequence's new token (key / value of `dtype`,
 * [num_seqs][num_kv_heads][head_dim]) at position context_lens[s] - 1 with
 * the row-scaled quantisation above, codes and scales, inside the decode
 * launch.  Other arguments, results and errors as pa_paged_decode_fp8 and
 * pa_paged_decode_fp8_append.
 */
PA_API pa_status pa_reshape_and_cache_fp8_rowscale(
    const void* key, const void* value, void* k_cache, void* v_cache, float* k_scales,
    float* v_scales, const int64_t* slot_mapping, int32_t num_tokens, int32_t num_kv_heads,
    int32_t head_dim, int32_t block_size, int64_t num_blocks, pa_dtype dtype, int32_t* d_status,
    pa_stream_t stream);

PA_API pa_status pa_reshape_and_cache_int8_rowscale(
    const void* key, const void* value, void* k_cache, void* v_cache, float* k_scales,
    float* v_scales, const int64_t* slot_mapping, int32_t num_tokens, int32_t num_kv_heads,
    int32_t head_dim, int32_t block_size, int64_t num_blocks, pa_dtype dtype, int32_t* d_status,
    pa_stream_t stream);

PA_API pa_status pa_paged_decode_fp8_rowscale(
    void* out, const void* query, const void* k_cache, const void* v_cache, const float* k_scales,
    const float* v_scales, const int32_t* block_tables, const int32_t* context_lens,
    int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
    int32_t block_size, int32_t max_blocks_per_seq, int64_t num_blocks, int32_t max_context_len,
    float scale, int32_t partition_size, void* workspace, size_t workspace_bytes, pa_dtype dtype,
    int32_t* d_status, pa_stream_t stream);

PA_API pa_status pa_paged_decode_int8_rowscale(
    void* out, const void* query, const void* k_cache, const void* v_cache, const float* k_scales,
    const float* v_scales, const int32_t* block_tables, const int32_t* context_lens,
    int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
    int32_t block_size, int32_t max_blocks_per_seq, int64_t num_blocks, int32_t max_context_len,
    float scale, int32_t partition_size, void* workspace, size_t workspace_bytes, pa_dtype dtype,
    int32_t* d_status, pa_stream_t stream);

PA_API pa_status pa_paged_decode_fp8_rowscale_append(
    void* out, const void* query, const void* key, const void* value, void* k_cache,
    void* v_cache, float* k_scales, float* v_scales, const int32_t* block_tables,
    const int32_t* context_lens, int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
    int32_t head_dim, int32_t block_size, int32_t max_blocks_per_seq, int64_t num_blocks,
    int32_t max_context_len, float scale, int32_t partition_size, void* workspace,
    size_t workspace_bytes, pa_dtype dtype, int32_t* d_status, pa_stream_t stream);

PA_API pa_status pa_paged_decode_int8_rowscale_append(
    void* out, const void* query, const void* key, const void* value, void* k_cache,
    void* v_cache, float* k_scales, float* v_scales, const int32_t* block_tables,
    const int32_t* context_lens, int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
    int32_t head_dim, int32_t block_size, int32_t max_blocks_per_seq, int64_t num_blocks,
    int32_t max_context_len, float scale, int32_t partition_size, void* workspace,
    size_t workspace_bytes, pa_dtype dtype, int32_t* d_status, pa_stream_t stream);

/*
 * pa_paged_decode_shared_prefix -- pa_paged_decode for batches whose
 * sequences come in groups that share a stored prefix (the beams of one
 * prompt, parallel samples of one request).
 *
 * Defined by: [Practice §5.2 非连续KV访问优化] step 1 (process together the
 * queries that touch the same physical block) over the block sharing of
 * [VM-paging, 写时复制与块共享机制] and [Practice §4.1]: the members of a group
 * point at the same physical blocks for their first prefix_lens[g] tokens,
 * and those blocks are read from HBM once for all members.  The output is
 * that of pa_paged_decode on the same arguments (within rounding).
 *
 * Groups are group_size consecutive sequences: group g is sequences
 * [g * group_size, (g + 1) * group_size); num_seqs % group_size == 0.
 * prefix_lens    int32 [num_seqs / group_size], device: tokens group g shares,
 *                a multiple of block_size, at most every member's context
 *                length and at most max_prefix_len; 0 = nothing shared.  The
 *                members' block-table entries for those blocks must be equal.
 * max_prefix_len host: upper bound of prefix_lens (sizes the grid).
 * group_size * (num_q_heads / num_kv_heads) must be at most 8 and
 * block_size 16 or 32 (else PA_ERR_UNSUPPORTED).
 * Work split: each group's blocks form one list (the prefix blocks, then
 * every member's own blocks); one CTA covers a part of that list for one kv
 * head.  partition_size (0 = library's choice) is the part length in
 * tokens of that list; a group whose list fits one part is written
 * directly, others leave partials merged by a reduction kernel.
 * workspace      at least pa_paged_decode_shared_prefix_workspace_size(...)
 *                bytes, 16-byte aligned (may be NULL when that size is 0:
 *                every group's list fits one part).
 * d_status       as pa_paged_decode; a group whose prefix is not a whole
 *                number of blocks or is longer than a member's context (or
 *                max_prefix_len) sets PA_STATUS_BAD_CONTEXT and gets zero
 *                rows; members whose prefix block-table entries differ set
 *                PA_STATUS_BAD_BLOCK (their result is then unspecified).
 */
PA_API size_t pa_paged_decode_shared_prefix_workspace_size(
    int32_t num_seqs, int32_t group_size, int32_t num_q_heads, int32_t num_kv_heads,
    int32_t head_dim, int32_t block_size, int32_t max_context_len, int32_t max_prefix_len,
    int32_t partition_size);

PA_API pa_status pa_paged_decode_shared_prefix(
    void* out, const void* query, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, const int32_t* context_lens, const int32_t* prefix_lens,
    int32_t num_seqs, int32_t group_size, int32_t num_q_heads, int32_t num_kv_heads,
    int32_t head_dim, int32_t block_size, int32_t max_blocks_per_seq, int64_t num_blocks,
    int32_t max_context_len, int32_t max_prefix_len, float scale, int32_t partition_size,
    void* workspace, size_t workspace_bytes, pa_dtype dtype, int32_t* d_status,
    pa_stream_t stream);

/*
 * pa_paged_decode_no_alloc -- pa_paged_decode without a caller-supplied
 * workspace.
 *
 * The pages have no counterpart to this entry point.  It exists for callers
 * that cannot allocate device memory themselves: a plugin or custom operator
 * inside a host framework that owns every device allocation and hands the
 * plugin only its inputs and outputs, or code on a latency-critical path
 * that must not call cudaMalloc (which can synchronise the whole device) in
 * the middle of a step.
 *
 * Arguments and results are those of pa_paged_decode, minus `workspace` and
 * `workspace_bytes`.  The split-context scratch is instead a file-scope
 * device array of PA_NO_ALLOC_WORKSPACE_BYTES inside libpa.so; every GPU that
 * loads the library holds that memory until the process exits.  The call
 * allocates nothing: no cudaMalloc, no cudaFree, no allocating library call.
 *
 *  - A shape whose pa_paged_decode_workspace_size(...) is larger than
 *    PA_NO_ALLOC_WORKSPACE_BYTES is rejected with PA_ERR_INVALID_ARG before
 *    anything is enqueued; use pa_paged_decode with your own workspace (or a
 *    longer partition_size) for it.
 *  - Every call that needs the scratch looks up the array's device address
 *    in the current device's context (cudaGetSymbolAddress), so a device
 *    reset or another context never leaves a stale address behind.  The
 *    first such call on a device also loads the library's device code
 *    there: make that first call before any stream capture.
 *  - Every call shares the one array, which keeps the previous call's
 *    contents.  Nothing in it needs clearing (every value the reduction reads
 *    is written earlier in the same call), but calls that overlap on the GPU
 *    -- on different streams, or issued from different host threads -- race
 *    on it: order them.
 */
#define PA_NO_ALLOC_WORKSPACE_BYTES ((size_t)32 << 20)

PA_API pa_status pa_paged_decode_no_alloc(void* out, const void* query, const void* k_cache,
                                          const void* v_cache, const int32_t* block_tables,
                                          const int32_t* context_lens, int32_t num_seqs,
                                          int32_t num_q_heads, int32_t num_kv_heads,
                                          int32_t head_dim, int32_t block_size,
                                          int32_t max_blocks_per_seq, int64_t num_blocks,
                                          int32_t max_context_len, float scale,
                                          int32_t partition_size, pa_dtype dtype,
                                          int32_t* d_status, pa_stream_t stream);

/* Human-readable name of a pa_status (static string, never NULL). */
PA_API const char* pa_status_string(pa_status status);

/* Library version, e.g. "0.1.0" (static string). */
PA_API const char* pa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PA_H_ */
