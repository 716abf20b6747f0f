/*
 * pa_selftest.h -- test entry points of libpa.so's bounded waits.
 *
 * Every wait the decode kernels make for an asynchronous copy (an mbarrier
 * phase that completes when a block's K/V tiles have landed in shared
 * memory) gives up after a bounded time, sets PA_STATUS_TIMEOUT in the
 * device status word and lets the kernel finish, so that a copy that never
 * lands cannot hang the GPU.  Such a copy should never happen, so these
 * entry points make a wait run out on purpose, without any fault: they wait
 * on an mbarrier that nothing arrives on, with a short limit.  They serve
 * tests; a production caller has no use for them.
 *
 * The pages name graceful degradation when a part fails ("PagedAttention：
 * 大模型KV Cache分页管理优化实践" §6.3 实际部署建议, item 4); this is its device
 * half: a stuck wait turns into a status bit the host reads.
 *
 * Conventions (memory, errors, streams) as in pa.h.
 */
#ifndef PA_SELFTEST_H_
#define PA_SELFTEST_H_

#include "pa.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * pa_selftest_bounded_wait -- num_ctas CTAs of 128 threads each wait on an
 * mbarrier that nothing arrives on, with the library's warp-uniform bounded
 * wait and a limit of wait_limit_us microseconds; every warp that gives up
 * ORs PA_STATUS_TIMEOUT into *d_status.  The kernel then returns normally.
 *
 * d_status      device int32, required (the caller clears it).
 * d_wait_ns     optional device int64 [num_ctas]: each CTA's measured wait
 *               (global timer, nanoseconds) until its warps gave up.
 * wait_limit_us 1 .. 1000000; num_ctas 1 .. 1024 (else PA_ERR_INVALID_ARG).
 */
PA_API pa_status pa_selftest_bounded_wait(int32_t* d_status, int64_t* d_wait_ns,
                                          uint32_t wait_limit_us, int32_t num_ctas,
                                          pa_stream_t stream);

/*
 * pa_selftest_decode_abort -- pa_paged_decode (kv_dtype == dtype), or
 * pa_paged_decode_fp8 / _int8 with both scales 1 (kv_dtype
 * PA_DTYPE_FP8_E4M3 / PA_DTYPE_INT8), on the same kernels and launch
 * configuration, except that the first wait of every warp that has blocks
 * to read goes to an mbarrier that nothing completes, with a limit of
 * wait_limit_us microseconds (1 .. 1000000).  So every CTA runs the abort
 * path of a timed-out copy for real:
 *   - the warp sets PA_STATUS_TIMEOUT and waits again, bounded, for the
 *     copies it had already started (they land);
 *   - the CTA never reads or reuses that shared memory: it writes "no
 *     result" through global memory and returns -- zero output rows for a
 *     context that fits one partition, else an empty partial (max -inf,
 *     exp-sum 0) that the reduction weighs with 0.
 * Result: every output row is zero and *d_status is PA_STATUS_TIMEOUT
 * (plus whatever data errors the inputs carry).  Arguments and checks
 * otherwise as pa_paged_decode.
 */
PA_API pa_status pa_selftest_decode_abort(
    void* out, const void* query, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, const int32_t* context_lens, int32_t num_seqs,
    int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
    int32_t max_blocks_per_seq, int64_t num_blocks, int32_t max_context_len, float scale,
    int32_t partition_size, void* workspace, size_t workspace_bytes, pa_dtype dtype,
    pa_dtype kv_dtype, uint32_t wait_limit_us, int32_t* d_status, pa_stream_t stream);

/*
 * pa_selftest_shared_prefix_abort -- the same for
 * pa_paged_decode_shared_prefix (same arguments plus wait_limit_us): every
 * group's rows come out zero and *d_status is PA_STATUS_TIMEOUT.
 */
PA_API pa_status pa_selftest_shared_prefix_abort(
    void* out, const void* query, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, const int32_t* context_lens, const int32_t* prefix_lens,
    int32_t num_seqs, int32_t group_size, int32_t num_q_heads, int32_t num_kv_heads,
    int32_t head_dim, int32_t block_size, int32_t max_blocks_per_seq, int64_t num_blocks,
    int32_t max_context_len, int32_t max_prefix_len, float scale, int32_t partition_size,
    void* workspace, size_t workspace_bytes, pa_dtype dtype, uint32_t wait_limit_us,
    int32_t* d_status, pa_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* PA_SELFTEST_H_ */
