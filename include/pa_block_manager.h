/*
 * pa_block_manager.h -- host-side KV block manager (C ABI, part of libpa.so).
 *
 * The layer directly above the kernels: it hands out the physical block ids
 * that pa_reshape_and_cache / pa_paged_decode address, keeps the block
 * tables, reference counts and the free pool, decides copy-on-write copies
 * (whose data copy is pa_copy_blocks) and, optionally, caches full blocks by
 * content so that a later request with the same prefix reuses them.
 *
 * Pages cited (title, then section):
 *   [VM-paging] "vLLM用虚拟内存分页思想管理KV Cache"
 *   [Practice]  "PagedAttention：大模型KV Cache分页管理优化实践"
 *   [Manager]   "深入解析 vLLM 的 KV Cache 管理器：从内存碎片到 PagedAttention 的完整技术剖析"
 *
 * Behaviour:
 *  - fixed-size blocks from one pool; a block table per sequence
 *    ([VM-paging, 虚拟内存分页机制到KV Cache的映射]; [Practice §3.2]);
 *  - on-demand allocation: a token goes into the last block when it has
 *    room, else into a new block taken from the head of the free queue
 *    ([Practice §3.3 按需分配策略]);
 *  - sharing raises reference counts; a sequence writing into a block whose
 *    count is above 1 gets a private copy (a (src, dst) pair for
 *    pa_copy_blocks) and drops one reference on the original; with a count
 *    of 1 it writes in place ([VM-paging, 写时复制与块共享机制]; [Practice §4.1]);
 *  - freeing drops one reference per block (last block first); a block whose
 *    count reaches 0 goes to the tail of the free queue
 *    ([VM-paging, 写时复制与块共享机制]);
 *  - the free queue is a doubly linked list, so a cached block can be taken
 *    out of the middle in O(1) when a prefix hits it
 *    ([Manager, 第四部分 FreeKVCacheBlockQueue]);
 *  - automatic prefix caching (optional): every full block gets the hash
 *    hash(parent block's hash, the block's tokens, extra key), a chain so
 *    that two sequences share block N only if all tokens up to it agree and
 *    the extra key (LoRA adapter id, multimodal content hash, ...) is equal
 *    ([Manager, 第三部分 哈希链的设计]); freed blocks keep their hash and stay
 *    findable until the allocator reuses them ([Manager, 第三部分 APC 的工作机制]);
 *    allocation pops the queue head and, if that block still carries a hash,
 *    evicts it from the cache then ([Manager, 第四部分 BlockPool]);
 *  - a request that needs more free blocks than there are fails with
 *    PA_BM_NO_SPACE and leaves every structure unchanged
 *    ([Manager, 第四部分 KVCacheManager 与 allocate_slots()]);
 *  - swapping (optional, with a host pool attached): a group of sequences
 *    (the beams of one request, say) moves to host blocks and back, the
 *    mechanism of evicting a waiting request's KV to CPU memory and
 *    restoring it when the request is scheduled again
 *    ([VM-paging, 显存管理与调度策略设计], the eviction paragraph; [Manager,
 *    第四部分]: the cache manager supplies the mechanism, the scheduler the
 *    policy).  The byte copies are pa_swap_blocks calls with the pairs the
 *    manager returns.
 *
 * Slots are physical_block * block_size + offset.  Sequence ids are any
 * int64 chosen by the caller.  The manager is not thread-safe: one caller at
 * a time.  Host memory only; no GPU call is made.
 */
#ifndef PA_BLOCK_MANAGER_H_
#define PA_BLOCK_MANAGER_H_

#include <stdint.h>

#include "pa.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct pa_block_manager pa_block_manager;

/* Return codes of the pa_bm_* calls. */
#define PA_BM_OK 0
#define PA_BM_NO_SPACE 1        /* not enough free blocks; nothing changed */
#define PA_BM_BAD_ARG 2         /* null pointer, bad size, unknown/duplicate sequence id */
#define PA_BM_CAPACITY 3        /* an output buffer is too small; nothing changed */

/* A manager over blocks [0, num_blocks) of block_size tokens; free queue in
 * id order.  prefix_caching != 0 enables the content cache of full blocks.
 * Returns NULL on bad arguments or allocation failure. */
PA_API pa_block_manager* pa_bm_create(int32_t num_blocks, int32_t block_size,
                                      int32_t prefix_caching);
PA_API void pa_bm_destroy(pa_block_manager* bm);

PA_API int32_t pa_bm_num_free_blocks(const pa_block_manager* bm);
/* Reference count of a block (-1 for an id outside the pool). */
PA_API int32_t pa_bm_ref_count(const pa_block_manager* bm, int32_t block);
/* Blocks currently findable by content (with or without users). */
PA_API int32_t pa_bm_num_cached_blocks(const pa_block_manager* bm);

/* Register sequence seq_id with its first num_tokens tokens and give them
 * slots.  tokens: the token ids (needed only with prefix caching, may be
 * NULL otherwise).  With prefix caching, leading full blocks whose hash
 * chain is cached are reused (their KV need not be recomputed) and
 * *num_cached receives how many leading tokens that covers -- always fewer
 * than num_tokens, so at least the last token is computed; else 0.
 * slots_out: num_tokens entries (may be NULL). */
PA_API int32_t pa_bm_add_sequence(pa_block_manager* bm, int64_t seq_id, const int32_t* tokens,
                                  int32_t num_tokens, int64_t extra_key, int64_t* slots_out,
                                  int32_t* num_cached);

/* child shares every block of parent (reference counts rise by one). */
PA_API int32_t pa_bm_fork(pa_block_manager* bm, int64_t parent, int64_t child);

/* Slots for the next n tokens of seq_id.  tokens: their ids (prefix caching
 * only, may be NULL otherwise).  cow_out: room for cow_capacity (src, dst)
 * pairs (int64 [cow_capacity][2]); *num_cow receives the number of block
 * copies that must run (pa_copy_blocks) before the tokens are written.  At
 * most one copy per call is ever needed, so cow_capacity >= 1 suffices. */
PA_API int32_t pa_bm_append_slots(pa_block_manager* bm, int64_t seq_id, const int32_t* tokens,
                                  int32_t n, int64_t* slots_out, int64_t* cow_out,
                                  int32_t cow_capacity, int32_t* num_cow);

/* Drop the sequence and one reference on each of its blocks. */
PA_API int32_t pa_bm_free_sequence(pa_block_manager* bm, int64_t seq_id);

/* The sequence's block table: *num_blocks entries written to table_out
 * (capacity entries available; PA_BM_CAPACITY if too small). */
PA_API int32_t pa_bm_block_table(const pa_block_manager* bm, int64_t seq_id, int32_t* table_out,
                                 int32_t capacity, int32_t* num_blocks);
/* Number of tokens of the sequence (-1 if unknown). */
PA_API int32_t pa_bm_context_len(const pa_block_manager* bm, int64_t seq_id);

/*
 * Watermark ([VM-paging, 显存管理与调度策略设计]: a share of the blocks, 5% say,
 * is held back so that the requests already running can keep growing when
 * free blocks run low).  After pa_bm_set_watermark(bm, r), pa_bm_add_sequence
 * and pa_bm_swap_in return PA_BM_NO_SPACE when they would leave fewer than r
 * free blocks; pa_bm_append_slots may use the reserve.  0 <= r <=
 * num_blocks (else PA_BM_BAD_ARG); the default is 0.
 */
PA_API int32_t pa_bm_set_watermark(pa_block_manager* bm, int32_t reserved_blocks);

/* pa_bm_add_sequence for a request that may draw on the watermark reserve
 * when high_priority != 0: the two-level allocation of [Practice §7
 * 演进方向与优化空间], where the reserve is a fast pool kept for high-priority
 * requests once utilisation is high.  With high_priority == 0 it is
 * pa_bm_add_sequence. */
PA_API int32_t pa_bm_add_sequence_priority(pa_block_manager* bm, int64_t seq_id,
                                           const int32_t* tokens, int32_t num_tokens,
                                           int64_t extra_key, int32_t high_priority,
                                           int64_t* slots_out, int32_t* num_cached);

/*
 * Swapping.  pa_bm_attach_host_pool gives the manager host blocks
 * [0, num_host_blocks) of a pinned host pool shaped like the device pool
 * (once per manager).  While a sequence is swapped out it has no device
 * blocks: pa_bm_append_slots, pa_bm_fork and pa_bm_block_table return
 * PA_BM_BAD_ARG for it, pa_bm_context_len still answers, and
 * pa_bm_free_sequence releases its host blocks.
 *
 * pa_bm_swap_out -- the group seq_ids[0 .. num_seqs) (distinct, all
 *   resident) moves to the host pool.  Every distinct device block of the
 *   group gets one host block, so blocks the group shares stay shared; the
 *   group's references on the device blocks are dropped, and blocks left
 *   without users return to the free queue (a full block keeps its hash, so
 *   a later prefix hit or swap-in can still find it).  pairs_out receives
 *   *num_pairs (device block, host block) pairs, int64 [capacity][2], for
 *   pa_swap_blocks from the device pools to the host pools; those copies
 *   must run before any kernel that writes a block allocated after this
 *   call (stream order does it when they are enqueued first).
 * pa_bm_swap_in -- the group (distinct, all swapped out) comes back.  Each
 *   distinct host block becomes one device block: a full block whose hash is
 *   still in the prefix cache is revived without a copy, any other block
 *   gets a fresh device block and a (host block, device block) pair for
 *   pa_swap_blocks from the host pools to the device pools, to run before the
 *   group's next decode.  Block tables are in the same order as before.
 * Both are all or nothing: PA_BM_NO_SPACE when the destination pool lacks
 * room, PA_BM_CAPACITY when pairs_out has fewer than the needed entries
 * (one per block of the group suffices), PA_BM_BAD_ARG for an unknown,
 * repeated or wrongly placed sequence or when no host pool is attached; in
 * each case nothing changes.
 */
PA_API int32_t pa_bm_attach_host_pool(pa_block_manager* bm, int32_t num_host_blocks);
PA_API int32_t pa_bm_num_free_host_blocks(const pa_block_manager* bm);
/* 1 if the sequence is swapped out, 0 if resident, -1 if unknown. */
PA_API int32_t pa_bm_is_swapped(const pa_block_manager* bm, int64_t seq_id);
PA_API int32_t pa_bm_swap_out(pa_block_manager* bm, const int64_t* seq_ids, int32_t num_seqs,
                              int64_t* pairs_out, int32_t capacity, int32_t* num_pairs);
PA_API int32_t pa_bm_swap_in(pa_block_manager* bm, const int64_t* seq_ids, int32_t num_seqs,
                             int64_t* pairs_out, int32_t capacity, int32_t* num_pairs);

/*
 * Monitoring ([Practice §6.3 实际部署建议]: watch the physical block
 * utilisation, above 90% as the target, and the hit rate).
 *   used_blocks     blocks with at least one user;
 *   stored_tokens   tokens held in them, a shared block counted once (its
 *                   fill is the most tokens any of its users keeps in it);
 *                   utilisation = stored_tokens / (used_blocks * block_size),
 *                   internal waste = 1 - utilisation;
 *   prefix_queries, prefix_hits   full prompt blocks that
 *                   pa_bm_add_sequence looked up in the prefix cache, and
 *                   how many it reused (prefix caching only; successful
 *                   calls only); hit rate = hits / queries.
 */
typedef struct pa_bm_stats_t {
    int32_t num_blocks, block_size;
    int32_t used_blocks, free_blocks, cached_blocks;
    int32_t num_seqs, swapped_seqs, free_host_blocks;
    int64_t stored_tokens;
    int64_t prefix_queries, prefix_hits;
} pa_bm_stats_t;

PA_API int32_t pa_bm_stats(const pa_block_manager* bm, pa_bm_stats_t* out);

/* Checks every invariant (counts equal table references, free queue holds
 * exactly the blocks with count 0, no cycles, cached hashes map back to
 * their blocks, internal waste <= block_size - 1, and for the host pool:
 * swapped sequences hold host blocks only, host counts equal references,
 * the host free list holds exactly the host blocks with count 0).  0 = all
 * hold, else a code naming the first violated one. */
PA_API int32_t pa_bm_check(const pa_block_manager* bm);

#ifdef __cplusplus
}
#endif

#endif /* PA_BLOCK_MANAGER_H_ */
