// block_manager.cpp -- host-side KV block manager (see include/pa_block_manager.h).
//
// Pages cited (title, then section):
//   [VM-paging] "vLLM用虚拟内存分页思想管理KV Cache"
//   [Practice]  "PagedAttention：大模型KV Cache分页管理优化实践"
//   [Manager]   "深入解析 vLLM 的 KV Cache 管理器：从内存碎片到 PagedAttention 的完整技术剖析"
#include "pa_block_manager.h"

#include <stdint.h>

#include <algorithm>
#include <new>
#include <unordered_map>
#include <vector>

namespace {

// 64-bit mixing step (the splitmix64 finaliser of Steele, Lea and Flood).
inline uint64_t mix64(uint64_t z)
{
    z += 0x9e3779b97f4a7c15ull;
    z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ull;
    z = (z ^ (z >> 27)) * 0x94d049bb133111ebull;
    return z ^ (z >> 31);
}

// Hash of a full block: its parent's hash, the extra key and its tokens
// ([Manager, 第三部分 哈希链的设计]).
inline uint64_t block_hash(uint64_t parent, int64_t extra_key, const int32_t* tokens, int n)
{
    uint64_t h = mix64(parent ^ mix64(static_cast<uint64_t>(extra_key)));
    for (int i = 0; i < n; ++i) h = mix64(h ^ static_cast<uint32_t>(tokens[i]));
    return h;
}

constexpr uint64_t kRootHash = 0x5041474544ull;   // parent of a sequence's first block

struct Block {
    int32_t ref = 0;
    int32_t prev = -1, next = -1;   // free-queue links
    bool in_free = false;
    bool hashed = false;
    uint64_t hash = 0;
};

struct Seq {
    std::vector<int32_t> table;       // device blocks (empty while swapped out)
    int32_t len = 0;
    int64_t extra_key = 0;
    std::vector<int32_t> tokens;    // kept only with prefix caching
    uint64_t last_full_hash = kRootHash;
    bool swapped = false;
    std::vector<int32_t> host_table;  // host blocks while swapped out
};

}  // namespace

struct pa_block_manager {
    int32_t num_blocks = 0, block_size = 0;
    bool caching = false;
    int32_t watermark = 0;      // free blocks that admissions must leave untouched
    int64_t prefix_queries = 0, prefix_hits = 0;   // full prompt blocks looked up / found
    std::vector<Block> blocks;
    int32_t head = -1, tail = -1, nfree = 0;
    std::unordered_map<uint64_t, int32_t> cache;     // hash -> block
    std::unordered_map<int64_t, Seq> seqs;
    // host pool for swapped-out sequences: reference counts and free ids
    int32_t num_host = 0;
    std::vector<int32_t> host_ref;
    std::vector<int32_t> host_free;                  // a stack; the top is taken first

    // ---- free queue: O(1) push at the tail, pop at the head, remove anywhere
    void push_back(int32_t b)
    {
        Block& x = blocks[b];
        x.prev = tail;
        x.next = -1;
        if (tail >= 0) blocks[tail].next = b; else head = b;
        tail = b;
        x.in_free = true;
        ++nfree;
    }
    void remove(int32_t b)
    {
        Block& x = blocks[b];
        if (x.prev >= 0) blocks[x.prev].next = x.next; else head = x.next;
        if (x.next >= 0) blocks[x.next].prev = x.prev; else tail = x.prev;
        x.prev = x.next = -1;
        x.in_free = false;
        --nfree;
    }
    // Allocation: the head of the free queue; a block that still carries a
    // hash is dropped from the cache now ([Manager, 第四部分 BlockPool]).
    int32_t take()
    {
        const int32_t b = head;
        remove(b);
        Block& x = blocks[b];
        if (x.hashed) {
            auto it = cache.find(x.hash);
            if (it != cache.end() && it->second == b) cache.erase(it);
            x.hashed = false;
        }
        x.ref = 1;
        return b;
    }
    void register_full_block(int32_t b, uint64_t h)
    {
        if (!caching || cache.count(h)) return;
        cache.emplace(h, b);
        blocks[b].hashed = true;
        blocks[b].hash = h;
    }
    int64_t slot_of(const Seq& q, int32_t pos) const
    {
        return static_cast<int64_t>(q.table[pos / block_size]) * block_size + pos % block_size;
    }
    // Hashes of a sequence's full blocks, from its tokens (prefix caching).
    std::vector<uint64_t> full_hashes(const Seq& q) const
    {
        std::vector<uint64_t> h;
        uint64_t parent = kRootHash;
        for (int32_t j = 0; j < q.len / block_size; ++j) {
            parent = block_hash(parent, q.extra_key,
                                q.tokens.data() + static_cast<int64_t>(j) * block_size,
                                block_size);
            h.push_back(parent);
        }
        return h;
    }
    // The distinct sequences of a group, each known and in the given swap
    // state; nullptr entries never returned.
    bool group(const int64_t* ids, int32_t n, bool swapped, std::vector<Seq*>* out)
    {
        if (ids == nullptr || n <= 0 || num_host == 0) return false;
        for (int32_t i = 0; i < n; ++i) {
            auto it = seqs.find(ids[i]);
            if (it == seqs.end() || it->second.swapped != swapped) return false;
            if (std::find(out->begin(), out->end(), &it->second) != out->end()) return false;
            out->push_back(&it->second);
        }
        return true;
    }
};

extern "C" pa_block_manager* pa_bm_create(int32_t num_blocks, int32_t block_size,
                                          int32_t prefix_caching)
{
    if (num_blocks <= 0 || block_size <= 0) return nullptr;
    pa_block_manager* bm = new (std::nothrow) pa_block_manager();
    if (!bm) return nullptr;
    try {
        bm->num_blocks = num_blocks;
        bm->block_size = block_size;
        bm->caching = prefix_caching != 0;
        bm->blocks.resize(num_blocks);
        for (int32_t b = 0; b < num_blocks; ++b) bm->push_back(b);
    } catch (...) {
        delete bm;
        return nullptr;
    }
    return bm;
}

extern "C" void pa_bm_destroy(pa_block_manager* bm) { delete bm; }

extern "C" int32_t pa_bm_num_free_blocks(const pa_block_manager* bm) { return bm ? bm->nfree : 0; }

extern "C" int32_t pa_bm_ref_count(const pa_block_manager* bm, int32_t block)
{
    if (!bm || block < 0 || block >= bm->num_blocks) return -1;
    return bm->blocks[block].ref;
}

extern "C" int32_t pa_bm_num_cached_blocks(const pa_block_manager* bm)
{
    return bm ? static_cast<int32_t>(bm->cache.size()) : 0;
}

static int32_t add_sequence(pa_block_manager* bm, int64_t seq_id, const int32_t* tokens,
                            int32_t num_tokens, int64_t extra_key, bool may_use_reserve,
                            int64_t* slots_out, int32_t* num_cached)
{
    if (!bm || num_tokens < 0 || bm->seqs.count(seq_id)) return PA_BM_BAD_ARG;
    if (bm->caching && num_tokens > 0 && tokens == nullptr) return PA_BM_BAD_ARG;
    const int32_t B = bm->block_size;
    const int32_t nblk = (num_tokens + B - 1) / B;
    const int32_t nfull = num_tokens / B;

    // prefix hits: leading full blocks whose hash chain is cached
    // ([Manager, 第三部分 APC 的工作机制]); always leave the last token to compute
    std::vector<uint64_t> hashes;
    std::vector<int32_t> hits;
    if (bm->caching) {
        uint64_t parent = kRootHash;
        for (int32_t j = 0; j < nfull; ++j) {
            parent = block_hash(parent, extra_key, tokens + static_cast<int64_t>(j) * B, B);
            hashes.push_back(parent);
        }
        for (int32_t j = 0; j < nfull; ++j) {
            auto it = bm->cache.find(hashes[j]);
            if (it == bm->cache.end()) break;
            hits.push_back(it->second);
        }
        if (!hits.empty() && static_cast<int64_t>(hits.size()) * B >= num_tokens) hits.pop_back();
    }
    int32_t revived = 0;
    for (int32_t b : hits) revived += bm->blocks[b].ref == 0;
    const int32_t fresh = nblk - static_cast<int32_t>(hits.size());
    const int32_t reserve = may_use_reserve ? 0 : bm->watermark;
    if (fresh + revived > bm->nfree - reserve) return PA_BM_NO_SPACE;

    Seq q;
    q.extra_key = extra_key;
    q.len = num_tokens;
    try {
        q.table.reserve(nblk);
        for (int32_t b : hits) {
            if (bm->blocks[b].ref == 0) bm->remove(b);
            ++bm->blocks[b].ref;
            q.table.push_back(b);
        }
        for (int32_t j = static_cast<int32_t>(hits.size()); j < nblk; ++j) {
            const int32_t b = bm->take();
            q.table.push_back(b);
            if (j < nfull && bm->caching) bm->register_full_block(b, hashes[j]);
        }
        if (bm->caching) {
            q.tokens.assign(tokens, tokens + num_tokens);
            q.last_full_hash = nfull > 0 ? hashes[nfull - 1] : kRootHash;
        }
        if (slots_out)
            for (int32_t i = 0; i < num_tokens; ++i) slots_out[i] = bm->slot_of(q, i);
        bm->seqs.emplace(seq_id, std::move(q));
    } catch (...) {
        return PA_BM_BAD_ARG;
    }
    if (num_cached) *num_cached = static_cast<int32_t>(hits.size()) * B;
    if (bm->caching) {
        bm->prefix_queries += nfull;
        bm->prefix_hits += static_cast<int64_t>(hits.size());
    }
    return PA_BM_OK;
}

extern "C" int32_t pa_bm_add_sequence(pa_block_manager* bm, int64_t seq_id, const int32_t* tokens,
                                      int32_t num_tokens, int64_t extra_key, int64_t* slots_out,
                                      int32_t* num_cached)
{
    return add_sequence(bm, seq_id, tokens, num_tokens, extra_key, false, slots_out, num_cached);
}

// The two-level allocation of [Practice §7 演进方向与优化空间]: the watermark
// reserve is the fast pool that only high-priority requests may draw on.
extern "C" int32_t pa_bm_add_sequence_priority(pa_block_manager* bm, int64_t seq_id,
                                               const int32_t* tokens, int32_t num_tokens,
                                               int64_t extra_key, int32_t high_priority,
                                               int64_t* slots_out, int32_t* num_cached)
{
    return add_sequence(bm, seq_id, tokens, num_tokens, extra_key, high_priority != 0, slots_out,
                        num_cached);
}

extern "C" int32_t pa_bm_fork(pa_block_manager* bm, int64_t parent, int64_t child)
{
    if (!bm || parent == child) return PA_BM_BAD_ARG;
    auto it = bm->seqs.find(parent);
    if (it == bm->seqs.end() || it->second.swapped || bm->seqs.count(child)) return PA_BM_BAD_ARG;
    try {
        Seq q = it->second;
        for (int32_t b : q.table) ++bm->blocks[b].ref;
        bm->seqs.emplace(child, std::move(q));
    } catch (...) {
        return PA_BM_BAD_ARG;
    }
    return PA_BM_OK;
}

extern "C" int32_t pa_bm_append_slots(pa_block_manager* bm, int64_t seq_id, const int32_t* tokens,
                                      int32_t n, int64_t* slots_out, int64_t* cow_out,
                                      int32_t cow_capacity, int32_t* num_cow)
{
    if (!bm || n < 0) return PA_BM_BAD_ARG;
    auto it = bm->seqs.find(seq_id);
    if (it == bm->seqs.end() || it->second.swapped) return PA_BM_BAD_ARG;
    if (bm->caching && n > 0 && tokens == nullptr) return PA_BM_BAD_ARG;
    Seq& q = it->second;
    const int32_t B = bm->block_size;
    int32_t need = 0;
    bool cow = false;
    if (n > 0) {
        need = (q.len + n + B - 1) / B - (q.len + B - 1) / B;
        cow = q.len % B != 0 && bm->blocks[q.table.back()].ref > 1;
        need += cow;
    }
    if (need > bm->nfree) return PA_BM_NO_SPACE;
    if (cow && (cow_out == nullptr || cow_capacity < 1)) return PA_BM_CAPACITY;
    int32_t pairs = 0;
    try {
        if (bm->caching) q.tokens.reserve(q.tokens.size() + n);
        q.table.reserve((q.len + n + B - 1) / B);
        for (int32_t i = 0; i < n; ++i) {
            const int32_t pos = q.len;
            if (pos % B == 0) {
                q.table.push_back(bm->take());
            } else {
                const int32_t last = q.table.back();
                if (bm->blocks[last].ref > 1) {          // copy on write
                    const int32_t fresh = bm->take();
                    cow_out[2 * pairs] = last;
                    cow_out[2 * pairs + 1] = fresh;
                    ++pairs;
                    --bm->blocks[last].ref;
                    q.table.back() = fresh;
                }
            }
            if (slots_out) slots_out[i] = bm->slot_of(q, pos);
            q.len = pos + 1;
            if (bm->caching) {
                q.tokens.push_back(tokens[i]);
                if (q.len % B == 0) {                    // the block just filled up
                    const uint64_t h = block_hash(q.last_full_hash, q.extra_key,
                                                  q.tokens.data() + (q.len - B), B);
                    q.last_full_hash = h;
                    bm->register_full_block(q.table.back(), h);
                }
            }
        }
    } catch (...) {
        return PA_BM_BAD_ARG;
    }
    if (num_cow) *num_cow = pairs;
    return PA_BM_OK;
}

extern "C" int32_t pa_bm_free_sequence(pa_block_manager* bm, int64_t seq_id)
{
    if (!bm) return PA_BM_BAD_ARG;
    auto it = bm->seqs.find(seq_id);
    if (it == bm->seqs.end()) return PA_BM_BAD_ARG;
    const std::vector<int32_t>& t = it->second.table;
    for (auto r = t.rbegin(); r != t.rend(); ++r) {       // last block first
        Block& x = bm->blocks[*r];
        if (--x.ref == 0) bm->push_back(*r);
    }
    for (auto r = it->second.host_table.rbegin(); r != it->second.host_table.rend(); ++r)
        if (--bm->host_ref[*r] == 0) bm->host_free.push_back(*r);
    bm->seqs.erase(it);
    return PA_BM_OK;
}

extern "C" int32_t pa_bm_block_table(const pa_block_manager* bm, int64_t seq_id,
                                     int32_t* table_out, int32_t capacity, int32_t* num_blocks)
{
    if (!bm) return PA_BM_BAD_ARG;
    auto it = bm->seqs.find(seq_id);
    if (it == bm->seqs.end() || it->second.swapped) return PA_BM_BAD_ARG;
    const std::vector<int32_t>& t = it->second.table;
    if (num_blocks) *num_blocks = static_cast<int32_t>(t.size());
    if (static_cast<int64_t>(t.size()) > capacity || (!t.empty() && table_out == nullptr))
        return PA_BM_CAPACITY;
    for (size_t i = 0; i < t.size(); ++i) table_out[i] = t[i];
    return PA_BM_OK;
}

extern "C" int32_t pa_bm_context_len(const pa_block_manager* bm, int64_t seq_id)
{
    if (!bm) return -1;
    auto it = bm->seqs.find(seq_id);
    return it == bm->seqs.end() ? -1 : it->second.len;
}

// The watermark of [VM-paging, 显存管理与调度策略设计]: a reserve of free blocks
// that new (and resumed) requests may not take, so that running requests can
// still grow when memory is tight.
extern "C" int32_t pa_bm_set_watermark(pa_block_manager* bm, int32_t reserved_blocks)
{
    if (!bm || reserved_blocks < 0 || reserved_blocks > bm->num_blocks) return PA_BM_BAD_ARG;
    bm->watermark = reserved_blocks;
    return PA_BM_OK;
}

extern "C" int32_t pa_bm_attach_host_pool(pa_block_manager* bm, int32_t num_host_blocks)
{
    if (!bm || bm->num_host != 0 || num_host_blocks <= 0) return PA_BM_BAD_ARG;
    try {
        bm->host_ref.assign(num_host_blocks, 0);
        bm->host_free.reserve(num_host_blocks);
        for (int32_t h = num_host_blocks - 1; h >= 0; --h) bm->host_free.push_back(h);
    } catch (...) {
        bm->host_ref.clear();
        bm->host_free.clear();
        return PA_BM_BAD_ARG;
    }
    bm->num_host = num_host_blocks;
    return PA_BM_OK;
}

extern "C" int32_t pa_bm_num_free_host_blocks(const pa_block_manager* bm)
{
    return bm ? static_cast<int32_t>(bm->host_free.size()) : 0;
}

extern "C" int32_t pa_bm_is_swapped(const pa_block_manager* bm, int64_t seq_id)
{
    if (!bm) return -1;
    auto it = bm->seqs.find(seq_id);
    return it == bm->seqs.end() ? -1 : (it->second.swapped ? 1 : 0);
}

// Evict a group to the host pool ([VM-paging, 显存管理与调度策略设计]: the KV of
// waiting requests moves to CPU memory under pressure).  Each distinct device
// block of the group gets one host block, so blocks the group shares stay
// shared on the host; the group's references on the device blocks are then
// dropped (last block first, sequence by sequence), and blocks left without
// users return to the free queue with their hashes.
extern "C" int32_t pa_bm_swap_out(pa_block_manager* bm, const int64_t* seq_ids, int32_t num_seqs,
                                  int64_t* pairs_out, int32_t capacity, int32_t* num_pairs)
{
    if (!bm) return PA_BM_BAD_ARG;
    try {
        std::vector<Seq*> g;
        if (!bm->group(seq_ids, num_seqs, false, &g)) return PA_BM_BAD_ARG;
        std::unordered_map<int32_t, int32_t> host_of;  // device block -> host block
        std::vector<int32_t> order;                    // distinct device blocks, first use first
        for (Seq* q : g)
            for (int32_t b : q->table)
                if (host_of.emplace(b, -1).second) order.push_back(b);
        const int32_t need = static_cast<int32_t>(order.size());
        if (need > static_cast<int32_t>(bm->host_free.size())) return PA_BM_NO_SPACE;
        if (need > capacity || (need > 0 && pairs_out == nullptr)) return PA_BM_CAPACITY;
        for (Seq* q : g) q->host_table.reserve(q->table.size());
        for (int32_t i = 0; i < need; ++i) {
            const int32_t h = bm->host_free.back();
            bm->host_free.pop_back();
            host_of[order[i]] = h;
            pairs_out[2 * i] = order[i];
            pairs_out[2 * i + 1] = h;
        }
        for (Seq* q : g) {
            for (int32_t b : q->table) {
                const int32_t h = host_of[b];
                ++bm->host_ref[h];
                q->host_table.push_back(h);
            }
            for (auto r = q->table.rbegin(); r != q->table.rend(); ++r)
                if (--bm->blocks[*r].ref == 0) bm->push_back(*r);
            q->table.clear();
            q->swapped = true;
        }
        if (num_pairs) *num_pairs = need;
    } catch (...) {
        return PA_BM_BAD_ARG;
    }
    return PA_BM_OK;
}

// Bring a swapped-out group back.  Each distinct host block becomes one
// device block: a full block whose hash is still in the prefix cache is
// revived in place (its bytes never left the device), any other block gets
// a fresh device block and a (host, device) copy.  All or nothing.
extern "C" int32_t pa_bm_swap_in(pa_block_manager* bm, const int64_t* seq_ids, int32_t num_seqs,
                                 int64_t* pairs_out, int32_t capacity, int32_t* num_pairs)
{
    if (!bm) return PA_BM_BAD_ARG;
    try {
        std::vector<Seq*> g;
        if (!bm->group(seq_ids, num_seqs, true, &g)) return PA_BM_BAD_ARG;
        struct Need {
            int32_t host;
            bool full;
            uint64_t hash;
            int32_t revive;       // cached device block, or -1
        };
        std::unordered_map<int32_t, int32_t> index;    // host block -> position in needs
        std::vector<Need> needs;
        for (Seq* q : g) {
            const std::vector<uint64_t> hashes = bm->caching ? bm->full_hashes(*q)
                                                             : std::vector<uint64_t>();
            for (size_t j = 0; j < q->host_table.size(); ++j) {
                const int32_t h = q->host_table[j];
                if (!index.emplace(h, static_cast<int32_t>(needs.size())).second) continue;
                Need n{h, j < hashes.size(), j < hashes.size() ? hashes[j] : 0, -1};
                if (n.full) {
                    auto c = bm->cache.find(n.hash);
                    if (c != bm->cache.end()) n.revive = c->second;
                }
                needs.push_back(n);
            }
        }
        int32_t fresh = 0, from_free = 0;
        std::vector<int32_t> revived;
        for (const Need& n : needs) {
            if (n.revive < 0) {
                ++fresh;
            } else if (std::find(revived.begin(), revived.end(), n.revive) == revived.end()) {
                revived.push_back(n.revive);
                from_free += bm->blocks[n.revive].ref == 0;
            }
        }
        if (fresh + from_free > bm->nfree - bm->watermark) return PA_BM_NO_SPACE;
        if (fresh > capacity || (fresh > 0 && pairs_out == nullptr)) return PA_BM_CAPACITY;
        for (Seq* q : g) q->table.reserve(q->host_table.size());

        std::vector<int32_t> dev(needs.size());
        for (int32_t b : revived)
            if (bm->blocks[b].ref == 0) bm->remove(b);  // out of the queue before any take()
        int32_t pairs = 0;
        for (size_t i = 0; i < needs.size(); ++i) {
            const Need& n = needs[i];
            if (n.revive >= 0) {
                dev[i] = n.revive;
                continue;
            }
            const int32_t b = bm->take();
            bm->blocks[b].ref = 0;                     // counted per table entry below
            if (n.full) bm->register_full_block(b, n.hash);
            dev[i] = b;
            pairs_out[2 * pairs] = n.host;
            pairs_out[2 * pairs + 1] = b;
            ++pairs;
        }
        for (Seq* q : g) {
            for (int32_t h : q->host_table) {
                const int32_t b = dev[index[h]];
                ++bm->blocks[b].ref;
                q->table.push_back(b);
            }
            for (auto r = q->host_table.rbegin(); r != q->host_table.rend(); ++r)
                if (--bm->host_ref[*r] == 0) bm->host_free.push_back(*r);
            q->host_table.clear();
            q->swapped = false;
        }
        if (num_pairs) *num_pairs = pairs;
    } catch (...) {
        return PA_BM_BAD_ARG;
    }
    return PA_BM_OK;
}

// The monitoring figures of [Practice §6.3 实际部署建议] (block utilisation,
// hit rate).  A block's fill is the most tokens any of its users holds in it.
extern "C" int32_t pa_bm_stats(const pa_block_manager* bm, pa_bm_stats_t* out)
{
    if (!bm || !out) return PA_BM_BAD_ARG;
    try {
        const int32_t B = bm->block_size;
        std::vector<int32_t> fill(bm->num_blocks, 0);
        int32_t swapped = 0;
        for (const auto& kv : bm->seqs) {
            const Seq& q = kv.second;
            swapped += q.swapped;
            for (size_t j = 0; j < q.table.size(); ++j) {
                const int32_t n = std::min<int32_t>(B, q.len - static_cast<int32_t>(j) * B);
                fill[q.table[j]] = std::max(fill[q.table[j]], n);
            }
        }
        pa_bm_stats_t st = {};
        st.num_blocks = bm->num_blocks;
        st.block_size = B;
        for (int32_t b = 0; b < bm->num_blocks; ++b) {
            if (bm->blocks[b].ref == 0) continue;
            ++st.used_blocks;
            st.stored_tokens += fill[b];
        }
        st.free_blocks = bm->nfree;
        st.cached_blocks = static_cast<int32_t>(bm->cache.size());
        st.prefix_queries = bm->prefix_queries;
        st.prefix_hits = bm->prefix_hits;
        st.num_seqs = static_cast<int32_t>(bm->seqs.size());
        st.swapped_seqs = swapped;
        st.free_host_blocks = static_cast<int32_t>(bm->host_free.size());
        *out = st;
    } catch (...) {
        return PA_BM_BAD_ARG;
    }
    return PA_BM_OK;
}

extern "C" int32_t pa_bm_check(const pa_block_manager* bm)
{
    if (!bm) return 1;
    const int32_t nb = bm->num_blocks, B = bm->block_size;
    std::vector<int32_t> refs(nb, 0), host_refs(bm->num_host, 0);
    for (const auto& kv : bm->seqs) {
        const Seq& q = kv.second;
        const std::vector<int32_t>& t = q.swapped ? q.host_table : q.table;
        if (q.swapped && !q.table.empty()) return 10;             // swapped: host blocks only
        if (!q.swapped && !q.host_table.empty()) return 10;
        const int64_t waste = static_cast<int64_t>(t.size()) * B - q.len;
        if (waste < 0 || waste > B - 1) return 2;                 // internal waste bound
        for (int32_t b : t) {
            if (b < 0 || b >= (q.swapped ? bm->num_host : nb)) return 3;
            ++(q.swapped ? host_refs : refs)[b];
        }
    }
    for (int32_t h = 0; h < bm->num_host; ++h)
        if (host_refs[h] != bm->host_ref[h]) return 11;          // host counts == references
    std::vector<char> listed(bm->num_host, 0);
    for (int32_t h : bm->host_free) {
        if (h < 0 || h >= bm->num_host || listed[h] || bm->host_ref[h] != 0) return 12;
        listed[h] = 1;
    }
    for (int32_t h = 0; h < bm->num_host; ++h)
        if ((bm->host_ref[h] == 0) != (listed[h] != 0)) return 12;  // host free <=> count 0
    for (int32_t b = 0; b < nb; ++b)
        if (refs[b] != bm->blocks[b].ref) return 4;               // counts == references
    int32_t count = 0, prev = -1;
    for (int32_t b = bm->head; b >= 0; b = bm->blocks[b].next) {
        if (++count > nb) return 5;                               // cycle
        if (bm->blocks[b].prev != prev || !bm->blocks[b].in_free || bm->blocks[b].ref != 0) return 6;
        prev = b;
    }
    if (prev != bm->tail || count != bm->nfree) return 7;
    for (int32_t b = 0; b < nb; ++b)
        if ((bm->blocks[b].ref == 0) != bm->blocks[b].in_free) return 8;   // free <=> count 0
    for (const auto& kv : bm->cache) {
        const Block& x = bm->blocks[kv.second];
        if (!x.hashed || x.hash != kv.first) return 9;
    }
    return 0;
}
