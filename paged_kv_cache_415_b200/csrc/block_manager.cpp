// block_manager.cpp -- host-side KV block manager (see include/pa_block_manager.h).
//
// Pages cited (title, then section):
//   [VM-paging] "vLLM用虚拟内存分页思想管理KV Cache"
//   [Practice]  "PagedAttention：大模型KV Cache分页管理优化实践"
//   [Manager]   "深入解析 vLLM 的 KV Cache 管理器：从内存碎片到 PagedAttention 的完整技术剖析"
#include "pa_block_manager.h"

#include <stdint.h>

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
    std::vector<int32_t> table;
    int32_t len = 0;
    int64_t extra_key = 0;
    std::vector<int32_t> tokens;    // kept only with prefix caching
    uint64_t last_full_hash = kRootHash;
};

}  // namespace

struct pa_block_manager {
    int32_t num_blocks = 0, block_size = 0;
    bool caching = false;
    std::vector<Block> blocks;
    int32_t head = -1, tail = -1, nfree = 0;
    std::unordered_map<uint64_t, int32_t> cache;     // hash -> block
    std::unordered_map<int64_t, Seq> seqs;

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

extern "C" int32_t pa_bm_add_sequence(pa_block_manager* bm, int64_t seq_id, const int32_t* tokens,
                                      int32_t num_tokens, int64_t extra_key, int64_t* slots_out,
                                      int32_t* num_cached)
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
    if (fresh + revived > bm->nfree) return PA_BM_NO_SPACE;

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
    return PA_BM_OK;
}

extern "C" int32_t pa_bm_fork(pa_block_manager* bm, int64_t parent, int64_t child)
{
    if (!bm || parent == child) return PA_BM_BAD_ARG;
    auto it = bm->seqs.find(parent);
    if (it == bm->seqs.end() || bm->seqs.count(child)) return PA_BM_BAD_ARG;
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
    if (it == bm->seqs.end()) return PA_BM_BAD_ARG;
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
    bm->seqs.erase(it);
    return PA_BM_OK;
}

extern "C" int32_t pa_bm_block_table(const pa_block_manager* bm, int64_t seq_id,
                                     int32_t* table_out, int32_t capacity, int32_t* num_blocks)
{
    if (!bm) return PA_BM_BAD_ARG;
    auto it = bm->seqs.find(seq_id);
    if (it == bm->seqs.end()) return PA_BM_BAD_ARG;
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

extern "C" int32_t pa_bm_check(const pa_block_manager* bm)
{
    if (!bm) return 1;
    const int32_t nb = bm->num_blocks, B = bm->block_size;
    std::vector<int32_t> refs(nb, 0);
    for (const auto& kv : bm->seqs) {
        const Seq& q = kv.second;
        const int64_t waste = static_cast<int64_t>(q.table.size()) * B - q.len;
        if (waste < 0 || waste > B - 1) return 2;                 // internal waste bound
        for (int32_t b : q.table) {
            if (b < 0 || b >= nb) return 3;
            ++refs[b];
        }
    }
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
