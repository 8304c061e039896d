// allocator.cpp -- host block allocator behind the pa_alloc_* C ABI.
//
// A global free pool of fixed-size physical KV blocks with one reference count per block;
// each sequence owns a list of block ids (its block table) and a length.  Blocks are taken
// only when the previous one is full ("深度解构 LLM 推理优化…" section 2.2); forked sequences
// share their parent's blocks by reference count (intelliparadigm sections 2.1-2.2, "零拷贝
// 共享"); the first write into a partly filled shared block copies it ("深度解构…" section
// 2.3; intelliparadigm section 3.1); a finished sequence releases its blocks ("vLLM 推理原理…"
// generation flow).  Policy details the pages leave open are stated in pa.h.
//
// Prefix caching ("vLLM 推理原理…" section 前缀缓存能省掉哪部分工作: requests that start with the
// same text reuse the KV of the common prefix, on an exact match only): every full block of a
// prompt inserted with pa_alloc_new_seq_prefix is registered under (the physical block before it
// and that block's generation, the block's token ids).  A later prompt walks its blocks from the
// first one and shares every block found; the first miss ends the walk.  Cached blocks whose
// count drops to zero stay cached and become evictable, least recently released first, when the
// free pool runs dry; evicting a block bumps its generation, so entries that named it as their
// predecessor can no longer match.
#include <algorithm>
#include <cstdint>
#include <list>
#include <map>
#include <new>
#include <numeric>
#include <unordered_map>
#include <unordered_set>
#include <vector>

#include "pa.h"

namespace {

// SplitMix64 (S. Vigna): the free pool's initial shuffle is drawn from this stream.
uint64_t splitmix64_next(uint64_t &state)
{
    state += 0x9E3779B97F4A7C15ull;
    uint64_t z = state;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

struct Sequence {
    std::vector<int32_t> blocks;
    int64_t len = 0;
};

// Identity of a cached block: its predecessor (physical id and generation; -1 for the first block
// of a prompt) and its token ids.
struct PrefixKey {
    int32_t parent = -1;
    uint32_t parent_gen = 0;
    std::vector<int32_t> tokens;
    bool operator<(const PrefixKey &o) const
    {
        if (parent != o.parent) return parent < o.parent;
        if (parent_gen != o.parent_gen) return parent_gen < o.parent_gen;
        return tokens < o.tokens;
    }
};

}  // namespace

struct pa_alloc {
    int num_blocks = 0;
    int block_size = 0;
    std::vector<int32_t> free_stack;          // back() is handed out next
    std::vector<int32_t> refcnt;
    std::unordered_map<int64_t, Sequence> seqs;
    int64_t next_id = 0;
    // prefix cache
    std::map<PrefixKey, int32_t> cache;                // key -> block
    std::vector<const PrefixKey *> key_of;             // block -> its key in `cache`, or null
    std::vector<uint32_t> gen;                         // block -> generation (bumped on eviction)
    std::list<int32_t> evictable;                      // cached blocks with count 0, oldest first
    std::vector<std::list<int32_t>::iterator> lru_pos; // block -> position in `evictable`
    std::vector<char> in_lru;
    int64_t hit_tokens = 0, miss_tokens = 0;

    int64_t available() const { return (int64_t)free_stack.size() + (int64_t)evictable.size(); }

    // A block for new data: the free pool first, else the least recently released cached block,
    // which leaves the cache.  Caller has checked available() > 0.
    int32_t take()
    {
        int32_t b;
        if (!free_stack.empty()) {
            b = free_stack.back();
            free_stack.pop_back();
        } else {
            b = evictable.front();
            evictable.pop_front();
            in_lru[b] = 0;
            cache.erase(cache.find(*key_of[b]));
            key_of[b] = nullptr;
            ++gen[b];
        }
        refcnt[b] = 1;
        return b;
    }

    void release(int32_t b)
    {
        if (--refcnt[b] == 0) {
            if (key_of[b] != nullptr) {
                lru_pos[b] = evictable.insert(evictable.end(), b);
                in_lru[b] = 1;
            } else {
                free_stack.push_back(b);
            }
        }
    }

    // Another holder for block b (a prefix hit): an evictable block leaves the LRU list.
    void retain(int32_t b)
    {
        if (refcnt[b] == 0 && in_lru[b]) {
            evictable.erase(lru_pos[b]);
            in_lru[b] = 0;
        }
        ++refcnt[b];
    }

    // Fresh blocks needed to grow `s` by n tokens, and whether the first write copies.
    int64_t blocks_needed(const Sequence &s, int64_t n, bool &cow) const
    {
        const int64_t total = (s.len + n + block_size - 1) / block_size;
        cow = n > 0 && s.len % block_size != 0 && refcnt[s.blocks.back()] > 1;
        return total - (int64_t)s.blocks.size() + (cow ? 1 : 0);
    }

    // Caller has checked capacity.
    void grow(Sequence &s, int64_t n, int64_t *slots, int64_t *cow_src, int64_t *cow_dst)
    {
        bool cow = false;
        blocks_needed(s, n, cow);
        int64_t src = -1, dst = -1;
        if (cow) {
            const int32_t old = s.blocks.back();
            const int32_t fresh = take();
            --refcnt[old];                    // other holders remain, so it stays > 0
            s.blocks.back() = fresh;
            src = old;
            dst = fresh;
        }
        for (int64_t k = 0; k < n; ++k) {
            const int64_t pos = s.len;
            if (pos % block_size == 0) s.blocks.push_back(take());
            if (slots) slots[k] = (int64_t)s.blocks[pos / block_size] * block_size + pos % block_size;
            ++s.len;
        }
        if (cow_src) *cow_src = src;
        if (cow_dst) *cow_dst = dst;
    }
};

extern "C" {

pa_alloc *pa_alloc_create(int num_blocks, int block_size, uint64_t seed)
{
    if (num_blocks <= 0 || block_size <= 0) return nullptr;
    pa_alloc *a = new (std::nothrow) pa_alloc();
    if (!a) return nullptr;
    a->num_blocks = num_blocks;
    a->block_size = block_size;
    a->refcnt.assign(num_blocks, 0);
    a->key_of.assign(num_blocks, nullptr);
    a->gen.assign(num_blocks, 0);
    a->lru_pos.resize(num_blocks);
    a->in_lru.assign(num_blocks, 0);
    std::vector<int32_t> order(num_blocks);
    for (int i = 0; i < num_blocks; ++i) order[i] = i;
    if (seed != 0) {
        uint64_t st = seed;
        for (int i = num_blocks - 1; i > 0; --i) {
            const uint64_t j = splitmix64_next(st) % (uint64_t)(i + 1);
            std::swap(order[i], order[j]);
        }
    }
    a->free_stack.assign(order.rbegin(), order.rend());   // first pop yields order[0]
    return a;
}

void pa_alloc_destroy(pa_alloc *a) { delete a; }

int pa_alloc_new_seq(pa_alloc *a, int64_t *seq_id)
{
    if (!a || !seq_id) return PA_ERR_INVALID_ARG;
    const int64_t id = a->next_id++;
    a->seqs.emplace(id, Sequence{});
    *seq_id = id;
    return PA_OK;
}

int pa_alloc_append_n(pa_alloc *a, int64_t seq, int n, int64_t *slots, int64_t *cow_src, int64_t *cow_dst)
{
    if (!a || n < 0) return PA_ERR_INVALID_ARG;
    auto it = a->seqs.find(seq);
    if (it == a->seqs.end()) return PA_ERR_NOT_FOUND;
    bool cow = false;
    if (a->blocks_needed(it->second, n, cow) > a->available()) return PA_ERR_OOM;
    a->grow(it->second, n, slots, cow_src, cow_dst);
    return PA_OK;
}

int pa_alloc_append_slot(pa_alloc *a, int64_t seq, int64_t *slot, int64_t *cow_src, int64_t *cow_dst)
{
    if (!slot) return PA_ERR_INVALID_ARG;
    return pa_alloc_append_n(a, seq, 1, slot, cow_src, cow_dst);
}

int pa_alloc_append_batch(pa_alloc *a, const int64_t *seqs, int n, int64_t *slots, int64_t *cow_pairs,
                          int *num_cow)
{
    if (!a || n < 0 || (n > 0 && (!seqs || !slots || !cow_pairs)) || !num_cow) return PA_ERR_INVALID_ARG;
    // Dry run: the same decisions grow() will take, in order, on a copy of the affected counts.
    std::unordered_set<int64_t> seen;
    std::unordered_map<int32_t, int32_t> dropped;       // block -> holders that moved away
    int64_t need = 0;
    for (int i = 0; i < n; ++i) {
        auto it = a->seqs.find(seqs[i]);
        if (it == a->seqs.end()) return PA_ERR_NOT_FOUND;
        if (!seen.insert(seqs[i]).second) return PA_ERR_INVALID_ARG;   // one token per sequence
        const Sequence &s = it->second;
        if (s.len % a->block_size == 0) {
            ++need;
        } else {
            const int32_t b = s.blocks.back();
            if (a->refcnt[b] - dropped[b] > 1) {
                ++need;
                ++dropped[b];
            }
        }
    }
    if (need > a->available()) return PA_ERR_OOM;
    int ncow = 0;
    for (int i = 0; i < n; ++i) {
        int64_t src = -1, dst = -1;
        a->grow(a->seqs[seqs[i]], 1, slots + i, &src, &dst);
        if (src >= 0) {
            cow_pairs[2 * ncow] = src;
            cow_pairs[2 * ncow + 1] = dst;
            ++ncow;
        }
    }
    *num_cow = ncow;
    return PA_OK;
}

int pa_alloc_fork(pa_alloc *a, int64_t parent, int64_t *child)
{
    if (!a || !child) return PA_ERR_INVALID_ARG;
    auto it = a->seqs.find(parent);
    if (it == a->seqs.end()) return PA_ERR_NOT_FOUND;
    Sequence c = it->second;
    for (int32_t b : c.blocks) ++a->refcnt[b];
    const int64_t id = a->next_id++;
    a->seqs.emplace(id, std::move(c));
    *child = id;
    return PA_OK;
}

int pa_alloc_free_seq(pa_alloc *a, int64_t seq)
{
    if (!a) return PA_ERR_INVALID_ARG;
    auto it = a->seqs.find(seq);
    if (it == a->seqs.end()) return PA_ERR_NOT_FOUND;
    const std::vector<int32_t> &blocks = it->second.blocks;
    for (auto b = blocks.rbegin(); b != blocks.rend(); ++b) a->release(*b);
    a->seqs.erase(it);
    return PA_OK;
}

int pa_alloc_block_table(const pa_alloc *a, const int64_t *seqs, int num_seqs, int32_t *table, int max_blocks,
                         int32_t *context_lens)
{
    if (!a || num_seqs < 0 || max_blocks <= 0 || (num_seqs > 0 && (!seqs || !table))) return PA_ERR_INVALID_ARG;
    for (int r = 0; r < num_seqs; ++r) {
        auto it = a->seqs.find(seqs[r]);
        if (it == a->seqs.end()) return PA_ERR_NOT_FOUND;
        if ((int64_t)it->second.blocks.size() > max_blocks) return PA_ERR_INVALID_ARG;
        if (it->second.len > INT32_MAX) return PA_ERR_INVALID_ARG;
    }
    for (int r = 0; r < num_seqs; ++r) {
        const Sequence &s = a->seqs.find(seqs[r])->second;
        int32_t *row = table + (size_t)r * max_blocks;
        std::fill(row, row + max_blocks, -1);
        std::copy(s.blocks.begin(), s.blocks.end(), row);
        if (context_lens) context_lens[r] = (int32_t)s.len;
    }
    return PA_OK;
}

int pa_alloc_seq_len(const pa_alloc *a, int64_t seq, int64_t *len)
{
    if (!a || !len) return PA_ERR_INVALID_ARG;
    auto it = a->seqs.find(seq);
    if (it == a->seqs.end()) return PA_ERR_NOT_FOUND;
    *len = it->second.len;
    return PA_OK;
}

int pa_alloc_stats(const pa_alloc *a, int *free_blocks, int *used_blocks, int *shared_blocks, int64_t *frag_tokens)
{
    if (!a) return PA_ERR_INVALID_ARG;
    int used = 0, shared = 0;
    for (int32_t c : a->refcnt) {
        used += c > 0;
        shared += c > 1;
    }
    int64_t frag = 0;
    for (const auto &kv : a->seqs)
        frag += (int64_t)kv.second.blocks.size() * a->block_size - kv.second.len;
    if (free_blocks) *free_blocks = (int)a->available();
    if (used_blocks) *used_blocks = used;
    if (shared_blocks) *shared_blocks = shared;
    if (frag_tokens) *frag_tokens = frag;
    return PA_OK;
}

int pa_alloc_refcount(const pa_alloc *a, int block)
{
    if (!a || block < 0 || block >= a->num_blocks) return PA_ERR_INVALID_ARG;
    return a->refcnt[block];
}

int pa_alloc_new_seq_prefix(pa_alloc *a, const int32_t *tokens, int n, int64_t *seq_id, int64_t *slots,
                            int *cached_tokens)
{
    if (!a || n < 0 || (n > 0 && !tokens) || !seq_id || !cached_tokens) return PA_ERR_INVALID_ARG;
    const int bs = a->block_size;
    const int full = n / bs, total = (n + bs - 1) / bs;
    // walk the prompt's full blocks through the cache (no state change yet)
    std::vector<int32_t> hits;
    int64_t hit_evictable = 0;
    PrefixKey key;
    for (int k = 0; k < full; ++k) {
        key.tokens.assign(tokens + (size_t)k * bs, tokens + (size_t)(k + 1) * bs);
        auto it = a->cache.find(key);
        if (it == a->cache.end()) break;
        const int32_t b = it->second;
        hits.push_back(b);
        hit_evictable += a->refcnt[b] == 0;
        key.parent = b;
        key.parent_gen = a->gen[b];
    }
    const int64_t fresh = total - (int64_t)hits.size();
    if (fresh > a->available() - hit_evictable) return PA_ERR_OOM;

    Sequence s;
    for (int32_t b : hits) {
        a->retain(b);
        s.blocks.push_back(b);
    }
    for (int k = (int)hits.size(); k < total; ++k) {
        const int32_t b = a->take();
        s.blocks.push_back(b);
        if (k < full) {                           // a full prompt block: register it
            PrefixKey nk;
            nk.parent = k > 0 ? s.blocks[k - 1] : -1;
            nk.parent_gen = k > 0 ? a->gen[s.blocks[k - 1]] : 0;
            nk.tokens.assign(tokens + (size_t)k * bs, tokens + (size_t)(k + 1) * bs);
            auto ins = a->cache.emplace(std::move(nk), b);
            a->key_of[b] = &ins.first->first;
        }
    }
    s.len = n;
    if (slots)
        for (int t = 0; t < n; ++t) slots[t] = (int64_t)s.blocks[t / bs] * bs + t % bs;
    const int cached = (int)hits.size() * bs;
    a->hit_tokens += cached;
    a->miss_tokens += n - cached;
    const int64_t id = a->next_id++;
    a->seqs.emplace(id, std::move(s));
    *seq_id = id;
    *cached_tokens = cached;
    return PA_OK;
}

int pa_alloc_prefix_stats(const pa_alloc *a, int64_t *hit_tokens, int64_t *miss_tokens, int *cached_blocks,
                          int *evictable_blocks)
{
    if (!a) return PA_ERR_INVALID_ARG;
    if (hit_tokens) *hit_tokens = a->hit_tokens;
    if (miss_tokens) *miss_tokens = a->miss_tokens;
    if (cached_blocks) *cached_blocks = (int)a->cache.size();
    if (evictable_blocks) *evictable_blocks = (int)a->evictable.size();
    return PA_OK;
}

int pa_alloc_order_by_prefix(const pa_alloc *a, const int64_t *seqs, int n, int32_t *order)
{
    if (!a || n < 0 || (n > 0 && (!seqs || !order))) return PA_ERR_INVALID_ARG;
    std::vector<const Sequence *> sq(n);
    for (int i = 0; i < n; ++i) {
        auto it = a->seqs.find(seqs[i]);
        if (it == a->seqs.end()) return PA_ERR_NOT_FOUND;
        sq[i] = &it->second;
    }
    std::vector<int32_t> idx(n);
    std::iota(idx.begin(), idx.end(), 0);
    std::stable_sort(idx.begin(), idx.end(), [&](int32_t x, int32_t y) { return sq[x]->blocks < sq[y]->blocks; });
    std::copy(idx.begin(), idx.end(), order);
    return PA_OK;
}

}  // extern "C"
