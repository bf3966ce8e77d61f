// block_manager.cpp -- host-side manager of the paged KV-cache pool: free
// stack, reference counts, copy-on-write, the hash-chain prefix cache with
// LRU eviction, and swapping of whole sequences to a host pool, declared in
// include/pagedkv_block_manager.h.  Pure host C++.
#include <cstdint>
#include <cstring>
#include <list>
#include <new>
#include <unordered_map>
#include <vector>

#include "pagedkv_block_manager.h"

namespace {

// 64-bit mixing of the parent block's hash and a block's token ids
// (splitmix64 finaliser per word).  Equal content gives equal hashes; a hit is
// confirmed by comparing the stored parent hash and tokens, so a collision can
// only cost a cache miss.
uint64_t mix64(uint64_t x) {
    x += 0x9E3779B97F4A7C15ull;
    x = (x ^ (x >> 30)) * 0xBF58476D1CE4E5B9ull;
    x = (x ^ (x >> 27)) * 0x94D049BB133111EBull;
    return x ^ (x >> 31);
}

uint64_t block_hash(uint64_t parent, const int32_t* tokens, int n) {
    uint64_t h = mix64(parent ^ 0x5BD1E995u);
    for (int i = 0; i < n; ++i) h = mix64(h ^ static_cast<uint32_t>(tokens[i]));
    return h ? h : 1;  // 0 means "no hash"
}

struct CacheEntry {
    int32_t block;
    uint64_t parent;
    std::vector<int32_t> tokens;
};

struct Sequence {
    std::vector<int32_t> blocks;       // device blocks (empty while swapped out)
    std::vector<int32_t> host_blocks;  // host blocks while swapped out
    std::vector<int32_t> tail;  // token ids of the last, partial block
    int64_t num_tokens = 0;
    uint64_t last_full_hash = 0;  // hash of the last full block (0 = none)
    bool swapped = false;
};

}  // namespace

struct pkv_block_manager {
    int64_t num_blocks;
    int block_size;
    bool prefix_caching;
    std::vector<int32_t> free_stack;   // top = back
    std::vector<int32_t> ref;
    std::vector<uint64_t> hash_of;     // cache hash of a cached block, 0 if none
    std::unordered_map<uint64_t, CacheEntry> cache;
    std::list<int32_t> lru;            // cached blocks with ref 0, oldest first
    std::vector<std::list<int32_t>::iterator> lru_pos;
    std::vector<char> in_lru;
    std::unordered_map<int64_t, Sequence> seqs;
    std::vector<int32_t> host_free;    // host pool's free stack, top = back
    std::vector<int32_t> host_ref;     // swapped-out table entries per host block
    int64_t num_host_blocks = 0;
    int64_t swapped = 0;               // sequences swapped out
    int64_t hits = 0, evictions = 0, cows = 0;

    int32_t take_block() {
        if (!free_stack.empty()) {
            const int32_t b = free_stack.back();
            free_stack.pop_back();
            ref[b] = 1;
            return b;
        }
        if (!lru.empty()) {
            const int32_t b = lru.front();
            lru.pop_front();
            in_lru[b] = 0;
            cache.erase(hash_of[b]);
            hash_of[b] = 0;
            ++evictions;
            ref[b] = 1;
            return b;
        }
        return -1;
    }

    void release_block(int32_t b) {
        if (--ref[b] > 0) return;
        if (hash_of[b]) {
            lru.push_back(b);
            lru_pos[b] = std::prev(lru.end());
            in_lru[b] = 1;
        } else {
            free_stack.push_back(b);
        }
    }

    void acquire_cached(int32_t b) {
        if (ref[b] == 0 && in_lru[b]) {
            lru.erase(lru_pos[b]);
            in_lru[b] = 0;
        }
        ++ref[b];
    }

    // Register a just-filled block under its hash (if that hash is free).
    void register_full(Sequence& s, int32_t b, const int32_t* toks) {
        const uint64_t h = block_hash(s.last_full_hash, toks, block_size);
        if (prefix_caching && hash_of[b] == 0 && cache.find(h) == cache.end()) {
            cache.emplace(h, CacheEntry{b, s.last_full_hash, std::vector<int32_t>(toks, toks + block_size)});
            hash_of[b] = h;
        }
        s.last_full_hash = h;
    }

    int64_t available() const { return static_cast<int64_t>(free_stack.size() + lru.size()); }

    // Drop a swapped-out sequence's references to its host blocks, last to
    // first; a host block no sequence references any more goes back on top of
    // the host free stack.
    void release_host(Sequence& s) {
        for (auto h = s.host_blocks.rbegin(); h != s.host_blocks.rend(); ++h)
            if (--host_ref[*h] == 0) host_free.push_back(*h);
        s.host_blocks.clear();
    }

    // A live (not swapped-out) sequence, or nullptr.
    Sequence* resident(int64_t seq_id) {
        auto it = seqs.find(seq_id);
        return it == seqs.end() || it->second.swapped ? nullptr : &it->second;
    }
    const Sequence* resident(int64_t seq_id) const {
        auto it = seqs.find(seq_id);
        return it == seqs.end() || it->second.swapped ? nullptr : &it->second;
    }
};

extern "C" {

pkv_block_manager* pkv_bm_create(int64_t num_blocks, int block_size, int prefix_caching) {
    if (num_blocks <= 0 || num_blocks > INT32_MAX || block_size <= 0) return nullptr;
    pkv_block_manager* bm = new (std::nothrow) pkv_block_manager();
    if (!bm) return nullptr;
    bm->num_blocks = num_blocks;
    bm->block_size = block_size;
    bm->prefix_caching = prefix_caching != 0;
    bm->free_stack.resize(num_blocks);
    for (int64_t i = 0; i < num_blocks; ++i) bm->free_stack[i] = static_cast<int32_t>(num_blocks - 1 - i);
    bm->ref.assign(num_blocks, 0);
    bm->hash_of.assign(num_blocks, 0);
    bm->lru_pos.resize(num_blocks);
    bm->in_lru.assign(num_blocks, 0);
    return bm;
}

void pkv_bm_destroy(pkv_block_manager* bm) { delete bm; }

int pkv_bm_add_sequence(pkv_block_manager* bm, int64_t seq_id, const int32_t* tokens, int64_t num_tokens,
                        int64_t* num_cached_tokens) {
    if (!bm || num_tokens < 0 || (num_tokens > 0 && !tokens) || bm->seqs.count(seq_id)) return PKV_BM_EINVAL;
    const int B = bm->block_size;
    const int64_t full = num_tokens / B;
    const int64_t need = (num_tokens + B - 1) / B;
    // Plan first (which full blocks hit the cache), so that a failure changes nothing.
    std::vector<int32_t> hit_blocks;
    uint64_t parent = 0;
    if (bm->prefix_caching) {
        for (int64_t i = 0; i < full; ++i) {
            const int32_t* t = tokens + i * B;
            const uint64_t h = block_hash(parent, t, B);
            auto it = bm->cache.find(h);
            if (it == bm->cache.end() || it->second.parent != parent ||
                std::memcmp(it->second.tokens.data(), t, sizeof(int32_t) * B) != 0)
                break;
            hit_blocks.push_back(it->second.block);
            parent = h;
        }
    }
    // Blocks of the hit prefix that sit in the LRU list are not available for
    // the new blocks of this very sequence.
    int64_t hit_in_lru = 0;
    for (int32_t b : hit_blocks) hit_in_lru += bm->in_lru[b] ? 1 : 0;
    const int64_t fresh = need - static_cast<int64_t>(hit_blocks.size());
    if (fresh > bm->available() - hit_in_lru) return PKV_BM_ENOSPACE;

    Sequence s;
    for (int32_t b : hit_blocks) {
        bm->acquire_cached(b);
        s.blocks.push_back(b);
    }
    bm->hits += static_cast<int64_t>(hit_blocks.size());
    s.last_full_hash = parent;
    for (int64_t i = static_cast<int64_t>(hit_blocks.size()); i < need; ++i) {
        const int32_t b = bm->take_block();
        s.blocks.push_back(b);
        if (i < full) bm->register_full(s, b, tokens + i * B);
    }
    if (num_tokens > full * B) s.tail.assign(tokens + full * B, tokens + num_tokens);
    s.num_tokens = num_tokens;
    if (num_cached_tokens) *num_cached_tokens = static_cast<int64_t>(hit_blocks.size()) * B;
    bm->seqs.emplace(seq_id, std::move(s));
    return PKV_BM_OK;
}

int pkv_bm_append(pkv_block_manager* bm, int64_t seq_id, const int32_t* tokens, int64_t num_tokens,
                  int64_t* slots_out, int64_t* cow_pairs_out, int64_t max_pairs, int64_t* num_pairs) {
    if (!bm || num_tokens < 0 || (num_tokens > 0 && (!tokens || !slots_out))) return PKV_BM_EINVAL;
    Sequence* sp = bm->resident(seq_id);
    if (!sp) return PKV_BM_EINVAL;
    Sequence& s = *sp;
    const int B = bm->block_size;
    // Blocks needed: one copy if the partial last block is shared, plus the new ones.
    const int64_t off0 = s.num_tokens % B;
    const bool cow = num_tokens > 0 && off0 != 0 && bm->ref[s.blocks.back()] > 1;
    const int64_t new_blocks = (off0 + num_tokens + B - 1) / B - (off0 ? 1 : 0);
    const int64_t need = new_blocks + (cow ? 1 : 0);
    if (need > bm->available()) return PKV_BM_ENOSPACE;
    if (cow && (max_pairs < 1 || !cow_pairs_out)) return PKV_BM_EBUFFER;
    int64_t pairs = 0;
    if (cow) {
        const int32_t src = s.blocks.back();
        const int32_t dst = bm->take_block();
        bm->release_block(src);
        s.blocks.back() = dst;
        cow_pairs_out[0] = src;
        cow_pairs_out[1] = dst;
        pairs = 1;
        ++bm->cows;
    }
    for (int64_t i = 0; i < num_tokens; ++i) {
        const int64_t off = s.num_tokens % B;
        if (off == 0) s.blocks.push_back(bm->take_block());
        slots_out[i] = static_cast<int64_t>(s.blocks.back()) * B + off;
        s.tail.push_back(tokens[i]);
        ++s.num_tokens;
        if (s.num_tokens % B == 0) {
            bm->register_full(s, s.blocks.back(), s.tail.data());
            s.tail.clear();
        }
    }
    if (num_pairs) *num_pairs = pairs;
    return PKV_BM_OK;
}

int pkv_bm_append_batch(pkv_block_manager* bm, const int64_t* seq_ids, const int32_t* tokens, int64_t n,
                        int64_t* slots_out, int64_t* cow_pairs_out, int64_t max_pairs, int64_t* num_pairs,
                        int64_t* num_done) {
    if (!bm || n < 0 || (n > 0 && (!seq_ids || !tokens || !slots_out)) || max_pairs < 0) return PKV_BM_EINVAL;
    int64_t pairs = 0, i = 0;
    int rc = PKV_BM_OK;
    for (; i < n; ++i) {
        int64_t k = 0;
        rc = pkv_bm_append(bm, seq_ids[i], tokens + i, 1, slots_out + i, cow_pairs_out ? cow_pairs_out + 2 * pairs : nullptr,
                           max_pairs - pairs, &k);
        if (rc != PKV_BM_OK) break;
        pairs += k;
    }
    if (num_pairs) *num_pairs = pairs;
    if (num_done) *num_done = i;
    return rc;
}

int pkv_bm_fork(pkv_block_manager* bm, int64_t parent_id, int64_t child_id) {
    if (!bm || parent_id == child_id) return PKV_BM_EINVAL;
    const Sequence* parent = bm->resident(parent_id);
    if (!parent || bm->seqs.count(child_id)) return PKV_BM_EINVAL;
    Sequence child = *parent;
    for (int32_t b : child.blocks) ++bm->ref[b];
    bm->seqs.emplace(child_id, std::move(child));
    return PKV_BM_OK;
}

int pkv_bm_free(pkv_block_manager* bm, int64_t seq_id) {
    if (!bm) return PKV_BM_EINVAL;
    auto it = bm->seqs.find(seq_id);
    if (it == bm->seqs.end()) return PKV_BM_EINVAL;
    if (it->second.swapped) {
        bm->release_host(it->second);
        --bm->swapped;
    }
    // release from the last block to the first, so that the LRU list keeps a
    // prefix's deeper blocks older than its shallower ones (evicted first)
    const std::vector<int32_t>& blocks = it->second.blocks;
    for (auto b = blocks.rbegin(); b != blocks.rend(); ++b) bm->release_block(*b);
    bm->seqs.erase(it);
    return PKV_BM_OK;
}

int pkv_bm_set_host_blocks(pkv_block_manager* bm, int64_t num_host_blocks) {
    if (!bm || num_host_blocks < 0 || num_host_blocks > INT32_MAX || bm->swapped) return PKV_BM_EINVAL;
    bm->num_host_blocks = num_host_blocks;
    bm->host_ref.assign(num_host_blocks, 0);
    bm->host_free.resize(num_host_blocks);
    for (int64_t i = 0; i < num_host_blocks; ++i)
        bm->host_free[i] = static_cast<int32_t>(num_host_blocks - 1 - i);
    return PKV_BM_OK;
}

int pkv_bm_swap_out_group(pkv_block_manager* bm, const int64_t* seq_ids, int64_t n, int64_t* pairs_out,
                          int64_t max_pairs, int64_t* num_pairs) {
    if (!bm || n <= 0 || !seq_ids || max_pairs < 0) return PKV_BM_EINVAL;
    std::vector<Sequence*> group;
    for (int64_t g = 0; g < n; ++g) {
        Sequence* sp = bm->resident(seq_ids[g]);
        for (int64_t e = 0; e < g; ++e)
            if (seq_ids[e] == seq_ids[g]) sp = nullptr;
        if (!sp) return PKV_BM_EINVAL;
        group.push_back(sp);
    }
    // distinct device blocks of the group, in order of first appearance
    std::unordered_map<int32_t, int32_t> to_host;
    std::vector<int32_t> distinct;
    for (Sequence* sp : group)
        for (int32_t b : sp->blocks)
            if (to_host.emplace(b, -1).second) distinct.push_back(b);
    const int64_t k = static_cast<int64_t>(distinct.size());
    if (k > static_cast<int64_t>(bm->host_free.size())) return PKV_BM_ENOSPACE;
    if (k > max_pairs || (k > 0 && !pairs_out)) return PKV_BM_EBUFFER;
    for (int64_t i = 0; i < k; ++i) {
        const int32_t h = bm->host_free.back();
        bm->host_free.pop_back();
        to_host[distinct[i]] = h;
        pairs_out[2 * i] = distinct[i];
        pairs_out[2 * i + 1] = h;
    }
    for (Sequence* sp : group) {
        for (int32_t b : sp->blocks) {
            const int32_t h = to_host[b];
            sp->host_blocks.push_back(h);
            ++bm->host_ref[h];
        }
        for (auto b = sp->blocks.rbegin(); b != sp->blocks.rend(); ++b) bm->release_block(*b);
        sp->blocks.clear();
        sp->swapped = true;
        ++bm->swapped;
    }
    if (num_pairs) *num_pairs = k;
    return PKV_BM_OK;
}

int pkv_bm_swap_in_group(pkv_block_manager* bm, const int64_t* seq_ids, int64_t n, int64_t* pairs_out,
                         int64_t max_pairs, int64_t* num_pairs) {
    if (!bm || n <= 0 || !seq_ids || max_pairs < 0) return PKV_BM_EINVAL;
    std::vector<Sequence*> group;
    for (int64_t g = 0; g < n; ++g) {
        auto it = bm->seqs.find(seq_ids[g]);
        Sequence* sp = (it == bm->seqs.end() || !it->second.swapped) ? nullptr : &it->second;
        for (int64_t e = 0; e < g; ++e)
            if (seq_ids[e] == seq_ids[g]) sp = nullptr;
        if (!sp) return PKV_BM_EINVAL;
        group.push_back(sp);
    }
    std::unordered_map<int32_t, int32_t> to_dev;
    std::vector<int32_t> distinct;
    for (Sequence* sp : group)
        for (int32_t h : sp->host_blocks)
            if (to_dev.emplace(h, -1).second) distinct.push_back(h);
    const int64_t k = static_cast<int64_t>(distinct.size());
    if (k > bm->available()) return PKV_BM_ENOSPACE;
    if (k > max_pairs || (k > 0 && !pairs_out)) return PKV_BM_EBUFFER;
    for (int64_t i = 0; i < k; ++i) {
        const int32_t d = bm->take_block();
        bm->ref[d] = 0;  // counted below, one per table entry
        to_dev[distinct[i]] = d;
        pairs_out[2 * i] = distinct[i];
        pairs_out[2 * i + 1] = d;
    }
    for (Sequence* sp : group) {
        for (int32_t h : sp->host_blocks) {
            const int32_t d = to_dev[h];
            sp->blocks.push_back(d);
            ++bm->ref[d];
        }
        bm->release_host(*sp);
        sp->swapped = false;
        --bm->swapped;
    }
    if (num_pairs) *num_pairs = k;
    return PKV_BM_OK;
}

int pkv_bm_swap_out(pkv_block_manager* bm, int64_t seq_id, int64_t* pairs_out, int64_t max_pairs,
                    int64_t* num_pairs) {
    return pkv_bm_swap_out_group(bm, &seq_id, 1, pairs_out, max_pairs, num_pairs);
}

int pkv_bm_swap_in(pkv_block_manager* bm, int64_t seq_id, int64_t* pairs_out, int64_t max_pairs,
                   int64_t* num_pairs) {
    return pkv_bm_swap_in_group(bm, &seq_id, 1, pairs_out, max_pairs, num_pairs);
}

int pkv_bm_slots(const pkv_block_manager* bm, int64_t seq_id, int64_t start, int64_t count, int64_t* slots_out) {
    if (!bm || start < 0 || count < 0 || (count > 0 && !slots_out)) return PKV_BM_EINVAL;
    const Sequence* s = bm->resident(seq_id);
    if (!s || start + count > s->num_tokens) return PKV_BM_EINVAL;
    const int B = bm->block_size;
    for (int64_t i = 0; i < count; ++i) {
        const int64_t pos = start + i;
        slots_out[i] = static_cast<int64_t>(s->blocks[pos / B]) * B + pos % B;
    }
    return PKV_BM_OK;
}

int pkv_bm_block_table(const pkv_block_manager* bm, int64_t seq_id, int32_t* out, int64_t max_blocks,
                       int64_t* num_blocks) {
    if (!bm || max_blocks < 0 || (max_blocks > 0 && !out)) return PKV_BM_EINVAL;
    const Sequence* s = bm->resident(seq_id);
    if (!s) return PKV_BM_EINVAL;
    const std::vector<int32_t>& b = s->blocks;
    if (num_blocks) *num_blocks = static_cast<int64_t>(b.size());
    if (static_cast<int64_t>(b.size()) > max_blocks) return PKV_BM_EBUFFER;
    for (int64_t i = 0; i < max_blocks; ++i) out[i] = i < static_cast<int64_t>(b.size()) ? b[i] : -1;
    return PKV_BM_OK;
}

int64_t pkv_bm_num_tokens(const pkv_block_manager* bm, int64_t seq_id) {
    if (!bm) return PKV_BM_EINVAL;
    auto it = bm->seqs.find(seq_id);
    return it == bm->seqs.end() ? static_cast<int64_t>(PKV_BM_EINVAL) : it->second.num_tokens;
}

int pkv_bm_stats(const pkv_block_manager* bm, int64_t* out, int n) {
    if (!bm || n < 0 || (n > 0 && !out)) return PKV_BM_EINVAL;
    const int64_t v[9] = {static_cast<int64_t>(bm->free_stack.size()), static_cast<int64_t>(bm->lru.size()),
                          static_cast<int64_t>(bm->cache.size()), bm->hits, bm->evictions, bm->cows,
                          static_cast<int64_t>(bm->seqs.size()), static_cast<int64_t>(bm->host_free.size()),
                          bm->swapped};
    const int m = n < 9 ? n : 9;
    for (int i = 0; i < m; ++i) out[i] = v[i];
    return m;
}

int pkv_bm_ref_count(const pkv_block_manager* bm, int64_t block) {
    if (!bm || block < 0 || block >= bm->num_blocks) return PKV_BM_EINVAL;
    return bm->ref[block];
}

}  // extern "C"
