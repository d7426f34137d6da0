// block_manager.cpp -- host-side block bookkeeping of the paged KV cache: free list,
// reference counts, on-demand allocation, copy-on-write, prefix cache, swap.
//
// "KV cache, GQA, paging and continuous batching", section "PagedAttention": fixed-size
// blocks, a per-sequence block table, blocks allocated on demand; shared prefixes point at
// the same blocks, copy-on-write at divergence.  Section "The scheduler, and preemption":
// admission bounded by free blocks, preempted sequences swapped to host memory.
// "KV cache, continuous batching and paged attention", section "Prefix caching": KV blocks
// cached by a hash of the prefix.
#include <array>
#include <cstring>
#include <list>
#include <mutex>
#include <new>
#include <unordered_map>
#include <vector>

#include "../../include/pkv_block_manager.h"

namespace {

constexpr int kBS = PKV_BLOCK_SIZE;

// A full block's identity: the block before it (and that block's generation, so a key
// dies when its predecessor is reused) plus its own token ids.
struct Key {
    int32_t parent;
    uint32_t parent_gen;
    std::array<int32_t, kBS> tok;
    bool operator==(const Key& o) const
    {
        return parent == o.parent && parent_gen == o.parent_gen && tok == o.tok;
    }
};

struct KeyHash {
    size_t operator()(const Key& k) const
    {
        // 64-bit FNV-1a over the key's words; equality is checked exactly on every hit.
        uint64_t h = 1469598103934665603ull;
        auto mix = [&h](uint32_t w) {
            for (int i = 0; i < 4; ++i) {
                h ^= (w >> (8 * i)) & 0xFF;
                h *= 1099511628211ull;
            }
        };
        mix((uint32_t)k.parent);
        mix(k.parent_gen);
        for (int32_t t : k.tok) mix((uint32_t)t);
        return (size_t)h;
    }
};

struct Seq {
    std::vector<int32_t> blocks;      // block table
    int64_t len = 0;                  // tokens with reserved slots
    std::vector<int32_t> tail;        // token ids of the partly filled last block
    bool tokens_known = true;         // every token id so far was given
    bool swapped = false;
    int32_t swapped_blocks = 0;
};

}  // namespace

struct pkv_block_manager {
    int32_t N;
    bool prefix;
    std::vector<int32_t> ref;
    std::vector<uint32_t> gen;
    std::vector<int32_t> free_list;                        // stack; back() is taken first
    std::list<int32_t> lru;                                // unreferenced cached blocks, oldest first
    std::vector<std::list<int32_t>::iterator> lru_pos;
    std::vector<char> in_lru;
    std::vector<char> keyed;
    std::vector<Key> key_of;
    std::unordered_map<Key, int32_t, KeyHash> cache;
    std::unordered_map<int64_t, Seq> seqs;
    pkv_bm_stats st{};
    std::mutex mu;

    explicit pkv_block_manager(int32_t n, bool p)
        : N(n), prefix(p), ref(n, 0), gen(n, 0), lru_pos(n), in_lru(n, 0), keyed(n, 0), key_of(n)
    {
        free_list.reserve(n);
        for (int32_t b = n - 1; b >= 0; --b) free_list.push_back(b);
    }

    int64_t available() const { return (int64_t)free_list.size() + (int64_t)lru.size(); }

    void unkey(int32_t b)
    {
        if (!keyed[b]) return;
        auto it = cache.find(key_of[b]);
        if (it != cache.end() && it->second == b) cache.erase(it);
        keyed[b] = 0;
    }

    // A block for a new owner (reference count 1).  The caller checked available().
    int32_t take()
    {
        int32_t b;
        if (!free_list.empty()) {
            b = free_list.back();
            free_list.pop_back();
        } else {
            b = lru.front();
            lru.pop_front();
            in_lru[b] = 0;
            unkey(b);
            ++gen[b];
            ++st.evictions;
        }
        ref[b] = 1;
        return b;
    }

    void release(int32_t b)
    {
        if (--ref[b] > 0) return;
        if (keyed[b]) {   // stays findable until an allocation needs it
            lru.push_back(b);
            lru_pos[b] = std::prev(lru.end());
            in_lru[b] = 1;
        } else {
            ++gen[b];
            free_list.push_back(b);
        }
    }

    void acquire_cached(int32_t b)
    {
        if (ref[b] == 0 && in_lru[b]) {
            lru.erase(lru_pos[b]);
            in_lru[b] = 0;
        }
        ++ref[b];
    }

    Key key_for(const Seq& s, size_t j, const int32_t* tok) const
    {
        Key k;
        k.parent = j > 0 ? s.blocks[j - 1] : -1;
        k.parent_gen = j > 0 ? gen[s.blocks[j - 1]] : 0;
        std::memcpy(k.tok.data(), tok, sizeof(int32_t) * kBS);
        return k;
    }

    void register_full(const Seq& s, size_t j, const int32_t* tok)
    {
        const int32_t b = s.blocks[j];
        if (keyed[b]) return;
        Key k = key_for(s, j, tok);
        if (cache.find(k) != cache.end()) return;   // same prefix already cached in another block
        cache.emplace(k, b);
        key_of[b] = k;
        keyed[b] = 1;
    }

    int needed(const Seq& s, int64_t n) const
    {
        const int64_t have = (s.len + kBS - 1) / kBS;
        const int64_t want = (s.len + n + kBS - 1) / kBS;
        const bool cow = n > 0 && (s.len % kBS) != 0 && ref[s.blocks.back()] > 1;
        return (int)(want - have + (cow ? 1 : 0));
    }

    int check() const;
};

int pkv_block_manager::check() const
{
    std::vector<int64_t> count(N, 0);
    for (const auto& kv : seqs) {
        const Seq& s = kv.second;
        if (s.swapped) {
            if (!s.blocks.empty()) return PKV_ERR_STATE;
            continue;
        }
        if ((int64_t)s.blocks.size() != (s.len + kBS - 1) / kBS) return PKV_ERR_STATE;
        if ((int64_t)s.tail.size() > kBS - 1) return PKV_ERR_STATE;
        for (int32_t b : s.blocks) {
            if (b < 0 || b >= N) return PKV_ERR_STATE;
            ++count[b];
        }
    }
    std::vector<char> on_free(N, 0);
    for (int32_t b : free_list) {
        if (b < 0 || b >= N || on_free[b]) return PKV_ERR_STATE;
        on_free[b] = 1;
    }
    int64_t in_list = 0;
    for (int32_t b : lru) {
        if (b < 0 || b >= N || !in_lru[b] || !keyed[b]) return PKV_ERR_STATE;
        ++in_list;
    }
    int64_t used = 0, flagged = 0;
    for (int32_t b = 0; b < N; ++b) {
        if (ref[b] != count[b]) return PKV_ERR_STATE;
        const int states = (ref[b] > 0) + on_free[b] + (in_lru[b] ? 1 : 0);
        if (states != 1) return PKV_ERR_STATE;
        if (on_free[b] && keyed[b]) return PKV_ERR_STATE;
        used += ref[b] > 0;
        flagged += in_lru[b] ? 1 : 0;
    }
    if (flagged != in_list) return PKV_ERR_STATE;
    if (used + (int64_t)free_list.size() + (int64_t)lru.size() != N) return PKV_ERR_STATE;
    for (const auto& kv : cache) {
        const int32_t b = kv.second;
        if (b < 0 || b >= N || !keyed[b] || !(key_of[b] == kv.first)) return PKV_ERR_STATE;
    }
    return PKV_OK;
}

extern "C" {

int pkv_bm_create(int32_t num_blocks, int enable_prefix_cache, pkv_bm_t* out)
{
    if (!out) return PKV_ERR_NULL;
    *out = nullptr;
    if (num_blocks <= 0) return PKV_ERR_ARG;
    pkv_block_manager* bm = new (std::nothrow) pkv_block_manager(num_blocks, enable_prefix_cache != 0);
    if (!bm) return PKV_ERR_ARG;
    *out = bm;
    return PKV_OK;
}

int pkv_bm_destroy(pkv_bm_t bm)
{
    delete bm;
    return PKV_OK;
}

int64_t pkv_bm_free_blocks(pkv_bm_t bm)
{
    if (!bm) return PKV_ERR_NULL;
    std::lock_guard<std::mutex> g(bm->mu);
    return bm->available();
}

int pkv_bm_refcount(pkv_bm_t bm, int32_t block)
{
    if (!bm) return PKV_ERR_NULL;
    std::lock_guard<std::mutex> g(bm->mu);
    if (block < 0 || block >= bm->N) return PKV_ERR_ARG;
    return bm->ref[block];
}

int pkv_bm_add_sequence(pkv_bm_t bm, int64_t seq_id, const int32_t* prompt, int32_t n_prompt,
                        int32_t* num_cached_tokens)
{
    if (!bm) return PKV_ERR_NULL;
    if (num_cached_tokens) *num_cached_tokens = 0;
    if (n_prompt < 0) return PKV_ERR_ARG;
    std::lock_guard<std::mutex> g(bm->mu);
    if (bm->seqs.count(seq_id)) return PKV_ERR_STATE;
    Seq s;
    s.tokens_known = prompt != nullptr || n_prompt == 0;
    if (bm->prefix && prompt && n_prompt > 1) {
        const int32_t max_blocks = (n_prompt - 1) / kBS;
        for (int32_t j = 0; j < max_blocks; ++j) {
            ++bm->st.prefix_queries;
            auto it = bm->cache.find(bm->key_for(s, (size_t)j, prompt + (size_t)j * kBS));
            if (it == bm->cache.end()) break;
            ++bm->st.prefix_hits;
            bm->acquire_cached(it->second);
            s.blocks.push_back(it->second);
        }
    }
    s.len = (int64_t)s.blocks.size() * kBS;
    if (num_cached_tokens) *num_cached_tokens = (int32_t)s.len;
    bm->seqs.emplace(seq_id, std::move(s));
    return PKV_OK;
}

int pkv_bm_blocks_needed(pkv_bm_t bm, int64_t seq_id, int32_t n)
{
    if (!bm) return PKV_ERR_NULL;
    if (n < 0) return PKV_ERR_ARG;
    std::lock_guard<std::mutex> g(bm->mu);
    auto it = bm->seqs.find(seq_id);
    if (it == bm->seqs.end() || it->second.swapped) return PKV_ERR_STATE;
    return bm->needed(it->second, n);
}

int pkv_bm_append_slots(pkv_bm_t bm, int64_t seq_id, const int32_t* tokens, int32_t n, int32_t* slot_mapping,
                        int32_t* cow_src, int32_t* cow_dst, int32_t* num_cow)
{
    if (!bm) return PKV_ERR_NULL;
    if (num_cow) *num_cow = 0;
    if (n < 0) return PKV_ERR_ARG;
    if (n > 0 && !slot_mapping) return PKV_ERR_NULL;
    std::lock_guard<std::mutex> g(bm->mu);
    auto it = bm->seqs.find(seq_id);
    if (it == bm->seqs.end() || it->second.swapped) return PKV_ERR_STATE;
    Seq& s = it->second;
    if (n == 0) return PKV_OK;
    if (s.len + n > (int64_t)0x7fffffff) return PKV_ERR_ARG;
    const bool cow = (s.len % kBS) != 0 && bm->ref[s.blocks.back()] > 1;
    if (cow && (!cow_src || !cow_dst || !num_cow)) return PKV_ERR_NULL;
    if (bm->needed(s, n) > bm->available()) return PKV_ERR_NO_BLOCKS;
    if (cow) {
        const int32_t old = s.blocks.back();
        const int32_t fresh = bm->take();
        --bm->ref[old];   // still held by another table (> 0)
        s.blocks.back() = fresh;
        *cow_src = old;
        *cow_dst = fresh;
        *num_cow = 1;
        ++bm->st.cow_copies;
    }
    if (!tokens) {
        s.tokens_known = false;
        s.tail.clear();
    }
    for (int32_t i = 0; i < n; ++i) {
        const int64_t pos = s.len + i;
        const int64_t j = pos / kBS;
        const int off = (int)(pos % kBS);
        if (off == 0) s.blocks.push_back(bm->take());
        slot_mapping[i] = s.blocks[(size_t)j] * kBS + off;
        if (s.tokens_known) {
            s.tail.push_back(tokens[i]);
            if (off == kBS - 1) {
                if (bm->prefix) bm->register_full(s, (size_t)j, s.tail.data());
                s.tail.clear();
            }
        }
    }
    s.len += n;
    return PKV_OK;
}

int pkv_bm_fork(pkv_bm_t bm, int64_t parent_id, int64_t child_id)
{
    if (!bm) return PKV_ERR_NULL;
    std::lock_guard<std::mutex> g(bm->mu);
    auto it = bm->seqs.find(parent_id);
    if (it == bm->seqs.end() || it->second.swapped || bm->seqs.count(child_id)) return PKV_ERR_STATE;
    Seq child = it->second;
    for (int32_t b : child.blocks) ++bm->ref[b];
    bm->seqs.emplace(child_id, std::move(child));
    return PKV_OK;
}

int pkv_bm_free_sequence(pkv_bm_t bm, int64_t seq_id)
{
    if (!bm) return PKV_ERR_NULL;
    std::lock_guard<std::mutex> g(bm->mu);
    auto it = bm->seqs.find(seq_id);
    if (it == bm->seqs.end()) return PKV_ERR_STATE;
    Seq& s = it->second;
    for (size_t j = s.blocks.size(); j-- > 0;) bm->release(s.blocks[j]);
    bm->seqs.erase(it);
    return PKV_OK;
}

int pkv_bm_block_table(pkv_bm_t bm, int64_t seq_id, int32_t* table, int32_t capacity, int32_t* num_blocks,
                       int32_t* num_tokens)
{
    if (!bm) return PKV_ERR_NULL;
    std::lock_guard<std::mutex> g(bm->mu);
    auto it = bm->seqs.find(seq_id);
    if (it == bm->seqs.end()) return PKV_ERR_STATE;
    const Seq& s = it->second;
    const int32_t nb = (int32_t)s.blocks.size();
    if (num_blocks) *num_blocks = nb;
    if (num_tokens) *num_tokens = (int32_t)s.len;
    if (nb > capacity) return PKV_ERR_ARG;
    if (nb > 0 && !table) return PKV_ERR_NULL;
    for (int32_t j = 0; j < nb; ++j) table[j] = s.blocks[(size_t)j];
    return PKV_OK;
}

int pkv_bm_swap_out(pkv_bm_t bm, int64_t seq_id, int32_t* blocks, int32_t capacity, int32_t* num_blocks)
{
    if (!bm) return PKV_ERR_NULL;
    std::lock_guard<std::mutex> g(bm->mu);
    auto it = bm->seqs.find(seq_id);
    if (it == bm->seqs.end() || it->second.swapped) return PKV_ERR_STATE;
    Seq& s = it->second;
    const int32_t nb = (int32_t)s.blocks.size();
    if (num_blocks) *num_blocks = nb;
    if (nb > capacity) return PKV_ERR_ARG;
    if (nb > 0 && !blocks) return PKV_ERR_NULL;
    for (int32_t j = 0; j < nb; ++j) blocks[j] = s.blocks[(size_t)j];
    for (size_t j = s.blocks.size(); j-- > 0;) bm->release(s.blocks[j]);
    s.blocks.clear();
    s.swapped = true;
    s.swapped_blocks = nb;
    return PKV_OK;
}

int pkv_bm_swap_in(pkv_bm_t bm, int64_t seq_id, int32_t* blocks, int32_t capacity, int32_t* num_blocks)
{
    if (!bm) return PKV_ERR_NULL;
    std::lock_guard<std::mutex> g(bm->mu);
    auto it = bm->seqs.find(seq_id);
    if (it == bm->seqs.end() || !it->second.swapped) return PKV_ERR_STATE;
    Seq& s = it->second;
    const int32_t nb = s.swapped_blocks;
    if (num_blocks) *num_blocks = nb;
    if (nb > capacity) return PKV_ERR_ARG;
    if (nb > 0 && !blocks) return PKV_ERR_NULL;
    if (nb > bm->available()) return PKV_ERR_NO_BLOCKS;
    for (int32_t j = 0; j < nb; ++j) {
        const int32_t b = bm->take();
        s.blocks.push_back(b);
        blocks[j] = b;
    }
    s.swapped = false;
    s.swapped_blocks = 0;
    return PKV_OK;
}

int pkv_bm_get_stats(pkv_bm_t bm, pkv_bm_stats* out)
{
    if (!bm || !out) return PKV_ERR_NULL;
    std::lock_guard<std::mutex> g(bm->mu);
    pkv_bm_stats s = bm->st;
    s.num_blocks = bm->N;
    s.free_blocks = (int64_t)bm->free_list.size();
    s.cached_blocks = (int64_t)bm->lru.size();
    s.used_blocks = 0;
    s.shared_blocks = 0;
    for (int32_t b = 0; b < bm->N; ++b) {
        s.used_blocks += bm->ref[b] > 0;
        s.shared_blocks += bm->ref[b] > 1;
    }
    s.num_sequences = (int64_t)bm->seqs.size();
    *out = s;
    return PKV_OK;
}

int pkv_bm_check(pkv_bm_t bm)
{
    if (!bm) return PKV_ERR_NULL;
    std::lock_guard<std::mutex> g(bm->mu);
    return bm->check();
}

}  // extern "C"
