// Prefix-block manager: block-granular KV reuse across requests over the
// paged pool the decode kernels read.
//
// "xinfer-ai" package docs, "Prefix Cache (KV Reuse)": finished sequences
// contribute their full KV blocks to a global prefix cache; a new request
// finds the longest cached block-aligned prefix and reuses those blocks; the
// remaining tokens are prefilled as usual, their KV written after the cached
// prefix.  Only full blocks are reused: a common prefix that ends inside a
// block has that block's tail recomputed, and a prompt cached entirely at
// block boundaries recomputes its last block so that the prefill step is
// never empty.  The cache shares the pool with the live sequences and is
// capped at a number of tokens rounded down to whole blocks.
//
// Here a block is one page of the pool (page_size tokens).  A cached block
// is a node of a trie whose edges are the blocks' token ids: the node of a
// prefix of k blocks is reached from the root through the k blocks in
// order, so a block is reused only after the same tokens in the same
// position.  Pages are reference counted: one reference per live sequence
// whose page table holds the page, one while the page is a cached block.  A
// page with no reference is free.  When a fresh page is needed and none is
// free, or when the cache is over its cap, the least recently used cached
// block that no live sequence holds and that has no cached children is
// evicted.  Everything here is host code; the caller copies the page tables
// it receives to the device for tq_quantize_append and tq_paged_decode.
#include <algorithm>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <new>
#include <unordered_map>
#include <vector>

#include "../../include/tq.h"

#define TQ_API extern "C" __attribute__((visibility("default")))

namespace {

struct Node {
    int32_t page = -1;              // the block's page (-1 for the root)
    int32_t parent = -1;
    int32_t nchild = 0;             // cached children
    uint64_t last_use = 0;
    uint64_t key = 0;               // hash of the block's token ids
    std::vector<int32_t> tokens;    // the block's token ids (collision check)
    bool live = false;              // in the trie
};

struct Seq {
    bool active = false;
    std::vector<int32_t> pages;     // its page table
    std::vector<int32_t> nodes;     // nodes of its reused prefix blocks
};

uint64_t block_hash(const int32_t* t, int n)
{
    uint64_t h = 1469598103934665603ull;                 // FNV-1a over the 4 bytes of each id
    for (int i = 0; i < n; ++i) {
        uint32_t x = (uint32_t)t[i];
        for (int b = 0; b < 4; ++b) {
            h ^= (x >> (8 * b)) & 0xffu;
            h *= 1099511628211ull;
        }
    }
    return h;
}

}  // namespace

struct tq_prefix_cache {
    int32_t num_pages = 0, page_size = 0;
    int64_t cap_blocks = 0;
    std::vector<int32_t> refs;                          // per page
    std::vector<int32_t> free_pages;                    // stack
    std::vector<Node> nodes;                            // [0] is the root
    std::vector<int32_t> free_nodes;
    // (parent node, block hash) -> child nodes with that hash
    std::unordered_multimap<uint64_t, int32_t> children;
    std::vector<Seq> seqs;
    std::vector<int32_t> free_seqs;
    int64_t cached_blocks = 0;
    uint64_t tick = 0;
    int64_t hit_tokens = 0, prompt_tokens = 0, evictions = 0;
    std::mutex mu;

    static uint64_t edge(int32_t parent, uint64_t key)
    {
        return key ^ (0x9e3779b97f4a7c15ull * (uint64_t)(parent + 1));
    }

    int32_t find_child(int32_t parent, const int32_t* t) const
    {
        const uint64_t key = block_hash(t, page_size);
        auto range = children.equal_range(edge(parent, key));
        for (auto it = range.first; it != range.second; ++it) {
            const Node& n = nodes[it->second];
            if (n.live && n.parent == parent && n.key == key &&
                std::equal(n.tokens.begin(), n.tokens.end(), t))
                return it->second;
        }
        return -1;
    }

    void unlink(int32_t id)
    {
        Node& n = nodes[id];
        auto range = children.equal_range(edge(n.parent, n.key));
        for (auto it = range.first; it != range.second; ++it)
            if (it->second == id) {
                children.erase(it);
                break;
            }
        if (n.parent > 0) nodes[n.parent].nchild--;
        n.live = false;
        n.tokens.clear();
        free_nodes.push_back(id);
    }

    void release(int32_t page)
    {
        if (--refs[page] == 0) free_pages.push_back(page);
    }

    // Evict the least recently used cached block that no sequence holds and
    // that has no cached children.  False when there is none.
    bool evict_one()
    {
        int32_t best = -1;
        for (int32_t i = 1; i < (int32_t)nodes.size(); ++i) {
            const Node& n = nodes[i];
            if (!n.live || n.nchild != 0 || refs[n.page] != 1) continue;
            if (best < 0 || n.last_use < nodes[best].last_use) best = i;
        }
        if (best < 0) return false;
        const int32_t page = nodes[best].page;
        unlink(best);
        cached_blocks--;
        evictions++;
        release(page);
        return true;
    }

    int32_t alloc_page()
    {
        while (free_pages.empty())
            if (!evict_one()) return -1;
        const int32_t p = free_pages.back();
        free_pages.pop_back();
        refs[p] = 1;
        return p;
    }

    // A cached block for `page` under `parent`.  Everything that can throw
    // (host allocation) happens before any state changes.
    int32_t new_node(int32_t parent, int32_t page, const int32_t* t)
    {
        const bool reuse = !free_nodes.empty();
        if (!reuse) {
            nodes.emplace_back();                       // an unused slot if a later step throws
            free_nodes.reserve(nodes.size());           // unlink() never reallocates
        }
        const int32_t id = reuse ? free_nodes.back() : (int32_t)nodes.size() - 1;
        std::vector<int32_t> tk(t, t + page_size);
        const uint64_t key = block_hash(t, page_size);
        children.emplace(edge(parent, key), id);
        if (reuse) free_nodes.pop_back();
        Node& n = nodes[id];
        n.page = page;
        n.parent = parent;
        n.nchild = 0;
        n.last_use = ++tick;
        n.key = key;
        n.tokens = std::move(tk);
        n.live = true;
        if (parent > 0) nodes[parent].nchild++;
        cached_blocks++;
        return id;
    }

    void enforce_cap()
    {
        while (cached_blocks > cap_blocks)
            if (!evict_one()) break;
    }
};

TQ_API tq_prefix_cache* tq_prefix_cache_create(int32_t num_pages, int32_t page_size,
                                               int64_t max_cached_tokens)
{
    if (num_pages <= 0 || page_size <= 0) return nullptr;
    tq_prefix_cache* pc = new (std::nothrow) tq_prefix_cache();
    if (!pc) return nullptr;
    try {
        pc->num_pages = num_pages;
        pc->page_size = page_size;
        pc->cap_blocks = max_cached_tokens > 0 ? max_cached_tokens / page_size : num_pages / 2;
        pc->refs.assign(num_pages, 0);
        pc->free_pages.reserve(num_pages);
        for (int32_t p = num_pages - 1; p >= 0; --p) pc->free_pages.push_back(p);  // 0 first
        pc->nodes.emplace_back();                                                // root
    } catch (...) {
        delete pc;
        return nullptr;
    }
    return pc;
}

TQ_API void tq_prefix_cache_destroy(tq_prefix_cache* pc) { delete pc; }

TQ_API tq_status tq_prefix_cache_begin(tq_prefix_cache* pc, const int32_t* tokens,
                                       int32_t num_tokens, int32_t* page_table, int32_t max_pages,
                                       int32_t* cached_tokens, int32_t* seq)
{
    if (!pc || num_tokens <= 0 || !tokens || !page_table || !cached_tokens || !seq)
        return TQ_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(pc->mu);
    const int32_t P = pc->page_size;
    const int32_t npages = (num_tokens + P - 1) / P;
    if (npages > max_pages) return TQ_ERR_INVALID_ARG;
    Seq s;
    int32_t id = -1;
    try {
        // host allocations first, so that nothing below can throw
        s.pages.reserve(npages);
        s.nodes.reserve(num_tokens / P);
        if (pc->free_seqs.empty()) {
            pc->seqs.emplace_back();                    // a spare record if we fail later
            pc->free_seqs.reserve(pc->seqs.size());     // finish() never reallocates
        }
    } catch (...) {
        return TQ_ERR_NO_PAGES;
    }
    // longest cached prefix of whole blocks; a prompt cached entirely at
    // block boundaries gives back its last block, to be recomputed
    int32_t at = 0;
    for (int32_t i = 0; i < num_tokens / P; ++i) {
        const int32_t c = pc->find_child(at, tokens + (int64_t)i * P);
        if (c < 0) break;
        s.nodes.push_back(c);
        at = c;
    }
    if (!s.nodes.empty() && (int64_t)s.nodes.size() * P == num_tokens) s.nodes.pop_back();
    s.active = true;
    for (int32_t c : s.nodes) {
        Node& n = pc->nodes[c];
        n.last_use = ++pc->tick;
        pc->refs[n.page]++;
        s.pages.push_back(n.page);
    }
    while ((int32_t)s.pages.size() < npages) {
        const int32_t p = pc->alloc_page();
        if (p < 0) {                                   // give everything back
            for (int32_t q : s.pages) pc->release(q);
            return TQ_ERR_NO_PAGES;
        }
        s.pages.push_back(p);
    }
    if (!pc->free_seqs.empty()) {
        id = pc->free_seqs.back();
        pc->free_seqs.pop_back();
    } else {
        id = (int32_t)pc->seqs.size() - 1;              // the record made above
    }
    std::copy(s.pages.begin(), s.pages.end(), page_table);
    *cached_tokens = (int32_t)s.nodes.size() * P;
    *seq = id;
    pc->hit_tokens += (int64_t)s.nodes.size() * P;
    pc->prompt_tokens += num_tokens;
    pc->seqs[id] = std::move(s);
    return TQ_OK;
}

TQ_API tq_status tq_prefix_cache_extend(tq_prefix_cache* pc, int32_t seq, int32_t new_len,
                                        int32_t* page_table, int32_t max_pages)
{
    if (!pc || !page_table || new_len < 0) return TQ_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(pc->mu);
    if (seq < 0 || seq >= (int32_t)pc->seqs.size() || !pc->seqs[seq].active)
        return TQ_ERR_INVALID_ARG;
    Seq& s = pc->seqs[seq];
    const int32_t need = (new_len + pc->page_size - 1) / pc->page_size;
    if (need > max_pages) return TQ_ERR_INVALID_ARG;
    const size_t had = s.pages.size();
    try {
        while ((int32_t)s.pages.size() < need) {
            const int32_t p = pc->alloc_page();
            if (p < 0) {
                while (s.pages.size() > had) {
                    pc->release(s.pages.back());
                    s.pages.pop_back();
                }
                return TQ_ERR_NO_PAGES;
            }
            s.pages.push_back(p);
        }
    } catch (...) {
        return TQ_ERR_NO_PAGES;
    }
    std::copy(s.pages.begin(), s.pages.end(), page_table);
    return TQ_OK;
}

TQ_API tq_status tq_prefix_cache_finish(tq_prefix_cache* pc, int32_t seq, const int32_t* tokens,
                                        int32_t num_tokens)
{
    if (!pc || num_tokens < 0 || (num_tokens > 0 && !tokens)) return TQ_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(pc->mu);
    if (seq < 0 || seq >= (int32_t)pc->seqs.size() || !pc->seqs[seq].active)
        return TQ_ERR_INVALID_ARG;
    Seq& s = pc->seqs[seq];
    const int32_t P = pc->page_size;
    if ((int64_t)num_tokens > (int64_t)s.pages.size() * P) return TQ_ERR_INVALID_ARG;
    // the sequence's full blocks join the cache along its own chain; a block
    // already cached (reused, or computed by another sequence) keeps its
    // cached page and this sequence's copy is given back
    const int32_t full = num_tokens / P;
    int32_t at = 0;
    size_t i = 0;
    try {
        for (; i < s.pages.size(); ++i) {
            const int32_t page = s.pages[i];
            if (i < s.nodes.size()) {                   // reused: cached already
                at = s.nodes[i];
                pc->nodes[at].last_use = ++pc->tick;
                pc->release(page);
                continue;
            }
            if ((int32_t)i < full && at >= 0) {
                const int32_t* t = tokens + (int64_t)i * P;
                const int32_t c = pc->find_child(at, t);
                if (c >= 0) {
                    pc->nodes[c].last_use = ++pc->tick;
                    pc->release(page);
                    at = c;
                } else {
                    at = pc->new_node(at, page, t);     // the sequence's reference moves to the cache
                }
                continue;
            }
            at = -1;
            pc->release(page);                          // partial block or beyond the tokens
        }
    } catch (...) {
        // out of host memory inserting block i: it and the rest go back
        for (; i < s.pages.size(); ++i) pc->release(s.pages[i]);
    }
    s.active = false;
    s.pages.clear();
    s.nodes.clear();
    pc->free_seqs.push_back(seq);
    pc->enforce_cap();
    return TQ_OK;
}

TQ_API tq_status tq_prefix_cache_stats(tq_prefix_cache* pc, tq_prefix_stats* out)
{
    if (!pc || !out) return TQ_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(pc->mu);
    int64_t live = 0;
    for (const Seq& s : pc->seqs)
        if (s.active) live++;
    out->free_pages = (int64_t)pc->free_pages.size();
    out->cached_blocks = pc->cached_blocks;
    out->live_sequences = live;
    out->hit_tokens = pc->hit_tokens;
    out->prompt_tokens = pc->prompt_tokens;
    out->evictions = pc->evictions;
    return TQ_OK;
}

TQ_API int32_t tq_prefix_cache_page_refs(tq_prefix_cache* pc, int32_t page)
{
    if (!pc || page < 0 || page >= pc->num_pages) return -1;
    std::lock_guard<std::mutex> lock(pc->mu);
    return pc->refs[page];
}
