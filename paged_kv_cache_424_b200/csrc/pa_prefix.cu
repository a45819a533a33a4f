// pa_prefix.cu -- host side of prefix caching: the table that finds, for a
// new request's token ids, the physical KV blocks that already hold the same
// prefix, and the order in which decode visits sequences so that sequences
// sharing blocks run together.
//
// Method: "vLLM PagedAttention 大模型推理架构深度实战" section 7.3 (automatic
// prefix caching: requests with an identical prefix are recognised and share
// KV-cache blocks; later turns of a chat reuse the earlier turns' KV) and
// section 2.3 (a block's reference count is the number of sequences that map
// it).  Host code only: no kernel lives here.
//
// A cached block is identified by its content: the 16 token ids it holds and
// the block holding the 16 tokens before them (its parent), so equal keys
// mean equal prefixes.  Parents are named by (block id, generation); a
// block's generation changes when it is evicted, so a child of an evicted
// block can never be matched through a reused id.  Lookups hash the key but
// always compare it in full.
#include <algorithm>
#include <array>
#include <cstdint>
#include <cstring>
#include <list>
#include <new>
#include <unordered_map>
#include <vector>

#include "../../include/pa.h"
#include "pa_decode.h"

namespace {

constexpr int kBlockTokens = 16;

struct Key {
    int64_t parent;  // parent block id << 24 | generation (low 24 bits), -1 for the first block
    std::array<int32_t, kBlockTokens> tokens;
    bool operator==(const Key &o) const { return parent == o.parent && tokens == o.tokens; }
};

// 64-bit mixing of the key's words (a multiply-xorshift finaliser per word).
struct KeyHash {
    static uint64_t mix(uint64_t h, uint64_t w) {
        h ^= w + 0x9e3779b97f4a7c15ull + (h << 6) + (h >> 2);
        h ^= h >> 31;
        h *= 0xbf58476d1ce4e5b9ull;
        h ^= h >> 29;
        return h;
    }
    size_t operator()(const Key &k) const {
        uint64_t h = mix(0x243f6a8885a308d3ull, (uint64_t)k.parent);
        for (int32_t t : k.tokens) h = mix(h, (uint32_t)t);
        return (size_t)h;
    }
};

struct BlockInfo {
    bool cached = false;
    int32_t refs = 0;
    uint32_t generation = 0;
    Key key{};
    std::list<int32_t>::iterator lru_pos{};  // valid while cached and refs == 0
};

int64_t parent_name(int32_t block, uint32_t generation) {
    return ((int64_t)block << 24) | (int64_t)(generation & 0xffffffu);
}

Key make_key(int64_t parent, const int32_t *tokens) {
    Key k;
    k.parent = parent;
    std::memcpy(k.tokens.data(), tokens, sizeof(int32_t) * kBlockTokens);
    return k;
}

}  // namespace

struct pa_prefix_cache {
    std::vector<BlockInfo> blocks;
    std::unordered_map<Key, int32_t, KeyHash> table;
    std::list<int32_t> lru;  // cached blocks with no user, least recently released first
    int64_t hits = 0, lookups = 0;

    void unuse(int32_t b) {
        BlockInfo &bi = blocks[b];
        if (--bi.refs == 0) bi.lru_pos = lru.insert(lru.end(), b);
    }
    void use(int32_t b) {
        BlockInfo &bi = blocks[b];
        if (bi.refs++ == 0) lru.erase(bi.lru_pos);
    }
};

extern "C" {

pa_prefix_cache *pa_prefix_cache_create(int64_t num_blocks) {
    if (num_blocks <= 0 || num_blocks > ((int64_t)1 << 31) - 1) {
        pa::set_last_error(PA_ERR_SHAPE, "pa_prefix_cache_create: num_blocks must be in [1, 2^31)");
        return nullptr;
    }
    pa_prefix_cache *c = new (std::nothrow) pa_prefix_cache();
    if (!c) {
        pa::set_last_error(PA_ERR_MEMORY, "pa_prefix_cache_create: out of host memory");
        return nullptr;
    }
    try {
        c->blocks.resize((size_t)num_blocks);
    } catch (...) {
        delete c;
        pa::set_last_error(PA_ERR_MEMORY, "pa_prefix_cache_create: out of host memory");
        return nullptr;
    }
    return c;
}

void pa_prefix_cache_destroy(pa_prefix_cache *c) { delete c; }

int32_t pa_prefix_cache_match(pa_prefix_cache *c, const int32_t *tokens, int32_t num_tokens, int32_t *blocks_out,
                              int32_t max_blocks) {
    if (!c || (num_tokens > 0 && !tokens) || (max_blocks > 0 && !blocks_out))
        return pa::set_last_error(PA_ERR_NULL, "pa_prefix_cache_match: a required pointer is NULL");
    if (num_tokens < 0 || max_blocks < 0)
        return pa::set_last_error(PA_ERR_SHAPE, "pa_prefix_cache_match: negative size");
    const int32_t full = std::min(num_tokens / kBlockTokens, max_blocks);
    int64_t parent = -1;
    int32_t n = 0;
    for (; n < full; ++n) {
        ++c->lookups;
        auto it = c->table.find(make_key(parent, tokens + (int64_t)n * kBlockTokens));
        if (it == c->table.end()) break;
        ++c->hits;
        const int32_t b = it->second;
        blocks_out[n] = b;
        parent = parent_name(b, c->blocks[b].generation);
    }
    for (int32_t i = 0; i < n; ++i) c->use(blocks_out[i]);
    return n;
}

pa_status pa_prefix_cache_insert(pa_prefix_cache *c, const int32_t *tokens, int32_t num_tokens,
                                 const int32_t *blocks, int32_t num_blocks) {
    if (!c || (num_tokens > 0 && !tokens) || (num_blocks > 0 && !blocks))
        return pa::set_last_error(PA_ERR_NULL, "pa_prefix_cache_insert: a required pointer is NULL");
    if (num_tokens < 0 || num_blocks < 0)
        return pa::set_last_error(PA_ERR_SHAPE, "pa_prefix_cache_insert: negative size");
    const int32_t full = std::min(num_tokens / kBlockTokens, num_blocks);
    for (int32_t i = 0; i < full; ++i)
        if (blocks[i] < 0 || (size_t)blocks[i] >= c->blocks.size())
            return pa::set_last_error(PA_ERR_SHAPE, "pa_prefix_cache_insert: block id outside the pool");
    int64_t parent = -1;
    for (int32_t i = 0; i < full; ++i) {
        const Key k = make_key(parent, tokens + (int64_t)i * kBlockTokens);
        const int32_t b = blocks[i];
        auto it = c->table.find(k);
        int32_t canonical = b;
        if (it != c->table.end()) {
            canonical = it->second;  // the same prefix is cached already: keep that block
        } else if (!c->blocks[b].cached) {
            BlockInfo &bi = c->blocks[b];
            bi.cached = true;
            bi.key = k;
            bi.refs = 1;  // the inserting sequence maps it
            c->table.emplace(k, b);
        }
        parent = parent_name(canonical, c->blocks[canonical].generation);
    }
    return PA_OK;
}

int32_t pa_prefix_cache_release(pa_prefix_cache *c, const int32_t *blocks, int32_t num_blocks) {
    if (!c || (num_blocks > 0 && !blocks))
        return pa::set_last_error(PA_ERR_NULL, "pa_prefix_cache_release: a required pointer is NULL");
    if (num_blocks < 0) return pa::set_last_error(PA_ERR_SHAPE, "pa_prefix_cache_release: negative size");
    int32_t n = 0;
    for (int32_t i = 0; i < num_blocks; ++i) {
        const int32_t b = blocks[i];
        if (b < 0 || (size_t)b >= c->blocks.size() || !c->blocks[b].cached || c->blocks[b].refs <= 0) continue;
        c->unuse(b);
        ++n;
    }
    return n;
}

int32_t pa_prefix_cache_evict(pa_prefix_cache *c, int32_t max_blocks, int32_t *blocks_out) {
    if (!c || (max_blocks > 0 && !blocks_out))
        return pa::set_last_error(PA_ERR_NULL, "pa_prefix_cache_evict: a required pointer is NULL");
    if (max_blocks < 0) return pa::set_last_error(PA_ERR_SHAPE, "pa_prefix_cache_evict: negative size");
    int32_t n = 0;
    while (n < max_blocks && !c->lru.empty()) {
        const int32_t b = c->lru.front();
        c->lru.pop_front();
        BlockInfo &bi = c->blocks[b];
        c->table.erase(bi.key);
        bi.cached = false;
        bi.generation = (bi.generation + 1) & 0xffffffu;  // children of the old content become unreachable
        blocks_out[n++] = b;
    }
    return n;
}

pa_status pa_prefix_cache_stats(const pa_prefix_cache *c, int64_t *cached, int64_t *evictable, int64_t *hits,
                                int64_t *lookups) {
    if (!c) return pa::set_last_error(PA_ERR_NULL, "pa_prefix_cache_stats: cache is NULL");
    if (cached) *cached = (int64_t)c->table.size();
    if (evictable) *evictable = (int64_t)c->lru.size();
    if (hits) *hits = c->hits;
    if (lookups) *lookups = c->lookups;
    return PA_OK;
}

pa_status pa_prefix_order(const int32_t *block_tables, const int32_t *context_lens, int32_t num_seqs,
                          int32_t max_blocks_per_seq, int32_t *order) {
    if (num_seqs < 0 || max_blocks_per_seq < 0)
        return pa::set_last_error(PA_ERR_SHAPE, "pa_prefix_order: negative size");
    if (num_seqs == 0) return PA_OK;
    if (!context_lens || !order || (!block_tables && max_blocks_per_seq > 0))
        return pa::set_last_error(PA_ERR_NULL, "pa_prefix_order: a required pointer is NULL");
    // Sequences that share a prefix share its first block: sort by (first
    // block, sequence index); sequences with an empty context go last.
    std::vector<std::pair<int64_t, int32_t>> keyed((size_t)num_seqs);
    for (int32_t s = 0; s < num_seqs; ++s) {
        const bool has = context_lens[s] > 0 && max_blocks_per_seq > 0;
        const int64_t first = has ? (int64_t)block_tables[(int64_t)s * max_blocks_per_seq] : INT64_MAX;
        keyed[(size_t)s] = {first, s};
    }
    std::sort(keyed.begin(), keyed.end());
    for (int32_t i = 0; i < num_seqs; ++i) order[i] = keyed[(size_t)i].second;
    return PA_OK;
}

}  // extern "C"
