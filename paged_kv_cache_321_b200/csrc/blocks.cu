// Host block manager: per-layer block allocation with prefix caching, the
// bookkeeping that turns requests' token streams into the block tables the
// kernels read. Host code only (no device work).
//
// Method: PagedKVCache in makarna/pkg/kvcache/paged_cache.go
// (ensureCapacityLocked, AppendToken, AllocateForTokens, Commit, Free,
// LayerBlockIDs) over its BlockPool (AllocateBlocks, FreeBlocks,
// FindCachedBlocks, TouchBlocks, CacheBlocks), whose bodies the page does not
// show; the pool below takes the plainest reading of those calls:
//  * a block is free, held (reference count > 0: one per sequence holding
//    it, its owner and every borrower), or cached and unheld (its content is
//    known by its hash; it stays findable until it is needed again);
//  * AllocateBlocks takes free blocks first, then evicts the least recently
//    released cached ones; it takes all n or nothing;
//  * FreeBlocks drops one reference per block; a block reaching zero goes to
//    the cached list if it has a hash, else to the free list;
//  * FindCachedBlocks walks a hash chain from its start and stops at the first
//    hash with no cached block; TouchBlocks takes a reference (a borrow);
//  * CacheBlocks gives blocks their hashes unless a hash already has a block.
// Block hashes chain a parent hash and a full block of token ids through
// 64-bit FNV-1a (the page does not show ComputeBlockHash).
#include <stdint.h>
#include <stdlib.h>

#include <list>
#include <mutex>
#include <unordered_map>
#include <vector>

#include "common.cuh"

struct kvp_blocks {
    struct Block {
        int refs = 0;
        bool hashed = false;
        uint64_t hash = 0;
        std::list<int>::iterator lru;  // position in `cached` while unheld and hashed
        bool in_lru = false;
    };
    struct Layer {
        std::vector<Block> blocks;
        std::vector<int> free_list;  // popped from the back
        std::list<int> cached;       // unheld hashed blocks, least recently released first
        std::unordered_map<uint64_t, int> by_hash;
    };
    int num_layers = 0, num_blocks = 0, block_size = 0, max_seq_len = 0;
    std::vector<Layer> layers;
    std::mutex mu;
};

struct kvp_seq {
    kvp_blocks *pool = nullptr;
    std::vector<int32_t> tokens;
    std::vector<uint64_t> hashes;           // one per full block of tokens
    std::vector<std::vector<int>> ids;      // [layer][block index]
    std::vector<std::vector<char>> owned;   // [layer][block index]: 0 = borrowed
    int computed = 0, written = 0;
    uint64_t epoch = 0;                     // bumped whenever the blocks are replaced
    std::vector<uint64_t> synced_epoch;     // [layer]: epoch of the last delta (~0: never)
    std::vector<int> synced;                // [layer]: entries handed out by the last delta
};

namespace {

using kvp::set_error;

uint64_t block_hash(const int32_t *tok, int n, const uint64_t *parent)
{
    uint64_t h = 0xcbf29ce484222325ull;  // FNV-1a 64 offset basis
    auto mix = [&](uint8_t byte) {
        h ^= byte;
        h *= 0x100000001b3ull;  // FNV-1a 64 prime
    };
    mix(parent ? 1 : 0);
    if (parent)
        for (int b = 0; b < 8; ++b) mix(static_cast<uint8_t>(*parent >> (8 * b)));
    for (int i = 0; i < n; ++i)
        for (int b = 0; b < 4; ++b) mix(static_cast<uint8_t>(static_cast<uint32_t>(tok[i]) >> (8 * b)));
    return h;
}

// AllocateBlocks: n blocks of `layer`, all or none.
bool allocate(kvp_blocks *p, int layer, int n, std::vector<int> &out)
{
    kvp_blocks::Layer &L = p->layers[layer];
    if (static_cast<size_t>(n) > L.free_list.size() + L.cached.size()) return false;
    for (int i = 0; i < n; ++i) {
        int id;
        if (!L.free_list.empty()) {
            id = L.free_list.back();
            L.free_list.pop_back();
        } else {  // evict the least recently released cached block
            id = L.cached.front();
            L.cached.pop_front();
            kvp_blocks::Block &b = L.blocks[id];
            b.in_lru = false;
            L.by_hash.erase(b.hash);
            b.hashed = false;
        }
        L.blocks[id].refs = 1;
        out.push_back(id);
    }
    return true;
}

// FreeBlocks: one reference less per block.
void release(kvp_blocks *p, int layer, const std::vector<int> &ids)
{
    kvp_blocks::Layer &L = p->layers[layer];
    for (int id : ids) {
        kvp_blocks::Block &b = L.blocks[id];
        if (b.refs <= 0) continue;
        if (--b.refs == 0) {
            if (b.hashed) {
                b.lru = L.cached.insert(L.cached.end(), id);
                b.in_lru = true;
            } else {
                L.free_list.push_back(id);
            }
        }
    }
}

// FindCachedBlocks: the longest cached prefix of the hash chain.
void find_cached(kvp_blocks *p, int layer, const std::vector<uint64_t> &hashes, size_t limit, std::vector<int> &out)
{
    kvp_blocks::Layer &L = p->layers[layer];
    for (size_t i = 0; i < hashes.size() && i < limit; ++i) {
        auto it = L.by_hash.find(hashes[i]);
        if (it == L.by_hash.end()) break;
        out.push_back(it->second);
    }
}

// TouchBlocks: a reference per block (a borrow), taken off the cached list.
void touch(kvp_blocks *p, int layer, const std::vector<int> &ids)
{
    kvp_blocks::Layer &L = p->layers[layer];
    for (int id : ids) {
        kvp_blocks::Block &b = L.blocks[id];
        if (b.in_lru) {
            L.cached.erase(b.lru);
            b.in_lru = false;
        }
        ++b.refs;
    }
}

// CacheBlocks: publish blocks under their hashes (first block per hash wins).
void cache(kvp_blocks *p, int layer, const int *ids, const uint64_t *hashes, int n)
{
    kvp_blocks::Layer &L = p->layers[layer];
    for (int i = 0; i < n; ++i) {
        kvp_blocks::Block &b = L.blocks[ids[i]];
        if (b.hashed || L.by_hash.count(hashes[i])) continue;
        b.hashed = true;
        b.hash = hashes[i];
        L.by_hash.emplace(hashes[i], ids[i]);
    }
}

// ensureCapacityLocked: every layer holds at least `required` blocks; on a
// failure the blocks taken by this call in earlier layers go back.
int ensure_capacity(kvp_seq *s, int required)
{
    kvp_blocks *p = s->pool;
    const int cur = static_cast<int>(s->ids[0].size());
    if (required <= cur) return KVP_OK;
    const int need = required - cur;
    std::vector<std::vector<int>> taken(p->num_layers);
    for (int l = 0; l < p->num_layers; ++l) {
        if (!allocate(p, l, need, taken[l])) {
            for (int k = 0; k < l; ++k) {
                release(p, k, taken[k]);
                s->ids[k].resize(cur);
                s->owned[k].resize(cur);
            }
            return set_error(KVP_ERANGE, "layer %d: no %d free blocks", l, need);
        }
        s->ids[l].insert(s->ids[l].end(), taken[l].begin(), taken[l].end());
        s->owned[l].insert(s->owned[l].end(), taken[l].size(), 1);
    }
    return KVP_OK;
}

void free_all(kvp_seq *s)
{
    for (int l = 0; l < static_cast<int>(s->ids.size()); ++l) release(s->pool, l, s->ids[l]);
    for (auto &v : s->ids) v.clear();
    for (auto &v : s->owned) v.clear();
    s->tokens.clear();
    s->hashes.clear();
    s->computed = s->written = 0;
    ++s->epoch;
}

}  // namespace

extern "C" uint64_t kvp_block_hash(const int32_t *tokens, int n, const uint64_t *parent)
{
    return block_hash(tokens, n < 0 ? 0 : n, parent);
}

extern "C" int kvp_blocks_create(int num_layers, int num_blocks, int block_size, int max_seq_len, kvp_blocks **out)
{
    if (!out) return set_error(KVP_EINVAL, "kvp_blocks_create: out is NULL");
    *out = nullptr;
    if (num_layers <= 0 || num_blocks <= 0 || block_size <= 0 || max_seq_len < 0)
        return set_error(KVP_EINVAL, "kvp_blocks_create: bad sizes (%d layers, %d blocks, block size %d)",
                         num_layers, num_blocks, block_size);
    kvp_blocks *p = new kvp_blocks;
    p->num_layers = num_layers, p->num_blocks = num_blocks, p->block_size = block_size, p->max_seq_len = max_seq_len;
    p->layers.resize(num_layers);
    for (auto &L : p->layers) {
        L.blocks.resize(num_blocks);
        L.free_list.reserve(num_blocks);
        for (int i = num_blocks - 1; i >= 0; --i) L.free_list.push_back(i);  // block 0 handed out first
    }
    *out = p;
    return KVP_OK;
}

extern "C" int kvp_blocks_destroy(kvp_blocks *p)
{
    delete p;
    return KVP_OK;
}

extern "C" int kvp_blocks_count(kvp_blocks *p, int layer, int *free_blocks, int *cached_blocks, int *held_blocks)
{
    if (!p || layer < 0 || layer >= p->num_layers) return set_error(KVP_EINVAL, "kvp_blocks_count: bad pool or layer");
    std::lock_guard<std::mutex> lock(p->mu);
    const kvp_blocks::Layer &L = p->layers[layer];
    int held = 0;
    for (const auto &b : L.blocks) held += b.refs > 0;
    if (free_blocks) *free_blocks = static_cast<int>(L.free_list.size());
    if (cached_blocks) *cached_blocks = static_cast<int>(L.cached.size());
    if (held_blocks) *held_blocks = held;
    return KVP_OK;
}

extern "C" int kvp_blocks_refs(kvp_blocks *p, int layer, int block)
{
    if (!p || layer < 0 || layer >= p->num_layers || block < 0 || block >= p->num_blocks)
        return set_error(KVP_EINVAL, "kvp_blocks_refs: bad pool, layer or block");
    std::lock_guard<std::mutex> lock(p->mu);
    return p->layers[layer].blocks[block].refs;
}

extern "C" int kvp_seq_create(kvp_blocks *p, kvp_seq **out)
{
    if (!p || !out) return set_error(KVP_EINVAL, "kvp_seq_create: NULL argument");
    kvp_seq *s = new kvp_seq;
    s->pool = p;
    s->ids.resize(p->num_layers);
    s->owned.resize(p->num_layers);
    s->synced_epoch.assign(p->num_layers, ~0ull);
    s->synced.assign(p->num_layers, 0);
    *out = s;
    return KVP_OK;
}

extern "C" int kvp_seq_destroy(kvp_seq *s)
{
    if (!s) return KVP_OK;
    {
        std::lock_guard<std::mutex> lock(s->pool->mu);
        free_all(s);
    }
    delete s;
    return KVP_OK;
}

extern "C" int kvp_seq_free(kvp_seq *s)
{
    if (!s) return set_error(KVP_EINVAL, "kvp_seq_free: NULL sequence");
    std::lock_guard<std::mutex> lock(s->pool->mu);
    free_all(s);
    return KVP_OK;
}

extern "C" int kvp_seq_allocate_for_tokens(kvp_seq *s, const int32_t *tokens, int n, int *computed)
{
    if (!s || (n > 0 && !tokens) || n < 0) return set_error(KVP_EINVAL, "kvp_seq_allocate_for_tokens: bad arguments");
    kvp_blocks *p = s->pool;
    if (p->max_seq_len > 0 && n > p->max_seq_len)
        return set_error(KVP_EOVERFLOW, "prompt length %d exceeds max_seq_len %d", n, p->max_seq_len);
    std::lock_guard<std::mutex> lock(p->mu);
    free_all(s);  // a new prompt replaces whatever the sequence held
    s->tokens.assign(tokens, tokens + n);
    const int bs = p->block_size, nfull = n / bs;
    s->hashes.resize(nfull);
    for (int i = 0; i < nfull; ++i) s->hashes[i] = block_hash(tokens + i * bs, bs, i ? &s->hashes[i - 1] : nullptr);
    if (nfull > 0) {
        // the prefix every layer has cached (layers are published together,
        // but a layer may have evicted part of it)
        size_t hit = s->hashes.size();
        std::vector<std::vector<int>> cached(p->num_layers);
        for (int l = 0; l < p->num_layers; ++l) {
            find_cached(p, l, s->hashes, hit, cached[l]);
            hit = cached[l].size();
        }
        for (int l = 0; l < p->num_layers; ++l) {
            cached[l].resize(hit);
            touch(p, l, cached[l]);
            s->ids[l] = cached[l];
            s->owned[l].assign(hit, 0);
        }
        const int fresh = nfull - static_cast<int>(hit);
        for (int l = 0; l < p->num_layers && fresh > 0; ++l) {
            std::vector<int> got;
            if (!allocate(p, l, fresh, got)) {
                // everything this call took, borrowed or new, goes back
                for (int k = 0; k < p->num_layers; ++k) release(p, k, s->ids[k]);
                for (auto &v : s->ids) v.clear();
                for (auto &v : s->owned) v.clear();
                s->tokens.clear();
                s->hashes.clear();
                return set_error(KVP_ERANGE, "layer %d: no %d free blocks", l, fresh);
            }
            s->ids[l].insert(s->ids[l].end(), got.begin(), got.end());
            s->owned[l].insert(s->owned[l].end(), got.size(), 1);
        }
        s->computed = static_cast<int>(hit) * bs;
    }
    // the last prompt token is always computed (its logits are needed)
    if (s->computed >= n) s->computed = n > 0 ? n - 1 : 0;
    s->written = s->computed;
    if (computed) *computed = s->computed;
    return KVP_OK;
}

extern "C" int kvp_seq_append_token(kvp_seq *s, int32_t token)
{
    if (!s) return set_error(KVP_EINVAL, "kvp_seq_append_token: NULL sequence");
    kvp_blocks *p = s->pool;
    std::lock_guard<std::mutex> lock(p->mu);
    s->tokens.push_back(token);
    const int bs = p->block_size, n = static_cast<int>(s->tokens.size());
    if (n % bs != 0) return KVP_OK;
    const int bi = n / bs - 1;
    int rc = ensure_capacity(s, bi + 1);
    const uint64_t *parent = bi > 0 && bi - 1 < static_cast<int>(s->hashes.size()) ? &s->hashes[bi - 1] : nullptr;
    const uint64_t h = block_hash(s->tokens.data() + bi * bs, bs, parent);
    if (bi < static_cast<int>(s->hashes.size())) s->hashes[bi] = h;
    else s->hashes.push_back(h);
    return rc;
}

extern "C" int kvp_seq_reserve(kvp_seq *s, int num_tokens)
{
    if (!s || num_tokens < 0) return set_error(KVP_EINVAL, "kvp_seq_reserve: bad arguments");
    kvp_blocks *p = s->pool;
    if (p->max_seq_len > 0 && num_tokens > p->max_seq_len)
        return set_error(KVP_EOVERFLOW, "%d tokens exceed max_seq_len %d", num_tokens, p->max_seq_len);
    std::lock_guard<std::mutex> lock(p->mu);
    return ensure_capacity(s, (num_tokens + p->block_size - 1) / p->block_size);
}

extern "C" int kvp_seq_commit(kvp_seq *s, int new_tokens)
{
    if (!s || new_tokens < 0) return set_error(KVP_EINVAL, "kvp_seq_commit: bad arguments");
    kvp_blocks *p = s->pool;
    std::lock_guard<std::mutex> lock(p->mu);
    const int old = s->computed;
    s->computed += new_tokens;
    if (s->written < s->computed) s->written = s->computed;
    const int bs = p->block_size;
    const int ob = old / bs;
    int nb = s->computed / bs;
    nb = nb < static_cast<int>(s->hashes.size()) ? nb : static_cast<int>(s->hashes.size());
    for (int l = 0; l < p->num_layers && nb > ob; ++l) {
        const int upto = nb < static_cast<int>(s->ids[l].size()) ? nb : static_cast<int>(s->ids[l].size());
        if (upto > ob) cache(p, l, s->ids[l].data() + ob, s->hashes.data() + ob, upto - ob);
    }
    return KVP_OK;
}

extern "C" int kvp_seq_len(const kvp_seq *s) { return s ? s->computed : KVP_EINVAL; }

extern "C" int kvp_seq_num_blocks(const kvp_seq *s)
{
    return s ? static_cast<int>(s->ids.empty() ? 0 : s->ids[0].size()) : KVP_EINVAL;
}

extern "C" int kvp_seq_block_table(const kvp_seq *s, int layer, int32_t *out, int max_blocks, uint8_t *owned)
{
    if (!s || !out || max_blocks < 0 || layer < 0 || layer >= static_cast<int>(s->ids.size()))
        return set_error(KVP_EINVAL, "kvp_seq_block_table: bad arguments");
    std::lock_guard<std::mutex> lock(s->pool->mu);
    const std::vector<int> &ids = s->ids[layer];
    const int n = static_cast<int>(ids.size());
    if (n > max_blocks) return set_error(KVP_ERANGE, "sequence holds %d blocks, row has %d entries", n, max_blocks);
    for (int i = 0; i < max_blocks; ++i) {
        out[i] = i < n ? ids[i] : -1;
        if (owned) owned[i] = i < n ? static_cast<uint8_t>(s->owned[layer][i]) : 0;
    }
    return n;
}

extern "C" int kvp_seq_block_table_delta(kvp_seq *s, int layer, int32_t *row, int max_blocks, int *first, int *end)
{
    if (!s || !row || !first || !end || max_blocks < 0 || layer < 0 || layer >= static_cast<int>(s->ids.size()))
        return set_error(KVP_EINVAL, "kvp_seq_block_table_delta: bad arguments");
    std::lock_guard<std::mutex> lock(s->pool->mu);
    const std::vector<int> &ids = s->ids[layer];
    const int n = static_cast<int>(ids.size());
    if (n > max_blocks) return set_error(KVP_ERANGE, "sequence holds %d blocks, row has %d entries", n, max_blocks);
    if (s->synced_epoch[layer] != s->epoch) {  // first call, or the blocks were replaced: the whole row
        for (int i = 0; i < max_blocks; ++i) row[i] = i < n ? ids[i] : -1;
        *first = 0, *end = max_blocks;
    } else if (n > s->synced[layer]) {  // growth: only the new entries
        for (int i = s->synced[layer]; i < n; ++i) row[i] = ids[i];
        *first = s->synced[layer], *end = n;
    } else {
        *first = *end = 0;
    }
    s->synced_epoch[layer] = s->epoch;
    s->synced[layer] = n;
    return KVP_OK;
}
