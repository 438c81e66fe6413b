// block_manager.cpp -- host-side allocator of a paged KV cache's blocks, with
// prefix caching (content-addressed reuse of full blocks) and eviction.
//
// "Inference From Scratch", ch. 10 (a block pool, one block table per
// sequence, a slot mapping for every new token) and ch. 11 (prefix caching:
// hash-based reuse of the KV blocks of a common prefix); "The Project: Serve
// Your Own LLM", M13c (a pool smaller than the worst case, so that the engine
// has to preempt).
//
// A sequence owns a list of block ids.  A block that holds block_size tokens
// is *published* under a key made of its tokens and the key of the block
// before it (the whole prefix up to it, chained), so a later sequence whose
// prompt starts with the same tokens reuses it instead of recomputing it.
// Keys are compared exactly (the tokens are stored), so a hash collision can
// never make two different prefixes share a block.  Blocks are reference
// counted; a published block whose last user leaves stays cached, in
// least-recently-released order, until the pool needs it.  A partial block
// is always private, so appending to it never touches another sequence's
// tokens.
//
// The block manager is plain host C++ with no CUDA; it is not thread safe
// (one owner, as in an engine's scheduler loop).
#include <climits>
#include <stdint.h>

#include <algorithm>
#include <cstring>
#include <iterator>
#include <list>
#include <new>
#include <unordered_map>
#include <vector>

#include "../../include/pkv.h"
#include "pkv_internal.h"

namespace pkv {
namespace {

// 64-bit key of a block's content given its parent key (splitmix-style mix).
uint64_t mix64(uint64_t x) {
    x += 0x9e3779b97f4a7c15ull;
    x = (x ^ (x >> 30)) * 0xbf58476d1ce4e5b9ull;
    x = (x ^ (x >> 27)) * 0x94d049bb133111ebull;
    return x ^ (x >> 31);
}

uint64_t block_key(uint64_t parent, const int32_t* tokens, int n) {
    uint64_t h = mix64(parent ^ 0x5851f42d4c957f2dull);
    for (int i = 0; i < n; ++i) h = mix64(h ^ (uint64_t)(uint32_t)tokens[i]);
    return h;
}

struct Block {
    int32_t refs = 0;
    bool published = false;
    uint64_t key = 0;
    uint64_t parent = 0;                 // key of the previous block (0: first block)
    int32_t parent_block = -1;           // the previous block's id (exact-match check)
    std::vector<int32_t> tokens;         // published blocks: their tokens (exact-match check)
    std::list<int32_t>::iterator lru;    // position in the evictable list
    bool in_lru = false;
};

struct Sequence {
    std::vector<int32_t> blocks;
    std::vector<int32_t> tail;           // tokens of the partial last block
    int64_t num_tokens = 0;
    uint64_t last_key = 0;               // key of the last full block
    int32_t shared_tokens = 0;           // leading tokens in reused blocks
    std::vector<int64_t> prompt_slots;   // slot of each prompt token, -1 when reused
};

struct BlockManager {
    int32_t num_blocks, block_size;
    std::vector<Block> blocks;
    std::vector<int32_t> free_list;                      // never-published free blocks
    std::list<int32_t> evictable;                        // published, unreferenced (LRU first)
    std::unordered_multimap<uint64_t, int32_t> cache;    // key -> published block
    std::unordered_map<int64_t, Sequence> seqs;

    BlockManager(int32_t nb, int32_t bs) : num_blocks(nb), block_size(bs), blocks(nb) {
        free_list.reserve(nb);
        for (int32_t i = nb - 1; i >= 0; --i) free_list.push_back(i);
    }

    void unpublish(int32_t id) {
        Block& b = blocks[id];
        auto range = cache.equal_range(b.key);
        for (auto it = range.first; it != range.second; ++it)
            if (it->second == id) {
                cache.erase(it);
                break;
            }
        b.published = false;
        b.tokens.clear();
    }

    // A block for new tokens: a free one, else the least recently released
    // cached one (evicted from the cache); -1 when every block is in use.
    int32_t allocate() {
        int32_t id = -1;
        if (!free_list.empty()) {
            id = free_list.back();
            free_list.pop_back();
        } else if (!evictable.empty()) {
            id = evictable.front();
            evictable.pop_front();
            blocks[id].in_lru = false;
            unpublish(id);
        } else {
            return -1;
        }
        Block& b = blocks[id];
        b.refs = 1;
        b.published = false;
        b.parent_block = -1;
        return id;
    }

    void release(int32_t id) {
        Block& b = blocks[id];
        if (--b.refs > 0) return;
        if (b.published) {
            evictable.push_back(id);
            b.lru = std::prev(evictable.end());
            b.in_lru = true;
        } else {
            free_list.push_back(id);
        }
    }

    void acquire_cached(int32_t id) {
        Block& b = blocks[id];
        if (b.refs++ == 0 && b.in_lru) {
            evictable.erase(b.lru);
            b.in_lru = false;
        }
    }

    // A published block with exactly this content after this parent block.
    int32_t lookup(uint64_t key, int32_t parent_block, const int32_t* tokens) const {
        auto range = cache.equal_range(key);
        for (auto it = range.first; it != range.second; ++it) {
            const Block& b = blocks[it->second];
            if (b.parent_block == parent_block &&
                std::memcmp(b.tokens.data(), tokens, sizeof(int32_t) * block_size) == 0)
                return it->second;
        }
        return -1;
    }

    // Block `id` has just been filled with `tokens` after parent block `parent_block`.
    void publish(int32_t id, uint64_t key, uint64_t parent, int32_t parent_block,
                 const int32_t* tokens) {
        if (lookup(key, parent_block, tokens) >= 0) return;  // an identical block is cached
        Block& b = blocks[id];
        b.published = true;
        b.key = key;
        b.parent = parent;
        b.parent_block = parent_block;
        b.tokens.assign(tokens, tokens + block_size);
        cache.emplace(key, id);
    }
};

}  // namespace
}  // namespace pkv

using pkv::BlockManager;

extern "C" {

pkv_block_manager* pkv_bm_create(int32_t num_blocks, int32_t block_size) {
    pkv::set_last_error("");
    if (num_blocks <= 0 || block_size <= 0) {
        pkv::set_last_error("num_blocks and block_size must be > 0");
        return nullptr;
    }
    try {
        return reinterpret_cast<pkv_block_manager*>(new BlockManager(num_blocks, block_size));
    } catch (const std::bad_alloc&) {
        pkv::set_last_error("out of host memory");
        return nullptr;
    }
}

void pkv_bm_destroy(pkv_block_manager* bm) { delete reinterpret_cast<BlockManager*>(bm); }

pkv_status pkv_bm_add_sequence(pkv_block_manager* handle, int64_t seq_id, const int32_t* tokens,
                               int64_t num_tokens, int32_t* shared_tokens) {
    pkv::set_last_error("");
    auto* bm = reinterpret_cast<BlockManager*>(handle);
    if (!bm || num_tokens < 0 || (num_tokens > 0 && !tokens)) {
        pkv::set_last_error("invalid argument");
        return PKV_ERR_INVALID_ARG;
    }
    if (bm->seqs.count(seq_id)) {
        pkv::set_last_error("sequence %lld already exists", (long long)seq_id);
        return PKV_ERR_INVALID_ARG;
    }
    const int32_t bs = bm->block_size;
    pkv::Sequence s;
    s.prompt_slots.assign((size_t)num_tokens, -1);
    // reuse: the longest run of full prompt blocks that is cached
    int64_t t = 0;
    uint64_t parent = 0;
    int32_t parent_block = -1;
    while (t + bs <= num_tokens) {
        const uint64_t key = pkv::block_key(parent, tokens + t, bs);
        const int32_t id = bm->lookup(key, parent_block, tokens + t);
        if (id < 0) break;
        bm->acquire_cached(id);
        s.blocks.push_back(id);
        parent = key;
        parent_block = id;
        t += bs;
    }
    s.shared_tokens = (int32_t)t;
    // fresh blocks for the rest; full ones are published as they are filled
    bool ok = true;
    for (; t < num_tokens; t += bs) {
        const int32_t id = bm->allocate();
        if (id < 0) {
            ok = false;
            break;
        }
        s.blocks.push_back(id);
        const int64_t n = std::min<int64_t>(bs, num_tokens - t);
        for (int64_t i = 0; i < n; ++i) s.prompt_slots[(size_t)(t + i)] = (int64_t)id * bs + i;
        if (n == bs) {
            const uint64_t key = pkv::block_key(parent, tokens + t, bs);
            bm->publish(id, key, parent, parent_block, tokens + t);
            parent = key;
            parent_block = id;
        } else {
            s.tail.assign(tokens + t, tokens + t + n);
        }
    }
    if (!ok) {
        for (int32_t id : s.blocks) bm->release(id);
        pkv::set_last_error("out of KV blocks: free a sequence (preempt) and retry");
        return PKV_ERR_WORKSPACE;
    }
    s.num_tokens = num_tokens;
    s.last_key = parent;
    if (shared_tokens) *shared_tokens = s.shared_tokens;
    bm->seqs.emplace(seq_id, std::move(s));
    return PKV_OK;
}

pkv_status pkv_bm_prompt_slots(const pkv_block_manager* handle, int64_t seq_id, int64_t* slots,
                               int64_t max_tokens) {
    pkv::set_last_error("");
    auto* bm = reinterpret_cast<const BlockManager*>(handle);
    if (!bm || !slots) return PKV_ERR_INVALID_ARG;
    auto it = bm->seqs.find(seq_id);
    if (it == bm->seqs.end()) {
        pkv::set_last_error("unknown sequence %lld", (long long)seq_id);
        return PKV_ERR_INVALID_ARG;
    }
    const auto& ps = it->second.prompt_slots;
    if ((int64_t)ps.size() > max_tokens) {
        pkv::set_last_error("prompt has %zu tokens, room for %lld", ps.size(), (long long)max_tokens);
        return PKV_ERR_INVALID_ARG;
    }
    std::copy(ps.begin(), ps.end(), slots);
    return PKV_OK;
}

pkv_status pkv_bm_append(pkv_block_manager* handle, int64_t seq_id, int32_t token, int64_t* slot) {
    pkv::set_last_error("");
    auto* bm = reinterpret_cast<BlockManager*>(handle);
    if (!bm || !slot) return PKV_ERR_INVALID_ARG;
    auto it = bm->seqs.find(seq_id);
    if (it == bm->seqs.end()) {
        pkv::set_last_error("unknown sequence %lld", (long long)seq_id);
        return PKV_ERR_INVALID_ARG;
    }
    pkv::Sequence& s = it->second;
    const int32_t bs = bm->block_size;
    const int64_t off = s.num_tokens % bs;
    if (off == 0) {
        const int32_t id = bm->allocate();
        if (id < 0) {
            pkv::set_last_error("out of KV blocks: free a sequence (preempt) and retry");
            return PKV_ERR_WORKSPACE;
        }
        s.blocks.push_back(id);
        s.tail.clear();
    }
    const int32_t id = s.blocks.back();
    *slot = (int64_t)id * bs + off;
    s.tail.push_back(token);
    ++s.num_tokens;
    if ((int64_t)s.tail.size() == bs) {
        // the block is full: publish it for later prompts with this prefix
        const int32_t parent_block = s.blocks.size() >= 2 ? s.blocks[s.blocks.size() - 2] : -1;
        const uint64_t key = pkv::block_key(s.last_key, s.tail.data(), bs);
        bm->publish(id, key, s.last_key, parent_block, s.tail.data());
        s.last_key = key;
        s.tail.clear();
    }
    return PKV_OK;
}

pkv_status pkv_bm_free_sequence(pkv_block_manager* handle, int64_t seq_id) {
    pkv::set_last_error("");
    auto* bm = reinterpret_cast<BlockManager*>(handle);
    if (!bm) return PKV_ERR_INVALID_ARG;
    auto it = bm->seqs.find(seq_id);
    if (it == bm->seqs.end()) {
        pkv::set_last_error("unknown sequence %lld", (long long)seq_id);
        return PKV_ERR_INVALID_ARG;
    }
    // release the last blocks first, so that a prefix outlives its continuations
    for (auto b = it->second.blocks.rbegin(); b != it->second.blocks.rend(); ++b) bm->release(*b);
    bm->seqs.erase(it);
    return PKV_OK;
}

pkv_status pkv_bm_block_table(const pkv_block_manager* handle, int64_t seq_id, int32_t* table,
                              int32_t max_blocks, int32_t* num_blocks, int64_t* num_tokens) {
    pkv::set_last_error("");
    auto* bm = reinterpret_cast<const BlockManager*>(handle);
    if (!bm) return PKV_ERR_INVALID_ARG;
    auto it = bm->seqs.find(seq_id);
    if (it == bm->seqs.end()) {
        pkv::set_last_error("unknown sequence %lld", (long long)seq_id);
        return PKV_ERR_INVALID_ARG;
    }
    const auto& blocks = it->second.blocks;
    if (num_blocks) *num_blocks = (int32_t)blocks.size();
    if (num_tokens) *num_tokens = it->second.num_tokens;
    if (table) {
        if ((int32_t)blocks.size() > max_blocks) {
            pkv::set_last_error("sequence has %zu blocks, room for %d", blocks.size(), max_blocks);
            return PKV_ERR_INVALID_ARG;
        }
        std::copy(blocks.begin(), blocks.end(), table);
        for (int32_t j = (int32_t)blocks.size(); j < max_blocks; ++j) table[j] = -1;
    }
    return PKV_OK;
}

int32_t pkv_bm_shared_tokens(const pkv_block_manager* handle, int64_t seq_id) {
    auto* bm = reinterpret_cast<const BlockManager*>(handle);
    if (!bm) return -1;
    auto it = bm->seqs.find(seq_id);
    return it == bm->seqs.end() ? -1 : it->second.shared_tokens;
}

int32_t pkv_bm_free_blocks(const pkv_block_manager* handle) {
    auto* bm = reinterpret_cast<const BlockManager*>(handle);
    if (!bm) return -1;
    return (int32_t)(bm->free_list.size() + bm->evictable.size());
}

int32_t pkv_bm_cached_blocks(const pkv_block_manager* handle) {
    auto* bm = reinterpret_cast<const BlockManager*>(handle);
    if (!bm) return -1;
    return (int32_t)bm->cache.size();
}

// KV memory accounting ("Efficient LLM Inference", From KV Elements to Memory
// Accounting and Admission Budgets): every cached token holds a key and a
// value vector per kv head per layer, and the paged cache hands out whole
// blocks, so a request of L tokens occupies ceil(L / block_size) blocks.
int64_t pkv_kv_request_bytes(int64_t num_layers, int64_t num_kv_heads, int64_t head_dim,
                             int64_t block_size, int64_t tokens, int32_t kv_dtype) {
    const int64_t esz = kv_dtype == PKV_DTYPE_F32 ? 4
                        : kv_dtype == PKV_DTYPE_BF16 ? 2
                        : kv_dtype == PKV_DTYPE_E4M3 ? 1 : 0;
    if (esz == 0 || num_layers <= 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
        tokens < 0)
        return -1;
    const int64_t blocks = (tokens + block_size - 1) / block_size;
    const int64_t per_block = num_layers * 2 * num_kv_heads * block_size * head_dim * esz;
    if (blocks > 0 && per_block > INT64_MAX / blocks) return -1;
    return blocks * per_block;
}

int64_t pkv_kv_admission_capacity(int64_t pool_bytes, int64_t num_layers, int64_t num_kv_heads,
                                  int64_t head_dim, int64_t block_size, int64_t tokens,
                                  int32_t kv_dtype) {
    const int64_t per = pkv_kv_request_bytes(num_layers, num_kv_heads, head_dim, block_size,
                                             tokens, kv_dtype);
    if (per < 0 || pool_bytes < 0) return -1;
    if (per == 0) return INT64_MAX;
    return pool_bytes / per;
}

}  // extern "C"
