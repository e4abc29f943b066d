// Host block manager: the CPU-side half of paging.
//
// The KV tensors live on the GPU, the bookkeeping of which physical block
// holds which logical block of which sequence lives here (page "Nano-vLLM로
// 배우는 vLLM 추론 엔진 작동 원리 한눈에 정리", section "KV 캐시와 Block
// Manager").  Blocks are handed out only when a token needs one and return to
// the pool when no table holds them (page "vLLM — PagedAttention으로 LLM 추론
// 성능을 2~4배 끌어올린 서빙 엔진", section "PagedAttention — OS 가상 메모리에서
// 영감").
//
// Every operation is O(blocks it touches); the table is a dense
// [max_seqs][max_blocks_per_seq] int32 array so that it can be copied to the
// device as is (whole, or only the rows reported dirty).
//
// Prefix caching (Nano-vLLM page, section "KV 캐시와 Block Manager": blocks of a
// shared prompt prefix are identified by a hash and reused): a full block is
// identified by the 64-bit FNV-1a hash of its parent's hash (8 little-endian
// bytes) followed by its Bs token ids (4 little-endian bytes each), the first
// block's parent being 0, and a hit also requires equal token ids.  Copy-on-
// write (the OS paging the vLLM overview page likens the pool to, section
// "PagedAttention — OS 가상 메모리에서 영감"): an append into a block that
// several tables hold gives the writer a fresh block and reports the copy.
// The free blocks form one list: blocks without a hash return to its top
// (so without hashes it is the plain stack), hashed blocks to its bottom,
// tail first; allocation takes the top and evicts a taken block's hash.
#include <algorithm>
#include <cstdint>
#include <cstring>
#include <new>
#include <unordered_map>
#include <vector>

#include "pa.h"

namespace {
constexpr int64_t kNoId = INT64_MIN;   // token id not known (appended without one)

uint64_t fnv1a64_bytes(uint64_t h, const uint8_t* p, size_t n) {
    for (size_t i = 0; i < n; ++i) {
        h ^= p[i];
        h *= 0x100000001B3ull;
    }
    return h;
}

// Hash of a full block: FNV-1a over (parent hash, 8 bytes LE) then each id (4 bytes LE).
uint64_t block_hash(uint64_t parent, const int64_t* ids, int32_t n) {
    uint8_t buf[8];
    for (int k = 0; k < 8; ++k) buf[k] = (uint8_t)(parent >> (8 * k));
    uint64_t h = fnv1a64_bytes(0xCBF29CE484222325ull, buf, 8);
    for (int32_t i = 0; i < n; ++i) {
        const uint32_t u = (uint32_t)(int32_t)ids[i];
        for (int k = 0; k < 4; ++k) buf[k] = (uint8_t)(u >> (8 * k));
        h = fnv1a64_bytes(h, buf, 4);
    }
    return h;
}
}  // namespace

// Free list over block ids (prev/next links): top = where allocation takes from.
struct FreeList {
    std::vector<int32_t> prev, next;   // prev: towards the bottom, next: towards the top
    std::vector<uint8_t> in;
    int32_t top = -1, bottom = -1;
    size_t count = 0;
    void init(int32_t n) {
        prev.assign(n, -1);
        next.assign(n, -1);
        in.assign(n, 0);
    }
    size_t size() const { return count; }
    void push_top(int32_t b) {
        prev[b] = top;
        next[b] = -1;
        if (top >= 0) next[top] = b; else bottom = b;
        top = b;
        in[b] = 1;
        ++count;
    }
    void push_bottom(int32_t b) {
        next[b] = bottom;
        prev[b] = -1;
        if (bottom >= 0) prev[bottom] = b; else top = b;
        bottom = b;
        in[b] = 1;
        ++count;
    }
    void remove(int32_t b) {
        if (prev[b] >= 0) next[prev[b]] = next[b]; else bottom = next[b];
        if (next[b] >= 0) prev[next[b]] = prev[b]; else top = prev[b];
        prev[b] = next[b] = -1;
        in[b] = 0;
        --count;
    }
    int32_t pop_top() {
        const int32_t b = top;
        remove(b);
        return b;
    }
};

struct pa_block_manager {
    int32_t num_blocks = 0;
    int32_t block_size = 0;
    int32_t max_seqs = 0;
    int32_t max_blocks = 0;
    FreeList free_list;
    std::vector<int32_t> refcount;     // per physical block
    std::vector<int32_t> tables;       // [max_seqs][max_blocks], -1 beyond
    std::vector<int32_t> nblocks;      // blocks held per row
    std::vector<int32_t> lens;         // tokens per row
    std::vector<uint8_t> live;
    std::vector<uint8_t> dirty;
    std::vector<int32_t> dirty_list;
    // prefix caching
    std::unordered_map<uint64_t, int32_t> cache;   // hash -> block
    std::vector<uint64_t> bhash;                   // a block's registered hash
    std::vector<uint8_t> has_hash;
    std::vector<int64_t> ids;                      // [num_blocks][block_size] token ids (kNoId)
    std::vector<uint64_t> chain;                   // per sequence: hash of its last full block
    std::vector<uint8_t> hashable;                 // per sequence: every token has an id

    int32_t* row(int32_t seq) { return tables.data() + (size_t)seq * max_blocks; }

    void mark(int32_t seq) {
        if (!dirty[seq]) {
            dirty[seq] = 1;
            dirty_list.push_back(seq);
        }
    }
    int64_t* block_ids(int32_t b) { return ids.data() + (size_t)b * block_size; }
    int32_t pop() {
        const int32_t b = free_list.pop_top();
        if (has_hash[b]) {                         // evict
            cache.erase(bhash[b]);
            has_hash[b] = 0;
        }
        refcount[b] = 1;
        std::fill(block_ids(b), block_ids(b) + block_size, kNoId);
        return b;
    }
    // Drops one reference of each block; freed ones without a hash go on top in order,
    // freed hashed ones to the bottom, last block first.
    void release_blocks(const int32_t* blocks, int32_t n) {
        freed.clear();
        for (int32_t i = 0; i < n; ++i)
            if (--refcount[blocks[i]] == 0) freed.push_back(blocks[i]);
        for (int32_t b : freed)
            if (!has_hash[b]) free_list.push_top(b);
        for (size_t i = freed.size(); i-- > 0;)
            if (has_hash[freed[i]]) free_list.push_bottom(freed[i]);
    }
    void register_block(int32_t b, uint64_t h) {
        if (!has_hash[b] && cache.find(h) == cache.end()) {
            cache.emplace(h, b);
            bhash[b] = h;
            has_hash[b] = 1;
        }
    }
    std::vector<int32_t> freed;
    bool valid_seq(int32_t seq) const { return seq >= 0 && seq < max_seqs; }
};

static int32_t ceil_div(int64_t a, int64_t b) { return (int32_t)((a + b - 1) / b); }

extern "C" int pa_bm_create(int32_t num_blocks, int32_t block_size, int32_t max_seqs,
                            int32_t max_blocks_per_seq, const int32_t* free_order,
                            int32_t num_free, pa_block_manager** out) {
    if (!out || num_blocks <= 0 || block_size <= 0 || max_seqs <= 0 || max_blocks_per_seq <= 0 ||
        num_free < 0 || num_free > num_blocks || (num_free > 0 && !free_order))
        return PA_ERR_INVALID;
    *out = nullptr;
    pa_block_manager* bm = new (std::nothrow) pa_block_manager();
    if (!bm) return PA_ERR_INVALID;
    bm->num_blocks = num_blocks;
    bm->block_size = block_size;
    bm->max_seqs = max_seqs;
    bm->max_blocks = max_blocks_per_seq;
    bm->refcount.assign(num_blocks, 0);
    // validate: ids in range, no duplicates
    std::vector<uint8_t> seen(num_blocks, 0);
    for (int32_t i = 0; i < num_free; ++i) {
        const int32_t b = free_order[i];
        if (b < 0 || b >= num_blocks || seen[b]) {
            delete bm;
            return PA_ERR_INVALID;
        }
        seen[b] = 1;
    }
    bm->free_list.init(num_blocks);
    for (int32_t i = num_free - 1; i >= 0; --i) bm->free_list.push_top(free_order[i]);
    bm->bhash.assign(num_blocks, 0);
    bm->has_hash.assign(num_blocks, 0);
    bm->ids.assign((size_t)num_blocks * block_size, kNoId);
    bm->chain.assign(max_seqs, 0);
    bm->hashable.assign(max_seqs, 0);
    bm->tables.assign((size_t)max_seqs * max_blocks_per_seq, -1);
    bm->nblocks.assign(max_seqs, 0);
    bm->lens.assign(max_seqs, 0);
    bm->live.assign(max_seqs, 0);
    bm->dirty.assign(max_seqs, 0);
    *out = bm;
    return PA_OK;
}

extern "C" void pa_bm_destroy(pa_block_manager* bm) { delete bm; }

extern "C" int pa_bm_import_seq(pa_block_manager* bm, int32_t seq, int32_t num_tokens,
                                const int32_t* blocks) {
    if (!bm || !bm->valid_seq(seq) || bm->live[seq] || num_tokens < 0) return PA_ERR_INVALID;
    const int32_t nb = ceil_div(num_tokens, bm->block_size);
    if (nb > bm->max_blocks || (nb > 0 && !blocks)) return PA_ERR_INVALID;
    for (int32_t i = 0; i < nb; ++i)
        if (blocks[i] < 0 || blocks[i] >= bm->num_blocks || bm->free_list.in[blocks[i]]) return PA_ERR_INVALID;
    int32_t* r = bm->row(seq);
    for (int32_t i = 0; i < nb; ++i) {
        r[i] = blocks[i];
        bm->refcount[blocks[i]] += 1;
    }
    bm->nblocks[seq] = nb;
    bm->lens[seq] = num_tokens;
    bm->live[seq] = 1;
    bm->hashable[seq] = 0;
    bm->mark(seq);
    return PA_OK;
}

extern "C" int pa_bm_add_seq(pa_block_manager* bm, int32_t seq, int32_t num_tokens) {
    if (!bm || !bm->valid_seq(seq) || bm->live[seq] || num_tokens < 0) return PA_ERR_INVALID;
    const int32_t nb = ceil_div(num_tokens, bm->block_size);
    if (nb > bm->max_blocks) return PA_ERR_INVALID;
    if ((size_t)nb > bm->free_list.size()) return PA_ERR_OOM_BLOCKS;
    int32_t* r = bm->row(seq);
    for (int32_t i = 0; i < nb; ++i) r[i] = bm->pop();
    bm->nblocks[seq] = nb;
    bm->lens[seq] = num_tokens;
    bm->live[seq] = 1;
    bm->hashable[seq] = 0;
    bm->mark(seq);
    return PA_OK;
}

extern "C" int pa_bm_fork_seq(pa_block_manager* bm, int32_t seq, int32_t src,
                              int32_t num_shared_blocks, int32_t num_tokens) {
    if (!bm || !bm->valid_seq(seq) || !bm->valid_seq(src) || seq == src || bm->live[seq] ||
        !bm->live[src] || num_shared_blocks < 0 || num_tokens < 0)
        return PA_ERR_INVALID;
    const int32_t Bs = bm->block_size;
    // only full blocks of the source can be shared, and the new sequence must cover them
    if ((int64_t)num_shared_blocks * Bs > bm->lens[src] ||
        (int64_t)num_shared_blocks * Bs > num_tokens)
        return PA_ERR_INVALID;
    const int32_t nb = ceil_div(num_tokens, Bs);
    if (nb > bm->max_blocks) return PA_ERR_INVALID;
    if ((size_t)(nb - num_shared_blocks) > bm->free_list.size()) return PA_ERR_OOM_BLOCKS;
    int32_t* r = bm->row(seq);
    const int32_t* s = bm->row(src);
    for (int32_t i = 0; i < num_shared_blocks; ++i) {
        r[i] = s[i];
        bm->refcount[s[i]] += 1;
    }
    for (int32_t i = num_shared_blocks; i < nb; ++i) r[i] = bm->pop();
    bm->nblocks[seq] = nb;
    bm->lens[seq] = num_tokens;
    bm->live[seq] = 1;
    bm->hashable[seq] = 0;
    bm->mark(seq);
    return PA_OK;
}

extern "C" int pa_bm_free_seq(pa_block_manager* bm, int32_t seq) {
    if (!bm || !bm->valid_seq(seq) || !bm->live[seq]) return PA_ERR_INVALID;
    int32_t* r = bm->row(seq);
    bm->release_blocks(r, bm->nblocks[seq]);
    std::fill(r, r + bm->nblocks[seq], -1);
    bm->nblocks[seq] = 0;
    bm->lens[seq] = 0;
    bm->live[seq] = 0;
    bm->hashable[seq] = 0;
    bm->chain[seq] = 0;
    bm->mark(seq);
    return PA_OK;
}

extern "C" int pa_bm_append_tokens(pa_block_manager* bm, const int32_t* seqs, int32_t n,
                                   int64_t* slots) {
    if (!bm || n < 0 || (n > 0 && (!seqs || !slots))) return PA_ERR_INVALID;
    const int32_t Bs = bm->block_size;
    // First pass: validate and count the new blocks, so that failure changes nothing.
    size_t need = 0;
    for (int32_t i = 0; i < n; ++i) {
        const int32_t s = seqs[i];
        if (!bm->valid_seq(s) || !bm->live[s]) return PA_ERR_INVALID;
        const int32_t p = bm->lens[s];
        if (p % Bs == 0) {
            if (p / Bs >= bm->max_blocks) return PA_ERR_INVALID;
            ++need;
        } else if (bm->refcount[bm->row(s)[p / Bs]] > 1) {
            return PA_ERR_SHARED_BLOCK;
        }
    }
    if (need > bm->free_list.size()) return PA_ERR_OOM_BLOCKS;
    for (int32_t i = 0; i < n; ++i) {
        const int32_t s = seqs[i];
        const int32_t p = bm->lens[s];
        int32_t* r = bm->row(s);
        if (p % Bs == 0) {
            r[p / Bs] = bm->pop();
            bm->nblocks[s] += 1;
            bm->mark(s);
        }
        slots[i] = (int64_t)r[p / Bs] * Bs + p % Bs;
        bm->lens[s] = p + 1;
        bm->hashable[s] = 0;   // a token without an id: this sequence's blocks are not hashed
    }
    return PA_OK;
}

extern "C" int pa_bm_add_seq_tokens(pa_block_manager* bm, int32_t seq, const int32_t* token_ids,
                                    int32_t num_tokens, int32_t* num_cached_tokens) {
    if (!bm || !bm->valid_seq(seq) || bm->live[seq] || num_tokens < 0 || (num_tokens > 0 && !token_ids))
        return PA_ERR_INVALID;
    const int32_t Bs = bm->block_size;
    const int32_t full = num_tokens / Bs, nb = ceil_div(num_tokens, Bs);
    if (nb > bm->max_blocks) return PA_ERR_INVALID;
    std::vector<int64_t> chunk(Bs);
    auto load = [&](int32_t i) {
        for (int32_t k = 0; k < Bs; ++k) {
            const int32_t t = i * Bs + k;
            chunk[k] = t < num_tokens ? (int64_t)token_ids[t] : kNoId;
        }
    };
    // longest cached prefix of full blocks (hash chain, ids compared)
    std::vector<int32_t> hits;
    uint64_t parent = 0;
    for (int32_t i = 0; i < full; ++i) {
        load(i);
        const uint64_t h = block_hash(parent, chunk.data(), Bs);
        const auto it = bm->cache.find(h);
        if (it == bm->cache.end() ||
            !std::equal(chunk.begin(), chunk.end(), bm->block_ids(it->second)))
            break;
        hits.push_back(it->second);
        parent = h;
    }
    size_t free_hits = 0;
    for (int32_t b : hits) free_hits += bm->refcount[b] == 0;
    if ((size_t)(nb - (int32_t)hits.size()) > bm->free_list.size() - free_hits) return PA_ERR_OOM_BLOCKS;
    int32_t* r = bm->row(seq);
    for (size_t i = 0; i < hits.size(); ++i) {
        const int32_t b = hits[i];
        if (bm->refcount[b] == 0) bm->free_list.remove(b);
        bm->refcount[b] += 1;
        r[i] = b;
    }
    for (int32_t i = (int32_t)hits.size(); i < nb; ++i) {
        const int32_t b = bm->pop();
        load(i);
        std::copy(chunk.begin(), chunk.end(), bm->block_ids(b));
        if (i < full) {
            const uint64_t h = block_hash(parent, chunk.data(), Bs);
            bm->register_block(b, h);
            parent = h;
        }
        r[i] = b;
    }
    bm->nblocks[seq] = nb;
    bm->lens[seq] = num_tokens;
    bm->live[seq] = 1;
    bm->hashable[seq] = 1;
    bm->chain[seq] = parent;
    bm->mark(seq);
    if (num_cached_tokens) *num_cached_tokens = (int32_t)hits.size() * Bs;
    return PA_OK;
}

extern "C" int pa_bm_fork_all(pa_block_manager* bm, int32_t seq, int32_t src) {
    if (!bm || !bm->valid_seq(seq) || !bm->valid_seq(src) || seq == src || bm->live[seq] ||
        !bm->live[src])
        return PA_ERR_INVALID;
    const int32_t nb = bm->nblocks[src];
    int32_t* r = bm->row(seq);
    const int32_t* sr = bm->row(src);
    for (int32_t i = 0; i < nb; ++i) {
        r[i] = sr[i];
        bm->refcount[sr[i]] += 1;
    }
    bm->nblocks[seq] = nb;
    bm->lens[seq] = bm->lens[src];
    bm->live[seq] = 1;
    bm->hashable[seq] = bm->hashable[src];
    bm->chain[seq] = bm->chain[src];
    bm->mark(seq);
    return PA_OK;
}

extern "C" int pa_bm_append_token_ids(pa_block_manager* bm, const int32_t* seqs,
                                      const int32_t* token_ids, int32_t n, int64_t* slots,
                                      int32_t* copies, int32_t* num_copies) {
    if (!bm || n < 0 || (n > 0 && (!seqs || !token_ids || !slots || !copies)) || !num_copies)
        return PA_ERR_INVALID;
    const int32_t Bs = bm->block_size;
    size_t need = 0;   // new blocks: one per block boundary crossed, one per shared block written
    for (int32_t i = 0; i < n; ++i) {
        const int32_t s = seqs[i];
        if (!bm->valid_seq(s) || !bm->live[s]) return PA_ERR_INVALID;
        const int32_t p = bm->lens[s];
        if (p % Bs == 0) {
            if (p / Bs >= bm->max_blocks) return PA_ERR_INVALID;
            ++need;
        } else if (bm->refcount[bm->row(s)[p / Bs]] > 1) {
            ++need;
        }
    }
    if (need > bm->free_list.size()) return PA_ERR_OOM_BLOCKS;
    int32_t nc = 0;
    for (int32_t i = 0; i < n; ++i) {
        const int32_t s = seqs[i];
        const int32_t p = bm->lens[s];
        int32_t* r = bm->row(s);
        if (p % Bs == 0) {
            r[p / Bs] = bm->pop();
            bm->nblocks[s] += 1;
            bm->mark(s);
        } else if (bm->refcount[r[p / Bs]] > 1) {   // copy-on-write
            const int32_t old = r[p / Bs];
            const int32_t fresh = bm->pop();
            std::copy(bm->block_ids(old), bm->block_ids(old) + Bs, bm->block_ids(fresh));
            copies[2 * nc] = old;
            copies[2 * nc + 1] = fresh;
            ++nc;
            r[p / Bs] = fresh;
            bm->release_blocks(&old, 1);
            bm->mark(s);
        }
        const int32_t b = r[p / Bs];
        bm->block_ids(b)[p % Bs] = token_ids[i];
        slots[i] = (int64_t)b * Bs + p % Bs;
        bm->lens[s] = p + 1;
        if ((p + 1) % Bs == 0 && bm->hashable[s]) {   // the block is full: register it
            const uint64_t h = block_hash(bm->chain[s], bm->block_ids(b), Bs);
            bm->register_block(b, h);
            bm->chain[s] = h;
        }
    }
    *num_copies = nc;
    return PA_OK;
}

extern "C" int32_t pa_bm_num_cached_blocks(const pa_block_manager* bm) {
    return bm ? (int32_t)bm->cache.size() : -1;
}

extern "C" int32_t pa_bm_num_free(const pa_block_manager* bm) {
    return bm ? (int32_t)bm->free_list.size() : -1;
}

extern "C" int32_t pa_bm_refcount(const pa_block_manager* bm, int32_t block) {
    if (!bm || block < 0 || block >= bm->num_blocks) return -1;
    return bm->refcount[block];
}

extern "C" const int32_t* pa_bm_block_tables(const pa_block_manager* bm) {
    return bm ? bm->tables.data() : nullptr;
}

extern "C" const int32_t* pa_bm_context_lens(const pa_block_manager* bm) {
    return bm ? bm->lens.data() : nullptr;
}

extern "C" int32_t pa_bm_take_dirty_rows(pa_block_manager* bm, int32_t* rows, int32_t cap) {
    if (!bm || cap < 0 || (cap > 0 && !rows)) return -1;
    std::sort(bm->dirty_list.begin(), bm->dirty_list.end());
    const int32_t n = std::min<int32_t>(cap, (int32_t)bm->dirty_list.size());
    for (int32_t i = 0; i < n; ++i) {
        rows[i] = bm->dirty_list[i];
        bm->dirty[rows[i]] = 0;
    }
    bm->dirty_list.erase(bm->dirty_list.begin(), bm->dirty_list.begin() + n);
    return n;
}

extern "C" int pa_slot_mapping(const int32_t* block_tables, int32_t max_blocks_per_seq,
                               const int32_t* lengths, int32_t num_seqs, int32_t block_size,
                               int64_t* slots) {
    if (num_seqs < 0 || block_size <= 0 || max_blocks_per_seq <= 0) return PA_ERR_INVALID;
    if (num_seqs > 0 && (!block_tables || !lengths || !slots)) return PA_ERR_INVALID;
    for (int32_t b = 0; b < num_seqs; ++b) {
        const int32_t len = lengths[b];
        if (len <= 0) {
            slots[b] = -1;
            continue;
        }
        const int32_t p = len - 1;
        if (p / block_size >= max_blocks_per_seq) return PA_ERR_INVALID;
        const int32_t blk = block_tables[(size_t)b * max_blocks_per_seq + p / block_size];
        slots[b] = blk < 0 ? -1 : (int64_t)blk * block_size + p % block_size;
    }
    return PA_OK;
}
