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
#include <algorithm>
#include <cstdint>
#include <cstring>
#include <new>
#include <vector>

#include "pa.h"

struct pa_block_manager {
    int32_t num_blocks = 0;
    int32_t block_size = 0;
    int32_t max_seqs = 0;
    int32_t max_blocks = 0;
    std::vector<int32_t> free_stack;   // top = back()
    std::vector<int32_t> refcount;     // per physical block
    std::vector<int32_t> tables;       // [max_seqs][max_blocks], -1 beyond
    std::vector<int32_t> nblocks;      // blocks held per row
    std::vector<int32_t> lens;         // tokens per row
    std::vector<uint8_t> live;
    std::vector<uint8_t> dirty;
    std::vector<int32_t> dirty_list;

    int32_t* row(int32_t seq) { return tables.data() + (size_t)seq * max_blocks; }

    void mark(int32_t seq) {
        if (!dirty[seq]) {
            dirty[seq] = 1;
            dirty_list.push_back(seq);
        }
    }
    int32_t pop() {
        const int32_t b = free_stack.back();
        free_stack.pop_back();
        refcount[b] = 1;
        return b;
    }
    void release(int32_t b) {
        if (--refcount[b] == 0) free_stack.push_back(b);
    }
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
    bm->free_stack.reserve(num_blocks);
    for (int32_t i = num_free - 1; i >= 0; --i) bm->free_stack.push_back(free_order[i]);
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
    std::vector<uint8_t> on_stack(bm->num_blocks, 0);
    for (int32_t b : bm->free_stack) on_stack[b] = 1;
    for (int32_t i = 0; i < nb; ++i)
        if (blocks[i] < 0 || blocks[i] >= bm->num_blocks || on_stack[blocks[i]]) return PA_ERR_INVALID;
    int32_t* r = bm->row(seq);
    for (int32_t i = 0; i < nb; ++i) {
        r[i] = blocks[i];
        bm->refcount[blocks[i]] += 1;
    }
    bm->nblocks[seq] = nb;
    bm->lens[seq] = num_tokens;
    bm->live[seq] = 1;
    bm->mark(seq);
    return PA_OK;
}

extern "C" int pa_bm_add_seq(pa_block_manager* bm, int32_t seq, int32_t num_tokens) {
    if (!bm || !bm->valid_seq(seq) || bm->live[seq] || num_tokens < 0) return PA_ERR_INVALID;
    const int32_t nb = ceil_div(num_tokens, bm->block_size);
    if (nb > bm->max_blocks) return PA_ERR_INVALID;
    if ((size_t)nb > bm->free_stack.size()) return PA_ERR_OOM_BLOCKS;
    int32_t* r = bm->row(seq);
    for (int32_t i = 0; i < nb; ++i) r[i] = bm->pop();
    bm->nblocks[seq] = nb;
    bm->lens[seq] = num_tokens;
    bm->live[seq] = 1;
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
    if ((size_t)(nb - num_shared_blocks) > bm->free_stack.size()) return PA_ERR_OOM_BLOCKS;
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
    bm->mark(seq);
    return PA_OK;
}

extern "C" int pa_bm_free_seq(pa_block_manager* bm, int32_t seq) {
    if (!bm || !bm->valid_seq(seq) || !bm->live[seq]) return PA_ERR_INVALID;
    int32_t* r = bm->row(seq);
    for (int32_t i = 0; i < bm->nblocks[seq]; ++i) {
        bm->release(r[i]);
        r[i] = -1;
    }
    bm->nblocks[seq] = 0;
    bm->lens[seq] = 0;
    bm->live[seq] = 0;
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
    if (need > bm->free_stack.size()) return PA_ERR_OOM_BLOCKS;
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
    }
    return PA_OK;
}

extern "C" int32_t pa_bm_num_free(const pa_block_manager* bm) {
    return bm ? (int32_t)bm->free_stack.size() : -1;
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
