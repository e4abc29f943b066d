// Per-block pool: the allocator half of paging, without per-sequence tables.
//
// The KV cache is a pool of fixed-size physical blocks handed out one at a time as tokens
// arrive, and a block may be held by several block tables at once (page "vLLM —
// PagedAttention으로 LLM 추론 성능을 2~4배 끌어올린 서빙 엔진", section "PagedAttention — OS 가상
// 메모리에서 영감"; page "Nano-vLLM로 배우는 vLLM 추론 엔진 작동 원리 한눈에 정리", section "KV
// 캐시와 Block Manager": shared prefix blocks).  This object keeps only that: a stack of free
// block ids and a reference count per block.  Callers that keep their own block tables use it
// directly; pa_bm_* (block_manager.cpp) is the same policy with the tables kept for them.
//
// Policy (the same as pa_bm_*): the free ids form a stack, free_order[0] on top (handed out
// first); alloc takes from the top and sets the count to 1; share adds one holder; free drops
// one, and a block whose count reaches zero goes back on top of the stack.
#include <cstdint>
#include <new>
#include <vector>

#include "pa.h"

struct pa_block_pool {
    std::vector<int32_t> stack;      // free ids, top = back()
    std::vector<int32_t> refcount;   // 0 = free
};

extern "C" int pa_pool_create(int32_t num_blocks, const int32_t* free_order, int32_t num_free,
                              pa_block_pool** out) {
    if (!out || num_blocks <= 0 || num_free < 0 || num_free > num_blocks) return PA_ERR_INVALID;
    if (num_free > 0 && !free_order) return PA_ERR_INVALID;
    *out = nullptr;
    pa_block_pool* p = new (std::nothrow) pa_block_pool;
    if (!p) return PA_ERR_INVALID;
    try {
        // every block not listed as free starts out held once (a caller's reserved blocks)
        p->refcount.assign(num_blocks, 1);
        p->stack.reserve(num_blocks);
        for (int32_t i = num_free - 1; i >= 0; --i) {
            const int32_t b = free_order[i];
            if (b < 0 || b >= num_blocks || p->refcount[b] == 0) {
                delete p;
                return PA_ERR_INVALID;   // out of range or listed twice
            }
            p->refcount[b] = 0;
            p->stack.push_back(b);
        }
    } catch (...) {
        delete p;
        return PA_ERR_INVALID;
    }
    *out = p;
    return PA_OK;
}

extern "C" void pa_pool_destroy(pa_block_pool* pool) { delete pool; }

extern "C" int pa_pool_alloc(pa_block_pool* pool, int32_t n, int32_t* blocks) {
    if (!pool || n < 0 || (n > 0 && !blocks)) return PA_ERR_INVALID;
    if ((size_t)n > pool->stack.size()) return PA_ERR_OOM_BLOCKS;   // all or nothing
    for (int32_t i = 0; i < n; ++i) {
        const int32_t b = pool->stack.back();
        pool->stack.pop_back();
        pool->refcount[b] = 1;
        blocks[i] = b;
    }
    return PA_OK;
}

extern "C" int pa_pool_share(pa_block_pool* pool, int32_t block) {
    if (!pool || block < 0 || block >= (int32_t)pool->refcount.size()) return PA_ERR_INVALID;
    if (pool->refcount[block] == 0) return PA_ERR_INVALID;   // nobody holds a free block
    ++pool->refcount[block];
    return PA_OK;
}

extern "C" int pa_pool_free(pa_block_pool* pool, int32_t block) {
    if (!pool || block < 0 || block >= (int32_t)pool->refcount.size()) return PA_ERR_INVALID;
    if (pool->refcount[block] == 0) return PA_ERR_INVALID;   // already free
    if (--pool->refcount[block] == 0) pool->stack.push_back(block);
    return PA_OK;
}

extern "C" int32_t pa_pool_num_free(const pa_block_pool* pool) {
    return pool ? (int32_t)pool->stack.size() : -1;
}

extern "C" int32_t pa_pool_refcount(const pa_block_pool* pool, int32_t block) {
    if (!pool || block < 0 || block >= (int32_t)pool->refcount.size()) return -1;
    return pool->refcount[block];
}
