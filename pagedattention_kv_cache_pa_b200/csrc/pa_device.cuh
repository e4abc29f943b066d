// Device-side helpers shared by the decode kernels: bf16 packing, the split
// bookkeeping, and the log-sum-exp merge of split partial states.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "pa_internal.h"

namespace pa {

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// float -> bf16 bits, round to nearest even (finite inputs; NaN kept quiet).
__device__ __forceinline__ uint16_t f32_to_bf16_rn(float f) {
    uint16_t r;
    asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(r) : "f"(f));
    return r;
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void raise_status(int32_t* status, int32_t bit) {
    if (status) atomicOr(status, bit);
}

// Context length of sequence b after clipping to what the grid and the table cover.
__device__ __forceinline__ int32_t clipped_length(const DecodeParams& p, int32_t b) {
    int32_t L = p.context_lens[b];
    const int32_t table_cap = p.max_blocks_per_seq * p.block_size;
    const int32_t cap = p.max_context_len < table_cap ? p.max_context_len : table_cap;
    if (L < 0 || L > cap) {
        raise_status(p.status, kStatusBadLength);
        L = L < 0 ? 0 : cap;
    }
    return L;
}

// Writes zeros for the query heads of (b, kv head): the output of an empty context.
__device__ __forceinline__ void store_zero_group(const DecodeParams& p, int32_t b, int32_t kvh) {
    uint16_t* o = p.out + ((size_t)b * p.num_q_heads + (size_t)kvh * p.group) * p.head_dim;
    for (int32_t i = threadIdx.x; i < p.group * p.head_dim; i += blockDim.x) o[i] = 0;
}

// Merge of the nsplit partial states of (b, kv head) into bf16 output:
//   M = max_s lse_s,  w_s = 2^(lse_s - M),  out = sum_s w_s o_s / sum_s w_s
// (log2-domain log-sum-exp).  Reads bypass L1: the partials were written by
// other CTAs of this launch.
__device__ __forceinline__ void merge_splits(const DecodeParams& p, int32_t b, int32_t kvh,
                                             int32_t nsplit) {
    const int32_t G = p.group, D = p.head_dim;
    const size_t base = ((size_t)b * p.num_kv_heads + kvh) * p.max_splits;
    uint16_t* out = p.out + ((size_t)b * p.num_q_heads + (size_t)kvh * G) * D;
    for (int32_t i = threadIdx.x; i < G * D; i += blockDim.x) {
        const int32_t h = i / D, d = i - h * D;
        float M = -INFINITY;
        for (int32_t s = 0; s < nsplit; ++s) M = fmaxf(M, __ldcg(p.part_lse + (base + s) * G + h));
        float W = 0.f, acc = 0.f;
        for (int32_t s = 0; s < nsplit; ++s) {
            const float w = fast_exp2(__ldcg(p.part_lse + (base + s) * G + h) - M);
            W += w;
            acc += w * __ldcg(p.part_o + ((base + s) * G + h) * D + d);
        }
        out[(size_t)h * D + d] = f32_to_bf16_rn(acc / W);
    }
}

// Called by every thread of a split CTA after it has written its partial
// state.  Returns true in the one CTA that arrives last for (b, kv head); that
// CTA has merged the splits and reset the counter.  The writer side fences
// before the arrival; the last arriver fences before reading.
__device__ __forceinline__ void arrive_and_maybe_merge(const DecodeParams& p, int32_t b,
                                                       int32_t kvh, int32_t nsplit) {
    __shared__ int32_t s_last;
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        int32_t* ctr = p.counters + (size_t)b * p.num_kv_heads + kvh;
        const int32_t prev = atomicAdd(ctr, 1);
        s_last = (prev == nsplit - 1);
        if (s_last) {
            *ctr = 0;  // self-reset for the next launch (kernel boundary orders it)
            __threadfence();
        }
    }
    __syncthreads();
    if (s_last) merge_splits(p, b, kvh, nsplit);
}

}  // namespace pa
