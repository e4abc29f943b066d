// KV-cache append: scatter each new token's K/V rows into its slot.
//
// The KV cache keeps the K/V projections of earlier tokens so a decode step
// does not recompute them (Tiny-vLLM summary page, section "고성능 추론을 위한
// 고급 최적화 기법"; dev.to vLLM page, section "KV Cache가 왜 병목인가").  With
// paging, a token's storage is a slot: block s / Bs, offset s % Bs of the pool
// (dev.to page, section "PagedAttention — OS 가상 메모리에서 영감").
//
// One thread moves one 16-byte chunk of K and the same chunk of V, so a warp
// writes whole 128-byte rows (D = 64) with coalesced 16-byte stores.  Pure
// copy: the result is bit-identical to the input rows.
#include <cuda_runtime.h>
#include <stdint.h>

#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {
namespace {

__global__ void __launch_bounds__(256) append_kv_kernel(
    const uint4* __restrict__ k, const uint4* __restrict__ v, const int64_t* __restrict__ slots,
    int64_t chunks, int32_t chunks_per_row, int32_t num_kv_heads, int32_t block_size,
    int64_t num_slots, uint4* __restrict__ k_cache, uint4* __restrict__ v_cache) {
    allow_dependents();   // a decode launched early may plan while the rows are written
    const int64_t per_token = (int64_t)num_kv_heads * chunks_per_row;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < chunks;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = i / per_token;
        const int64_t within = i - t * per_token;          // h * chunks_per_row + c
        const int64_t slot = slots[t];
        if (slot < 0 || slot >= num_slots) continue;
        const int64_t blk = slot / block_size;
        const int64_t off = slot - blk * block_size;
        const int64_t h = within / chunks_per_row;
        const int64_t c = within - h * chunks_per_row;
        const int64_t dst = ((blk * num_kv_heads + h) * block_size + off) * chunks_per_row + c;
        const uint4 kk = __ldg(k + i);
        const uint4 vv = __ldg(v + i);
        k_cache[dst] = kk;
        v_cache[dst] = vv;
    }
}

// Append of each sequence's newest token at position context_lens[b]-1 of its
// table row (the fused append + decode call on the kernels that do not fuse it).
__global__ void __launch_bounds__(256) append_at_end_kernel(const DecodeParams p) {
    const int32_t chunks_per_row = p.head_dim / 8;
    const int64_t per_seq = (int64_t)p.num_kv_heads * chunks_per_row;
    const int64_t total = per_seq * p.num_seqs;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int32_t b = (int32_t)(i / per_seq);
        const int64_t within = i - (int64_t)b * per_seq;
        const int32_t L = p.context_lens[b];
        const int32_t cap = p.max_blocks_per_seq * p.block_size;
        if (L <= 0 || L > cap || L > p.max_context_len) continue;
        const int32_t pos = L - 1;
        const int32_t blk = p.block_tables[(size_t)b * p.max_blocks_per_seq + pos / p.block_size];
        if (blk < 0 || blk >= p.num_blocks) continue;
        const int64_t h = within / chunks_per_row, c = within - h * chunks_per_row;
        const int64_t dst = (((int64_t)blk * p.num_kv_heads + h) * p.block_size + pos % p.block_size) *
                                chunks_per_row + c;
        reinterpret_cast<uint4*>(const_cast<uint16_t*>(p.k_cache))[dst] =
            __ldg(reinterpret_cast<const uint4*>(p.k_new) + i);
        reinterpret_cast<uint4*>(const_cast<uint16_t*>(p.v_cache))[dst] =
            __ldg(reinterpret_cast<const uint4*>(p.v_new) + i);
    }
}

// E4M3 append: like append_kv_kernel, each 16-byte chunk of 8 bf16 becomes 8 codes
// of value * inv_scale (a float product, then nearest even with saturation at +-448).
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}
__device__ __forceinline__ uint2 quantize8(uint4 x, float inv) {
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
    uint32_t c[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        c[i] = f32x2_to_e4m3x2(__fmul_rn(bf16_lo(w[i]), inv), __fmul_rn(bf16_hi(w[i]), inv));
    return make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
}

__global__ void __launch_bounds__(256) append_e4m3_kernel(
    const uint4* __restrict__ k, const uint4* __restrict__ v, const int64_t* __restrict__ slots,
    int64_t chunks, int32_t chunks_per_row, int32_t num_kv_heads, int32_t block_size,
    int64_t num_slots, float k_inv, float v_inv, uint2* __restrict__ k_cache, uint2* __restrict__ v_cache) {
    allow_dependents();
    const int64_t per_token = (int64_t)num_kv_heads * chunks_per_row;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < chunks;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = i / per_token;
        const int64_t within = i - t * per_token;
        const int64_t slot = slots[t];
        if (slot < 0 || slot >= num_slots) continue;
        const int64_t blk = slot / block_size, off = slot - blk * block_size;
        const int64_t h = within / chunks_per_row, c = within - h * chunks_per_row;
        const int64_t dst = ((blk * num_kv_heads + h) * block_size + off) * chunks_per_row + c;
        k_cache[dst] = quantize8(__ldg(k + i), k_inv);
        v_cache[dst] = quantize8(__ldg(v + i), v_inv);
    }
}

// Copy-on-write on the device: pair k copies block copies[2k] onto block copies[2k+1] in
// both caches (a block is Hkv x Bs x D contiguous elements), 16 bytes per thread.
__global__ void __launch_bounds__(256) copy_blocks_kernel(uint4* __restrict__ k_cache,
                                                          uint4* __restrict__ v_cache,
                                                          const int32_t* __restrict__ copies,
                                                          int32_t n, int64_t chunks_per_block,
                                                          int32_t num_blocks) {
    allow_dependents();
    const int64_t total = (int64_t)n * chunks_per_block;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t pair = i / chunks_per_block, c = i - pair * chunks_per_block;
        const int32_t src = copies[2 * pair], dst = copies[2 * pair + 1];
        if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) continue;
        k_cache[dst * chunks_per_block + c] = k_cache[src * chunks_per_block + c];
        v_cache[dst * chunks_per_block + c] = v_cache[src * chunks_per_block + c];
    }
}

}  // namespace

cudaError_t launch_append_e4m3(const pa_bf16* k, const pa_bf16* v, const int64_t* slots, int32_t T,
                               float k_inv_scale, float v_inv_scale, uint8_t* k_cache,
                               uint8_t* v_cache, const pa_cache_desc& d, cudaStream_t stream) {
    const int32_t chunks_per_row = d.head_dim / 8;
    const int64_t chunks = (int64_t)T * d.num_kv_heads * chunks_per_row;
    if (chunks == 0) return cudaSuccess;
    int64_t blocks = (chunks + 255) / 256;
    if (blocks > 148 * 32) blocks = 148 * 32;
    append_e4m3_kernel<<<(unsigned)blocks, 256, 0, stream>>>(
        reinterpret_cast<const uint4*>(k), reinterpret_cast<const uint4*>(v), slots, chunks,
        chunks_per_row, d.num_kv_heads, d.block_size, (int64_t)d.num_blocks * d.block_size,
        k_inv_scale, v_inv_scale, reinterpret_cast<uint2*>(k_cache), reinterpret_cast<uint2*>(v_cache));
    return cudaGetLastError();
}

cudaError_t launch_copy_blocks(pa_bf16* k_cache, pa_bf16* v_cache, const int32_t* copies, int32_t n,
                               const pa_cache_desc& d, cudaStream_t stream) {
    const int64_t cpb = (int64_t)d.num_kv_heads * d.block_size * d.head_dim / 8;
    const int64_t total = (int64_t)n * cpb;
    if (total == 0) return cudaSuccess;
    int64_t blocks = (total + 255) / 256;
    if (blocks > 148 * 32) blocks = 148 * 32;
    copy_blocks_kernel<<<(unsigned)blocks, 256, 0, stream>>>(
        reinterpret_cast<uint4*>(k_cache), reinterpret_cast<uint4*>(v_cache), copies, n, cpb,
        d.num_blocks);
    return cudaGetLastError();
}

cudaError_t launch_append_at_end(const DecodeParams& p, cudaStream_t stream) {
    const int64_t total = (int64_t)p.num_seqs * p.num_kv_heads * (p.head_dim / 8);
    if (total == 0) return cudaSuccess;
    int64_t blocks = (total + 255) / 256;
    if (blocks > 148 * 32) blocks = 148 * 32;
    append_at_end_kernel<<<(unsigned)blocks, 256, 0, stream>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_append(const pa_bf16* k, const pa_bf16* v, const int64_t* slots, int32_t T,
                          pa_bf16* k_cache, pa_bf16* v_cache, const pa_cache_desc& d,
                          cudaStream_t stream) {
    const int32_t chunks_per_row = d.head_dim / 8;
    const int64_t chunks = (int64_t)T * d.num_kv_heads * chunks_per_row;
    if (chunks == 0) return cudaSuccess;
    const int threads = 256;
    int64_t blocks = (chunks + threads - 1) / threads;
    if (blocks > 148 * 32) blocks = 148 * 32;  // grid-stride beyond 32 CTAs per SM
    append_kv_kernel<<<(unsigned)blocks, threads, 0, stream>>>(
        reinterpret_cast<const uint4*>(k), reinterpret_cast<const uint4*>(v), slots, chunks,
        chunks_per_row, d.num_kv_heads, d.block_size, (int64_t)d.num_blocks * d.block_size,
        reinterpret_cast<uint4*>(k_cache), reinterpret_cast<uint4*>(v_cache));
    return cudaGetLastError();
}

}  // namespace pa
