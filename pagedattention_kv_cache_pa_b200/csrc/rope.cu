// RoPE (rotary position embedding) fused with the KV append.
//
// RoPE is one of the per-layer operations of the Llama 3.2 1B model the
// Tiny-vLLM summary page targets (section "핵심 LLM 연산의 CUDA 커널 구현"); in a
// decode step it turns q and the new token's K at the token's position just
// before K is cached.  The page gives no formula; this library applies
// RoFormer's rotation in the rotate-half pairing with the caller's frequency
// base theta: pair (x[i], x[i + D/2]) turns by pos * theta^(-2i/D).  Rotated
// rows are rounded to nearest-even bf16, the format q and the caches hold.
//
// One CTA per token (grid-stride): the token's D/2 cos/sin pairs go to shared
// memory once, then each thread rotates an 8-pair chunk of one q or K head
// (16-byte loads of both halves) or copies one 16-byte chunk of V.
#include <cuda_runtime.h>
#include <stdint.h>

#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {
namespace {

constexpr int kThreads = 256;

struct RopeArgs {
    const uint16_t* q;
    uint16_t* q_out;
    const uint16_t* k;
    const uint16_t* v;
    const int32_t* positions;    // slot-mapping mode: position of each token
    const int64_t* slots;        // slot-mapping mode: slot of each token (< 0: not written)
    int32_t T, Hq, Hkv, D, Bs;
    int64_t num_slots;
    float theta;
    uint16_t* k_cache;
    uint16_t* v_cache;
};

template <bool kAtEnd>
__global__ void __launch_bounds__(kThreads) rope_append_kernel(const RopeArgs a, const DecodeParams p) {
    allow_dependents();
    __shared__ double s_inv[64];
    __shared__ float s_c[64], s_s[64];
    const int32_t half = a.D / 2, hc = a.D / 16, vc = a.D / 8;
    for (int32_t i = threadIdx.x; i < half; i += blockDim.x) s_inv[i] = rope_inv_freq(i, a.D, a.theta);
    const int32_t items = (a.Hq + a.Hkv) * hc + a.Hkv * vc;
    for (int32_t t = blockIdx.x; t < a.T; t += gridDim.x) {
        int32_t pos;
        int64_t slot = -1;
        if (kAtEnd) {
            const int32_t L = clipped_length(p, t);
            pos = L > 0 ? L - 1 : 0;
            if (L > 0) {
                const int32_t blk = p.block_tables[(size_t)t * p.max_blocks_per_seq + pos / a.Bs];
                if (blk >= 0 && blk < p.num_blocks) slot = (int64_t)blk * a.Bs + pos % a.Bs;
            }
        } else {
            pos = a.positions[t];
            slot = a.slots[t];
            if (slot >= a.num_slots) slot = -1;
        }
        __syncthreads();   // the previous token's cos/sin are no longer read
        for (int32_t i = threadIdx.x; i < half; i += blockDim.x) rope_cos_sin(pos, s_inv[i], &s_c[i], &s_s[i]);
        __syncthreads();
        const int64_t blk = slot >= 0 ? slot / a.Bs : 0, off = slot >= 0 ? slot % a.Bs : 0;
        for (int32_t w = threadIdx.x; w < items; w += blockDim.x) {
            if (w < (a.Hq + a.Hkv) * hc) {
                const bool is_q = w < a.Hq * hc;
                const int32_t r = is_q ? w : w - a.Hq * hc;
                const int32_t h = r / hc, c = r - h * hc;
                if (!is_q && slot < 0) continue;
                const uint16_t* src = is_q ? a.q + ((size_t)t * a.Hq + h) * a.D
                                           : a.k + ((size_t)t * a.Hkv + h) * a.D;
                uint4 x1 = *reinterpret_cast<const uint4*>(src + c * 8);
                uint4 x2 = *reinterpret_cast<const uint4*>(src + half + c * 8);
                rope_rotate8(x1, x2, s_c + c * 8, s_s + c * 8);
                uint16_t* dst = is_q ? a.q_out + ((size_t)t * a.Hq + h) * a.D
                                     : a.k_cache + ((blk * a.Hkv + h) * a.Bs + off) * a.D;
                *reinterpret_cast<uint4*>(dst + c * 8) = x1;
                *reinterpret_cast<uint4*>(dst + half + c * 8) = x2;
            } else {
                if (slot < 0) continue;
                const int32_t r = w - (a.Hq + a.Hkv) * hc;
                const int32_t h = r / vc, c = r - h * vc;
                *reinterpret_cast<uint4*>(a.v_cache + ((blk * a.Hkv + h) * a.Bs + off) * a.D + c * 8) =
                    *reinterpret_cast<const uint4*>(a.v + ((size_t)t * a.Hkv + h) * a.D + c * 8);
            }
        }
    }
}

unsigned grid_for(int32_t T) { return (unsigned)(T < 148 * 8 ? T : 148 * 8); }

}  // namespace

cudaError_t launch_rope_append(const pa_bf16* q, pa_bf16* q_out, const pa_bf16* k, const pa_bf16* v,
                               const int32_t* positions, const int64_t* slots, int32_t T, float theta,
                               pa_bf16* k_cache, pa_bf16* v_cache, const pa_cache_desc& d,
                               cudaStream_t stream) {
    if (T == 0) return cudaSuccess;
    RopeArgs a{};
    a.q = q;
    a.q_out = q_out;
    a.k = k;
    a.v = v;
    a.positions = positions;
    a.slots = slots;
    a.T = T;
    a.Hq = d.num_q_heads;
    a.Hkv = d.num_kv_heads;
    a.D = d.head_dim;
    a.Bs = d.block_size;
    a.num_slots = (int64_t)d.num_blocks * d.block_size;
    a.theta = theta;
    a.k_cache = k_cache;
    a.v_cache = v_cache;
    DecodeParams unused{};
    rope_append_kernel<false><<<grid_for(T), kThreads, 0, stream>>>(a, unused);
    return cudaGetLastError();
}

cudaError_t launch_rope_append_at_end(const DecodeParams& p, uint16_t* q_out, cudaStream_t stream) {
    if (p.num_seqs == 0) return cudaSuccess;
    RopeArgs a{};
    a.q = p.q;
    a.q_out = q_out;
    a.k = p.k_new;
    a.v = p.v_new;
    a.T = p.num_seqs;
    a.Hq = p.num_q_heads;
    a.Hkv = p.num_kv_heads;
    a.D = p.head_dim;
    a.Bs = p.block_size;
    a.num_slots = (int64_t)p.num_blocks * p.block_size;
    a.theta = p.rope_theta;
    a.k_cache = const_cast<uint16_t*>(p.k_cache);
    a.v_cache = const_cast<uint16_t*>(p.v_cache);
    rope_append_kernel<true><<<grid_for(p.num_seqs), kThreads, 0, stream>>>(a, p);
    return cudaGetLastError();
}

}  // namespace pa
