// Paged decode attention on CUDA cores (the plain variant).
//
// One CTA of four warps per (sequence, kv head, split of the context).  Each
// warp walks every fourth token of the split: it looks up the token's
// physical block in the table, loads the K row (one 4- or 8-byte piece per
// lane: the row is read by the warp as one coalesced 128/256-byte access),
// forms q.K for every query head of the GQA group (warp-shuffle sum), updates
// that head's running max / sum / output (online softmax, fp32, log2 domain),
// and accumulates p * V the same way.  The four warps' states are combined in
// shared memory, then either stored (one split) or written as a partial state
// for the merge kernel.
//
// It serves as the CUDA-core reference for the tensor-core kernel: every K/V
// element is widened to fp32 once, but the per-token shuffle reductions make
// it ALU- and latency-bound rather than HBM-bound.
#include <cuda_runtime.h>
#include <stdint.h>

#include "pa_device.cuh"

namespace pa {
namespace {

constexpr int kWarps = 4;

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

template <int D, int EPL>
__device__ __forceinline__ void load_row(const uint16_t* row, float (&f)[EPL]) {
    if constexpr (EPL == 2) {
        const uint32_t w = __ldg(reinterpret_cast<const uint32_t*>(row));
        f[0] = bf16_lo(w);
        f[1] = bf16_hi(w);
    } else {
        const uint2 w = __ldg(reinterpret_cast<const uint2*>(row));
        f[0] = bf16_lo(w.x);
        f[1] = bf16_hi(w.x);
        f[2] = bf16_lo(w.y);
        f[3] = bf16_hi(w.y);
    }
}

template <int D, int GM>
__global__ void __launch_bounds__(kWarps * 32) decode_simt_kernel(const DecodeParams p) {
    constexpr int EPL = D / 32;  // head-dim elements per lane
    const int32_t split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
    const int32_t L = clipped_length(p, b);
    if (L == 0) {
        if (split == 0) store_zero_group(p, b, kvh, threadIdx.x, blockDim.x);
        return;
    }
    const int32_t C = p.split_tokens;
    const int32_t nsplit = (L + C - 1) / C;
    if (split >= nsplit) return;
    const int32_t t0 = split * C;
    const int32_t t1 = min(L, t0 + C);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int32_t G = p.group;
    const int32_t Bs = p.block_size;

    float q[GM][EPL];
    const uint16_t* qbase = p.q + ((size_t)b * p.num_q_heads + (size_t)kvh * G) * D;
#pragma unroll
    for (int h = 0; h < GM; ++h) {
        if (h < G) {
            load_row<D, EPL>(qbase + (size_t)h * D + lane * EPL, q[h]);
        } else {
#pragma unroll
            for (int e = 0; e < EPL; ++e) q[h][e] = 0.f;
        }
    }
    float m[GM], l[GM], acc[GM][EPL];
#pragma unroll
    for (int h = 0; h < GM; ++h) {
        m[h] = -INFINITY;
        l[h] = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc[h][e] = 0.f;
    }

    const int32_t* table = p.block_tables + (size_t)b * p.max_blocks_per_seq;
    for (int32_t j = t0 + warp; j < t1; j += kWarps) {
        const int32_t blk = __ldg(table + j / Bs);
        const int32_t off = j % Bs;
        float kf[EPL], vf[EPL];
        if (blk < 0 || blk >= p.num_blocks) {
            if (lane == 0) raise_status(p.status, kStatusBadBlock);
#pragma unroll
            for (int e = 0; e < EPL; ++e) kf[e] = vf[e] = 0.f;
        } else {
            const size_t row = (((size_t)blk * p.num_kv_heads + kvh) * Bs + off) * D + lane * EPL;
            load_row<D, EPL>(p.k_cache + row, kf);
            load_row<D, EPL>(p.v_cache + row, vf);
        }
#pragma unroll
        for (int h = 0; h < GM; ++h) {
            if (h < G) {
                float s = 0.f;
#pragma unroll
                for (int e = 0; e < EPL; ++e) s += q[h][e] * kf[e];
                s = warp_sum(s) * p.scale_log2;
                const float mn = fmaxf(m[h], s);
                const float alpha = fast_exp2(m[h] - mn);
                const float pr = fast_exp2(s - mn);
                l[h] = l[h] * alpha + pr;
#pragma unroll
                for (int e = 0; e < EPL; ++e) acc[h][e] = acc[h][e] * alpha + pr * vf[e];
                m[h] = mn;
            }
        }
    }

    // Combine the four warps' running states.
    __shared__ float s_m[kWarps][GM], s_l[kWarps][GM];
    __shared__ float s_acc[kWarps][GM][D];
#pragma unroll
    for (int h = 0; h < GM; ++h) {
        if (lane == 0) {
            s_m[warp][h] = m[h];
            s_l[warp][h] = l[h];
        }
#pragma unroll
        for (int e = 0; e < EPL; ++e) s_acc[warp][h][lane * EPL + e] = acc[h][e];
    }
    __syncthreads();
    const size_t part = (((size_t)b * p.num_kv_heads + kvh) * p.max_splits + split) * G;
    uint16_t* out = p.out + ((size_t)b * p.num_q_heads + (size_t)kvh * G) * D;
    for (int i = threadIdx.x; i < G * D; i += kWarps * 32) {
        const int h = i / D, d = i - h * D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) M = fmaxf(M, s_m[w][h]);
        float lsum = 0.f, osum = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            const float sc = fast_exp2(s_m[w][h] - M);
            lsum += s_l[w][h] * sc;
            osum += s_acc[w][h][d] * sc;
        }
        if (nsplit == 1) {
            out[(size_t)h * D + d] = f32_to_bf16_rn(osum / lsum);
        } else {
            p.part_o[(part + h) * D + d] = osum / lsum;
            if (d == 0) p.part_lse[part + h] = M + __log2f(lsum);
        }
    }
}

template <int D>
cudaError_t launch_d(const DecodeParams& p, cudaStream_t stream) {
    const dim3 grid(p.max_splits, p.num_kv_heads, p.num_seqs);
    const dim3 block(kWarps * 32);
    if (p.group <= 1) decode_simt_kernel<D, 1><<<grid, block, 0, stream>>>(p);
    else if (p.group <= 2) decode_simt_kernel<D, 2><<<grid, block, 0, stream>>>(p);
    else if (p.group <= 4) decode_simt_kernel<D, 4><<<grid, block, 0, stream>>>(p);
    else if (p.group <= 8) decode_simt_kernel<D, 8><<<grid, block, 0, stream>>>(p);
    else decode_simt_kernel<D, 16><<<grid, block, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_simt(const DecodeParams& p, cudaStream_t stream) {
    if (p.head_dim == 64) return launch_d<64>(p, stream);
    if (p.head_dim == 128) return launch_d<128>(p, stream);
    return cudaErrorInvalidValue;
}

}  // namespace pa
