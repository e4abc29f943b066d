// Log-sum-exp merge of split-KV partial states (flash-decoding's second pass).
//
// A decode kernel that cut a sequence's context into pieces left, per piece s
// and query head h, the normalised output o_s[h][:] and the piece's log2-
// domain log-sum-exp lse_s[h].  The softmax over the whole context is
//   M = max_s lse_s,  w_s = 2^(lse_s - M),  out = sum_s w_s o_s / sum_s w_s,
// rounded once to bf16.  One CTA of D threads per (sequence, kv head, query
// head): the piece weights are computed once into shared memory, then each
// thread accumulates one head-dim element with its global loads in flight
// together.  The kernel runs as a programmatic dependent launch: its CTAs may
// start while the decode kernel drains and wait (griddepcontrol.wait) for the
// decode grid to complete before reading.
#include <cuda_runtime.h>
#include <stdint.h>

#include "pa_device.cuh"

namespace pa {
namespace {

constexpr int kSmemSplits = 2048;   // pieces whose weights fit in shared memory

template <int D, bool kStream>
__global__ void __launch_bounds__(D) merge_kernel(const DecodeParams p) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    __shared__ float s_w[kSmemSplits];
    __shared__ float s_red[D / 32];
    const int32_t b = blockIdx.x, kvh = blockIdx.y, h = blockIdx.z;
    const int32_t G = p.group, Hkv = p.num_kv_heads;
    const int tid = threadIdx.x;
    int32_t nsplit;
    size_t row0, row_step;       // row of piece k: first piece row0, then row0 + k * row_step
    int64_t first_row;           // stream layout: the first piece lives in its own row
    if (kStream) {
        const int4 dsc = reinterpret_cast<const int4*>(p.seq_desc)[(size_t)(kvh / 8) * p.num_seqs + b];
        nsplit = dsc.x;
        if (nsplit <= 1) return;
        // CTA i_first + k, slot 0 (k > 0); the first CTA used slot dsc.z
        first_row = (((int64_t)dsc.y * 2 + dsc.z) * Hkv + kvh) * G + h;
        row0 = (((size_t)(dsc.y + 1) * 2) * Hkv + kvh) * G + h;   // piece k >= 1: row0 + (k-1) * step
        row_step = (size_t)2 * Hkv * G;
    } else {
        const int32_t L = clipped_length(p, b);
        nsplit = (L + p.split_tokens - 1) / p.split_tokens;
        if (nsplit <= 1) return;
        first_row = (((int64_t)b * Hkv + kvh) * p.max_splits) * G + h;
        row0 = (size_t)first_row + G;
        row_step = (size_t)G;
    }
    auto row_of = [&](int32_t k) -> size_t {
        return k == 0 ? (size_t)first_row : row0 + (size_t)(k - 1) * row_step;
    };
    // block-wide max of the pieces' log-sum-exps
    float M = -INFINITY;
    for (int32_t k = tid; k < nsplit; k += D) M = fmaxf(M, __ldcg(p.part_lse + row_of(k)));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    if ((tid & 31) == 0) s_red[tid >> 5] = M;
    __syncthreads();
    M = s_red[0];
#pragma unroll
    for (int w = 1; w < D / 32; ++w) M = fmaxf(M, s_red[w]);
    const bool cached = nsplit <= kSmemSplits;
    if (cached) {
        for (int32_t k = tid; k < nsplit; k += D) s_w[k] = fast_exp2(__ldcg(p.part_lse + row_of(k)) - M);
        __syncthreads();
    }
    float W = 0.f, acc = 0.f;
#pragma unroll 8
    for (int32_t k = 0; k < nsplit; ++k) {
        const size_t r = row_of(k);
        const float w = cached ? s_w[k] : fast_exp2(__ldcg(p.part_lse + r) - M);
        W += w;
        acc += w * __ldcg(p.part_o + r * D + tid);
    }
    p.out[((size_t)b * p.num_q_heads + (size_t)kvh * G + h) * D + tid] = f32_to_bf16_rn(acc / W);
}

template <int D, bool kStream>
cudaError_t launch_m(const DecodeParams& p, bool pdl, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)p.num_seqs, (unsigned)p.num_kv_heads, (unsigned)p.group);
    cfg.blockDim = dim3(D);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, merge_kernel<D, kStream>, p);
}

}  // namespace

cudaError_t launch_merge(const DecodeParams& p, bool stream_layout, bool pdl, cudaStream_t stream) {
    if (p.head_dim == 64)
        return stream_layout ? launch_m<64, true>(p, pdl, stream) : launch_m<64, false>(p, pdl, stream);
    if (p.head_dim == 128)
        return stream_layout ? launch_m<128, true>(p, pdl, stream) : launch_m<128, false>(p, pdl, stream);
    return cudaErrorInvalidValue;
}

}  // namespace pa
