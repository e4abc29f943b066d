// Log-sum-exp merge of split-KV partial states (flash-decoding's second pass).
//
// A decode kernel that cut a sequence's context into pieces left, per piece s
// and query head h, the normalised output o_s[h][:] and the piece's log2-
// domain log-sum-exp lse_s[h].  The softmax over the whole context is
//   M = max_s lse_s,  w_s = 2^(lse_s - M),  out = sum_s w_s o_s / sum_s w_s,
// rounded once to bf16.  The pieces are spread over a CTA's threads and
// folded with a running max, so a merge costs one round of L2 reads (after the
// piece descriptor): one CTA per (sequence, kv head, query head), or, for a
// stream-partitioned decode of a large batch, one CTA per (sequence, kv head)
// holding the kv head's G query heads.  The kernels run as programmatic
// dependent launches: their CTAs may start while the decode kernel drains and
// wait (griddepcontrol.wait) for the decode grid to complete before reading.
#include <cuda_runtime.h>
#include <stdint.h>

#include "pa_device.cuh"

namespace pa {
namespace {

// One CTA of PG * D/4 threads per (sequence, kv head, query head): PG groups over
// the pieces (piece k goes to group k % PG) times D/4 float4 columns of the head
// dimension.  Each thread folds its pieces into a running (max, weight, sum)
// state as their lse and output arrive (independent loads), and the groups'
// states are merged the same way through shared memory.  Long contexts cut a
// sequence into many pieces: 16 groups keep each thread's chain short there.
// kStream: the stream partition's pieces (read from the sequence's descriptor);
// else the split kernels' fixed splits.
template <int D, bool kStream, int PG>
__global__ void __launch_bounds__(PG * D / 4) merge_kernel(const DecodeParams p) {
    constexpr int kCols = D / 4;
    constexpr int kPieceGroups = PG;
    allow_dependents();   // a next decode call launched early may plan while this runs
    wait_prerequisite();
    __shared__ float4 s_acc[kPieceGroups][kCols];
    __shared__ float s_m[kPieceGroups], s_w[kPieceGroups];
    const int32_t b = blockIdx.x, kvh = blockIdx.y, h = blockIdx.z;
    const int32_t G = p.group, Hkv = p.num_kv_heads;
    const int tid = threadIdx.x;
    int32_t nsplit;
    size_t first_row, row0, row_step;   // piece 0: first_row; piece k >= 1: row0 + (k-1) * row_step
    if (kStream) {
        const int4 dsc = reinterpret_cast<const int4*>(p.seq_desc)[(size_t)(kvh / 8) * p.num_seqs + b];
        nsplit = dsc.x;
        if (nsplit <= 1) return;
        // a descriptor this launch's decode did not write (it gave up on a timed-out wait)
        // may be left from an earlier call: read nothing outside this launch's partial rows
        if (dsc.y < 0 || dsc.z < 0 || dsc.z > 1 || (int64_t)dsc.y + nsplit > p.grid) return;
        // CTA i_first + k wrote slot 0 for k > 0; the first CTA used slot dsc.z
        first_row = (((size_t)dsc.y * 2 + dsc.z) * Hkv + kvh) * G + h;
        row0 = (((size_t)(dsc.y + 1) * 2) * Hkv + kvh) * G + h;
        row_step = (size_t)2 * Hkv * G;
    } else {
        const int32_t L = clipped_length(p, b);
        nsplit = (L + p.split_tokens - 1) / p.split_tokens;
        if (nsplit <= 1) return;
        first_row = (((size_t)b * Hkv + kvh) * p.max_splits) * G + h;
        row0 = first_row + G;
        row_step = (size_t)G;
    }
    const int kg = tid / kCols, col = tid - kg * kCols;
    float m = -INFINITY, W = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
    for (int32_t k = kg; k < nsplit; k += kPieceGroups) {
        const size_t r = k == 0 ? first_row : row0 + (size_t)(k - 1) * row_step;
        const float lse = __ldcg(p.part_lse + r);
        const float4 o = __ldcg(reinterpret_cast<const float4*>(p.part_o + r * D) + col);
        const float mn = fmaxf(m, lse);
        const float sc = fast_exp2(m - mn), w = fast_exp2(lse - mn);
        W = W * sc + w;
        acc.x = acc.x * sc + w * o.x;
        acc.y = acc.y * sc + w * o.y;
        acc.z = acc.z * sc + w * o.z;
        acc.w = acc.w * sc + w * o.w;
        m = mn;
    }
    s_acc[kg][col] = acc;
    if (col == 0) {
        s_m[kg] = m;
        s_w[kg] = W;
    }
    __syncthreads();
    if (tid < kCols) {
        float M = s_m[0];
#pragma unroll
        for (int g = 1; g < kPieceGroups; ++g) M = fmaxf(M, s_m[g]);
        float Wt = 0.f;
        float4 t = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int g = 0; g < kPieceGroups; ++g) {
            const float sc = fast_exp2(s_m[g] - M);   // a group with no piece has m = -inf: weight 0
            const float4 u = s_acc[g][tid];
            Wt += s_w[g] * sc;
            t.x += u.x * sc;
            t.y += u.y * sc;
            t.z += u.z * sc;
            t.w += u.w * sc;
        }
        const float inv = 1.f / Wt;
        uint2 packed;
        packed.x = pack_bf16x2(t.x * inv, t.y * inv);
        packed.y = pack_bf16x2(t.z * inv, t.w * inv);
        reinterpret_cast<uint2*>(p.out + ((size_t)b * p.num_q_heads + (size_t)kvh * G + h) * D)[tid] = packed;
    }
}

// The stream kernel's pieces of a large batch: one CTA per (sequence, kv head) with all G
// query heads of the kv head in it, PG groups of G * D/4 threads (piece k to group k % PG).  A
// sequence the decode did not cut costs its CTA one descriptor read, instead of G CTAs' worth.
// PG is chosen at launch so that the grid fills about one wave of the GPU.
template <int D>
__global__ void __launch_bounds__(1024) merge_stream_kernel(const DecodeParams p, int PG) {
    constexpr int kCols = D / 4;
    allow_dependents();   // a next decode call launched early may plan while this runs
    wait_prerequisite();
    extern __shared__ float4 s_dyn[];
    const int32_t b = blockIdx.x, kvh = blockIdx.y, G = p.group, Hkv = p.num_kv_heads;
    const int4 dsc = reinterpret_cast<const int4*>(p.seq_desc)[(size_t)(kvh / 8) * p.num_seqs + b];
    const int32_t nsplit = dsc.x;
    if (nsplit <= 1) return;
    // a descriptor this launch's decode did not write (it gave up on a timed-out wait) may be
    // left from an earlier call: read nothing outside this launch's partial rows
    if (dsc.y < 0 || dsc.z < 0 || dsc.z > 1 || (int64_t)dsc.y + nsplit > p.grid) return;
    const int32_t C = G * kCols, t = threadIdx.x, pg = t / C, rem = t - pg * C;
    const int32_t h = rem / kCols, col = rem - h * kCols;
    float4* s_acc = s_dyn;                                            // [PG][C]
    float2* s_mw = reinterpret_cast<float2*>(s_dyn + (size_t)PG * C);  // [PG][G] (max, weight)
    float m = -INFINITY, W = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (pg < PG) {
#pragma unroll 4
        for (int32_t k = pg; k < nsplit; k += PG) {
            // piece 0 in slot dsc.z of CTA dsc.y, piece k >= 1 in slot 0 of CTA dsc.y + k
            const size_t r = ((((size_t)dsc.y + k) * 2 + (k == 0 ? dsc.z : 0)) * Hkv + kvh) * G + h;
            const float lse = __ldcg(p.part_lse + r);
            const float4 o = __ldcg(reinterpret_cast<const float4*>(p.part_o + r * D) + col);
            const float mn = fmaxf(m, lse);
            const float sc = fast_exp2(m - mn), w = fast_exp2(lse - mn);
            W = W * sc + w;
            acc.x = acc.x * sc + w * o.x;
            acc.y = acc.y * sc + w * o.y;
            acc.z = acc.z * sc + w * o.z;
            acc.w = acc.w * sc + w * o.w;
            m = mn;
        }
        s_acc[(size_t)pg * C + rem] = acc;
        if (col == 0) s_mw[pg * G + h] = make_float2(m, W);
    }
    __syncthreads();
    if (pg != 0) return;
    float M = -INFINITY;
    for (int g = 0; g < PG; ++g) M = fmaxf(M, s_mw[g * G + h].x);
    float Wt = 0.f;
    float4 tot = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int g = 0; g < PG; ++g) {
        const float2 mw = s_mw[g * G + h];
        const float sc = fast_exp2(mw.x - M);   // a group with no piece has max -inf: weight 0
        const float4 u = s_acc[(size_t)g * C + rem];
        Wt += mw.y * sc;
        tot.x += u.x * sc;
        tot.y += u.y * sc;
        tot.z += u.z * sc;
        tot.w += u.w * sc;
    }
    const float inv = 1.f / Wt;
    uint2 packed;
    packed.x = pack_bf16x2(tot.x * inv, tot.y * inv);
    packed.y = pack_bf16x2(tot.z * inv, tot.w * inv);
    reinterpret_cast<uint2*>(p.out + ((size_t)b * p.num_q_heads + (size_t)kvh * G + h) * D)[col] = packed;
}

template <int D>
cudaError_t launch_ms(const DecodeParams& p, bool pdl, cudaStream_t stream) {
    int sms = 0;
    if (num_sms_current_device(&sms) != PA_OK) return cudaErrorInvalidDevice;
    const int C = p.group * (D / 4);
    const int64_t ctas = (int64_t)p.num_seqs * p.num_kv_heads;
    const int64_t per_cta = (int64_t)sms * 2048 / (ctas * C);   // threads per column for one wave
    int PG = 1;
    while (PG < 16 && 2 * PG * C <= 1024 && 2 * PG <= per_cta) PG *= 2;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)p.num_seqs, (unsigned)p.num_kv_heads);
    cfg.blockDim = dim3((unsigned)(PG * C));
    cfg.dynamicSmemBytes = (size_t)PG * C * sizeof(float4) + (size_t)PG * p.group * sizeof(float2);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, merge_stream_kernel<D>, p, PG);
}

template <int D, bool kStream, int PG>
cudaError_t launch_m(const DecodeParams& p, bool pdl, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)p.num_seqs, (unsigned)p.num_kv_heads, (unsigned)p.group);
    cfg.blockDim = dim3(PG * D / 4);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, merge_kernel<D, kStream, PG>, p);
}

template <int D, bool kStream>
cudaError_t launch_mg(const DecodeParams& p, bool pdl, cudaStream_t stream) {
    // contexts of 8K tokens and more are cut into many pieces per sequence
    return p.max_context_len >= 8192 ? launch_m<D, kStream, 16>(p, pdl, stream)
                                     : launch_m<D, kStream, 4>(p, pdl, stream);
}

// Stream partition: one CTA per query head while that grid stays within about two waves of
// small CTAs (C2: 2048, C3: 1024, C4: 256 CTAs); beyond it (C5: 8192, mostly sequences that
// were not cut) one CTA per kv head.  Measured per call: C5 88.0 -> 83.8 us with the
// per-kv-head CTAs, while C2, C3 and C4 were 1.4 to 7 us faster with the per-head ones.
template <int D>
cudaError_t launch_stream_merge(const DecodeParams& p, bool pdl, cudaStream_t stream) {
    int sms = 0;
    if (num_sms_current_device(&sms) != PA_OK) return cudaErrorInvalidDevice;
    const int64_t per_head_ctas = (int64_t)p.num_seqs * p.num_kv_heads * p.group;
    if (per_head_ctas <= (int64_t)sms * 16) return launch_mg<D, true>(p, pdl, stream);
    return launch_ms<D>(p, pdl, stream);
}

}  // namespace

cudaError_t launch_merge(const DecodeParams& p, bool stream_layout, bool pdl, cudaStream_t stream) {
    if (p.head_dim == 64)
        return stream_layout ? launch_stream_merge<64>(p, pdl, stream) : launch_mg<64, false>(p, pdl, stream);
    if (p.head_dim == 128)
        return stream_layout ? launch_stream_merge<128>(p, pdl, stream) : launch_mg<128, false>(p, pdl, stream);
    return cudaErrorInvalidValue;
}

}  // namespace pa
