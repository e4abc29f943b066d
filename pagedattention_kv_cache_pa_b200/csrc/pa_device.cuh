// Device-side helpers shared by the decode kernels: bf16 packing, fast exp2,
// the device status word and context-length clipping.
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

// Lets a programmatic dependent launch (the merge kernel, or a decode kernel
// launched early) be scheduled; it still waits for this grid to complete
// before it reads anything this grid writes.
__device__ __forceinline__ void allow_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Waits until the grid this one was launched as a programmatic dependent of has
// completed and its writes are visible; returns at once for a plain launch.
__device__ __forceinline__ void wait_prerequisite() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ void raise_status(int32_t* status, int32_t bit) {
    if (status) atomicOr(status, bit);
}

// A context length as the decode uses it: negative or past what the table (and the call's
// max_context_len) can hold is reported and clipped.
__device__ __forceinline__ int32_t clip_length(const DecodeParams& p, int32_t L) {
    const int32_t table_cap = p.max_blocks_per_seq * p.block_size;
    const int32_t cap = p.max_context_len < table_cap ? p.max_context_len : table_cap;
    if (L < 0 || L > cap) {
        raise_status(p.status, kStatusBadLength);
        L = L < 0 ? 0 : cap;
    }
    return L;
}

// Context length of sequence b after clipping to what the grid and the table cover.
__device__ __forceinline__ int32_t clipped_length(const DecodeParams& p, int32_t b) {
    return clip_length(p, p.context_lens[b]);
}

// RoPE: pair i (of D/2) at position pos turns by a = pos * theta^(-2i/D).  The
// inverse frequency theta^(-2i/D) is formed once per CTA in double; the angle
// is formed and reduced to [-pi, pi] in double (positions reach 2^17, where a
// float product would already be off by ~1e-2 rad), then cos/sin in float
// (errors ~5e-7, far below the bf16 rounding of the rotated values).
// The rotation of (x[i], x[i + D/2]) by a is (x[i] c - x[i + D/2] s, x[i] s + x[i + D/2] c).
__device__ __forceinline__ double rope_inv_freq(int32_t i, int32_t D, float theta) {
    return exp2(-2.0 * (double)i / (double)D * log2((double)theta));
}
__device__ __forceinline__ void rope_cos_sin(int32_t pos, double inv_freq, float* c, float* s) {
    const double a = (double)pos * inv_freq;
    const double two_pi = 6.283185307179586476925286766559;
    const double r = a - two_pi * rint(a * (1.0 / two_pi));
    __sincosf((float)r, s, c);   // on [-pi, pi] the hardware form is within ~5e-7 of cos/sin
}
// Rotates 8 pairs: x1 = elements [i0, i0 + 8), x2 = the same of the second half.
__device__ __forceinline__ void rope_rotate8(uint4& x1, uint4& x2, const float* c, const float* s) {
    uint32_t* a = reinterpret_cast<uint32_t*>(&x1);
    uint32_t* b = reinterpret_cast<uint32_t*>(&x2);
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        const float a0 = bf16_lo(a[w]), a1 = bf16_hi(a[w]), b0 = bf16_lo(b[w]), b1 = bf16_hi(b[w]);
        const int e = 2 * w;
        a[w] = pack_bf16x2(a0 * c[e] - b0 * s[e], a1 * c[e + 1] - b1 * s[e + 1]);
        b[w] = pack_bf16x2(a0 * s[e] + b0 * c[e], a1 * s[e + 1] + b1 * c[e + 1]);
    }
}

// Writes zeros for the query heads of (b, kv head): the output of an empty context.
__device__ __forceinline__ void store_zero_group(const DecodeParams& p, int32_t b, int32_t kvh,
                                                 int tid, int nthreads) {
    uint16_t* o = p.out + ((size_t)b * p.num_q_heads + (size_t)kvh * p.group) * p.head_dim;
    for (int32_t i = tid; i < p.group * p.head_dim; i += nthreads) o[i] = 0;
}

}  // namespace pa
