// Paged decode attention, stream-partitioned: the main tensor-core kernel.
//
// Shaped by two facts measured on the B200: HBM streams at full rate through
// TMA only when each request is large (about 16 KB: one 2 KB box per page and
// kv head, as in decode_tensor.cu, leaves the CTAs' request rate the limit),
// and a decode step is short, so any imbalance between CTAs is paid in full.
//
//  * A CTA covers a group of 8 kv heads at once.  In the pool layout
//    [block][kv head][token][head dim], the 16 tokens x 8 heads of a block are
//    one 16 KB (D=64) region, fetched by a single 3-D tiled TMA box (dims
//    head_dim x block_size x blocks*kv_heads, 128-byte swizzle, no multicast)
//    for K and one for V.  Eight consumer warps each own one kv head; one
//    producer warp feeds a ring of stages (16 tokens each) on mbarriers.
//  * Work is the concatenation, over kv groups and sequences, of 16-token
//    slabs (an empty sequence counts one slab).  The persistent grid (every
//    resident CTA slot) cuts that stream into equal slices, so CTAs differ by
//    at most one slab whatever the length mix.  A CTA walks its slice; each
//    maximal run of one sequence inside it is a segment.  A sequence lying in
//    one CTA is written out directly; one shared by several CTAs leaves one
//    fp32 partial state per CTA (at most two per CTA: the run it starts in and
//    the run it ends in), which the merge kernel (merge.cu) combines.
//  * Per warp and stage: q.K^T for the group's query heads as m16n8k16 bf16
//    MMAs (16 tokens = M, up to 8 heads = N per n-tile), fp32 online softmax
//    in the log2 domain on the accumulator, probabilities rounded to bf16 and
//    transposed in registers (movmatrix) into the B operand of V^T P.
//  * q rows of a segment arrive by a 1-D bulk copy into a two-slot ring.
//  * Every wait is bounded (2 s, then a status bit), so nothing can hang.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <atomic>

#include "pa_device.cuh"
#include "pa_ptx.cuh"

namespace pa {
namespace {

constexpr int kGroup = 8;                    // kv heads per CTA = consumer warps
constexpr int kThreads = (kGroup + 1) * 32;
constexpr int kSlab = 16;                    // tokens per stage (bf16 pools, E4M3 at D=128)
constexpr int kRowBytes = 128;               // 64 bf16 of head dim, one swizzled row
constexpr int kQSlots = 2;

template <int D, int NT, bool F8 = false>
struct SCfg {
    static constexpr int kHalves = D / 64;
    // tokens per stage: E4M3 stages at D=64 hold 32 (the 16 KB of a bf16 stage), so that the
    // per-stage waits, votes and releases are spread over twice the tokens
    static constexpr int kSlab = (F8 && D == 64) ? 32 : ::pa::kSlab;
    static constexpr int kMT = kSlab / 16;                           // 16-token M tiles per stage
    static constexpr int kHalfBytes = kGroup * kSlab * kRowBytes;   // 16 KB
    static constexpr int kTileBytes = kHalves * kHalfBytes;         // bf16 K (or V) of a stage
    // as loaded: bf16 in 128-byte swizzled rows (one box per 64 dims), or E4M3 in plain D-byte rows
    static constexpr int kLoadBoxes = F8 ? 1 : kHalves;
    static constexpr int kLoadRowBytes = F8 ? D : kRowBytes;
    static constexpr int kTileBytesIn = F8 ? kGroup * kSlab * D : kTileBytes;
    static constexpr int kStageBytes = 2 * kTileBytesIn;
    // E4M3 stages carry half the bytes: more of them keep as many bytes in flight, except at
    // D=128, G<=8, where two CTAs of two stages per SM beat one of five (a CTA retires TMA
    // requests at a bounded rate, so more CTAs issue more of them)
    static constexpr int kStages = F8 ? (D == 64 ? (NT == 1 ? 3 : 2) : (NT == 1 ? 2 : 4))
                                      : ((D == 128 && NT == 2) ? 2 : 3);
    static constexpr int kKSteps = D / 16;
    static constexpr int kMTiles = D / 16;
    static constexpr int kMinBlocks = ((D == 64 && NT == 1) || (F8 && D == 128 && NT == 1)) ? 2 : 1;
    // dynamic shared memory for query group size g
    static constexpr size_t smem_bytes(int g) {
        return (size_t)kStages * kStageBytes + (size_t)kQSlots * kGroup * g * D * 2 + 1024;
    }
};

// kNew: the segment that starts at this stage holds the sequence's newest token (fused append)
enum : int32_t { kFirst = 1, kLast = 2, kEmpty = 4, kEnd = 8, kNew = 16 };

// Lazy running max: a slab rescales O only when a score passes the running max by more than
// this (log2 domain); probabilities up to 2^8 keep bf16 / f16 P and the fp32 sums exact in
// relative terms.
constexpr float kLazyLog2 = 8.f;

// Slabs an early-launched CTA prefetches into L2 before it waits for the previous kernel.
constexpr int32_t kPrefetchSlabs = 2;

struct Hdr {
    int32_t b, kvh0, t0, valid;   // sequence, first kv head of the group, stage tokens [t0, t0+valid)
    int32_t flags, qslot;         // kFirst / kLast / kEmpty / kEnd / kNew; q ring slot of the segment
    int32_t nsplit, slot;         // CTAs sharing the sequence; this CTA's partial slot (0/1)
    int32_t i_first, first_slot;  // first CTA of the sequence and the slot it used
    int32_t rope_pos;             // position of the sequence's newest token (L-1)
    int32_t new_blk;              // fused append, on the stage holding that token: its physical
                                  // block (-1: none, or an id outside the pool)
};

// Row of (kv head hl, token t) inside a stage half-tile filled by boxes of tb tokens x 8 heads.
__device__ __forceinline__ int stage_row(int hl, int t, int tb) {
    return (t / tb) * (kGroup * tb) + hl * tb + (t % tb);
}

__device__ __forceinline__ uint32_t swz(uint32_t half_tile, int row, int chunk) {
    return half_tile + row * kRowBytes + (((chunk & 7) ^ (row & 7)) << 4);
}

template <int SL>
__device__ __forceinline__ int32_t nslabs(const DecodeParams& p, int32_t b) {
    const int32_t L = clipped_length(p, b);
    return L == 0 ? 1 : (L + SL - 1) / SL;
}

// CTA whose slice holds slab s (slices: [floor(i S / G), floor((i+1) S / G)) ).
__device__ __forceinline__ int32_t cta_of(int64_t s, int64_t S, int64_t G) {
    return (int32_t)(((s + 1) * G - 1) / S);
}

// Four E4M3 codes -> two f16 pairs (exact: every E4M3 value is an f16 value): codes 0,1 (low
// half-word) and codes 2,3 (high half-word), one conversion per half-word register.
__device__ __forceinline__ void e4m3x4_to_f16x2x2(uint32_t codes, uint32_t& lo, uint32_t& hi) {
    asm("{ .reg .b16 l, h; mov.b32 {l, h}, %2; cvt.rn.f16x2.e4m3x2 %0, l; cvt.rn.f16x2.e4m3x2 %1, h; }"
        : "=r"(lo), "=r"(hi)
        : "r"(codes));
}
// Byte offset of (row, 16-byte chunk) in an E4M3 tile as TMA writes it: 64-byte rows (D=64)
// under the 64B swizzle (chunk ^= (row >> 1) & 3), 128-byte rows (D=128) under the 128B one.
template <int D>
__device__ __forceinline__ uint32_t f8_off(int row, int chunk) {
    if constexpr (D == 64) return (uint32_t)(row * 64 + ((chunk ^ ((row >> 1) & 3)) << 4));
    else return (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4));
}
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}
// bf16 pair -> f16 pair (the E4M3 path multiplies in f16; exact for |x| in [2^-14, 65504])
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t w) { return pack_f16x2(bf16_lo(w), bf16_hi(w)); }
// MMA on the stage's element type: bf16 pools multiply bf16, E4M3 pools f16
template <bool F8>
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    if constexpr (F8) mma_f16_16816(d, a, b0, b1); else mma_bf16_16816(d, a, b0, b1);
}
template <bool F8>
__device__ __forceinline__ uint32_t pack_p(float lo, float hi) {
    if constexpr (F8) return pack_f16x2(lo, hi); else return pack_bf16x2(lo, hi);
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}
// Two floats -> two E4M3 codes (nearest even, saturating), the first in the low byte.
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

template <int D, int NT, bool F8>
__global__ void __launch_bounds__(kThreads, SCfg<D, NT, F8>::kMinBlocks)
    decode_stream_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap kmap,
                         const __grid_constant__ CUtensorMap vmap) {
    using C = SCfg<D, NT, F8>;
    extern __shared__ uint8_t smem_raw[];
    __shared__ Hdr s_hdr[C::kStages];
    __shared__ __align__(8) uint64_t full_bar[C::kStages];
    __shared__ __align__(8) uint64_t empty_bar[C::kStages];
    __shared__ __align__(8) uint64_t qfull_bar[kQSlots];
    __shared__ __align__(8) uint64_t qempty_bar[kQSlots];
    __shared__ double s_rope_inv[64];   // RoPE inverse frequencies of the D/2 pairs

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int32_t G = p.group;
    const int32_t Hkv = p.num_kv_heads;
    const uint32_t smem_base = (smem_u32(smem_raw) + 1023u) & ~1023u;
    uint8_t* smem_gen = smem_raw + (smem_base - smem_u32(smem_raw));
    const uint32_t q_base = smem_base + C::kStages * C::kStageBytes;   // q ring after the stages
    const uint32_t q_slot_bytes = (uint32_t)(kGroup * G * D * 2);
    allow_dependents();
    if (threadIdx.x == kGroup * 32) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&kmap)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&vmap)) : "memory");
    }

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(smem_u32(&full_bar[s]), 1);
            mbar_init(smem_u32(&empty_bar[s]), kGroup);
        }
        for (int s = 0; s < kQSlots; ++s) {
            mbar_init(smem_u32(&qfull_bar[s]), 1);
            mbar_init(smem_u32(&qempty_bar[s]), kGroup);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (p.rope_theta > 0.f)
        for (int i = threadIdx.x; i < D / 2; i += blockDim.x) s_rope_inv[i] = rope_inv_freq(i, D, p.rope_theta);
    __syncthreads();

    if (warp == kGroup && p.selftest_stall && blockIdx.x == 0) {
        // failure-handling self-test: this CTA's producer issues no copy and signals nothing,
        // so its consumers' first waits run out with no copy in flight
    } else if (warp == kGroup) {
        // ================================ producer ================================
        const int32_t B = p.num_seqs, Bs = p.block_size;
        constexpr int32_t SL = C::kSlab;
        const int32_t tb = Bs < SL ? Bs : SL;                   // tokens per TMA box
        const int32_t groups = Hkv / kGroup;
        const int32_t zmax = p.num_blocks * Hkv;                // z extent of the maps
        const uint64_t kv_policy = l2_evict_first_policy();      // K/V are read once
        // slabs per group of kv heads: S_seq = sum_b nslabs(b)
        // slabs per group of kv heads, S_seq = sum_b nslabs(b): lane i sums the contiguous
        // chunk of sequences [i cs, (i+1) cs) (independent loads), then one warp scan
        const int32_t cs = (B + 31) / 32;
        const int32_t c_lo = min(B, lane * cs), c_hi = min(B, c_lo + cs);
        int64_t lane_sum = 0;
#pragma unroll 4
        for (int32_t b = c_lo; b < c_hi; ++b) lane_sum += nslabs<SL>(p, b);
        int64_t incl = lane_sum;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int64_t v = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += v;
        }
        const int64_t S_seq = __shfl_sync(0xffffffffu, incl, 31);
        const int64_t S = S_seq * groups;
        // slices: CTA i < Gc takes slabs [i S / Gc, (i+1) S / Gc); never more slices than slabs,
        // so that every slice a sequence spans holds at least one of its slabs
        const int64_t Gc = S < (int64_t)gridDim.x ? S : (int64_t)gridDim.x, ci = blockIdx.x;
        const int64_t lo = ci < Gc ? ci * S / Gc : S, hi = ci < Gc ? (ci + 1) * S / Gc : S;
        uint32_t gtile = 0, qk = 0;
        bool alive = true;
        auto acquire = [&](uint64_t* bars, uint32_t k, uint32_t n, int& slot) -> bool {
            slot = (int)(k % n);
            if (k >= n) {
                bool ok = true;
                if (lane == 0) ok = mbar_wait(smem_u32(&bars[slot]), ((k / n) - 1) & 1, p.status, p.wait_ns);
                return __shfl_sync(0xffffffffu, ok, 0);
            }
            return true;
        };
        if (lo < hi) {
            // locate slab lo: kv group gi, sequence b, slab j of b; P = stream index of b's slab 0.
            // The lane whose chunk holds it walks its chunk (values still in L1).
            int32_t gi = (int32_t)(lo / S_seq);
            const int64_t r = lo - (int64_t)gi * S_seq;
            const int64_t excl = incl - lane_sum;
            const unsigned hit = __ballot_sync(0xffffffffu, r >= excl && r < incl);
            const int k = __ffs(hit) - 1;
            int32_t b = 0, j = 0;
            int64_t P = 0;
            if (lane == k) {
                int64_t acc = excl;
                for (int32_t bb = c_lo; bb < c_hi; ++bb) {
                    const int32_t n = nslabs<SL>(p, bb);
                    if (r < acc + n) {
                        b = bb;
                        j = (int32_t)(r - acc);
                        P = (int64_t)gi * S_seq + acc;
                        break;
                    }
                    acc += n;
                }
            }
            b = __shfl_sync(0xffffffffu, b, k);
            j = __shfl_sync(0xffffffffu, j, k);
            P = __shfl_sync(0xffffffffu, P, k);
            int32_t L = clipped_length(p, b);
            int32_t nb = L == 0 ? 1 : (L + SL - 1) / SL;
            // segment state
            int32_t seg_nsplit = 1, seg_slot = 0, seg_ifirst = 0, seg_fslot = 0, seg_q = 0;
            const int32_t* table = p.block_tables + (size_t)b * p.max_blocks_per_seq;
            // the first table window, fetched while a prerequisite grid may still run
            int32_t win_base = (j * SL) / Bs, win_entry = -1;
            if (win_base + lane < p.max_blocks_per_seq) win_entry = __ldg(table + win_base + lane);
            // Loads issued ahead so that no copy waits on one: the window after the current one
            // (nx_win2), and, once a slice reaches the next sequence of the stream, that
            // sequence's length and first window (nx_len, nx_win)
            int32_t nx_len = 0, nx_win = -1, nx_win2 = -1;
            bool have_win2 = false;
            auto prefetch_win2 = [&]() {
                have_win2 = (int64_t)(win_base + 32) * Bs < L;      // the sequence goes past it
                const int32_t idx = win_base + 32 + lane;
                if (have_win2) nx_win2 = idx < p.max_blocks_per_seq ? __ldg(table + idx) : -1;
            };
            auto refill = [&](int32_t lbk) {                         // warp-uniform
                if (have_win2 && lbk == win_base + 32) {
                    win_entry = nx_win2;
                } else {
                    const int32_t idx = lbk + lane;
                    win_entry = idx < p.max_blocks_per_seq ? __ldg(table + idx) : -1;
                }
                win_base = lbk;
                prefetch_win2();
            };
            prefetch_win2();
            int q_next = -1;                                 // q ring slot already requested
            auto issue_q = [&](int32_t bq, int32_t gq, int& slot) -> bool {
                if (!acquire(qempty_bar, qk, kQSlots, slot)) return false;
                if (lane == 0) {
                    const uint32_t bar = smem_u32(&qfull_bar[slot]);
                    mbar_arrive_expect_tx(bar, q_slot_bytes);
                    bulk_load(q_base + slot * q_slot_bytes,
                              p.q + ((size_t)bq * p.num_q_heads + (size_t)gq * kGroup * G) * D, q_slot_bytes, bar);
                }
                ++qk;
                return true;
            };
            if (p.early) {
                // launched early: pull the first slabs of the slice (inside the first sequence
                // and the fetched table window) into L2 while the previous kernel finishes
                const int32_t pf_end = min(min((int64_t)nb, (int64_t)j + (hi - lo)), (int64_t)j + kPrefetchSlabs);
                for (int32_t jj = j; jj < pf_end && L > 0; ++jj) {
                    const int32_t t0 = jj * SL, valid = min(SL, L - t0);
                    for (int32_t x = 0; x * tb < valid; ++x) {
                        const int32_t tok = t0 + x * tb, lbk = tok / Bs;
                        if (lbk - win_base >= 32) break;
                        const int32_t blk = __shfl_sync(0xffffffffu, win_entry, lbk - win_base);
                        if (lane == 0 && blk >= 0 && blk < p.num_blocks) {
#pragma unroll
                            for (int h = 0; h < C::kLoadBoxes; ++h) {
                                tma_prefetch_3d(&kmap, h * 64, tok - lbk * Bs, blk * Hkv + gi * kGroup);
                                tma_prefetch_3d(&vmap, h * 64, tok - lbk * Bs, blk * Hkv + gi * kGroup);
                            }
                        }
                    }
                }
            }
            // everything below reads or writes what the previous kernel on the stream may touch
            wait_prerequisite();
            for (int64_t s = lo; s < hi && alive; ++s) {
                const bool first = (s == lo) || (j == 0);
                const bool last = (s == hi - 1) || (j == nb - 1);
                bool seg_new = false;
                if (first) {
                    const int32_t i_first = cta_of(P, S, Gc), i_last = cta_of(P + nb - 1, S, Gc);
                    seg_nsplit = i_last - i_first + 1;
                    seg_slot = P < lo ? 0 : 1;
                    seg_ifirst = i_first;
                    seg_fslot = P < (int64_t)i_first * S / Gc ? 0 : 1;
                    if (P >= lo && lane == 0)   // this CTA holds the sequence's first slab
                        reinterpret_cast<int4*>(p.seq_desc)[(size_t)gi * B + b] =
                            make_int4(seg_nsplit, i_first, seg_fslot, 0);
                    if (s != lo) {                   // a new sequence: its window is in hand
                        table = p.block_tables + (size_t)b * p.max_blocks_per_seq;
                        win_base = 0;
                        win_entry = nx_win;
                        prefetch_win2();
                    }
                    if (s + (nb - j) < hi) {         // the slice reaches the next sequence
                        const int32_t bn = b + 1 == B ? 0 : b + 1;
                        nx_len = __ldg(p.context_lens + bn);
                        nx_win = lane < p.max_blocks_per_seq
                                     ? __ldg(p.block_tables + (size_t)bn * p.max_blocks_per_seq + lane)
                                     : -1;
                    }
                    // fused append: this segment holds the sequence's newest token
                    seg_new = p.k_new != nullptr && L > 0 && s + (nb - 1 - j) < hi;
                    // q of every segment (empty sequences' too): requested at the previous
                    // sequence's start when the slice ran on into this one, else now; then the
                    // next sequence's q, if the slice reaches it
                    if (q_next >= 0) {
                        seg_q = q_next;
                        q_next = -1;
                    } else if (!issue_q(b, gi, seg_q)) {
                        alive = false;
                        break;
                    }
                    if (s + (nb - j) < hi) {
                        const bool wrap = b + 1 == B;
                        if (!issue_q(wrap ? 0 : b + 1, wrap ? gi + 1 : gi, q_next)) {
                            alive = false;
                            break;
                        }
                    }
                }
                int st;
                if (!acquire(empty_bar, gtile, C::kStages, st)) { alive = false; break; }
                const int32_t t0 = j * SL;
                const int32_t valid = L == 0 ? 0 : min(SL, L - t0);
                const uint32_t fbar = smem_u32(&full_bar[st]);
                // fused append: the stage that holds the newest token (position L-1) carries its
                // physical block; the consumer warps write the new K/V rows to the pool and into
                // the staged tile, so no copy waits on those writes
                int32_t new_blk = -1;
                if (valid > 0 && p.k_new != nullptr && j == nb - 1) {
                    const int32_t lbn = (L - 1) / Bs, lb0 = t0 / Bs;
                    if (win_base < 0 || lbn >= win_base + 32) refill(lb0);
                    const int32_t blk = __shfl_sync(0xffffffffu, win_entry, lbn - win_base);
                    new_blk = blk >= 0 && blk < p.num_blocks ? blk : -1;
                }
                if (lane == 0) {
                    s_hdr[st] = Hdr{b, gi * kGroup, t0, valid,
                                    (first ? kFirst : 0) | (last ? kLast : 0) | (L == 0 ? kEmpty : 0) |
                                        (seg_new ? kNew : 0),
                                    seg_q, seg_nsplit, seg_slot, seg_ifirst, seg_fslot, L - 1, new_blk};
                }
                if (valid > 0) {
                    const int32_t nbox = (valid + tb - 1) / tb;
                    if (lane == 0)
                        mbar_arrive_expect_tx(fbar, (uint32_t)(nbox * kGroup * tb * C::kLoadRowBytes * C::kLoadBoxes * 2));
                    const uint32_t k_tile = smem_base + st * C::kStageBytes;
                    const uint32_t v_tile = k_tile + C::kTileBytesIn;
                    for (int32_t x = 0; x < nbox; ++x) {
                        const int32_t tok = t0 + x * tb;
                        const int32_t lbk = tok / Bs;
                        if (win_base < 0 || lbk >= win_base + 32) refill(lbk);
                        const int32_t blk = __shfl_sync(0xffffffffu, win_entry, lbk - win_base);
                        if (lane == 0) {
                            int32_t z;
                            if (blk < 0 || blk >= p.num_blocks) {
                                raise_status(p.status, kStatusBadBlock);
                                z = zmax;                                // outside the map: zeros
                            } else {
                                z = blk * Hkv + gi * kGroup;
                            }
                            const int32_t y = tok - lbk * Bs;
                            const uint32_t off = (uint32_t)(x * kGroup * tb * C::kLoadRowBytes);
#pragma unroll
                            for (int h = 0; h < C::kLoadBoxes; ++h) {
                                tma_load_3d_hint(k_tile + h * C::kHalfBytes + off, &kmap, h * 64, y, z, fbar, kv_policy);
                                tma_load_3d_hint(v_tile + h * C::kHalfBytes + off, &vmap, h * 64, y, z, fbar, kv_policy);
                            }
                        }
                    }
                } else if (lane == 0) {
                    mbar_arrive(fbar);
                }
                ++gtile;
                // advance to the next slab of the stream
                if (++j == nb) {
                    j = 0;
                    P += nb;
                    if (++b == B) {
                        b = 0;
                        ++gi;
                    }
                    if (s + 1 < hi) {
                        L = clip_length(p, nx_len);
                        nb = L == 0 ? 1 : (L + SL - 1) / SL;
                    }
                }
            }
        }
        int st;
        if (acquire(empty_bar, gtile, C::kStages, st) && lane == 0) {
            s_hdr[st].flags = kEnd;
            mbar_arrive(smem_u32(&full_bar[st]));
        }
    } else {
        // ================================ consumers ===============================
        wait_prerequisite();   // they write out / partials: not before the previous kernel ends
        // warp w owns kv head kvh0 + w of every stage
        const int r = lane >> 2, c = lane & 3;
        const int mi = lane >> 3, rr = lane & 7;
        constexpr int32_t SL = C::kSlab;
        const int32_t tb = p.block_size < SL ? p.block_size : SL;
        const float sl2 = p.scale_log2;
        uint32_t qf[NT][C::kKSteps][2];
        float m_run[NT][2], l_run[NT][2];
        float o_acc[NT][C::kMTiles][4];
        uint32_t qk = 0;
        // fused append: this warp's kv head's new K and V rows, lane i < D/4 holding dims
        // 2i, 2i+1 and D/2 + 2i, D/2 + 2i + 1 (the RoPE pairs of those dims), read when the
        // segment starts and written when the stage holding the token arrives
        uint32_t nk[2] = {0u, 0u}, nv[2] = {0u, 0u};
        // rows of this warp's 16 tokens: lane-provided ldmatrix row addresses
        // per 16-token M tile u of a stage: K rows of tokens 16u + rr (+8), V rows likewise
        int row_a[C::kMT], row_b[C::kMT];
#pragma unroll
        for (int u = 0; u < C::kMT; ++u) {
            row_a[u] = stage_row(warp, 16 * u + rr + ((mi & 1) << 3), tb);
            row_b[u] = stage_row(warp, 16 * u + rr + ((mi >> 1) << 3), tb);
        }
        for (uint32_t gtile = 0;; ++gtile) {
            const int st = gtile % C::kStages;
            if (!warp_wait(smem_u32(&full_bar[st]), (gtile / C::kStages) & 1, p.status, p.wait_ns)) break;
            const Hdr hd = s_hdr[st];
            if (hd.flags & kEnd) break;
            const int32_t kvh = hd.kvh0 + warp;
            if (hd.flags & kEmpty) {
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&empty_bar[st]));
                if (hd.flags & kFirst) {                     // its q slot, unread
                    const int qs = qk % kQSlots;
                    if (!warp_wait(smem_u32(&qfull_bar[qs]), (qk / kQSlots) & 1, p.status, p.wait_ns)) break;
                    __syncwarp();
                    if (lane == 0) mbar_arrive(smem_u32(&qempty_bar[qs]));
                    ++qk;
                }
                store_zero_group(p, hd.b, kvh, lane, 32);
                continue;
            }
            if (hd.flags & kFirst) {
                const int qs = qk % kQSlots;
                if (!warp_wait(smem_u32(&qfull_bar[qs]), (qk / kQSlots) & 1, p.status, p.wait_ns)) break;
                uint16_t* qsm = reinterpret_cast<uint16_t*>(
                    smem_gen + (q_base - smem_base) + qs * (size_t)(kGroup * G * D * 2)) + (size_t)warp * G * D;
                if (p.rope_theta > 0.f) {
                    // RoPE: turn this warp's G query rows at the newest token's position, in place
                    for (int i = lane; i < D / 2; i += 32) {
                        float cs, sn;
                        rope_cos_sin(hd.rope_pos, s_rope_inv[i], &cs, &sn);
                        for (int h = 0; h < G; ++h) {
                            const float x1 = __uint_as_float((uint32_t)qsm[h * D + i] << 16);
                            const float x2 = __uint_as_float((uint32_t)qsm[h * D + i + D / 2] << 16);
                            qsm[h * D + i] = f32_to_bf16_rn(x1 * cs - x2 * sn);
                            qsm[h * D + i + D / 2] = f32_to_bf16_rn(x1 * sn + x2 * cs);
                        }
                    }
                    // generic writes to a slot the bulk copy refills later: order them first
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    __syncwarp();
                }
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const int h = nt * 8 + r;
#pragma unroll
                    for (int ks = 0; ks < C::kKSteps; ++ks) {
                        const uint32_t* qr = reinterpret_cast<const uint32_t*>(qsm + h * D + ks * 16);
                        if constexpr (F8) {
                            // E4M3: the k-step's dims in the order the K fragments bring them
                            // (lane column c holds dims 4c..4c+3 of the 16-dim chunk)
                            qf[nt][ks][0] = h < G ? bf16x2_to_f16x2(qr[2 * c]) : 0u;
                            qf[nt][ks][1] = h < G ? bf16x2_to_f16x2(qr[2 * c + 1]) : 0u;
                        } else {
                            qf[nt][ks][0] = h < G ? qr[c] : 0u;
                            qf[nt][ks][1] = h < G ? qr[c + 4] : 0u;
                        }
                    }
                    m_run[nt][0] = m_run[nt][1] = -INFINITY;
                    l_run[nt][0] = l_run[nt][1] = 0.f;
#pragma unroll
                    for (int mt = 0; mt < C::kMTiles; ++mt)
#pragma unroll
                        for (int e = 0; e < 4; ++e) o_acc[nt][mt][e] = 0.f;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&qempty_bar[qs]));
                ++qk;
                if (hd.flags & kNew) {
                    const int i = lane < D / 4 ? lane : 0;
                    const size_t row = ((size_t)hd.b * Hkv + kvh) * D / 2;
                    const uint32_t* kn = reinterpret_cast<const uint32_t*>(p.k_new) + row;
                    const uint32_t* vn = reinterpret_cast<const uint32_t*>(p.v_new) + row;
                    nk[0] = __ldg(kn + i);
                    nk[1] = __ldg(kn + D / 4 + i);
                    nv[0] = __ldg(vn + i);
                    nv[1] = __ldg(vn + D / 4 + i);
                }
            }
            const int valid = hd.valid;
            uint32_t k_tile = smem_base + st * C::kStageBytes;
            uint32_t v_tile = k_tile + C::kTileBytes;
            if (hd.new_blk >= 0 && hd.rope_pos >= hd.t0 && hd.rope_pos < hd.t0 + valid) {
                // fused append: the stage holds the sequence's newest token.  Its K (turned by
                // RoPE at that position when the call asks for it) and V rows go to the pool and
                // over the staged copy, which may predate them.
                if (lane < D / 4) {
                    const int32_t pos = hd.rope_pos, Bs = p.block_size, t = pos - hd.t0;
                    const int row = stage_row(warp, t, tb);
                    const size_t grow = ((size_t)hd.new_blk * Hkv + kvh) * Bs + (pos - (pos / Bs) * Bs);
                    uint32_t ka = nk[0], kb = nk[1];
                    if (p.rope_theta > 0.f) {
                        float c0, s0, c1, s1;
                        rope_cos_sin(pos, s_rope_inv[2 * lane], &c0, &s0);
                        rope_cos_sin(pos, s_rope_inv[2 * lane + 1], &c1, &s1);
                        const float a0 = bf16_lo(ka), a1 = bf16_hi(ka), b0 = bf16_lo(kb), b1 = bf16_hi(kb);
                        ka = pack_bf16x2(a0 * c0 - b0 * s0, a1 * c1 - b1 * s1);
                        kb = pack_bf16x2(a0 * s0 + b0 * c0, a1 * s1 + b1 * c1);
                    }
                    const int d0 = 2 * lane, d1 = D / 2 + 2 * lane;
                    if constexpr (F8) {
                        const float ks = p.k_inv_scale, vs = p.v_inv_scale;
                        const uint32_t q0 = f32x2_to_e4m3x2(__fmul_rn(bf16_lo(ka), ks), __fmul_rn(bf16_hi(ka), ks));
                        const uint32_t q1 = f32x2_to_e4m3x2(__fmul_rn(bf16_lo(kb), ks), __fmul_rn(bf16_hi(kb), ks));
                        const uint32_t w0 = f32x2_to_e4m3x2(__fmul_rn(bf16_lo(nv[0]), vs), __fmul_rn(bf16_hi(nv[0]), vs));
                        const uint32_t w1 = f32x2_to_e4m3x2(__fmul_rn(bf16_lo(nv[1]), vs), __fmul_rn(bf16_hi(nv[1]), vs));
                        // the caches are the caller's writable buffers (pa_append_decode)
                        uint8_t* kq = reinterpret_cast<uint8_t*>(const_cast<uint16_t*>(p.k_cache)) + grow * D;
                        uint8_t* vq = reinterpret_cast<uint8_t*>(const_cast<uint16_t*>(p.v_cache)) + grow * D;
                        *reinterpret_cast<uint16_t*>(kq + d0) = (uint16_t)q0;
                        *reinterpret_cast<uint16_t*>(kq + d1) = (uint16_t)q1;
                        *reinterpret_cast<uint16_t*>(vq + d0) = (uint16_t)w0;
                        *reinterpret_cast<uint16_t*>(vq + d1) = (uint16_t)w1;
                        uint8_t* kt = smem_gen + (k_tile - smem_base);
                        uint8_t* vt = smem_gen + (k_tile + C::kTileBytesIn - smem_base);
                        *reinterpret_cast<uint16_t*>(kt + f8_off<D>(row, d0 / 16) + d0 % 16) = (uint16_t)q0;
                        *reinterpret_cast<uint16_t*>(kt + f8_off<D>(row, d1 / 16) + d1 % 16) = (uint16_t)q1;
                        *reinterpret_cast<uint16_t*>(vt + f8_off<D>(row, d0 / 16) + d0 % 16) = (uint16_t)w0;
                        *reinterpret_cast<uint16_t*>(vt + f8_off<D>(row, d1 / 16) + d1 % 16) = (uint16_t)w1;
                    } else {
                        uint32_t* kc = reinterpret_cast<uint32_t*>(const_cast<uint16_t*>(p.k_cache)) + grow * D / 2;
                        uint32_t* vc = reinterpret_cast<uint32_t*>(const_cast<uint16_t*>(p.v_cache)) + grow * D / 2;
                        kc[lane] = ka;
                        kc[D / 4 + lane] = kb;
                        vc[lane] = nv[0];
                        vc[D / 4 + lane] = nv[1];
                        auto at = [&](uint32_t tile, int d) {   // byte address of dim d in the row
                            const int ch = d / 8;
                            return swz(tile + (ch >> 3) * C::kHalfBytes, row, ch) + (uint32_t)((d % 8) * 2);
                        };
                        asm volatile("st.shared.b32 [%0], %1;" ::"r"(at(k_tile, d0)), "r"(ka) : "memory");
                        asm volatile("st.shared.b32 [%0], %1;" ::"r"(at(k_tile, d1)), "r"(kb) : "memory");
                        asm volatile("st.shared.b32 [%0], %1;" ::"r"(at(v_tile, d0)), "r"(nv[0]) : "memory");
                        asm volatile("st.shared.b32 [%0], %1;" ::"r"(at(v_tile, d1)), "r"(nv[1]) : "memory");
                    }
                }
                // generic writes to a stage the copy engine refills later: order them first
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncwarp();
            }
            if constexpr (F8) {
                if (valid < SL) {
                    // tokens past the sequence: zero their V bytes (0-probability rows add nothing)
                    const uint32_t f8v = k_tile + C::kTileBytesIn;
                    for (int i = lane; i < (SL - valid) * (D / 16); i += 32) {
                        const int t = valid + i / (D / 16), ch = i % (D / 16);
                        *reinterpret_cast<uint4*>(smem_gen + (f8v - smem_base) + f8_off<D>(stage_row(warp, t, tb), ch)) =
                            make_uint4(0, 0, 0, 0);
                    }
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    __syncwarp();
                }
            } else if (valid < SL) {
                // tokens past the sequence: zero V so that 0-probability rows add nothing
                for (int i = lane; i < (SL - valid) * 8 * C::kHalves; i += 32) {
                    const int t = valid + i / (8 * C::kHalves);
                    const int ch = i % (8 * C::kHalves);
                    const int row = stage_row(warp, t, tb);
                    *reinterpret_cast<uint4*>(smem_gen + (v_tile - smem_base) + (ch >> 3) * C::kHalfBytes +
                                              row * kRowBytes + (((ch & 7) ^ (row & 7)) << 4)) =
                        make_uint4(0, 0, 0, 0);
                }
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncwarp();
            }
            // ---- S = K q^T : 16 tokens x 8 heads per (M tile, n-tile) ----
            float sacc[C::kMT][NT][4];
#pragma unroll
            for (int u = 0; u < C::kMT; ++u) {
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) sacc[u][nt][e] = 0.f;
                if constexpr (F8) {
                    // E4M3 K straight from the tile: one ldmatrix.x4 brings 16 tokens x 32 dims of
                    // codes (lane (r, c): 4 codes, dims 4c..4c+3 of a chunk), widened to f16 pairs
    #pragma unroll
                    for (int ks = 0; ks < C::kKSteps; ks += 2) {
                        uint32_t w[4];
                        ldmatrix_x4(k_tile + f8_off<D>(row_a[u], ks + (mi >> 1)), w);
    #pragma unroll
                        for (int h2 = 0; h2 < 2; ++h2) {
                            uint32_t a[4];
                            e4m3x4_to_f16x2x2(w[2 * h2], a[0], a[2]);
                            e4m3x4_to_f16x2x2(w[2 * h2 + 1], a[1], a[3]);
    #pragma unroll
                            for (int nt = 0; nt < NT; ++nt)
                                mma_16816<F8>(sacc[u][nt], a, qf[nt][ks + h2][0], qf[nt][ks + h2][1]);
                        }
                    }
                } else {
    #pragma unroll
                    for (int ks = 0; ks < C::kKSteps; ++ks) {
                        const int ch = 2 * ks + (mi >> 1);
                        uint32_t a[4];
                        ldmatrix_x4(swz(k_tile + (ch >> 3) * C::kHalfBytes, row_a[u], ch), a);
    #pragma unroll
                        for (int nt = 0; nt < NT; ++nt) mma_16816<F8>(sacc[u][nt], a, qf[nt][ks][0], qf[nt][ks][1]);
                    }
                }
            }
            // ---- online softmax over the 16 rows (tokens) per head column ----
            // The running max m is kept lazily: while every score of the slab stays within
            // 2^kLazyLog2 of its head's m (log2 domain), the slab is weighted by 2^(s - m) as m
            // stands, with no cross-lane maximum and no rescale of O.  Otherwise (always on a
            // segment's first slab, where m = -inf) m moves to the maximum over the slab.
            float sv[C::kMT][NT][4], mx[NT][2];
            bool need = false;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) mx[nt][0] = mx[nt][1] = -INFINITY;
#pragma unroll
            for (int u = 0; u < C::kMT; ++u) {
                const bool v_lo = 16 * u + r < valid, v_hi = 16 * u + r + 8 < valid;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    sv[u][nt][0] = v_lo ? sacc[u][nt][0] * sl2 : -INFINITY;
                    sv[u][nt][1] = v_lo ? sacc[u][nt][1] * sl2 : -INFINITY;
                    sv[u][nt][2] = v_hi ? sacc[u][nt][2] * sl2 : -INFINITY;
                    sv[u][nt][3] = v_hi ? sacc[u][nt][3] * sl2 : -INFINITY;
                    mx[nt][0] = fmax3(mx[nt][0], sv[u][nt][0], sv[u][nt][2]);
                    mx[nt][1] = fmax3(mx[nt][1], sv[u][nt][1], sv[u][nt][3]);
                }
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
                need |= mx[nt][0] > m_run[nt][0] + kLazyLog2 || mx[nt][1] > m_run[nt][1] + kLazyLog2;
            if (__any_sync(0xffffffffu, need)) {
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    float mx0 = mx[nt][0], mx1 = mx[nt][1];
#pragma unroll
                    for (int off = 4; off < 32; off <<= 1) {
                        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
                        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
                    }
                    const float mn0 = fmaxf(m_run[nt][0], mx0), mn1 = fmaxf(m_run[nt][1], mx1);
                    const float al0 = fast_exp2(m_run[nt][0] - mn0), al1 = fast_exp2(m_run[nt][1] - mn1);
                    m_run[nt][0] = mn0;
                    m_run[nt][1] = mn1;
                    l_run[nt][0] *= al0;
                    l_run[nt][1] *= al1;
#pragma unroll
                    for (int mt = 0; mt < C::kMTiles; ++mt) {
                        o_acc[nt][mt][0] *= al0;
                        o_acc[nt][mt][1] *= al1;
                        o_acc[nt][mt][2] *= al0;
                        o_acc[nt][mt][3] *= al1;
                    }
                }
            }
            uint32_t pb[C::kMT][NT][2];
#pragma unroll
            for (int u = 0; u < C::kMT; ++u)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const float p0 = fast_exp2(sv[u][nt][0] - m_run[nt][0]), p1 = fast_exp2(sv[u][nt][1] - m_run[nt][1]);
                    const float p2 = fast_exp2(sv[u][nt][2] - m_run[nt][0]), p3 = fast_exp2(sv[u][nt][3] - m_run[nt][1]);
                    l_run[nt][0] += p0 + p2;
                    l_run[nt][1] += p1 + p3;
                    pb[u][nt][0] = movmatrix_trans(pack_p<F8>(p0, p1));   // tokens 16u + 0-7
                    pb[u][nt][1] = movmatrix_trans(pack_p<F8>(p2, p3));   // tokens 16u + 8-15
                }
            // ---- O^T += V^T P : 16 head-dim rows x 8 heads per (m-tile, n-tile), 16 tokens per
            // k step (one per M tile of the stage) ----
#pragma unroll
            for (int u = 0; u < C::kMT; ++u) {
                if constexpr (F8) {
                    // E4M3 V: ldmatrix.trans over byte pairs gives lane (r, c) tokens 2c, 2c+1 of dims
                    // 2r, 2r+1; byte permutes split even and odd dims into two m-tiles (o_acc[2j]:
                    // dims 32j + 2r (+16), o_acc[2j+1]: dims 32j + 2r + 1 (+16))
                    const uint32_t f8v = k_tile + C::kTileBytesIn;
    #pragma unroll
                    for (int j = 0; j < D / 32; ++j) {
                        uint32_t w[4];
                        ldmatrix_x4_trans(f8v + f8_off<D>(row_b[u], 2 * j + (mi & 1)), w);
                        uint32_t ae[4], ao[4];
    #pragma unroll
                        for (int i = 0; i < 4; ++i)   // bytes 0, 2 (even dims) low, 1, 3 (odd dims) high
                            e4m3x4_to_f16x2x2(__byte_perm(w[i], 0u, 0x3120u), ae[i], ao[i]);
    #pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
                            mma_16816<F8>(o_acc[nt][2 * j], ae, pb[u][nt][0], pb[u][nt][1]);
                            mma_16816<F8>(o_acc[nt][2 * j + 1], ao, pb[u][nt][0], pb[u][nt][1]);
                        }
                    }
                } else {
    #pragma unroll
                    for (int mt = 0; mt < C::kMTiles; ++mt) {
                        const int ch = 2 * mt + (mi & 1);
                        uint32_t a[4];
                        ldmatrix_x4_trans(swz(v_tile + (ch >> 3) * C::kHalfBytes, row_b[u], ch), a);
    #pragma unroll
                        for (int nt = 0; nt < NT; ++nt) mma_16816<F8>(o_acc[nt][mt], a, pb[u][nt][0], pb[u][nt][1]);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&empty_bar[st]));
            if (!(hd.flags & kLast)) continue;

            // ======== end of this warp's segment: store, or publish a partial ========
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int jj = 0; jj < 2; ++jj)
#pragma unroll
                    for (int off = 4; off < 32; off <<= 1)
                        l_run[nt][jj] += __shfl_xor_sync(0xffffffffu, l_run[nt][jj], off);
            const int32_t b = hd.b;
            if (hd.nsplit == 1) {
                uint16_t* out = p.out + ((size_t)b * p.num_q_heads + (size_t)kvh * G) * D;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int jj = 0; jj < 2; ++jj) {
                        const int h = nt * 8 + 2 * c + jj;
                        if (h >= G) continue;
                        const float inv = p.out_scale / l_run[nt][jj];
                        if constexpr (F8) {   // m-tiles 2j / 2j+1 hold dims 32j + 2r / + 1 (and + 16)
#pragma unroll
                            for (int j = 0; j < D / 32; ++j) {
                                uint32_t* o32 = reinterpret_cast<uint32_t*>(out + (size_t)h * D + 32 * j + 2 * r);
                                o32[0] = pack_bf16x2(o_acc[nt][2 * j][jj] * inv, o_acc[nt][2 * j + 1][jj] * inv);
                                o32[8] = pack_bf16x2(o_acc[nt][2 * j][jj + 2] * inv, o_acc[nt][2 * j + 1][jj + 2] * inv);
                            }
                        } else {
#pragma unroll
                            for (int mt = 0; mt < C::kMTiles; ++mt) {
                                out[(size_t)h * D + mt * 16 + r] = f32_to_bf16_rn(o_acc[nt][mt][jj] * inv);
                                out[(size_t)h * D + mt * 16 + r + 8] = f32_to_bf16_rn(o_acc[nt][mt][jj + 2] * inv);
                            }
                        }
                    }
                continue;
            }
            const size_t prow = (((size_t)blockIdx.x * 2 + hd.slot) * Hkv + kvh) * G;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int jj = 0; jj < 2; ++jj) {
                    const int h = nt * 8 + 2 * c + jj;
                    if (h >= G) continue;
                    const float inv = p.out_scale / l_run[nt][jj];
                    float* po = p.part_o + (prow + h) * D;
                    if constexpr (F8) {
#pragma unroll
                        for (int j = 0; j < D / 32; ++j) {
                            float2* p2 = reinterpret_cast<float2*>(po + 32 * j + 2 * r);
                            p2[0] = make_float2(o_acc[nt][2 * j][jj] * inv, o_acc[nt][2 * j + 1][jj] * inv);
                            p2[8] = make_float2(o_acc[nt][2 * j][jj + 2] * inv, o_acc[nt][2 * j + 1][jj + 2] * inv);
                        }
                    } else {
#pragma unroll
                        for (int mt = 0; mt < C::kMTiles; ++mt) {
                            po[mt * 16 + r] = o_acc[nt][mt][jj] * inv;
                            po[mt * 16 + r + 8] = o_acc[nt][mt][jj + 2] * inv;
                        }
                    }
                    if (r == 0) p.part_lse[prow + h] = m_run[nt][jj] + __log2f(l_run[nt][jj]);
                }
        }
    }
    __syncthreads();
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static std::atomic<EncodeTiledFn> fn{nullptr};
    EncodeTiledFn f = fn.load(std::memory_order_acquire);
    if (!f) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess) {
            f = reinterpret_cast<EncodeTiledFn>(ptr);
            fn.store(f, std::memory_order_release);
        }
    }
    return f;
}

// 3-D view [blocks * Hkv][block_size][head_dim]; box = 64 dims x tb tokens x 8 kv heads.
// bf16 pools: boxes of 64 dims in 128-byte swizzled rows; E4M3 pools: whole D-byte rows,
// 64-byte rows (D=64) under the 64B swizzle, 128-byte rows under the 128B one.
}  // namespace

int stream_slab_tokens(bool fp8, int head_dim) { return fp8 && head_dim == 64 ? 32 : kSlab; }

namespace {

bool make_map(CUtensorMap* map, const void* base, const DecodeParams& p) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t esize = p.kv_fp8 ? 1 : 2;
    const cuuint64_t dims[3] = {(cuuint64_t)p.head_dim, (cuuint64_t)p.block_size,
                                (cuuint64_t)p.num_blocks * p.num_kv_heads};
    const cuuint64_t strides[2] = {(cuuint64_t)p.head_dim * esize,
                                   (cuuint64_t)p.block_size * p.head_dim * esize};
    const int slab = stream_slab_tokens(p.kv_fp8, p.head_dim);
    const cuuint32_t box[3] = {p.kv_fp8 ? (cuuint32_t)p.head_dim : 64u,
                               (cuuint32_t)(p.block_size < slab ? p.block_size : slab), (cuuint32_t)kGroup};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUtensorMapSwizzle swz_mode = !p.kv_fp8          ? CU_TENSOR_MAP_SWIZZLE_128B
                                        : p.head_dim == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                           : CU_TENSOR_MAP_SWIZZLE_128B;
    return fn(map, p.kv_fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
              const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz_mode,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int NT, bool F8>
auto kernel_ptr() {
    return decode_stream_kernel<D, NT, F8>;
}

// The dynamic shared-memory opt-in is a per-kernel attribute: set it once per
// device to the instantiation's largest need (its largest query group), then
// size every launch by its own group.
template <int D, int NT, bool F8>
bool ensure_smem_attr() {
    static std::atomic<uint64_t> done{0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
    const uint64_t bit = 1ull << dev;
    if (done.load(std::memory_order_acquire) & bit) return true;
    if (cudaFuncSetAttribute(kernel_ptr<D, NT, F8>(), cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)SCfg<D, NT, F8>::smem_bytes(NT * 8)) != cudaSuccess)
        return false;
    done.fetch_or(bit, std::memory_order_acq_rel);
    return true;
}

// Resident CTAs per SM for this instantiation and query group size (cached per device).
template <int D, int NT, bool F8>
int occupancy(int g) {
    static std::atomic<int> cache[64][17];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64 || g < 1 || g > NT * 8) return 0;
    int occ = cache[dev][g].load(std::memory_order_acquire);
    if (occ > 0) return occ;
    if (!ensure_smem_attr<D, NT, F8>()) return 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel_ptr<D, NT, F8>(), kThreads,
                                                      SCfg<D, NT, F8>::smem_bytes(g)) != cudaSuccess)
        return 0;
    cache[dev][g].store(occ, std::memory_order_release);
    return occ;
}

template <bool F8>
int occupancy_for(int D, int g) {
    const bool two = g > 8;
    if (D == 64) return two ? occupancy<64, 2, F8>(g) : occupancy<64, 1, F8>(g);
    if (D == 128) return two ? occupancy<128, 2, F8>(g) : occupancy<128, 1, F8>(g);
    return 0;
}

template <int D, int NT, bool F8>
cudaError_t launch_s(const DecodeParams& p, int grid, const CUtensorMap& km, const CUtensorMap& vm,
                     bool pdl, cudaStream_t stream) {
    if (!ensure_smem_attr<D, NT, F8>() || occupancy<D, NT, F8>(p.group) <= 0)
        return cudaErrorInvalidConfiguration;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = SCfg<D, NT, F8>::smem_bytes(p.group);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, decode_stream_kernel<D, NT, F8>, p, km, vm);
}

template <bool F8>
cudaError_t launch_by_shape(const DecodeParams& p, int grid, const CUtensorMap& km, const CUtensorMap& vm,
                            bool pdl, cudaStream_t stream) {
    const bool two = p.group > 8;
    if (p.head_dim == 64)
        return two ? launch_s<64, 2, F8>(p, grid, km, vm, pdl, stream)
                   : launch_s<64, 1, F8>(p, grid, km, vm, pdl, stream);
    if (p.head_dim == 128)
        return two ? launch_s<128, 2, F8>(p, grid, km, vm, pdl, stream)
                   : launch_s<128, 1, F8>(p, grid, km, vm, pdl, stream);
    return cudaErrorInvalidValue;
}

}  // namespace

bool stream_kernel_supports(const pa_cache_desc& d) {
    const int g = d.num_q_heads / d.num_kv_heads;
    return (d.head_dim == 64 || d.head_dim == 128) && d.num_kv_heads % kGroup == 0 && g >= 1 &&
           g <= 16 && encode_fn() != nullptr;
}

int stream_kernel_grid(const pa_cache_desc& d, int max_ctas, bool fp8) {
    int sms = 0;
    if (num_sms_current_device(&sms) != PA_OK) return 0;
    const int g = d.num_q_heads / d.num_kv_heads;
    const int occ = fp8 ? occupancy_for<true>(d.head_dim, g) : occupancy_for<false>(d.head_dim, g);
    if (occ <= 0) return 0;
    int grid = sms * occ;
    if (max_ctas > 0 && max_ctas < grid) grid = max_ctas;
    return grid;
}

cudaError_t launch_decode_stream(const DecodeParams& p, int grid, bool pdl, cudaStream_t stream) {
    CUtensorMap km, vm;
    if (!make_map(&km, p.k_cache, p) || !make_map(&vm, p.v_cache, p)) return cudaErrorInvalidValue;
    return p.kv_fp8 ? launch_by_shape<true>(p, grid, km, vm, pdl, stream)
                    : launch_by_shape<false>(p, grid, km, vm, pdl, stream);
}

}  // namespace pa
