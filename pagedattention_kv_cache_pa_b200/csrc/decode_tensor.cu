// Paged decode attention: TMA-staged pages, q.K and p.V on tensor cores.
//
// What it computes is the same as the CUDA-core kernel (softmax(scale q K^T) V
// per query head over the sequence's paged K/V, grouped-query heads sharing a
// kv head); how it gets there is shaped by the B200:
//
//  * One CTA per (sequence, kv head, split): 1 producer warp + 4 consumer warps.
//  * The producer reads the split's block-table entries (32 at a time, one
//    coalesced load, handed around the warp by shuffles) and streams each page
//    of K and V from HBM into a 4-stage shared-memory ring with tiled TMA loads
//    (cp.async.bulk.tensor, no multicast) completing on mbarriers.  A stage
//    holds 64 tokens; pages smaller than 64 tokens are gathered into it page by
//    page, larger ones are cut into 64-token pieces.  The tensor maps use the
//    128-byte swizzle, so the tensor-core operand loads below are free of bank
//    conflicts.  A block id outside the pool is loaded from outside the tensor
//    map, which TMA fills with zeros.
//  * Each consumer warp owns 16 of the stage's tokens.  Scores for all query
//    heads of the group come from one m16n8k16 bf16 MMA per 16 head-dim
//    elements, with the 16 tokens as M and up to 8 heads as N (q fragments stay
//    in registers for the whole split).  The fp32 online softmax (log2 domain)
//    runs on the accumulator fragment; the probabilities are rounded to bf16,
//    transposed in registers (movmatrix) into the B operand of the p.V MMA,
//    whose A operand is V^T read with ldmatrix.trans.  Every K/V byte is read
//    from HBM once per kv head and shared by the whole query group.
//  * The four warps' (max, sum, output) states are combined through shared
//    memory; a split writes its partial state for the merge kernel (merge.cu).
//
// Tensor cores are used here because at g query heads per kv head the CUDA-core
// form needs 4 g fp32 FMAs per K/V element pair plus per-token shuffle
// reductions, which for g >= 4 rivals the B200's fp32 issue rate at full HBM
// bandwidth; the MMA form moves that work off the FMA pipe.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <atomic>
#include <mutex>

#include "pa_device.cuh"
#include "pa_ptx.cuh"

namespace pa {
namespace {

constexpr int kConsumerWarps = 4;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kTileTokens = 64;   // tokens per pipeline stage (16 per consumer warp)
constexpr int kRowBytes = 128;    // one swizzled row: 64 bf16 head-dim elements

template <int D, int NT>
struct Cfg {
    static constexpr int kHalves = D / 64;                                 // 128-byte column halves
    static constexpr int kHalfBytes = kTileTokens * kRowBytes;             // 8 KB
    static constexpr int kTileBytes = kHalves * kHalfBytes;                // K (or V) of one stage
    // ring depth: 4 stages (D=64, 3 CTAs per SM), 3 (D=128, g<=8) or 2 (D=128, g<=16), 2 CTAs per SM
    static constexpr int kStages = D == 64 ? 4 : (NT == 1 ? 3 : 2);
    static constexpr int kStageBytes = 2 * kTileBytes;                     // K + V
    static constexpr int kSmemBytes = kStages * kStageBytes + 1024;        // + alignment slack
    static constexpr int kKSteps = D / 16;                                 // k-steps of q.K
    static constexpr int kMTiles = D / 16;                                 // m-tiles of p.V
    static constexpr int kMinBlocks = (D == 64 && NT == 1) ? 3 : 2;        // resident CTAs per SM
};

// Address of 16-byte chunk `chunk` (0..D/8-1) of token row `row` (0..63) in a
// stage tile laid out by the 128-byte-swizzled TMA loads ([half][64 rows][128 B]).
__device__ __forceinline__ uint32_t tile_addr(uint32_t tile, int row, int chunk) {
    const int half = chunk >> 3;
    const int c = (chunk & 7) ^ (row & 7);
    return tile + half * (kTileTokens * kRowBytes) + row * kRowBytes + (c << 4);
}

// Barrier among the four consumer warps only (the producer keeps streaming),
// built on an mbarrier so that, like every other wait here, it gives up after
// the timeout instead of hanging.  Each warp keeps its own copy of the phase.
struct ConsumerBarrier {
    uint32_t bar;
    uint32_t phase;
    __device__ __forceinline__ bool sync(int lane, int32_t* status) {
        __syncwarp();
        if (lane == 0) mbar_arrive(bar);
        const bool ok = warp_wait(bar, phase, status);
        phase ^= 1u;
        return ok;
    }
};

// What a stage carries besides K/V: which item and which tokens of it.
struct StageHeader {
    int32_t b, kvh, split, nsplit;
    int32_t ts, te;      // tokens [ts, te) of the item live in this stage
    int32_t flags;
    int32_t pad;
};
enum : int32_t { kFirst = 1, kLast = 2, kEmpty = 4, kEnd = 8 };

// Work items (sequence, split, kv head), kv head fastest, handed out through an
// atomic counter; every CTA walks the sequences forward to decode its indices.
struct ItemWalk {
    int32_t b = 0, base = 0, count = 0, L = 0;
    __device__ __forceinline__ void load(const DecodeParams& p) {
        L = clipped_length(p, b);
        const int32_t ns = L == 0 ? 1 : (L + p.split_tokens - 1) / p.split_tokens;
        count = ns * p.num_kv_heads;
    }
    // false once `item` lies past the last sequence
    __device__ __forceinline__ bool seek(const DecodeParams& p, int32_t item) {
        while (item >= base + count) {
            base += count;
            if (++b >= p.num_seqs) return false;
            load(p);
        }
        return true;
    }
};

template <int D, int NT>
__global__ void __launch_bounds__(kThreads, Cfg<D, NT>::kMinBlocks)
    decode_tensor_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap kmap,
                         const __grid_constant__ CUtensorMap vmap) {
    using C = Cfg<D, NT>;
    constexpr int kHeads = NT * 8;
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(16) uint16_t s_q[C::kStages][kHeads * D];
    __shared__ StageHeader s_hdr[C::kStages];
    __shared__ __align__(8) uint64_t full_bar[C::kStages];
    __shared__ __align__(8) uint64_t empty_bar[C::kStages];
    __shared__ __align__(8) uint64_t cons_bar;
    __shared__ __align__(16) float s_cmb[2][kHeads * D];
    __shared__ float s_ml[kConsumerWarps][2][kHeads];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int32_t G = p.group;
    const uint32_t smem_base = (smem_u32(smem_raw) + 1023u) & ~1023u;
    uint8_t* smem_gen = smem_raw + (smem_base - smem_u32(smem_raw));
    allow_dependents();

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(smem_u32(&full_bar[s]), 1);
            mbar_init(smem_u32(&empty_bar[s]), kConsumerWarps);
        }
        mbar_init(smem_u32(&cons_bar), kConsumerWarps);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    if (warp == kConsumerWarps) {
        // ================================ producer ================================
        const int32_t Bs = p.block_size, Hkv = p.num_kv_heads, Cs = p.split_tokens;
        const int32_t seg = Bs < kTileTokens ? Bs : kTileTokens;    // tokens per TMA box
        const int32_t rows_total = p.num_blocks * Hkv * Bs;
        const uint32_t q_bytes = (uint32_t)(G * D * 2);
        ItemWalk walk;
        walk.load(p);
        int32_t next = 0;
        if (lane == 0) next = atomicAdd(p.work_counter, 1);
        uint32_t gtile = 0;
        bool alive = true;
        // Hands out stage gtile: waits until the consumers released it.
        auto acquire = [&](int& s) -> bool {
            s = gtile % C::kStages;
            if (gtile >= (uint32_t)C::kStages) {
                bool ok = true;
                if (lane == 0)
                    ok = mbar_wait(smem_u32(&empty_bar[s]), ((gtile / C::kStages) - 1) & 1, p.status);
                return __shfl_sync(0xffffffffu, ok, 0);
            }
            return true;
        };
        while (alive) {
            const int32_t cur = __shfl_sync(0xffffffffu, next, 0);
            if (lane == 0) next = atomicAdd(p.work_counter, 1);   // consumed one item later
            if (!walk.seek(p, cur)) break;
            const int32_t local = cur - walk.base;
            const int32_t split = local / Hkv, kvh = local - split * Hkv;
            const int32_t b = walk.b, L = walk.L;
            const int32_t nsplit = walk.count / Hkv;
            const int32_t t0 = split * Cs, t1 = min(L, t0 + Cs);
            const int32_t ntiles = L == 0 ? 0 : (t1 - t0 + kTileTokens - 1) / kTileTokens;
            if (ntiles == 0) {
                int s;
                if (!acquire(s)) break;
                if (lane == 0) {
                    s_hdr[s] = StageHeader{b, kvh, split, nsplit, 0, 0, kFirst | kLast | kEmpty, 0};
                    mbar_arrive(smem_u32(&full_bar[s]));
                }
                ++gtile;
                continue;
            }
            const int32_t* table = p.block_tables + (size_t)b * p.max_blocks_per_seq;
            int32_t win_base = -1, win_entry = -1;
            for (int32_t tile = 0; tile < ntiles; ++tile) {
                int s;
                if (!acquire(s)) {
                    alive = false;
                    break;
                }
                const int32_t ts = t0 + tile * kTileTokens;
                const int32_t te = min(t1, ts + kTileTokens);
                const int32_t nseg = (te - ts + seg - 1) / seg;
                const bool first = tile == 0;
                const uint32_t k_tile = smem_base + s * C::kStageBytes;
                const uint32_t v_tile = k_tile + C::kTileBytes;
                const uint32_t bar = smem_u32(&full_bar[s]);
                if (lane == 0) {
                    s_hdr[s] = StageHeader{b, kvh, split, nsplit, ts, te,
                                           (first ? kFirst : 0) | (tile == ntiles - 1 ? kLast : 0), 0};
                    mbar_arrive_expect_tx(bar, (uint32_t)(nseg * seg * kRowBytes * C::kHalves * 2) +
                                                   (first ? q_bytes : 0u));
                    if (first)
                        bulk_load(smem_u32(&s_q[s][0]),
                                  p.q + ((size_t)b * p.num_q_heads + (size_t)kvh * G) * D, q_bytes, bar);
                }
                for (int32_t g = 0; g < nseg; ++g) {
                    const int32_t tok = ts + g * seg;
                    const int32_t lb = tok / Bs;                      // logical block
                    if (win_base < 0 || lb >= win_base + 32) {        // warp-uniform refill
                        win_base = lb;
                        const int32_t idx = win_base + lane;
                        win_entry = idx < p.max_blocks_per_seq ? __ldg(table + idx) : -1;
                    }
                    const int32_t blk = __shfl_sync(0xffffffffu, win_entry, lb - win_base);
                    if (lane == 0) {
                        int32_t y;
                        if (blk < 0 || blk >= p.num_blocks) {
                            raise_status(p.status, kStatusBadBlock);
                            y = rows_total;                           // outside the map: zero fill
                        } else {
                            y = (blk * Hkv + kvh) * Bs + (tok - lb * Bs);
                        }
                        const uint32_t row_off = (uint32_t)(g * seg) * kRowBytes;
#pragma unroll
                        for (int h = 0; h < C::kHalves; ++h) {
                            tma_load_2d(k_tile + h * C::kHalfBytes + row_off, &kmap, h * 64, y, bar);
                            tma_load_2d(v_tile + h * C::kHalfBytes + row_off, &vmap, h * 64, y, bar);
                        }
                    }
                }
                ++gtile;
            }
        }
        // tell the consumers there is no more work
        int s;
        if (acquire(s) && lane == 0) {
            s_hdr[s] = StageHeader{0, 0, 0, 0, 0, 0, kEnd, 0};
            mbar_arrive(smem_u32(&full_bar[s]));
        }
    } else {
        // ================================ consumers ===============================
        const int r = lane >> 2, c = lane & 3;
        const int tid = threadIdx.x;                    // 0..127
        const int row0 = warp * 16;                     // this warp's rows in a stage tile
        const int mi = lane >> 3, rr = lane & 7;
        const float sl2 = p.scale_log2;
        uint32_t qf[NT][C::kKSteps][2];
        float m_run[NT][2], l_run[NT][2];
        float o_acc[NT][C::kMTiles][4];
        ConsumerBarrier cb{smem_u32(&cons_bar), 0u};
        for (uint32_t gtile = 0;; ++gtile) {
            const int s = gtile % C::kStages;
            if (!warp_wait(smem_u32(&full_bar[s]), (gtile / C::kStages) & 1, p.status)) break;
            const StageHeader hd = s_hdr[s];
            if (hd.flags & kEnd) break;
            if (hd.flags & kEmpty) {
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&empty_bar[s]));
                if (warp == 0) store_zero_group(p, hd.b, hd.kvh, lane, 32);
                continue;
            }
            if (hd.flags & kFirst) {
                // q fragments (B operand of q.K): head n = 8 nt + r, head-dim k = 16 ks + 2c (+8)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const int h = nt * 8 + r;
#pragma unroll
                    for (int ks = 0; ks < C::kKSteps; ++ks) {
                        const uint32_t* qr = reinterpret_cast<const uint32_t*>(&s_q[s][h * D + ks * 16]);
                        qf[nt][ks][0] = h < G ? qr[c] : 0u;
                        qf[nt][ks][1] = h < G ? qr[c + 4] : 0u;
                    }
                    m_run[nt][0] = m_run[nt][1] = -INFINITY;
                    l_run[nt][0] = l_run[nt][1] = 0.f;
#pragma unroll
                    for (int mt = 0; mt < C::kMTiles; ++mt)
#pragma unroll
                        for (int e = 0; e < 4; ++e) o_acc[nt][mt][e] = 0.f;
                }
            }
            const int valid = min(16, max(0, hd.te - (hd.ts + row0)));
            const uint32_t k_tile = smem_base + s * C::kStageBytes;
            const uint32_t v_tile = k_tile + C::kTileBytes;
            if (valid > 0) {
                if (valid < 16) {
                    // rows past the item: zero V so that 0-probability rows add nothing
                    uint8_t* v_gen = smem_gen + (v_tile - smem_base);
                    for (int i = lane; i < (16 - valid) * 8 * C::kHalves; i += 32) {
                        const int rw = row0 + valid + i / (8 * C::kHalves);
                        const int ch = i % (8 * C::kHalves);
                        *reinterpret_cast<uint4*>(v_gen + tile_addr(0, rw, ch)) = make_uint4(0, 0, 0, 0);
                    }
                    // order these generic-proxy writes before the TMA that refills the stage
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    __syncwarp();
                }
                // ---- S = K q^T : 16 tokens x 8 heads per n-tile ----
                float sacc[NT][4];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) sacc[nt][e] = 0.f;
#pragma unroll
                for (int ks = 0; ks < C::kKSteps; ++ks) {
                    uint32_t a[4];
                    ldmatrix_x4(tile_addr(k_tile, row0 + rr + ((mi & 1) << 3), 2 * ks + (mi >> 1)), a);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(sacc[nt], a, qf[nt][ks][0], qf[nt][ks][1]);
                }
                // ---- online softmax over the 16 rows (tokens) per head column ----
                const bool v_lo = r < valid, v_hi = (r + 8) < valid;
                uint32_t pb[NT][2];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const float s0 = v_lo ? sacc[nt][0] * sl2 : -INFINITY;
                    const float s1 = v_lo ? sacc[nt][1] * sl2 : -INFINITY;
                    const float s2 = v_hi ? sacc[nt][2] * sl2 : -INFINITY;
                    const float s3 = v_hi ? sacc[nt][3] * sl2 : -INFINITY;
                    float mx0 = fmaxf(s0, s2), mx1 = fmaxf(s1, s3);
#pragma unroll
                    for (int off = 4; off < 32; off <<= 1) {
                        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
                        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
                    }
                    const float mn0 = fmaxf(m_run[nt][0], mx0), mn1 = fmaxf(m_run[nt][1], mx1);
                    const float al0 = fast_exp2(m_run[nt][0] - mn0), al1 = fast_exp2(m_run[nt][1] - mn1);
                    m_run[nt][0] = mn0;
                    m_run[nt][1] = mn1;
                    const float p0 = fast_exp2(s0 - mn0), p1 = fast_exp2(s1 - mn1);
                    const float p2 = fast_exp2(s2 - mn0), p3 = fast_exp2(s3 - mn1);
                    l_run[nt][0] = l_run[nt][0] * al0 + (p0 + p2);
                    l_run[nt][1] = l_run[nt][1] * al1 + (p1 + p3);
#pragma unroll
                    for (int mt = 0; mt < C::kMTiles; ++mt) {
                        o_acc[nt][mt][0] *= al0;
                        o_acc[nt][mt][1] *= al1;
                        o_acc[nt][mt][2] *= al0;
                        o_acc[nt][mt][3] *= al1;
                    }
                    pb[nt][0] = movmatrix_trans(pack_bf16x2(p0, p1));   // tokens 0-7
                    pb[nt][1] = movmatrix_trans(pack_bf16x2(p2, p3));   // tokens 8-15
                }
                // ---- O^T += V^T P : 16 head-dim rows x 8 heads per (m-tile, n-tile) ----
#pragma unroll
                for (int mt = 0; mt < C::kMTiles; ++mt) {
                    uint32_t a[4];
                    ldmatrix_x4_trans(tile_addr(v_tile, row0 + rr + ((mi >> 1) << 3), 2 * mt + (mi & 1)), a);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(o_acc[nt][mt], a, pb[nt][0], pb[nt][1]);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&empty_bar[s]));
            if (!(hd.flags & kLast)) continue;

            // ======== item done: combine the four warps, store or publish a split ========
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int j = 0; j < 2; ++j) {
#pragma unroll
                    for (int off = 4; off < 32; off <<= 1)
                        l_run[nt][j] += __shfl_xor_sync(0xffffffffu, l_run[nt][j], off);
                    if (r == 0) {
                        s_ml[warp][0][nt * 8 + 2 * c + j] = m_run[nt][j];
                        s_ml[warp][1][nt * 8 + 2 * c + j] = l_run[nt][j];
                    }
                }
            if (!cb.sync(lane, p.status)) break;
            // scale this warp's output by its share of the item's softmax mass
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int h = nt * 8 + 2 * c + j;
                    float M = -INFINITY;
#pragma unroll
                    for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, s_ml[w][0][h]);
                    float Ls = 0.f;
#pragma unroll
                    for (int w = 0; w < kConsumerWarps; ++w) Ls += s_ml[w][1][h] * fast_exp2(s_ml[w][0][h] - M);
                    const float f = fast_exp2(m_run[nt][j] - M) / Ls;
#pragma unroll
                    for (int mt = 0; mt < C::kMTiles; ++mt) {
                        o_acc[nt][mt][j] *= f;
                        o_acc[nt][mt][j + 2] *= f;
                    }
                }
            // deterministic pairwise sum: (warp 0 + warp 1) + (warp 2 + warp 3)
            float* cmb = s_cmb[warp >> 1];
            const bool writer = (warp & 1) == 0;
            if (writer) {
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int mt = 0; mt < C::kMTiles; ++mt) {
                        const int h = nt * 8 + 2 * c, d = mt * 16 + r;
                        cmb[h * D + d] = o_acc[nt][mt][0];
                        cmb[(h + 1) * D + d] = o_acc[nt][mt][1];
                        cmb[h * D + d + 8] = o_acc[nt][mt][2];
                        cmb[(h + 1) * D + d + 8] = o_acc[nt][mt][3];
                    }
            }
            if (!cb.sync(lane, p.status)) break;
            if (!writer) {
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int mt = 0; mt < C::kMTiles; ++mt) {
                        const int h = nt * 8 + 2 * c, d = mt * 16 + r;
                        cmb[h * D + d] += o_acc[nt][mt][0];
                        cmb[(h + 1) * D + d] += o_acc[nt][mt][1];
                        cmb[h * D + d + 8] += o_acc[nt][mt][2];
                        cmb[(h + 1) * D + d + 8] += o_acc[nt][mt][3];
                    }
            }
            if (!cb.sync(lane, p.status)) break;
            const int32_t b = hd.b, kvh = hd.kvh, nsplit = hd.nsplit;
            const size_t part = (((size_t)b * p.num_kv_heads + kvh) * p.max_splits + hd.split) * G;
            uint16_t* out = p.out + ((size_t)b * p.num_q_heads + (size_t)kvh * G) * D;
            for (int i = tid; i < G * D; i += kConsumerWarps * 32) {
                const int h = i / D, d = i - h * D;
                const float v = s_cmb[0][h * D + d] + s_cmb[1][h * D + d];
                if (nsplit == 1) {
                    out[(size_t)h * D + d] = f32_to_bf16_rn(v);
                } else {
                    p.part_o[(part + h) * D + d] = v;
                    if (d == 0) {
                        float M = -INFINITY;
#pragma unroll
                        for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, s_ml[w][0][h]);
                        float Ls = 0.f;
#pragma unroll
                        for (int w = 0; w < kConsumerWarps; ++w) Ls += s_ml[w][1][h] * fast_exp2(s_ml[w][0][h] - M);
                        p.part_lse[part + h] = M + __log2f(Ls);
                    }
                }
            }
            if (!cb.sync(lane, p.status)) break;   // s_cmb / s_ml free for the next item
        }
    }

    // ---- the last CTA to finish re-arms the work counter for the next launch ----
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        if (atomicAdd(p.done_counter, 1) == (int32_t)gridDim.x - 1) {
            *p.work_counter = 0;
            *p.done_counter = 0;
            __threadfence();
        }
    }
}

// ---- host side ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
    });
    return fn;
}

// 2-D view of a cache tensor: rows = num_blocks * Hkv * Bs, each D bf16; box = 64 x seg rows.
bool make_cache_map(CUtensorMap* map, const void* base, const DecodeParams& p) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)p.head_dim,
                                (cuuint64_t)p.num_blocks * p.num_kv_heads * p.block_size};
    const cuuint64_t strides[1] = {(cuuint64_t)p.head_dim * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)(p.block_size < kTileTokens ? p.block_size : kTileTokens)};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int NT>
cudaError_t launch_t(const DecodeParams& p, const CUtensorMap& km, const CUtensorMap& vm,
                     cudaStream_t stream) {
    using C = Cfg<D, NT>;
    // per device: dynamic shared-memory opt-in and resident CTAs per SM
    static std::atomic<int> ctas_per_sm[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    int occ = ctas_per_sm[dev].load(std::memory_order_acquire);
    if (occ <= 0) {
        e = cudaFuncSetAttribute(decode_tensor_kernel<D, NT>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
        if (e != cudaSuccess) return e;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, decode_tensor_kernel<D, NT>, kThreads,
                                                          C::kSmemBytes);
        if (e != cudaSuccess) return e;
        if (occ <= 0) return cudaErrorInvalidConfiguration;
        ctas_per_sm[dev].store(occ, std::memory_order_release);
    }
    int sms = 0;
    if (num_sms_current_device(&sms) != PA_OK) return cudaErrorInvalidDevice;
    // persistent grid: every resident slot, but never more CTAs than work items
    const int64_t items = (int64_t)p.num_seqs * p.num_kv_heads * p.max_splits;
    const int64_t grid = std::min<int64_t>((int64_t)sms * occ, std::max<int64_t>(items, 1));
    decode_tensor_kernel<D, NT><<<(unsigned)grid, kThreads, C::kSmemBytes, stream>>>(p, km, vm);
    return cudaGetLastError();
}

}  // namespace

bool tensor_kernel_supports(const pa_cache_desc& d) {
    return (d.head_dim == 64 || d.head_dim == 128) && d.num_q_heads / d.num_kv_heads <= 16 &&
           encode_fn() != nullptr;
}

cudaError_t launch_decode_tensor(const DecodeParams& p, cudaStream_t stream) {
    CUtensorMap km, vm;
    if (!make_cache_map(&km, p.k_cache, p) || !make_cache_map(&vm, p.v_cache, p))
        return cudaErrorInvalidValue;
    const bool two = p.group > 8;
    if (p.head_dim == 64)
        return two ? launch_t<64, 2>(p, km, vm, stream) : launch_t<64, 1>(p, km, vm, stream);
    if (p.head_dim == 128)
        return two ? launch_t<128, 2>(p, km, vm, stream) : launch_t<128, 1>(p, km, vm, stream);
    return cudaErrorInvalidValue;
}

}  // namespace pa
