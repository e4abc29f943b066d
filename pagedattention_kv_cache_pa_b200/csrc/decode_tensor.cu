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
//    memory; a split writes its partial state and the last split of a
//    (sequence, kv head) to arrive merges them (pa_device.cuh).
//
// Tensor cores are used here because at g query heads per kv head the CUDA-core
// form needs 4 g fp32 FMAs per K/V element pair plus per-token shuffle
// reductions, which for g >= 4 rivals the B200's fp32 issue rate at full HBM
// bandwidth; the MMA form moves that work off the FMA pipe.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "pa_device.cuh"

namespace pa {
namespace {

constexpr int kConsumerWarps = 4;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kTileTokens = 64;   // tokens per pipeline stage (16 per consumer warp)
constexpr int kRowBytes = 128;    // one swizzled row: 64 bf16 head-dim elements
constexpr unsigned long long kWaitTimeoutNs = 2000000000ull;  // 2 s

template <int D>
struct Cfg {
    static constexpr int kHalves = D / 64;                                 // 128-byte column halves
    static constexpr int kHalfBytes = kTileTokens * kRowBytes;             // 8 KB
    static constexpr int kTileBytes = kHalves * kHalfBytes;                // K (or V) of one stage
    static constexpr int kStages = D == 64 ? 4 : 3;                      // 3 (D=64) / 2 (D=128) CTAs per SM
    static constexpr int kStageBytes = 2 * kTileBytes;                     // K + V
    static constexpr int kSmemBytes = kStages * kStageBytes + 1024;        // + alignment slack
    static constexpr int kKSteps = D / 16;                                 // k-steps of q.K
    static constexpr int kMTiles = D / 16;                                 // m-tiles of p.V
};

// ---- PTX wrappers ------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ unsigned long long globaltimer() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Bounded wait: false (and the timeout status bit) if the phase does not
// complete within kWaitTimeoutNs.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, int32_t* status) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer();
    for (uint32_t it = 0;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 255u) == 255u && globaltimer() - t0 > kWaitTimeoutNs) {
            raise_status(status, kStatusTimeout);
            return false;
        }
    }
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int32_t x,
                                            int32_t y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}

// D(16x8, f32) += A(16x16, bf16, row) * B(16x8, bf16, col)
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Address of 16-byte chunk `chunk` (0..D/8-1) of token row `row` (0..63) in a
// stage tile laid out by the 128-byte-swizzled TMA loads ([half][64 rows][128 B]).
__device__ __forceinline__ uint32_t tile_addr(uint32_t tile, int row, int chunk) {
    const int half = chunk >> 3;
    const int c = (chunk & 7) ^ (row & 7);
    return tile + half * (kTileTokens * kRowBytes) + row * kRowBytes + (c << 4);
}

template <int D, int NT>
__global__ void __launch_bounds__(kThreads, 2)
    decode_tensor_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap kmap,
                         const __grid_constant__ CUtensorMap vmap) {
    using C = Cfg<D>;
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t full_bar[C::kStages];
    __shared__ __align__(8) uint64_t empty_bar[C::kStages];

    const int32_t split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
    const int32_t L = clipped_length(p, b);
    if (L == 0) {
        if (split == 0) store_zero_group(p, b, kvh);
        return;
    }
    const int32_t Cs = p.split_tokens;
    const int32_t nsplit = (L + Cs - 1) / Cs;
    if (split >= nsplit) return;
    const int32_t t0 = split * Cs;
    const int32_t t1 = min(L, t0 + Cs);
    const int32_t ntiles = (t1 - t0 + kTileTokens - 1) / kTileTokens;
    const int32_t G = p.group;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const uint32_t smem_base = (smem_u32(smem_raw) + 1023u) & ~1023u;
    uint8_t* smem_gen = smem_raw + (smem_base - smem_u32(smem_raw));

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(smem_u32(&full_bar[s]), 1);
            mbar_init(smem_u32(&empty_bar[s]), kConsumerWarps);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    // Per-warp running state (consumers) -- declared here so the combine below sees it.
    float m_run[NT][2], l_run[NT][2];
    float o_acc[NT][C::kMTiles][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        m_run[nt][0] = m_run[nt][1] = -INFINITY;
        l_run[nt][0] = l_run[nt][1] = 0.f;
#pragma unroll
        for (int mt = 0; mt < C::kMTiles; ++mt)
#pragma unroll
            for (int e = 0; e < 4; ++e) o_acc[nt][mt][e] = 0.f;
    }

    if (warp == kConsumerWarps) {
        // ================================ producer ================================
        const int32_t Bs = p.block_size;
        const int32_t seg = Bs < kTileTokens ? Bs : kTileTokens;     // tokens per TMA box
        const int32_t rows_total = p.num_blocks * p.num_kv_heads * Bs;
        const int32_t* table = p.block_tables + (size_t)b * p.max_blocks_per_seq;
        int32_t win_base = -1, win_entry = -1;
        for (int32_t tile = 0; tile < ntiles; ++tile) {
            const int s = tile % C::kStages;
            if (tile >= C::kStages) {
                const uint32_t par = ((tile / C::kStages) - 1) & 1;
                bool ok = true;
                if (lane == 0) ok = mbar_wait(smem_u32(&empty_bar[s]), par, p.status);
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
            }
            const int32_t ts = t0 + tile * kTileTokens;
            const int32_t te = min(t1, ts + kTileTokens);
            const int32_t nseg = (te - ts + seg - 1) / seg;
            const uint32_t k_tile = smem_base + s * C::kStageBytes;
            const uint32_t v_tile = k_tile + C::kTileBytes;
            if (lane == 0)
                mbar_arrive_expect_tx(smem_u32(&full_bar[s]),
                                      (uint32_t)(nseg * seg * kRowBytes * C::kHalves * 2));
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
                        y = rows_total;                          // outside the map: zero fill
                    } else {
                        y = (blk * p.num_kv_heads + kvh) * Bs + (tok - lb * Bs);
                    }
                    const uint32_t row_off = (uint32_t)(g * seg) * kRowBytes;
                    const uint32_t bar = smem_u32(&full_bar[s]);
#pragma unroll
                    for (int h = 0; h < C::kHalves; ++h) {
                        tma_load_2d(k_tile + h * C::kHalfBytes + row_off, &kmap, h * 64, y, bar);
                        tma_load_2d(v_tile + h * C::kHalfBytes + row_off, &vmap, h * 64, y, bar);
                    }
                }
            }
        }
    } else {
        // ================================ consumers ===============================
        const int r = lane >> 2, c = lane & 3;
        // q fragments (B operand of q.K): head n = 8 nt + r, head-dim k = 16 ks + 2c (+8)
        uint32_t qf[NT][C::kKSteps][2];
        const uint16_t* qbase = p.q + ((size_t)b * p.num_q_heads + (size_t)kvh * G) * D;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int h = nt * 8 + r;
#pragma unroll
            for (int ks = 0; ks < C::kKSteps; ++ks) {
                if (h < G) {
                    const uint32_t* qr = reinterpret_cast<const uint32_t*>(qbase + (size_t)h * D + ks * 16);
                    qf[nt][ks][0] = __ldg(qr + c);
                    qf[nt][ks][1] = __ldg(qr + c + 4);
                } else {
                    qf[nt][ks][0] = qf[nt][ks][1] = 0u;
                }
            }
        }
        const float sl2 = p.scale_log2;
        const int row0 = warp * 16;                     // this warp's rows in a stage tile
        for (int32_t tile = 0; tile < ntiles; ++tile) {
            const int s = tile % C::kStages;
            const uint32_t par = (tile / C::kStages) & 1;
            bool ok = true;
            if (lane == 0) ok = mbar_wait(smem_u32(&full_bar[s]), par, p.status);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            const int32_t ts = t0 + tile * kTileTokens;
            const int valid = min(16, max(0, t1 - (ts + row0)));
            const uint32_t k_tile = smem_base + s * C::kStageBytes;
            const uint32_t v_tile = k_tile + C::kTileBytes;
            if (valid > 0) {
                if (valid < 16) {
                    // rows past the context: zero V so that 0-probability rows add nothing
                    uint8_t* v_gen = smem_gen + (v_tile - smem_base);
                    for (int i = lane; i < (16 - valid) * 8 * C::kHalves; i += 32) {
                        const int rr = row0 + valid + i / (8 * C::kHalves);
                        const int ch = i % (8 * C::kHalves);
                        *reinterpret_cast<uint4*>(v_gen + (tile_addr(0, rr, ch))) = make_uint4(0, 0, 0, 0);
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
                const int mi = lane >> 3, rr = lane & 7;
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
                    float s0 = v_lo ? sacc[nt][0] * sl2 : -INFINITY;
                    float s1 = v_lo ? sacc[nt][1] * sl2 : -INFINITY;
                    float s2 = v_hi ? sacc[nt][2] * sl2 : -INFINITY;
                    float s3 = v_hi ? sacc[nt][3] * sl2 : -INFINITY;
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
        }
        // full row sums: add the partial sums of the 8 lanes that share a head column
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int off = 4; off < 32; off <<= 1)
                    l_run[nt][j] += __shfl_xor_sync(0xffffffffu, l_run[nt][j], off);
    }

    // ---- combine the four consumer warps through shared memory (stages are drained) ----
    __syncthreads();
    float* s_o = reinterpret_cast<float*>(smem_gen);               // [4][NT*8][D]
    float* s_m = s_o + kConsumerWarps * NT * 8 * D;                // [4][NT*8]
    float* s_l = s_m + kConsumerWarps * NT * 8;                    // [4][NT*8]
    if (warp < kConsumerWarps) {
        const int r = lane >> 2, c = lane & 3;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int h0 = nt * 8 + 2 * c;
            if (r == 0) {
                s_m[warp * NT * 8 + h0] = m_run[nt][0];
                s_m[warp * NT * 8 + h0 + 1] = m_run[nt][1];
                s_l[warp * NT * 8 + h0] = l_run[nt][0];
                s_l[warp * NT * 8 + h0 + 1] = l_run[nt][1];
            }
#pragma unroll
            for (int mt = 0; mt < C::kMTiles; ++mt) {
                float* base = s_o + (size_t)(warp * NT * 8) * D;
                const int d = mt * 16 + r;
                base[(size_t)h0 * D + d] = o_acc[nt][mt][0];
                base[(size_t)(h0 + 1) * D + d] = o_acc[nt][mt][1];
                base[(size_t)h0 * D + d + 8] = o_acc[nt][mt][2];
                base[(size_t)(h0 + 1) * D + d + 8] = o_acc[nt][mt][3];
            }
        }
    }
    __syncthreads();
    const size_t part = (((size_t)b * p.num_kv_heads + kvh) * p.max_splits + split) * G;
    uint16_t* out = p.out + ((size_t)b * p.num_q_heads + (size_t)kvh * G) * D;
    for (int i = threadIdx.x; i < G * D; i += kThreads) {
        const int h = i / D, d = i - h * D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, s_m[w * NT * 8 + h]);
        float lsum = 0.f, osum = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) {
            const float sc = fast_exp2(s_m[w * NT * 8 + h] - M);
            lsum += s_l[w * NT * 8 + h] * sc;
            osum += s_o[((size_t)w * NT * 8 + h) * D + d] * sc;
        }
        if (nsplit == 1) {
            out[(size_t)h * D + d] = f32_to_bf16_rn(osum / lsum);
        } else {
            p.part_o[(part + h) * D + d] = osum / lsum;
            if (d == 0) p.part_lse[part + h] = M + __log2f(lsum);
        }
    }
    if (nsplit > 1) arrive_and_maybe_merge(p, b, kvh, nsplit);
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
    using C = Cfg<D>;
    // the dynamic shared-memory opt-in is per device
    static std::atomic<uint64_t> done_mask{0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = 1ull << (dev & 63);
    if (!(done_mask.load(std::memory_order_acquire) & bit)) {
        e = cudaFuncSetAttribute(decode_tensor_kernel<D, NT>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
        if (e != cudaSuccess) return e;
        done_mask.fetch_or(bit, std::memory_order_acq_rel);
    }
    const dim3 grid(p.max_splits, p.num_kv_heads, p.num_seqs);
    decode_tensor_kernel<D, NT><<<grid, kThreads, C::kSmemBytes, stream>>>(p, km, vm);
    return cudaGetLastError();
}

}  // namespace

bool tensor_kernel_supports(const DecodeParams& p) {
    return (p.head_dim == 64 || p.head_dim == 128) && p.group <= 16 &&
           p.split_tokens % kTileTokens == 0 && encode_fn() != nullptr;
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
