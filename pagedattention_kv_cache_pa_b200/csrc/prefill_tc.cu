// Paged (chunked) prefill attention on the fifth-generation tensor cores.
//
// Same operation as prefill.cu: sequence b holds context_lens[b] = L tokens after this
// step's append, its last Tq = cu_q[b+1] - cu_q[b] tokens are the queries (positions
// L-Tq .. L-1), and the query at position p attends to cache tokens 0..p (Nano-vLLM
// page, section "Prefill vs Decode"; causal mask: Tiny-vLLM summary page, section
// "고성능 추론을 위한 고급 최적화 기법").
//
// One CTA of 128 threads per (128 query rows, kv head, sequence); a row is a (query
// token, query head of the kv head's group) pair and thread i owns row i, which is
// tensor-memory lane i.  Per 64-key tile t:
//   S_t = Q K_t^T   tcgen05.mma, M=128 N=64, Q and K_t K-major in shared memory,
//                   fp32 S_t in tensor memory;
//   softmax         each thread loads its row of S_t, masks it causally, updates its
//                   running max and sum in the log2 domain, and writes P_t (bf16) as a
//                   K-major A operand into shared memory;
//   O_t = P_t V_t   tcgen05.mma, M=128 N=D, V_t read MN-major straight from its
//                   [key][dim] tile; each thread folds its row of O_t into fp32
//                   registers, O = alpha O + O_t.
// One thread issues P_t V_t and Q K_{t+1} together, so S_{t+1} is computed while the
// rows of O_t are folded in.  K and V tiles have two buffers each: K_{t+2} is requested
// once S_t is done, V_{t+2} once O_t is done, from block ids read a tile ahead.  When
// the block size tiles 64 keys (8, 16, 32, 64 or a multiple of 64) they move by TMA, one
// box of 64 dims x min(Bs, 64) tokens per block and 64-dim atom, swizzled by the copy
// engine: warp 1 issues the K boxes and warp 2 the V boxes, so that warp 0, whose
// thread 0 issues the MMAs, carries no copy work; otherwise every thread gathers them
// with 16-byte cp.async copies.
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <cstring>

#include "pa_device.cuh"
#include "pa_internal.h"
#include "pa_ptx.cuh"
#include "pa_umma.cuh"

namespace pa {
namespace {

constexpr int kTcRows = 128;     // query rows per CTA (tensor-memory lanes)
constexpr int kTcKeys = 64;      // keys per tile
constexpr int kTcThreads = 128;

template <int D>
struct TcCfg {
    static constexpr int kQBytes = kTcRows * D * 2;
    static constexpr int kKVBytes = kTcKeys * D * 2;       // one K (or V) tile
    static constexpr int kPBytes = kTcRows * kTcKeys * 2;
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kOffQ + kQBytes;           // 2 buffers
    static constexpr int kOffV = kOffK + 2 * kKVBytes;      // 2 buffers
    static constexpr int kOffP = kOffV + 2 * kKVBytes;
    static constexpr int kOffBar = kOffP + kPBytes;         // 6 mbarriers, tensor-memory address
    static constexpr int kSmem = kOffBar + 64;
    static constexpr int kColS = 0;                         // S: 64 fp32 columns
    static constexpr int kColO = 64;                        // O_t: D fp32 columns
    static constexpr uint32_t kTmemCols = D == 64 ? 128 : 256;
    static constexpr int kMinBlocks = D == 64 ? 3 : 2;      // by shared memory and tensor memory
};

// Byte offset of (row, 16-byte chunk c) in a tile of `rows` rows of bf16 stored as
// 128-byte-swizzled atoms: atom c / 8 holds 128 bytes of every row, rows at 128 bytes,
// chunk (c % 8) XOR (row % 8).  This is the canonical K-major layout of a tcgen05
// operand (and the MN-major one when the rows run along K, as for V).
template <int ROWS>
__device__ __forceinline__ uint32_t sw128(int row, int c) {
    return (uint32_t)((c >> 3) * (ROWS * 128) + row * 128 + ((((c & 7) ^ (row & 7))) << 4));
}

__device__ __forceinline__ void cp_async16_tc(uint32_t dst, const void* src, bool live) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(live ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit_tc() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait_tc() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

template <int D, bool kTma>
__global__ void __launch_bounds__(kTcThreads, TcCfg<D>::kMinBlocks)
    prefill_tc_kernel(const PrefillParams p, const __grid_constant__ CUtensorMap kmap,
                      const __grid_constant__ CUtensorMap vmap) {
    using C = TcCfg<D>;
    constexpr int kCh = D / 8;                               // 16-byte chunks per row
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t s_base = smem_u32(smem);
    const uint32_t s_q = s_base + C::kOffQ, s_k = s_base + C::kOffK, s_v = s_base + C::kOffV;
    const uint32_t s_p = s_base + C::kOffP;
    // S done, O done, K tile landed (2 buffers), V tile landed (2 buffers)
    const uint32_t bar_s = s_base + C::kOffBar, bar_o = bar_s + 8, bar_k = bar_s + 16, bar_v = bar_s + 32;
    const uint32_t s_tmem = bar_s + 48;

    const int b = blockIdx.z, kvh = blockIdx.y;
    const int G = p.group, Hq = p.num_q_heads, Hkv = p.num_kv_heads, Bs = p.block_size;
    const int q0 = p.cu_q[b], Tq = p.cu_q[b + 1] - q0;
    const int L = p.context_lens[b];
    const int cap = p.max_blocks_per_seq * Bs;
    if (Tq <= 0) return;
    if (L < Tq || L > cap || Tq > p.max_q_len) {             // fewer tokens than queries, past the table,
                                                             // or more queries than the grid holds
        if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.y == 0) raise_status(p.status, kStatusBadLength);
        return;
    }
    if (s_base & 1023u) {                                    // the swizzle needs 1024-byte-aligned tiles
        if (threadIdx.x == 0) raise_status(p.status, kStatusSmemAlign);
        return;
    }
    // the last row tiles of a chunk attend to the most keys: they take the first CTAs
    const int rows = Tq * G, ntile = (rows + kTcRows - 1) / kTcRows;
    const int tile = ntile - 1 - (int)blockIdx.x;
    if (tile < 0) return;
    const int r0 = tile * kTcRows;
    const int* table = p.block_tables + (size_t)b * p.max_blocks_per_seq;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    const int last_tok = min(rows - 1, r0 + kTcRows - 1) / G;
    const int kend = L - Tq + last_tok + 1;                  // keys needed: up to the last row's position
    const int ntiles = (kend + kTcKeys - 1) / kTcKeys;
    const int pos_first = L - Tq + r0 / G;                   // smallest position in the tile

    // ---- tensor memory and barriers ----
    if (warp == 0) {
        tmem_alloc(s_tmem, C::kTmemCols);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(bar_s, 1);
        mbar_init(bar_o, 1);
        for (int i = 0; i < 4; ++i) mbar_init(bar_k + 8 * i, 1);   // bar_k[0..1], bar_v[0..1]
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    uint32_t tmem;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(tmem) : "r"(s_tmem) : "memory");
    const uint32_t t_lane = tmem + ((uint32_t)(warp * 32) << 16);   // this warp's 32 lanes

    // ---- loads: Q (rows past the chunk are zeros), K and V tiles through the block table ----
    for (int i = tid; i < kTcRows * kCh; i += kTcThreads) {
        const int row = i / kCh, c = i - row * kCh, R = r0 + row;
        const bool live = R < rows;
        const int tok = live ? R / G : 0, g = live ? R - tok * G : 0;
        const uint16_t* src = p.q + (((size_t)(q0 + tok) * Hq + (size_t)kvh * G + g) * D + c * 8);
        cp_async16_tc(s_q + sw128<kTcRows>(row, c), src, live);
    }
    // Thread tid copies chunk c_ld of keys j0, j0 + kJStep, ... of every tile.  Their block
    // ids are fetched one tile ahead into registers (fetch_ids), so the table lookups'
    // latency hides behind a whole tile of work instead of stalling each copy.
    constexpr int kJStep = kTcThreads / kCh;                 // 16 (D = 64) or 8 (D = 128)
    constexpr int kKPT = kTcKeys / kJStep;                   // keys per thread per tile: 4 or 8
    const int j0 = tid / kCh, c_ld = tid - (tid / kCh) * kCh;
    int ids[kKPT];
    // TMA: lane i of warp 1 (K) and of warp 2 (V) moves slot i of a tile (rb tokens of one
    // block) with one box per 64-dim atom; slot_id is that block's id for the next tile to
    // request.
    const int rb = Bs < kTcKeys ? Bs : kTcKeys, nslot = kTcKeys / rb;
    int slot_id = 0;
    auto fetch_ids = [&](int t) {
        if constexpr (kTma) {
            const int kp = t * kTcKeys + lane * rb;
            if ((warp == 1 || warp == 2) && lane < nslot && kp < L) slot_id = __ldg(table + kp / Bs);
        } else {
#pragma unroll
            for (int k = 0; k < kKPT; ++k) {
                const int kp = t * kTcKeys + j0 + k * kJStep;
                ids[k] = kp < L ? __ldg(table + kp / Bs) : 0;
            }
        }
    };
    auto tma_tile = [&](const CUtensorMap* map, uint32_t dst, uint32_t bar, int t) {   // one warp
        const int kp = t * kTcKeys + lane * rb;
        bool valid = lane < nslot && kp < L;
        if (valid && (slot_id < 0 || slot_id >= p.num_blocks)) {
            raise_status(p.status, kStatusBadBlock);
            valid = false;
        }
        const unsigned m = __ballot_sync(0xffffffffu, valid);
        if (lane == 0) mbar_arrive_expect_tx(bar, (uint32_t)(__popc(m) * rb * 128 * (D / 64)));
        __syncwarp();
        if (valid) {
            const int z = slot_id * Hkv + kvh, y = Bs > kTcKeys ? kp % Bs : 0;
#pragma unroll
            for (int a = 0; a < D / 64; ++a)
                tma_load_3d(dst + a * (kTcKeys * 128) + lane * rb * 128, map, a * 64, y, z, bar);
        }
    };
    auto load_tile = [&](const uint16_t* cache, uint32_t dst, int t) {
#pragma unroll
        for (int k = 0; k < kKPT; ++k) {
            const int j = j0 + k * kJStep, kp = t * kTcKeys + j;
            bool live = kp < L;
            size_t off = 0;
            if (live) {
                if (ids[k] < 0 || ids[k] >= p.num_blocks) {
                    raise_status(p.status, kStatusBadBlock);
                    live = false;
                } else {
                    off = (((size_t)ids[k] * Hkv + kvh) * Bs + kp % Bs) * D + c_ld * 8;
                }
            }
            cp_async16_tc(dst + sw128<kTcKeys>(j, c_ld), cache + off, live);
        }
    };
    // request K_t into buffer t & 1 (TMA: barrier bar_k[t & 1]; cp.async: one group)
    // TMA tiles requested (every thread counts them) and waited for by thread 0: on an
    // aborted run thread 0 drains the difference before the CTA exits
    int k_req = -1, v_req = -1, k_seen = -1, v_seen = -1;
    auto request_k = [&](int t) {
        if constexpr (kTma) {
            k_req = t;
            if (warp == 1) tma_tile(&kmap, s_k + (t & 1) * C::kKVBytes, bar_k + 8 * (t & 1), t);
        } else {
            load_tile(p.k_cache, s_k + (t & 1) * C::kKVBytes, t);
        }
    };
    auto request_v = [&](int t) {
        if constexpr (kTma) {
            v_req = t;
            if (warp == 2) tma_tile(&vmap, s_v + (t & 1) * C::kKVBytes, bar_v + 8 * (t & 1), t);
        } else {
            load_tile(p.v_cache, s_v + (t & 1) * C::kKVBytes, t);
        }
    };
    // cp.async groups in issue order: {Q, K0, V0}, K1, V1, then K_{t+2} and V_{t+2} per
    // tile t (empty groups past the last tile keep the count uniform); with TMA only Q
    fetch_ids(0);
    request_k(0);
    request_v(0);
    cp_async_commit_tc();
    if (ntiles > 1) {
        fetch_ids(1);
        request_k(1);
    }
    cp_async_commit_tc();
    if (ntiles > 1) request_v(1);
    cp_async_commit_tc();
    if (ntiles > 2) fetch_ids(2);
    bool failed = false;
    // thread 0, before an MMA reads K_t or V_t: its TMA copies have landed
    auto wait_kv = [&](uint32_t bar, int t) {
        if constexpr (kTma) {
            if (!mbar_wait(bar + 8 * (t & 1), (uint32_t)((t >> 1) & 1), p.status)) failed = true;
            if (bar == bar_k) k_seen = t; else v_seen = t;
        }
    };

    constexpr uint32_t kIdescS = umma_idesc_bf16(kTcRows, kTcKeys, false);
    constexpr uint32_t kIdescO = umma_idesc_bf16(kTcRows, D, true);
    auto issue_s = [&](int t) {                              // S = Q K_t^T over D / 16 K steps
        const uint32_t kt = s_k + (t & 1) * C::kKVBytes;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            const uint64_t a = umma_desc_sw128(s_q + (ks >> 2) * (kTcRows * 128) + (ks & 3) * 32, 16, 1024);
            const uint64_t bd = umma_desc_sw128(kt + (ks >> 2) * (kTcKeys * 128) + (ks & 3) * 32, 16, 1024);
            umma_bf16_ss(tmem + C::kColS, a, bd, kIdescS, ks > 0);
        }
        umma_commit(bar_s);
    };
    auto issue_o = [&](int t) {                              // O_t = P V_t over 4 K steps of 16 keys
        const uint32_t vt = s_v + (t & 1) * C::kKVBytes;
#pragma unroll
        for (int kk = 0; kk < kTcKeys / 16; ++kk) {
            const uint64_t a = umma_desc_sw128(s_p + kk * 32, 16, 1024);
            // MN-major B: 8-key groups 1024 bytes apart, 64-dim atoms one tile of keys apart
            const uint64_t bd = umma_desc_sw128(vt + kk * 16 * 128, kTcKeys * 128, 1024);
            umma_bf16_ss(tmem + C::kColO, a, bd, kIdescO, kk > 0);
        }
        umma_commit(bar_o);
    };

    cp_async_wait_tc<2>();                                   // Q, K0, V0
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncthreads();
    if (tid == 0) {
        tc_fence_after_sync();
        wait_kv(bar_k, 0);
        issue_s(0);
    }

    const int R = r0 + tid;
    const int pos = R < rows ? L - Tq + R / G : L - 1;      // padded rows: computed, not written
    const float sl2 = p.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;
    float o[D];
#pragma unroll
    for (int j = 0; j < D; ++j) o[j] = 0.f;

    for (int t = 0; t < ntiles; ++t) {
        // ---- S_t ----
        if (!mbar_wait(bar_s, (uint32_t)(t & 1), p.status)) failed = true;
        tc_fence_after_sync();
        if (t + 2 < ntiles) request_k(t + 2);                  // K_t is consumed
        cp_async_commit_tc();
        uint32_t sr[64];
        tmem_ld64(t_lane + C::kColS, sr);
        const int k0 = t * kTcKeys;
        float mx = -INFINITY;
        if (k0 + kTcKeys - 1 > pos_first) {                  // a tile on the diagonal: mask
#pragma unroll
            for (int j = 0; j < 64; ++j) {
                const float v = k0 + j <= pos ? __uint_as_float(sr[j]) : -INFINITY;
                sr[j] = __float_as_uint(v);
                mx = fmaxf(mx, v);
            }
        } else {
#pragma unroll
            for (int j = 0; j < 64; ++j) mx = fmaxf(mx, __uint_as_float(sr[j]));
        }
        // key 0 is in every row's range, so m_new is finite from the first tile on
        const float m_new = fmaxf(m_run, mx * sl2);
        const float alpha = fast_exp2(m_run - m_new);
        m_run = m_new;
        float rsum = 0.f;
        uint32_t pk[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const float p0 = fast_exp2(fmaf(__uint_as_float(sr[2 * j]), sl2, -m_new));
            const float p1 = fast_exp2(fmaf(__uint_as_float(sr[2 * j + 1]), sl2, -m_new));
            rsum += p0 + p1;
            pk[j] = pack_bf16x2(p0, p1);
        }
        l_run = l_run * alpha + rsum;
        const uint32_t prow = s_p + tid * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c)
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(prow + ((c ^ (tid & 7)) << 4)),
                         "r"(pk[4 * c]), "r"(pk[4 * c + 1]), "r"(pk[4 * c + 2]), "r"(pk[4 * c + 3])
                         : "memory");
        // ---- P_t V_t and Q K_{t+1}: K_{t+1} and V_{t+1} must have landed ----
        cp_async_wait_tc<1>();
        if (kTma && L - k0 < kTcKeys) {
            // the last tile: V rows past the sequence (stale pool rows, or never copied) are
            // zeroed so that P = 0 there cannot meet a NaN pattern
            if (!mbar_wait(bar_v + 8 * (t & 1), (uint32_t)((t >> 1) & 1), p.status)) failed = true;
            const uint32_t vt = s_v + (t & 1) * C::kKVBytes;
            for (int i = tid; i < (kTcKeys - (L - k0)) * (D / 8); i += kTcThreads) {
                const int row = (L - k0) + i / (D / 8), c = i % (D / 8);
                asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(vt + sw128<kTcKeys>(row, c)),
                             "r"(0u)
                             : "memory");
            }
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        tc_fence_before_sync();
        if (__syncthreads_or(failed)) break;
        if (tid == 0) {
            tc_fence_after_sync();
            wait_kv(bar_v, t);
            issue_o(t);
            if (t + 1 < ntiles) {
                wait_kv(bar_k, t + 1);
                issue_s(t + 1);
            }
        }
        // ---- O = alpha O + O_t ----
        if (!mbar_wait(bar_o, (uint32_t)(t & 1), p.status)) failed = true;
        tc_fence_after_sync();
        if (t + 2 < ntiles) request_v(t + 2);                  // V_t is consumed
        cp_async_commit_tc();
        if (t + 3 < ntiles) fetch_ids(t + 3);
#pragma unroll
        for (int h = 0; h < D / 64; ++h) {
            uint32_t orow[64];
            tmem_ld64(t_lane + C::kColO + h * 64, orow);
#pragma unroll
            for (int j = 0; j < 64; ++j) o[h * 64 + j] = fmaf(o[h * 64 + j], alpha, __uint_as_float(orow[j]));
        }
        tc_fence_before_sync();
    }
    cp_async_wait_tc<0>();
    if (kTma && tid == 0) {                                  // only after an early exit: copies in flight
        for (int t = k_seen + 1; t <= k_req; ++t) wait_kv(bar_k, t);
        for (int t = v_seen + 1; t <= v_req; ++t) wait_kv(bar_v, t);
    }
    tc_fence_before_sync();
    const bool aborted = __syncthreads_or(failed);
    if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, C::kTmemCols);
    }
    if (aborted || R >= rows) return;
    // ---- out = O / l ----
    const int tok = R / G, g = R - tok * G;
    const float inv = 1.f / l_run;
    uint16_t* out = p.out + ((size_t)(q0 + tok) * Hq + (size_t)kvh * G + g) * D;
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {
        uint4 w;
        w.x = pack_bf16x2(o[8 * c + 0] * inv, o[8 * c + 1] * inv);
        w.y = pack_bf16x2(o[8 * c + 2] * inv, o[8 * c + 3] * inv);
        w.z = pack_bf16x2(o[8 * c + 4] * inv, o[8 * c + 5] * inv);
        w.w = pack_bf16x2(o[8 * c + 6] * inv, o[8 * c + 7] * inv);
        *reinterpret_cast<uint4*>(out + 8 * c) = w;
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
    static std::atomic<EncodeTiledFn> fn{nullptr};
    EncodeTiledFn f = fn.load(std::memory_order_acquire);
    if (!f) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess) {
            f = reinterpret_cast<EncodeTiledFn>(ptr);
            fn.store(f, std::memory_order_release);
        }
    }
    return f;
}

// The pool as a 3-D bf16 tensor [blocks * Hkv][block_size][head_dim]; box = 64 dims x
// min(block_size, 64) tokens x 1, in 128-byte-swizzled rows.
bool make_pool_map(CUtensorMap* map, const void* base, const PrefillParams& p) {
    EncodeTiledFn fn = encode_tiled();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)p.head_dim, (cuuint64_t)p.block_size,
                                (cuuint64_t)p.num_blocks * p.num_kv_heads};
    const cuuint64_t strides[2] = {(cuuint64_t)p.head_dim * 2, (cuuint64_t)p.block_size * p.head_dim * 2};
    const cuuint32_t box[3] = {64u, (cuuint32_t)(p.block_size < kTcKeys ? p.block_size : kTcKeys), 1u};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, bool kTma>
cudaError_t launch_pf_tc(const PrefillParams& p, int max_q_len, cudaStream_t stream) {
    constexpr size_t smem = TcCfg<D>::kSmem;
    static std::atomic<uint64_t> attr_set{0};               // one bit per device
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!(attr_set.load(std::memory_order_acquire) & (1ull << dev))) {
        const cudaError_t e = cudaFuncSetAttribute(prefill_tc_kernel<D, kTma>,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        attr_set.fetch_or(1ull << dev, std::memory_order_acq_rel);
    }
    const int tiles = (max_q_len * p.group + kTcRows - 1) / kTcRows;
    if (tiles <= 0) return cudaSuccess;
    CUtensorMap km, vm;
    memset(&km, 0, sizeof km);
    memset(&vm, 0, sizeof vm);
    if (kTma && (!make_pool_map(&km, p.k_cache, p) || !make_pool_map(&vm, p.v_cache, p)))
        return cudaErrorInvalidValue;
    dim3 grid((unsigned)tiles, (unsigned)p.num_kv_heads, (unsigned)p.num_seqs);
    prefill_tc_kernel<D, kTma><<<grid, kTcThreads, smem, stream>>>(p, km, vm);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_tc(const PrefillParams& p, int max_q_len, cudaStream_t stream) {
    // TMA boxes need the block size to tile the 64-key tile (8, 16, 32, 64) or be a
    // multiple of it; any other size takes the cp.async gather
    const int bs = p.block_size;
    const bool tma = bs % kTcKeys == 0 || (bs >= 8 && kTcKeys % bs == 0);
    if (p.head_dim == 64) return tma ? launch_pf_tc<64, true>(p, max_q_len, stream)
                                     : launch_pf_tc<64, false>(p, max_q_len, stream);
    if (p.head_dim == 128) return tma ? launch_pf_tc<128, true>(p, max_q_len, stream)
                                      : launch_pf_tc<128, false>(p, max_q_len, stream);
    return cudaErrorInvalidValue;
}

}  // namespace pa
