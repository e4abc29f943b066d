// Paged (chunked) prefill attention on the fifth-generation tensor cores, warp-specialized.
//
// The operation is the one of prefill_tc.cu: sequence b holds L = context_lens[b] tokens
// after this step's append, its last Tq = cu_q[b+1] - cu_q[b] tokens are the queries
// (positions L-Tq .. L-1), and the query at position p attends to cache tokens 0..p
// (Nano-vLLM page, section "Prefill vs Decode"; causal mask: Tiny-vLLM summary page,
// section "고성능 추론을 위한 고급 최적화 기법").
//
// Persistent CTAs, as many as fit on the GPU at once.  The work items are (128 query rows, kv
// head, sequence), ordered row tile by row tile from the end of every chunk, so the items
// with the most keys come first; the CTAs take them round by round in zigzag.  Tile
// counters, barrier phases and tensor-memory buffers run on across a CTA's items, so an
// item's Q load and first scores overlap the previous item's last tiles.  6 warps with one
// job each hand work to one another through mbarriers only (no CTA-wide barrier inside the
// loop):
//   warps 0-3  softmax: thread i owns row i (tensor-memory lane i).  Per 64-key tile t it
//              reads its row of S_t from tensor memory, masks it causally, and writes the
//              probabilities P_t (bf16, two to a 32-bit column) back to tensor memory, where
//              the P V MMA takes them as its A operand (no shared-memory round trip).
//   warp 4     MMA issue (one thread): S_t = Q K_t^T into one of two score buffers in tensor
//              memory two tiles ahead, and, once P_t is written, O += P_t V_t, accumulated in
//              tensor memory across tiles.  The scores of the next tile are ready before the
//              softmax warps finish this one, so no MMA latency sits between two tiles.
//   warp 5     TMA: K and V tiles of 64 keys into a ring of stages, one box of 64 dims x
//              min(Bs, 64) tokens per block and 64-dim atom, swizzled by the copy engine; a
//              stage is refilled once the MMAs that read it have completed.
//   Q: two buffers.  The softmax warps request the next item's Q rows (cp.async, zeros past
//   the chunk) when an item starts and publish them when it ends.
//   An item's first P V, which overwrites O, waits until the softmax warps have read the
//   previous item's O out of tensor memory.
// Online softmax with O in tensor memory: a row keeps its running max m until a tile raises
// it by more than 8 (log2 domain); only then is the row's O scaled by 2^(m - m_new) in
// tensor memory (load, scale, store), after the P V of the previous tile has completed, and m
// replaced.  In between, probabilities are 2^(s - m) <= 2^8, which bf16 and the fp32 sums
// carry without loss of relative precision.  P has two tensor-memory buffers: P_t is written
// once the P V of tile t-2, which read the same buffer, has completed.
// Tensor memory per CTA: S 2 x 64 columns, O D columns, P 2 x 32 columns (256 columns at
// D = 64, two CTAs per SM; 512 at D = 128, one CTA per SM).
//
// Every wait is bounded (2 s, then the timeout status bit).  On a timeout each warp leaves
// its loop; the MMA thread drains the TMA copies it has not seen land and waits for its own
// MMAs, and the tensor memory is freed before the CTA exits.
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <atomic>
#include <cstring>

#include "pa_device.cuh"
#include "pa_internal.h"
#include "pa_ptx.cuh"
#include "pa_umma.cuh"

namespace pa {
namespace {

constexpr int kWsRows = 128;     // query rows per CTA (tensor-memory lanes)
constexpr int kWsKeys = 64;      // keys per tile
constexpr int kWsThreads = 192;  // 4 softmax warps, the MMA warp, the TMA warp
constexpr float kRescaleLog2 = 8.f;

template <int D>
struct WsCfg {
    // K/V ring.  Shared memory also bounds residency, so that no CTA's tensor-memory allocation
    // waits for a neighbour's: D = 64 needs 96 KB (three CTAs would not fit in 228 KB, and two
    // allocate 2 x 256 columns), D = 128 needs 160 KB (one CTA, 512 columns)
    static constexpr int kStages = D == 64 ? 4 : 3;
    static constexpr int kQBytes = kWsRows * D * 2;
    static constexpr int kKVBytes = kWsKeys * D * 2;       // one K (or V) tile
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kOffQ + 2 * kQBytes;      // Q: two buffers (this item's, the next's)
    static constexpr int kOffV = kOffK + kStages * kKVBytes;
    static constexpr int kOffBar = kOffV + kStages * kKVBytes;
    // barriers (8 bytes each): s_full[2], p_full, o_done[2], drain, q_full[2], o_free,
    // k_full[S], v_full[S], kv_empty[S]; then the tensor-memory address and the last tile the
    // TMA warp requested
    static constexpr int kBars = 9 + 3 * kStages;
    static constexpr int kSmem = kOffBar + kBars * 8 + 16;
    static constexpr int kColS = 0;                         // S: two buffers of 64 fp32 columns
    static constexpr int kColO = 128;                       // O: D fp32 columns
    static constexpr int kColP = kColO + D;                 // P: two buffers of 64 bf16 (32 columns)
    static constexpr uint32_t kTmemCols = D == 64 ? 256 : 512;
    // D = 64: two CTAs per SM (each softmax thread keeps its row of S in 64 registers while it
    // scales its row of O, which three CTAs of six warps would spill); D = 128: one
    static constexpr int kMinBlocks = D == 64 ? 2 : 1;
    static_assert(kMinBlocks * (kSmem + 1024) <= 228 * 1024 && (kMinBlocks + 1) * (kSmem + 1024) > 228 * 1024,
                  "shared memory must hold exactly kMinBlocks CTAs per SM");
    static_assert(kMinBlocks * kTmemCols <= 512, "tensor memory of the resident CTAs");
};

template <int ROWS>
__device__ __forceinline__ uint32_t ws_sw128(int row, int c) {
    return (uint32_t)((c >> 3) * (ROWS * 128) + row * 128 + ((((c & 7) ^ (row & 7))) << 4));
}

__device__ __forceinline__ void ws_cp_async16(uint32_t dst, const void* src, bool live) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(live ? 16 : 0)
                 : "memory");
}

// Row arithmetic two lanes at a time: three-input maximum and packed fp32 pairs (one
// instruction for two FMAs or two adds).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}
__device__ __forceinline__ uint64_t f2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2_split(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// 32 columns of this thread's lane of tensor memory, scaled by a and stored back.
__device__ __forceinline__ void tmem_scale32(uint32_t taddr, float a) {
    uint32_t r[32];
    tmem_ld32(taddr, r);
#pragma unroll
    for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(__uint_as_float(r[j]) * a);
    tmem_st32(taddr, r);
}

// The item a CTA takes in its round r: rounds of grid items in order, CTAs in zigzag (forward
// in even rounds, backward in odd ones), so that with items in decreasing size every CTA's
// total comes out close to the mean.
__device__ __forceinline__ long long ws_index(long long r) {
    return r * gridDim.x + ((r & 1) ? gridDim.x - 1 - blockIdx.x : blockIdx.x);
}

// One work item: 128 query rows (a row tile) of one kv head of one sequence.
struct WsItem {
    int b, kvh, q0, Tq, L, rows, r0, ntiles, pos_first;
};

// Item i: the t-th row tile from the end of every chunk for t = i / (B Hkv) (the last row
// tiles attend to the most keys, so every sequence's longest items come first), then the
// sequence, then the kv head.  Returns 1 for an item to run, 0 for none (a chunk with fewer
// row tiles, or no queries), -1 for a sequence whose lengths cannot hold its queries (fewer
// tokens than queries, past the table, or more queries than max_q_len).
__device__ __forceinline__ int ws_item(const PrefillParams& p, long long i, WsItem& it, bool& tile0) {
    const long long nsh = (long long)p.num_seqs * p.num_kv_heads;
    int t_rev, rem;
    if (i <= 0x7fffffffLL && nsh <= 0x7fffffffLL) {          // 32-bit division where it fits
        t_rev = (int)((unsigned)i / (unsigned)nsh);
        rem = (int)((unsigned)i - (unsigned)t_rev * (unsigned)nsh);
    } else {
        t_rev = (int)(i / nsh);
        rem = (int)(i - (long long)t_rev * nsh);
    }
    it.b = rem / p.num_kv_heads;
    it.kvh = rem - it.b * p.num_kv_heads;
    tile0 = t_rev == 0 && it.kvh == 0;
    it.q0 = p.cu_q[it.b];
    it.Tq = p.cu_q[it.b + 1] - it.q0;
    it.L = p.context_lens[it.b];
    if (it.Tq <= 0) return 0;
    if (it.L < it.Tq || it.L > p.max_blocks_per_seq * p.block_size || it.Tq > p.max_q_len) return -1;
    it.rows = it.Tq * p.group;
    const int tile = (it.rows + kWsRows - 1) / kWsRows - 1 - t_rev;
    if (tile < 0) return 0;
    it.r0 = tile * kWsRows;
    const int last_tok = min(it.rows - 1, it.r0 + kWsRows - 1) / p.group;
    it.ntiles = (it.L - it.Tq + last_tok + 1 + kWsKeys - 1) / kWsKeys;   // keys up to the last row's position
    it.pos_first = it.L - it.Tq + it.r0 / p.group;
    return 1;
}

template <int D>
__global__ void __launch_bounds__(kWsThreads, WsCfg<D>::kMinBlocks)
    prefill_ws_kernel(const PrefillParams p, const __grid_constant__ CUtensorMap kmap,
                      const __grid_constant__ CUtensorMap vmap) {
    using C = WsCfg<D>;
    constexpr int kCh = D / 8;                               // 16-byte chunks per row
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t s_base = smem_u32(smem);
    const uint32_t s_q = s_base + C::kOffQ, s_k = s_base + C::kOffK, s_v = s_base + C::kOffV;
    constexpr int ST = C::kStages;
    // barriers: s_full[2], p_full, o_done[2], drain, q_full[2], o_free, then per stage k_full,
    // v_full, kv_empty
    const uint32_t bar_s = s_base + C::kOffBar, bar_p = bar_s + 16, bar_o = bar_s + 24, bar_drain = bar_s + 40,
                   bar_qf = bar_s + 48, bar_of = bar_s + 64, bar_k = bar_s + 72,
                   bar_v = bar_k + 8 * ST, bar_e = bar_v + 8 * ST;
    const uint32_t s_tmem = bar_s + C::kBars * 8;
    volatile int* s_kreq = reinterpret_cast<volatile int*>(smem + C::kOffBar + C::kBars * 8 + 4);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = p.group, Hq = p.num_q_heads, Hkv = p.num_kv_heads, Bs = p.block_size;
    const long long n_items =
        (long long)p.num_seqs * Hkv * ((p.max_q_len * (long long)G + kWsRows - 1) / kWsRows);

    if (s_base & 1023u) {                                    // the swizzle needs 1024-byte-aligned tiles
        if (tid == 0) raise_status(p.status, kStatusSmemAlign);
        return;
    }
    if (warp == 0) {
        tmem_alloc(s_tmem, C::kTmemCols);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(bar_s, 1);
        mbar_init(bar_s + 8, 1);
        mbar_init(bar_p, 4);                                 // one arrival per softmax warp
        mbar_init(bar_o, 1);
        mbar_init(bar_o + 8, 1);
        mbar_init(bar_drain, 1);
        mbar_init(bar_qf, 4);                                // one arrival per softmax warp
        mbar_init(bar_qf + 8, 4);
        mbar_init(bar_of, 4);                                // one arrival per softmax warp
        for (int i = 0; i < ST; ++i) {
            mbar_init(bar_k + 8 * i, 1);
            mbar_init(bar_v + 8 * i, 1);
            mbar_init(bar_e + 8 * i, 1);
        }
        *s_kreq = -1;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    uint32_t tmem;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(tmem) : "r"(s_tmem) : "memory");
    bool failed = false;
    int k_seen = -1, v_seen = -1;                            // MMA thread: last K / V tile seen landed
    WsItem it;
    bool tile0;

    if (warp == 5) {
        // ================================ TMA ================================
        // Per item its K and V tiles into the ring; tile counter g runs over items.
        const int rb = Bs < kWsKeys ? Bs : kWsKeys, nslot = kWsKeys / rb;
        int g = 0;
        for (long long r = 0, i = ws_index(0); i < n_items && !failed; i = ws_index(++r)) {
            const int st_item = ws_item(p, i, it, tile0);
            if (st_item < 0 && tile0 && lane == 0) raise_status(p.status, kStatusBadLength);
            if (st_item <= 0) continue;
            const int* table = p.block_tables + (size_t)it.b * p.max_blocks_per_seq;
            for (int t = 0; t < it.ntiles; ++t, ++g) {
                const int st = g % ST;
                if (g >= ST) {                               // the MMAs of tile g - ST have completed
                    bool ok = true;
                    if (lane == 0) ok = mbar_wait(bar_e + 8 * st, (uint32_t)((g / ST - 1) & 1), p.status);
                    if (!__shfl_sync(0xffffffffu, ok, 0)) {
                        failed = true;
                        break;
                    }
                }
                const int kp = t * kWsKeys + lane * rb;
                bool valid = lane < nslot && kp < it.L;
                int id = valid ? __ldg(table + kp / Bs) : 0;
                if (valid && (id < 0 || id >= p.num_blocks)) {
                    raise_status(p.status, kStatusBadBlock);
                    valid = false;
                }
                const unsigned m = __ballot_sync(0xffffffffu, valid);
                const uint32_t bytes = (uint32_t)(__popc(m) * rb * 128 * (D / 64));
                if (lane == 0) {
                    mbar_arrive_expect_tx(bar_k + 8 * st, bytes);
                    mbar_arrive_expect_tx(bar_v + 8 * st, bytes);
                    *s_kreq = g;
                }
                __syncwarp();
                if (valid) {
                    const int z = id * Hkv + it.kvh, y = Bs > kWsKeys ? kp % Bs : 0;
#pragma unroll
                    for (int a = 0; a < D / 64; ++a) {
                        const uint32_t off = a * (kWsKeys * 128) + lane * rb * 128;
                        tma_load_3d(s_k + st * C::kKVBytes + off, &kmap, a * 64, y, z, bar_k + 8 * st);
                        tma_load_3d(s_v + st * C::kKVBytes + off, &vmap, a * 64, y, z, bar_v + 8 * st);
                    }
                }
            }
        }
    } else if (warp == 4) {
        // ================================ MMA ================================
        if (lane == 0) {
            constexpr uint32_t kIdescS = umma_idesc_bf16(kWsRows, kWsKeys, false);
            constexpr uint32_t kIdescO = umma_idesc_bf16(kWsRows, D, true);
            auto wait_k = [&](int gg) {
                if (!mbar_wait(bar_k + 8 * (gg % ST), (uint32_t)((gg / ST) & 1), p.status)) return false;
                k_seen = gg;
                return true;
            };
            auto wait_v = [&](int gg) {
                if (!mbar_wait(bar_v + 8 * (gg % ST), (uint32_t)((gg / ST) & 1), p.status)) return false;
                v_seen = gg;
                return true;
            };
            auto issue_s = [&](int gg, uint32_t qbuf) {      // S buffer gg & 1 = Q K^T over D / 16 K steps
                const uint32_t kt = s_k + (gg % ST) * C::kKVBytes;
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const uint64_t a = umma_desc_sw128(qbuf + (ks >> 2) * (kWsRows * 128) + (ks & 3) * 32, 16, 1024);
                    const uint64_t bd = umma_desc_sw128(kt + (ks >> 2) * (kWsKeys * 128) + (ks & 3) * 32, 16, 1024);
                    umma_bf16_ss(tmem + C::kColS + (gg & 1) * 64, a, bd, kIdescS, ks > 0);
                }
                umma_commit(bar_s + 8 * (gg & 1));
            };
            auto issue_o = [&](int gg, bool first) {         // O (+)= P V over 4 K steps of 16 keys
                const uint32_t vt = s_v + (gg % ST) * C::kKVBytes;
                const uint32_t pt = tmem + C::kColP + (gg & 1) * (kWsKeys / 2);   // P in tensor memory
#pragma unroll
                for (int kk = 0; kk < kWsKeys / 16; ++kk) {
                    const uint64_t bd = umma_desc_sw128(vt + kk * 16 * 128, kWsKeys * 128, 1024);
                    umma_bf16_ts(tmem + C::kColO, pt + kk * 8, bd, kIdescO, (!first || kk > 0) ? 1u : 0u);
                }
                umma_commit(bar_e + 8 * (gg % ST));          // K and V of the tile are free once these land
                umma_commit(bar_o + 8 * (gg & 1));
            };
            // per item: the scores of its first two tiles, then per tile P V and the scores two
            // tiles ahead; the first P V of an item waits until the softmax warps have read the
            // previous item's O out of tensor memory
            int g = 0, k = 0;
            bool ok = true;
            for (long long r = 0, i = ws_index(0); i < n_items && ok; i = ws_index(++r)) {
                if (ws_item(p, i, it, tile0) <= 0) continue;
                const int qb = k & 1, nt = it.ntiles;
                const uint32_t qbuf = s_q + qb * C::kQBytes;
                ok = mbar_wait(bar_qf + 8 * qb, (uint32_t)((k >> 1) & 1), p.status) && wait_k(g);
                if (!ok) break;
                tc_fence_after_sync();
                issue_s(g, qbuf);
                if (nt > 1) {
                    if (!(ok = wait_k(g + 1))) break;
                    issue_s(g + 1, qbuf);
                }
                for (int t = 0; t < nt && ok; ++t) {
                    const int gg = g + t;
                    ok = mbar_wait(bar_p, (uint32_t)(gg & 1), p.status) && wait_v(gg) &&
                         (t > 0 || k == 0 || mbar_wait(bar_of, (uint32_t)((k - 1) & 1), p.status));
                    if (!ok) break;
                    tc_fence_after_sync();
                    issue_o(gg, t == 0);
                    if (t + 2 < nt) {
                        if (!(ok = wait_k(gg + 2))) break;
                        issue_s(gg + 2, qbuf);
                    }
                }
                g += nt;
                ++k;
            }
            if (!ok) failed = true;
        }
        __syncwarp();
    } else {
        // ============================== softmax ==============================
        const uint32_t t_lane = tmem + ((uint32_t)(warp * 32) << 16);   // this warp's 32 lanes
        const float sl2 = p.scale_log2;
        // P V of tile gg: its barrier (buffer gg & 1) completes once per use
        auto wait_o = [&](int gg) {
            return warp_wait(bar_o + 8 * (gg & 1), (uint32_t)((gg >> 1) & 1), p.status);
        };
        // Q of an item into buffer k & 1, requested by these warps when the item before it
        // starts (that buffer's last reader, the S MMAs of item k - 2, finished before any
        // score of item k - 1 reached these warps); complete and published when that item ends
        // thread tid copies chunk tid % kCh of rows tid / kCh + j * (128 / kCh): one division
        // for its first row, then a carry per step of 128 / kCh rows
        constexpr int kRowStep = 128 / kCh;
        auto load_q = [&](const WsItem& w, int qb) {
            const uint32_t qbuf = s_q + qb * C::kQBytes;
            const int tok_step = kRowStep / G, g_step = kRowStep - tok_step * G;
            const int ch = tid % kCh;
            int row = tid / kCh, R = w.r0 + row, tok = R / G, gq = R - tok * G;
#pragma unroll 4
            for (int j = 0; j < kWsRows / kRowStep; ++j) {
                const bool live = R < w.rows;
                const uint16_t* src =
                    p.q + (((size_t)(w.q0 + (live ? tok : 0)) * Hq + (size_t)w.kvh * G + (live ? gq : 0)) * D + ch * 8);
                ws_cp_async16(qbuf + ws_sw128<kWsRows>(row, ch), src, live);
                row += kRowStep;
                R += kRowStep;
                tok += tok_step;
                gq += g_step;
                if (gq >= G) {
                    gq -= G;
                    ++tok;
                }
            }
        };
        auto publish_q = [&](int qb) {
            asm volatile("cp.async.wait_all;" ::: "memory");
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_qf + 8 * qb);
        };
        auto next_item = [&](long long& r, WsItem& w) {      // the CTA's next item with work
            for (long long i = ws_index(++r); i < n_items; i = ws_index(++r))
                if (ws_item(p, i, w, tile0) > 0) return true;
            return false;
        };
        long long r = -1;
        WsItem nx;
        bool has = next_item(r, it);
        if (has) {
            load_q(it, 0);
            publish_q(0);
        }
        int g = 0, k = 0;
        while (has && !failed) {
            const bool has_nx = next_item(r, nx);
            if (has_nx) load_q(nx, (k + 1) & 1);
            const int R = it.r0 + tid, L = it.L;
            const int pos = R < it.rows ? L - it.Tq + R / G : L - 1;   // padded rows: computed, not written
            float m_run = -INFINITY, l_run = 0.f;
            for (int t = 0; t < it.ntiles; ++t) {
                const int gg = g + t;
                if (!warp_wait(bar_s + 8 * (gg & 1), (uint32_t)((gg >> 1) & 1), p.status)) {
                    failed = true;
                    break;
                }
                tc_fence_after_sync();
                uint32_t sr[64];
                tmem_ld64(t_lane + C::kColS + (gg & 1) * 64, sr);
                const int k0 = t * kWsKeys;
                if (k0 + kWsKeys - 1 > it.pos_first) {       // a tile on the diagonal: mask
#pragma unroll
                    for (int j = 0; j < 64; ++j)
                        if (k0 + j > pos) sr[j] = __float_as_uint(-INFINITY);
                }
                // the row max over four independent chains of three-input maxima (a single
                // chain of dependent maxima would sit on the tile's critical path)
                float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                for (int j = 0; j < 64; j += 2)
                    mq[(j >> 1) & 3] = fmax3(mq[(j >> 1) & 3], __uint_as_float(sr[j]), __uint_as_float(sr[j + 1]));
                const float mx = fmax3(mq[0], mq[1], fmaxf(mq[2], mq[3]));
                // key 0 is in every row's range, so the max is finite from the first tile on
                const float m_new = fmaxf(m_run, mx * sl2);
                if (t == 0) {
                    m_run = m_new;
                } else {
                    const bool need = m_new > m_run + kRescaleLog2;
                    if (__any_sync(0xffffffffu, need)) {
                        // once O holds the previous tile in full, scale this row
                        if (!wait_o(gg - 1)) {
                            failed = true;
                            break;
                        }
                        tc_fence_after_sync();
                        const float a = need ? fast_exp2(m_run - m_new) : 1.f;
#pragma unroll
                        for (int h = 0; h < D / 32; ++h) tmem_scale32(t_lane + C::kColO + h * 32, a);
                        if (need) {
                            l_run *= a;
                            m_run = m_new;
                        }
                    }
                }
                // p = 2^(s sl2 - m) for two keys per packed FMA; the row sum in two independent
                // packed partial sums
                const uint64_t sc2 = f2(sl2, sl2), nm2 = f2(-m_run, -m_run);
                uint64_t rs2[2] = {f2(0.f, 0.f), f2(0.f, 0.f)};
                uint32_t pk[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    float x0, x1;
                    f2_split(f2_fma(f2(__uint_as_float(sr[2 * j]), __uint_as_float(sr[2 * j + 1])), sc2, nm2), x0, x1);
                    const float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
                    rs2[j & 1] = f2_add(rs2[j & 1], f2(p0, p1));
                    pk[j] = pack_bf16x2(p0, p1);
                }
                float r0a, r0b, r1a, r1b;
                f2_split(rs2[0], r0a, r0b);
                f2_split(rs2[1], r1a, r1b);
                l_run += (r0a + r1a) + (r0b + r1b);
                if (gg >= 2 && !wait_o(gg - 2)) {            // the P V that read this P buffer is done
                    failed = true;
                    break;
                }
                tmem_st32(t_lane + C::kColP + (gg & 1) * (kWsKeys / 2), pk);   // P: this row's 64 bf16
                if (L - k0 < kWsKeys) {
                    // the last tile: V rows past the sequence (stale pool rows, or never copied)
                    // are zeroed so that P = 0 there cannot meet a NaN pattern; the MMA reads V
                    // only after all four warps' arrivals below, so each warp zeroes its share
                    if (!warp_wait(bar_v + 8 * (gg % ST), (uint32_t)((gg / ST) & 1), p.status)) {
                        failed = true;
                        break;
                    }
                    const uint32_t vt = s_v + (gg % ST) * C::kKVBytes;
                    for (int c = tid; c < (kWsKeys - (L - k0)) * (D / 8); c += 128) {
                        const int row = (L - k0) + c / (D / 8), ch = c % (D / 8);
                        asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(vt + ws_sw128<kWsKeys>(row, ch)),
                                     "r"(0u)
                                     : "memory");
                    }
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                }
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_p);
            }
            if (failed || !wait_o(g + it.ntiles - 1)) {
                failed = true;
                break;
            }
            // O of this item out of tensor memory, then free it for the next item's first P V
            tc_fence_after_sync();
            const int tok = R / G, gq = R - tok * G;
            const float inv = 1.f / l_run;
            uint16_t* out = p.out + ((size_t)(it.q0 + tok) * Hq + (size_t)it.kvh * G + gq) * D;
#pragma unroll
            for (int h = 0; h < D / 32; ++h) {
                uint32_t o[32];
                tmem_ld32(t_lane + C::kColO + h * 32, o);   // warp-wide: padded rows join the load
                if (R < it.rows) {
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        uint4 w;
                        w.x = pack_bf16x2(__uint_as_float(o[8 * c + 0]) * inv, __uint_as_float(o[8 * c + 1]) * inv);
                        w.y = pack_bf16x2(__uint_as_float(o[8 * c + 2]) * inv, __uint_as_float(o[8 * c + 3]) * inv);
                        w.z = pack_bf16x2(__uint_as_float(o[8 * c + 4]) * inv, __uint_as_float(o[8 * c + 5]) * inv);
                        w.w = pack_bf16x2(__uint_as_float(o[8 * c + 6]) * inv, __uint_as_float(o[8 * c + 7]) * inv);
                        *reinterpret_cast<uint4*>(out + h * 32 + 8 * c) = w;
                    }
                }
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_of);
            if (has_nx) publish_q((k + 1) & 1);
            g += it.ntiles;
            ++k;
            it = nx;
            has = has_nx;
        }
        asm volatile("cp.async.wait_all;" ::: "memory");     // nothing left in flight at exit
    }
    // every role is done issuing: the MMA thread drains what may still be in flight (after a
    // timed-out wait: copies requested but never seen to land), then its own MMAs
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 4 && lane == 0) {
        const int req = *s_kreq;
        for (int t = k_seen + 1; t <= req; ++t) mbar_wait(bar_k + 8 * (t % ST), (uint32_t)((t / ST) & 1), p.status);
        for (int t = v_seen + 1; t <= req; ++t) mbar_wait(bar_v + 8 * (t % ST), (uint32_t)((t / ST) & 1), p.status);
        umma_commit(bar_drain);
        mbar_wait(bar_drain, 0u, p.status);
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn ws_encode_tiled() {
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
bool ws_pool_map(CUtensorMap* map, const void* base, const PrefillParams& p) {
    EncodeTiledFn fn = ws_encode_tiled();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)p.head_dim, (cuuint64_t)p.block_size,
                                (cuuint64_t)p.num_blocks * p.num_kv_heads};
    const cuuint64_t strides[2] = {(cuuint64_t)p.head_dim * 2, (cuuint64_t)p.block_size * p.head_dim * 2};
    const cuuint32_t box[3] = {64u, (cuuint32_t)(p.block_size < kWsKeys ? p.block_size : kWsKeys), 1u};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
cudaError_t launch_ws(const PrefillParams& p, int max_q_len, cudaStream_t stream) {
    constexpr size_t smem = WsCfg<D>::kSmem;
    static std::atomic<uint64_t> attr_set{0};               // one bit per device
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!(attr_set.load(std::memory_order_acquire) & (1ull << dev))) {
        const cudaError_t e = cudaFuncSetAttribute(prefill_ws_kernel<D>,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        attr_set.fetch_or(1ull << dev, std::memory_order_acq_rel);
    }
    const int tiles = (max_q_len * p.group + kWsRows - 1) / kWsRows;
    if (tiles <= 0) return cudaSuccess;
    CUtensorMap km, vm;
    memset(&km, 0, sizeof km);
    memset(&vm, 0, sizeof vm);
    if (!ws_pool_map(&km, p.k_cache, p) || !ws_pool_map(&vm, p.v_cache, p)) return cudaErrorInvalidValue;
    // persistent: as many CTAs as fit at once, each taking every grid-th work item
    int sms = 0;
    if (num_sms_current_device(&sms) != PA_OK || sms <= 0) return cudaErrorInvalidDevice;
    const long long items = (long long)p.num_seqs * p.num_kv_heads * tiles;
    const long long ctas = std::min<long long>(items, (long long)sms * WsCfg<D>::kMinBlocks);
    dim3 grid((unsigned)ctas);
    prefill_ws_kernel<D><<<grid, kWsThreads, smem, stream>>>(p, km, vm);
    return cudaGetLastError();
}

}  // namespace

bool prefill_ws_supports(int block_size) {
    // TMA boxes: the block size tiles the 64-key tile (8, 16, 32, 64) or is a multiple of it
    return block_size % kWsKeys == 0 || (block_size >= 8 && kWsKeys % block_size == 0);
}

cudaError_t launch_prefill_ws(const PrefillParams& p, int max_q_len, cudaStream_t stream) {
    if (p.head_dim == 64) return launch_ws<64>(p, max_q_len, stream);
    if (p.head_dim == 128) return launch_ws<128>(p, max_q_len, stream);
    return cudaErrorInvalidValue;
}

}  // namespace pa
