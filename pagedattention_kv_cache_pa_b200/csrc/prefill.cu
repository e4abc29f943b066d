// Paged (chunked) prefill attention: every new token of a sequence attends, causally,
// to the sequence's paged KV cache.
//
// Prefill processes a prompt (or a chunk of it) at once, where decode processes one
// token (Nano-vLLM page, section "Prefill vs Decode"); the causal mask lets a token see
// only itself and earlier tokens (Tiny-vLLM summary page, section "고성능 추론을 위한 고급
// 최적화 기법").  Sequence b holds context_lens[b] = L tokens after this step's append; its
// last Tq = cu_q[b+1] - cu_q[b] tokens are the queries (positions L-Tq .. L-1).
//
// FlashAttention-style tiles, one CTA per (64 query rows, kv head, sequence): a row is a
// (query token, query head of the kv head's group) pair, so the G heads that share a kv
// head share its K/V tiles.  Four warps own 16 rows each.  K/V tiles of 64 keys are
// gathered through the block table with 16-byte cp.async copies, double-buffered, into
// 128-byte-swizzled rows; S = Q K^T and O += P V run on mma.sync m16n8k16 bf16 with
// ldmatrix fragments (P goes from the S accumulators straight into A operands), with an
// fp32 online softmax in the log2 domain and the causal mask on every tile.
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "pa_device.cuh"
#include "pa_internal.h"
#include "pa_ptx.cuh"

namespace pa {
namespace {

constexpr int kRows = 64;        // query rows per CTA
constexpr int kKeys = 64;        // keys per tile
constexpr int kWarps = 4;
constexpr int kThreadsPf = kWarps * 32;

// Byte offset of (row, 16-byte chunk) in a tile of rows of D bf16: 128-byte groups of
// chunks, chunk index XOR (row & 7) inside each group, so ldmatrix reads are conflict-free.
template <int D>
__device__ __forceinline__ uint32_t toff(int row, int chunk) {
    return (uint32_t)(row * (2 * D) + ((chunk >> 3) << 7) + (((chunk & 7) ^ (row & 7)) << 4));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool live) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(live ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <int D>
__global__ void __launch_bounds__(kThreadsPf) prefill_kernel(const PrefillParams p) {
    constexpr int kCh = D / 8;                           // 16-byte chunks per row
    constexpr int kTile = kKeys * D * 2;                 // bytes of a K (or V) tile
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t s_base = smem_u32(smem);
    const uint32_t s_q = s_base;                         // Q tile: kRows x D
    const uint32_t s_k = s_q + kRows * D * 2;            // K tiles: 2 x kTile
    const uint32_t s_v = s_k + 2 * kTile;                // V tiles: 2 x kTile

    const int b = blockIdx.z, kvh = blockIdx.y;
    const int G = p.group, Hq = p.num_q_heads, Hkv = p.num_kv_heads, Bs = p.block_size;
    const int q0 = p.cu_q[b], Tq = p.cu_q[b + 1] - q0;
    const int L = p.context_lens[b];
    const int cap = p.max_blocks_per_seq * Bs;
    if (Tq <= 0) return;
    if (L < Tq || L > cap || Tq > p.max_q_len) {         // fewer tokens than queries, past the table,
                                                         // or more queries than the grid holds
        if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.y == 0) raise_status(p.status, kStatusBadLength);
        return;
    }
    // the last row tiles of a chunk attend to the most keys: they take the first CTAs
    const int rows = Tq * G, ntile = (rows + kRows - 1) / kRows;
    const int tile = ntile - 1 - (int)blockIdx.x;
    if (tile < 0) return;
    const int r0 = tile * kRows;
    const int* table = p.block_tables + (size_t)b * p.max_blocks_per_seq;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    // keys needed: up to the last row's position
    const int last_tok = min(rows - 1, r0 + kRows - 1) / G;
    const int kend = L - Tq + last_tok + 1;
    const int ntiles = (kend + kKeys - 1) / kKeys;

    // ---- Q tile (rows past the chunk are zeros) ----
    for (int i = tid; i < kRows * kCh; i += kThreadsPf) {
        const int row = i / kCh, c = i - row * kCh, R = r0 + row;
        const bool live = R < rows;
        const int tok = live ? R / G : 0, g = live ? R - tok * G : 0;
        const uint16_t* src = p.q + (((size_t)(q0 + tok) * Hq + (size_t)kvh * G + g) * D + c * 8);
        cp_async16(s_q + toff<D>(row, c), src, live);
    }
    auto load_kv = [&](int t, int buf) {
        const int k0 = t * kKeys;
        for (int i = tid; i < kKeys * kCh; i += kThreadsPf) {
            const int j = i / kCh, c = i - j * kCh, kp = k0 + j;
            bool live = kp < L;
            size_t off = 0;
            if (live) {
                const int blk = __ldg(table + kp / Bs);
                if (blk < 0 || blk >= p.num_blocks) {
                    raise_status(p.status, kStatusBadBlock);
                    live = false;
                } else {
                    off = (((size_t)blk * Hkv + kvh) * Bs + kp % Bs) * D + c * 8;
                }
            }
            cp_async16(s_k + buf * kTile + toff<D>(j, c), p.k_cache + off, live);
            cp_async16(s_v + buf * kTile + toff<D>(j, c), p.v_cache + off, live);
        }
        cp_async_commit();
    };
    load_kv(0, 0);                                       // commits Q and tile 0 together

    // per-thread rows: r and r + 8 of the warp's 16; their positions
    const int r = lane >> 2, c = lane & 3, mi = lane >> 3, rr = lane & 7;
    int pos[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        const int R = r0 + warp * 16 + r + 8 * e;
        pos[e] = R < rows ? L - Tq + R / G : L - 1;      // padded rows: computed, not written
    }
    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
    float o_acc[D / 8][4];
#pragma unroll
    for (int n = 0; n < D / 8; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) o_acc[n][e] = 0.f;
    uint32_t qa[D / 16][4];
    const float sl2 = p.scale_log2;

    for (int t = 0; t < ntiles; ++t) {
        const int buf = t & 1;
        if (t + 1 < ntiles) {
            load_kv(t + 1, buf ^ 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        if (t == 0) {
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks)
                ldmatrix_x4(s_q + toff<D>(warp * 16 + ((mi & 1) << 3) + rr, 2 * ks + (mi >> 1)), qa[ks]);
        }
        const uint32_t kt = s_k + buf * kTile, vt = s_v + buf * kTile;
        // ---- S = Q K^T : 16 rows x 64 keys (8 n-tiles) ----
        float s[8][4];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) s[nt][e] = 0.f;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)
#pragma unroll
            for (int nt = 0; nt < 8; nt += 2) {
                uint32_t kb[4];
                ldmatrix_x4(kt + toff<D>((nt + (mi >> 1)) * 8 + rr, 2 * ks + (mi & 1)), kb);
                mma_bf16_16816(s[nt], qa[ks], kb[0], kb[1]);
                mma_bf16_16816(s[nt + 1], qa[ks], kb[2], kb[3]);
            }
        // ---- causal mask and online softmax (rows r and r + 8; a row's 4 lanes share it) ----
        const int k0 = t * kKeys;
        float mx[2] = {m_run[0], m_run[1]};
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int key = k0 + nt * 8 + 2 * c + (e & 1), hr = e >> 1;
                s[nt][e] = key <= pos[hr] ? s[nt][e] * sl2 : -INFINITY;
                mx[hr] = fmaxf(mx[hr], s[nt][e]);
            }
        float alpha[2], base[2];
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
            mx[hr] = fmaxf(mx[hr], __shfl_xor_sync(0xffffffffu, mx[hr], 1));
            mx[hr] = fmaxf(mx[hr], __shfl_xor_sync(0xffffffffu, mx[hr], 2));
            base[hr] = mx[hr] == -INFINITY ? 0.f : mx[hr];
            alpha[hr] = fast_exp2(m_run[hr] - base[hr]);
            m_run[hr] = mx[hr];
        }
        float rsum[2] = {0.f, 0.f};
        uint32_t pa_[4][4];                              // P as A operands: 4 k-steps of 16 keys
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            const float p0 = fast_exp2(s[nt][0] - base[0]), p1 = fast_exp2(s[nt][1] - base[0]);
            const float p2 = fast_exp2(s[nt][2] - base[1]), p3 = fast_exp2(s[nt][3] - base[1]);
            rsum[0] += p0 + p1;
            rsum[1] += p2 + p3;
            pa_[nt >> 1][(nt & 1) * 2 + 0] = pack_bf16x2(p0, p1);   // row r
            pa_[nt >> 1][(nt & 1) * 2 + 1] = pack_bf16x2(p2, p3);   // row r + 8
        }
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
            rsum[hr] += __shfl_xor_sync(0xffffffffu, rsum[hr], 1);
            rsum[hr] += __shfl_xor_sync(0xffffffffu, rsum[hr], 2);
            l_run[hr] = l_run[hr] * alpha[hr] + rsum[hr];
        }
#pragma unroll
        for (int n = 0; n < D / 8; ++n) {
            o_acc[n][0] *= alpha[0];
            o_acc[n][1] *= alpha[0];
            o_acc[n][2] *= alpha[1];
            o_acc[n][3] *= alpha[1];
        }
        // ---- O += P V : A = P (rows x 16 keys), B = V (16 keys x 8 dims) via ldmatrix.trans ----
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            // A fragment order: (row r, keys 2c..), (row r+8, keys 2c..), (row r, keys 8+2c..), (row r+8, ..)
            const uint32_t a[4] = {pa_[kk][0], pa_[kk][1], pa_[kk][2], pa_[kk][3]};
#pragma unroll
            for (int nd = 0; nd < D / 8; nd += 2) {
                uint32_t vb[4];
                ldmatrix_x4_trans(vt + toff<D>(16 * kk + ((mi & 1) << 3) + rr, nd + (mi >> 1)), vb);
                mma_bf16_16816(o_acc[nd], a, vb[0], vb[1]);
                mma_bf16_16816(o_acc[nd + 1], a, vb[2], vb[3]);
            }
        }
        __syncthreads();                                 // this buffer is refilled next
    }
    // ---- out = O / l ----
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
        const int R = r0 + warp * 16 + r + 8 * hr;
        if (R >= rows) continue;
        const int tok = R / G, g = R - tok * G;
        const float inv = 1.f / l_run[hr];
        uint16_t* o = p.out + ((size_t)(q0 + tok) * Hq + (size_t)kvh * G + g) * D;
#pragma unroll
        for (int n = 0; n < D / 8; ++n)
            *reinterpret_cast<uint32_t*>(o + n * 8 + 2 * c) =
                pack_bf16x2(o_acc[n][2 * hr] * inv, o_acc[n][2 * hr + 1] * inv);
    }
}

template <int D>
cudaError_t launch_pf(const PrefillParams& p, int max_q_len, cudaStream_t stream) {
    const size_t smem = (size_t)kRows * D * 2 + 4 * (size_t)kKeys * D * 2;
    static std::atomic<uint64_t> attr_set{0};           // one bit per device
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!(attr_set.load(std::memory_order_acquire) & (1ull << dev))) {
        const cudaError_t e = cudaFuncSetAttribute(prefill_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   (int)smem);
        if (e != cudaSuccess) return e;
        attr_set.fetch_or(1ull << dev, std::memory_order_acq_rel);
    }
    const int tiles = (max_q_len * p.group + kRows - 1) / kRows;
    if (tiles <= 0) return cudaSuccess;
    dim3 grid((unsigned)tiles, (unsigned)p.num_kv_heads, (unsigned)p.num_seqs);
    prefill_kernel<D><<<grid, kThreadsPf, smem, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill(const PrefillParams& p, int max_q_len, cudaStream_t stream) {
    if (p.head_dim == 64) return launch_pf<64>(p, max_q_len, stream);
    if (p.head_dim == 128) return launch_pf<128>(p, max_q_len, stream);
    return cudaErrorInvalidValue;
}

}  // namespace pa
