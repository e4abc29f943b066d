// Internal declarations shared by the libpa translation units (host side).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "pa.h"

namespace pa {

// Bits of the device status word (first int32 of the decode workspace).
enum : int32_t {
    kStatusBadBlock = 1,
    kStatusBadLength = 2,
    kStatusTimeout = 4,
    kStatusSmemAlign = 8,   // shared memory off the 1024-byte boundary a swizzled operand needs
};

// Everything a decode kernel reads; passed by value as the kernel parameter.
struct DecodeParams {
    const uint16_t* q;             // [B][Hq][D]
    const uint16_t* k_cache;       // [N][Hkv][Bs][D]
    const uint16_t* v_cache;
    const int32_t* block_tables;   // [B][MB]
    const int32_t* context_lens;   // [B]
    const uint16_t* k_new;         // fused append: [B][Hkv][D] row of each sequence's newest
    const uint16_t* v_new;         //   token (position context_lens[b]-1), or null
    uint16_t* out;                 // [B][Hq][D]
    int32_t* status;               // device status word (workspace word 0)
    int32_t* work_counter;         // next work item to hand out (word 1, self-resetting)
    int32_t* done_counter;         // CTAs that have finished (word 2, self-resetting)
    int32_t* seq_desc;             // stream kernel: [Hkv/8][B] int4 {pieces, first CTA, first slot, 0}
    float* part_lse;               // [B][Hkv][S][G] log2-domain log-sum-exp
    float* part_o;                 // [B][Hkv][S][G][D] normalised partial outputs
    int32_t num_seqs;
    int32_t num_blocks;
    int32_t block_size;
    int32_t num_kv_heads;
    int32_t num_q_heads;
    int32_t head_dim;
    int32_t group;                 // Hq / Hkv
    int32_t max_blocks_per_seq;
    int32_t max_context_len;
    int32_t split_tokens;          // C: tokens per split (multiple of 64)
    int32_t max_splits;            // S = ceil(max_context_len / C)
    float scale_log2;              // scale * log2(e): scores are kept in the log2 domain
    int32_t early;                 // launched early (PA_FLAG_PDL): prefetch before the wait
    float rope_theta;              // > 0: rotate q and the new K rows at position L-1 (fused append)
    int32_t kv_fp8;                // caches hold E4M3 codes (uint8), values = code * scale
    float k_inv_scale, v_inv_scale;  // E4M3: float(1/scale) applied when quantizing new rows
    float out_scale;               // multiplies the normalised output (E4M3: the V scale; else 1)
    int32_t grid;                  // stream kernel: CTAs of the launch (bounds the merge's reads)

    int32_t selftest_stall;        // PA_FLAG_SELFTEST_STALL: CTA 0 of the stream kernel idles
    unsigned long long wait_ns;    // limit of every bounded wait in the stream kernel
};

// Which decode kernel a plan runs.
enum class DecodeKernel : int32_t {
    kSimt = 0,     // CUDA cores, one CTA per (sequence, kv head, split)
    kSplit = 1,    // tensor cores, persistent CTAs over (sequence, kv head, split) items
    kStream = 2,   // tensor cores, 8 kv heads per CTA, stream-partitioned slabs
};

struct DecodePlan {
    DecodeKernel kernel;
    int32_t split_tokens;          // kSimt / kSplit: tokens per split
    int32_t max_splits;            // kSimt / kSplit: splits per (sequence, kv head) at most
    int32_t grid;                  // kStream: persistent CTAs (partial slots: 2 per CTA)
    size_t off_desc, off_lse, off_o, off_qrot, bytes;
};

// Paged prefill: sequence b's last cu_q[b+1] - cu_q[b] tokens attend causally to its
// context_lens[b] cached tokens.
struct PrefillParams {
    const uint16_t* q;             // [total_q][Hq][D]
    const uint16_t* k_cache;
    const uint16_t* v_cache;
    const int32_t* block_tables;
    const int32_t* cu_q;           // [B + 1]
    const int32_t* context_lens;   // [B]
    uint16_t* out;                 // [total_q][Hq][D]
    int32_t* status;
    int32_t num_seqs, num_blocks, block_size, num_kv_heads, num_q_heads, head_dim, group;
    int32_t max_blocks_per_seq;
    int32_t max_q_len;             // the caller's bound on every sequence's query count
    float scale_log2;
};
cudaError_t launch_prefill(const PrefillParams& p, int max_q_len, cudaStream_t stream);
cudaError_t launch_prefill_tc(const PrefillParams& p, int max_q_len, cudaStream_t stream);
// warp-specialized tcgen05 prefill (TMA block sizes only: 8, 16, 32, 64 or multiples of 64)
cudaError_t launch_prefill_ws(const PrefillParams& p, int max_q_len, cudaStream_t stream);
bool prefill_ws_supports(int block_size);

constexpr size_t kWorkspaceAlign = 256;
// Limits of the decode kernels' bounded waits: normal calls, and PA_FLAG_SELFTEST_STALL calls
// (whose stalled waits are meant to run out quickly).
constexpr unsigned long long kDecodeWaitNs = 2000000000ull;   // 2 s
constexpr unsigned long long kSelftestWaitNs = 10000000ull;   // 10 ms

int num_sms_current_device(int* out);
int make_decode_plan(int32_t num_seqs, int32_t max_context_len, const pa_cache_desc& d,
                     const pa_decode_options* opt, DecodePlan* plan);

cudaError_t launch_append(const pa_bf16* k, const pa_bf16* v, const int64_t* slots, int32_t T,
                          pa_bf16* k_cache, pa_bf16* v_cache, const pa_cache_desc& d,
                          cudaStream_t stream);
cudaError_t launch_append_at_end(const DecodeParams& p, cudaStream_t stream);
// E4M3 append: codes of value * inv_scale (float product, nearest even, saturating).
cudaError_t launch_append_e4m3(const pa_bf16* k, const pa_bf16* v, const int64_t* slots, int32_t T,
                               float k_inv_scale, float v_inv_scale, uint8_t* k_cache,
                               uint8_t* v_cache, const pa_cache_desc& d, cudaStream_t stream);
cudaError_t launch_copy_blocks(pa_bf16* k_cache, pa_bf16* v_cache, const int32_t* copies, int32_t n,
                               const pa_cache_desc& d, cudaStream_t stream);
// RoPE + append through the slot mapping (pa_rope_append_kv).
cudaError_t launch_rope_append(const pa_bf16* q, pa_bf16* q_out, const pa_bf16* k, const pa_bf16* v,
                               const int32_t* positions, const int64_t* slots, int32_t T, float theta,
                               pa_bf16* k_cache, pa_bf16* v_cache, const pa_cache_desc& d,
                               cudaStream_t stream);
// RoPE + append of each sequence's newest token at position L-1 through the table, with the
// rotated q written to q_out (the fused call on the kernels that do not fuse it).
cudaError_t launch_rope_append_at_end(const DecodeParams& p, uint16_t* q_out, cudaStream_t stream);
cudaError_t launch_decode_simt(const DecodeParams& p, cudaStream_t stream);
cudaError_t launch_decode_tensor(const DecodeParams& p, cudaStream_t stream);
bool tensor_kernel_supports(const pa_cache_desc& d);
// pdl: launch as a programmatic dependent of the previous kernel on the stream.
cudaError_t launch_decode_stream(const DecodeParams& p, int grid, bool pdl, cudaStream_t stream);
cudaError_t launch_merge(const DecodeParams& p, bool stream_layout, bool pdl, cudaStream_t stream);
// Tokens per stage (the unit of the stream partition): 32 for E4M3 pools at head_dim 64, else 16.
int stream_slab_tokens(bool fp8, int head_dim);
bool stream_kernel_supports(const pa_cache_desc& d);
int stream_kernel_grid(const pa_cache_desc& d, int max_ctas, bool fp8);

}  // namespace pa
