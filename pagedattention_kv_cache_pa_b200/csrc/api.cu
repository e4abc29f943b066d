// C-ABI entry points of libpa: argument checks, the split plan, dispatch.
// The kernels themselves live in append.cu, decode_simt.cu and decode_tensor.cu.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include <atomic>

#include "pa.h"
#include "pa_internal.h"

namespace pa {

namespace {

constexpr int kMaxDevices = 64;
std::atomic<int> g_sm_count[kMaxDevices];

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

bool supported_block_size(int32_t bs) {
    return bs == 8 || bs == 16 || bs == 32 || bs == 64 || bs == 128 || bs == 256;
}

int check_desc(const pa_cache_desc* d) {
    if (!d) return PA_ERR_INVALID;
    if (d->num_blocks <= 0 || d->block_size <= 0 || d->num_kv_heads <= 0 ||
        d->num_q_heads <= 0 || d->head_dim <= 0 || d->max_blocks_per_seq <= 0)
        return PA_ERR_INVALID;
    if (d->num_q_heads % d->num_kv_heads != 0) return PA_ERR_INVALID;
    if ((int64_t)d->num_blocks * d->num_kv_heads * d->block_size > (int64_t)INT32_MAX)
        return PA_ERR_UNSUPPORTED;  // row index of the pool must fit in 32 bits
    return PA_OK;
}

// Optional override of the automatic split size, for tuning sweeps.
int32_t env_split_tokens() {
    static int32_t v = [] {
        const char* s = getenv("PA_SPLIT_TOKENS");
        return s ? (int32_t)atoi(s) : 0;
    }();
    return v;
}

int32_t env_kernel() {
    static int32_t v = [] {
        const char* s = getenv("PA_DECODE_KERNEL");
        if (!s) return (int32_t)PA_KERNEL_AUTO;
        if (!strcmp(s, "simt")) return (int32_t)PA_KERNEL_SIMT;
        if (!strcmp(s, "tensor")) return (int32_t)PA_KERNEL_TENSOR;
        if (!strcmp(s, "split")) return (int32_t)PA_KERNEL_TENSOR_SPLIT;
        return (int32_t)PA_KERNEL_AUTO;
    }();
    return v;
}

}  // namespace

int num_sms_current_device(int* out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return PA_ERR_CUDA;
    if (dev >= 0 && dev < kMaxDevices) {
        const int cached = g_sm_count[dev].load(std::memory_order_relaxed);
        if (cached > 0) {
            *out = cached;
            return PA_OK;
        }
    }
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        return PA_ERR_CUDA;
    if (dev >= 0 && dev < kMaxDevices) g_sm_count[dev].store(n, std::memory_order_relaxed);
    *out = n;
    return PA_OK;
}

// Decode plan: which kernel runs and how its workspace is laid out.
//  * kStream (tensor cores, Hkv a multiple of 8): persistent grid of every
//    resident CTA slot (or options->max_ctas); partial states: 2 per CTA.
//  * kSplit / kSimt: C tokens per split (a multiple of 64), a split grid of
//    ceil(max_context_len / C) per (sequence, kv head).  Automatic C: enough
//    work items for about 32 per SM if every sequence were max_context_len
//    long, never below 128 tokens.
// Workspace: [0, 256) status word and work counters; (kStream) one piece
// descriptor per (kv group, sequence); partial log-sum-exps; partial outputs.
int make_decode_plan(int32_t num_seqs, int32_t max_context_len, const pa_cache_desc& d,
                     const pa_decode_options* opt, DecodePlan* plan) {
    int32_t kernel = opt ? opt->kernel : PA_KERNEL_AUTO;
    if (kernel == PA_KERNEL_AUTO) kernel = env_kernel();
    if (kernel == PA_KERNEL_AUTO) kernel = PA_KERNEL_TENSOR;
    const int32_t G = d.num_q_heads / d.num_kv_heads;
    const size_t pairs = (size_t)num_seqs * d.num_kv_heads;
    auto up = [](size_t x) { return (x + kWorkspaceAlign - 1) / kWorkspaceAlign * kWorkspaceAlign; };
    plan->off_desc = kWorkspaceAlign;
    plan->off_lse = plan->off_desc;
    plan->off_qrot = 0;
    plan->grid = 0;
    plan->split_tokens = 0;
    plan->max_splits = 1;

    const bool fp8 = opt && opt->kv_dtype == PA_KV_E4M3;
    if (fp8 && !(kernel == PA_KERNEL_TENSOR && stream_kernel_supports(d)))
        return PA_ERR_UNSUPPORTED;   // E4M3 pools: the whole-group tensor kernel only
    if (kernel == PA_KERNEL_TENSOR && stream_kernel_supports(d)) {
        plan->kernel = DecodeKernel::kStream;
        plan->grid = stream_kernel_grid(d, opt ? opt->max_ctas : 0, fp8);
        if (plan->grid <= 0) return PA_ERR_CUDA;
        plan->off_lse = plan->off_desc + up((size_t)(d.num_kv_heads / 8) * num_seqs * 16);
        const size_t rows = (size_t)plan->grid * 2 * d.num_kv_heads * G;
        plan->off_o = plan->off_lse + up(rows * sizeof(float));
        plan->bytes = plan->off_o + up(rows * (size_t)d.head_dim * sizeof(float));
        return PA_OK;
    }
    if (kernel == PA_KERNEL_TENSOR || kernel == PA_KERNEL_TENSOR_SPLIT) {
        if (!tensor_kernel_supports(d)) return PA_ERR_UNSUPPORTED;
        plan->kernel = DecodeKernel::kSplit;
    } else if (kernel == PA_KERNEL_SIMT) {
        plan->kernel = DecodeKernel::kSimt;
    } else {
        return PA_ERR_INVALID;
    }
    int32_t C = opt ? opt->split_tokens : 0;
    if (C == 0) C = env_split_tokens();
    if (C < 0 || C % 64 != 0) return PA_ERR_INVALID;
    if (C == 0) {
        int sms = 0;
        const int rc = num_sms_current_device(&sms);
        if (rc != PA_OK) return rc;
        const int64_t work = (int64_t)num_seqs * d.num_kv_heads * (max_context_len > 0 ? max_context_len : 1);
        int64_t c = ceil_div(work, (int64_t)sms * 32);
        c = ceil_div(c, 64) * 64;
        if (c < 128) c = 128;
        C = (int32_t)(c > (1 << 30) ? (1 << 30) : c);
    }
    plan->split_tokens = C;
    plan->max_splits = (int32_t)(max_context_len > 0 ? ceil_div(max_context_len, C) : 1);
    if (plan->max_splits > 1) {
        plan->off_o = plan->off_lse + up(pairs * plan->max_splits * G * sizeof(float));
        plan->bytes = plan->off_o + up(pairs * plan->max_splits * G * (size_t)d.head_dim * sizeof(float));
    } else {
        plan->off_o = plan->off_lse;
        plan->bytes = plan->off_lse;
    }
    if (opt && opt->rope_theta > 0.f) {   // the rotated q of the fused call, from the rotation kernel
        plan->off_qrot = plan->bytes;
        plan->bytes += up((size_t)num_seqs * d.num_q_heads * d.head_dim * sizeof(uint16_t));
    }
    return PA_OK;
}

}  // namespace pa

using namespace pa;

extern "C" const char* pa_status_string(int status) {
    switch (status) {
        case PA_OK: return "PA_OK";
        case PA_ERR_INVALID: return "PA_ERR_INVALID: invalid argument";
        case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED: shape not built";
        case PA_ERR_CUDA: return "PA_ERR_CUDA: CUDA runtime error";
        case PA_ERR_WORKSPACE: return "PA_ERR_WORKSPACE: workspace missing, misaligned or too small";
        case PA_ERR_OOM_BLOCKS: return "PA_ERR_OOM_BLOCKS: not enough free blocks";
        case PA_ERR_SHARED_BLOCK: return "PA_ERR_SHARED_BLOCK: append into a shared block";
        case PA_ERR_BAD_BLOCK: return "PA_ERR_BAD_BLOCK: block id outside the pool";
        case PA_ERR_BAD_LENGTH: return "PA_ERR_BAD_LENGTH: context length beyond the bound";
        case PA_ERR_TIMEOUT: return "PA_ERR_TIMEOUT: a bounded wait in a kernel gave up";
        default: return "unknown status";
    }
}

extern "C" int pa_append_kv(const pa_bf16* k, const pa_bf16* v, const int64_t* slot_mapping,
                            int32_t num_tokens, pa_bf16* k_cache, pa_bf16* v_cache,
                            const pa_cache_desc* desc, void* stream) {
    int rc = check_desc(desc);
    if (rc != PA_OK) return rc;
    if (num_tokens < 0) return PA_ERR_INVALID;
    if (num_tokens == 0) return PA_OK;
    if (!k || !v || !slot_mapping || !k_cache || !v_cache) return PA_ERR_INVALID;
    if (desc->head_dim % 8 != 0) return PA_ERR_INVALID;
    if (!aligned(k, 16) || !aligned(v, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
        !aligned(slot_mapping, 8))
        return PA_ERR_INVALID;
    const cudaError_t e = launch_append(k, v, slot_mapping, num_tokens, k_cache, v_cache, *desc,
                                        (cudaStream_t)stream);
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

extern "C" int pa_rope_append_kv(const pa_bf16* q, pa_bf16* q_out, const pa_bf16* k, const pa_bf16* v,
                                 const int32_t* positions, const int64_t* slot_mapping,
                                 int32_t num_tokens, float rope_theta, pa_bf16* k_cache,
                                 pa_bf16* v_cache, const pa_cache_desc* desc, void* stream) {
    int rc = check_desc(desc);
    if (rc != PA_OK) return rc;
    if (num_tokens < 0 || !(rope_theta > 0.f) || !(rope_theta < INFINITY)) return PA_ERR_INVALID;
    if (desc->head_dim != 64 && desc->head_dim != 128) return PA_ERR_UNSUPPORTED;
    if (num_tokens == 0) return PA_OK;
    if (!q || !q_out || !k || !v || !positions || !slot_mapping || !k_cache || !v_cache)
        return PA_ERR_INVALID;
    if (!aligned(q, 16) || !aligned(q_out, 16) || !aligned(k, 16) || !aligned(v, 16) ||
        !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(slot_mapping, 8) ||
        !aligned(positions, 4))
        return PA_ERR_INVALID;
    const cudaError_t e = launch_rope_append(q, q_out, k, v, positions, slot_mapping, num_tokens,
                                             rope_theta, k_cache, v_cache, *desc, (cudaStream_t)stream);
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

extern "C" int pa_append_kv_e4m3(const pa_bf16* k, const pa_bf16* v, const int64_t* slot_mapping,
                                 int32_t num_tokens, float k_scale, float v_scale, uint8_t* k_cache,
                                 uint8_t* v_cache, const pa_cache_desc* desc, void* stream) {
    int rc = check_desc(desc);
    if (rc != PA_OK) return rc;
    if (num_tokens < 0 || desc->head_dim % 8 != 0 || !(k_scale > 0.f) || !(k_scale < INFINITY) ||
        !(v_scale > 0.f) || !(v_scale < INFINITY))
        return PA_ERR_INVALID;
    if (num_tokens == 0) return PA_OK;
    if (!k || !v || !slot_mapping || !k_cache || !v_cache || !aligned(k, 16) || !aligned(v, 16) ||
        !aligned(k_cache, 8) || !aligned(v_cache, 8) || !aligned(slot_mapping, 8))
        return PA_ERR_INVALID;
    const cudaError_t e = launch_append_e4m3(k, v, slot_mapping, num_tokens, 1.f / k_scale, 1.f / v_scale,
                                             k_cache, v_cache, *desc, (cudaStream_t)stream);
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

extern "C" int pa_prefill(const pa_bf16* q, const pa_bf16* k_cache, const pa_bf16* v_cache,
                          const int32_t* block_tables, const int32_t* cu_seqlens_q,
                          const int32_t* context_lens, int32_t num_seqs, int32_t max_q_len, float scale,
                          pa_bf16* out, void* workspace, size_t workspace_bytes,
                          const pa_cache_desc* desc, int32_t kernel, void* stream) {
    int rc = check_desc(desc);
    if (rc != PA_OK) return rc;
    if (num_seqs < 0 || num_seqs > 65535 || max_q_len < 0 || !(scale > 0.f) || !(scale < INFINITY))
        return PA_ERR_INVALID;
    if (kernel != PA_PREFILL_AUTO && kernel != PA_PREFILL_TCGEN05 && kernel != PA_PREFILL_MMA &&
        kernel != PA_PREFILL_TCGEN05_WS)
        return PA_ERR_INVALID;
    if (kernel == PA_PREFILL_TCGEN05_WS && !prefill_ws_supports(desc->block_size)) return PA_ERR_UNSUPPORTED;
    if (desc->head_dim != 64 && desc->head_dim != 128) return PA_ERR_UNSUPPORTED;
    if (desc->num_kv_heads > 65535) return PA_ERR_UNSUPPORTED;
    if (num_seqs == 0 || max_q_len == 0) return PA_OK;
    if ((int64_t)max_q_len * (desc->num_q_heads / desc->num_kv_heads) > (int64_t)64 * 65535)
        return PA_ERR_UNSUPPORTED;
    if (!q || !k_cache || !v_cache || !block_tables || !cu_seqlens_q || !context_lens || !out)
        return PA_ERR_INVALID;
    if (!aligned(q, 16) || !aligned(out, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
        !aligned(block_tables, 4) || !aligned(cu_seqlens_q, 4) || !aligned(context_lens, 4))
        return PA_ERR_INVALID;
    if (!workspace || !aligned(workspace, kWorkspaceAlign) || workspace_bytes < kWorkspaceAlign)
        return PA_ERR_WORKSPACE;
    PrefillParams p;
    p.q = q;
    p.k_cache = k_cache;
    p.v_cache = v_cache;
    p.block_tables = block_tables;
    p.cu_q = cu_seqlens_q;
    p.context_lens = context_lens;
    p.out = out;
    p.status = static_cast<int32_t*>(workspace);
    p.num_seqs = num_seqs;
    p.num_blocks = desc->num_blocks;
    p.block_size = desc->block_size;
    p.num_kv_heads = desc->num_kv_heads;
    p.num_q_heads = desc->num_q_heads;
    p.head_dim = desc->head_dim;
    p.group = desc->num_q_heads / desc->num_kv_heads;
    p.max_blocks_per_seq = desc->max_blocks_per_seq;
    p.max_q_len = max_q_len;
    p.scale_log2 = scale * 1.4426950408889634f;
    const cudaStream_t st = (cudaStream_t)stream;
    // automatic: the warp-specialized kernel where its TMA boxes tile the block size
    if (kernel == PA_PREFILL_AUTO)
        kernel = prefill_ws_supports(desc->block_size) ? PA_PREFILL_TCGEN05_WS : PA_PREFILL_TCGEN05;
    const cudaError_t e = kernel == PA_PREFILL_MMA          ? launch_prefill(p, max_q_len, st)
                          : kernel == PA_PREFILL_TCGEN05_WS ? launch_prefill_ws(p, max_q_len, st)
                                                            : launch_prefill_tc(p, max_q_len, st);
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

extern "C" int pa_copy_blocks(pa_bf16* k_cache, pa_bf16* v_cache, const int32_t* copies, int32_t n,
                              const pa_cache_desc* desc, void* stream) {
    int rc = check_desc(desc);
    if (rc != PA_OK) return rc;
    if (n < 0 || desc->head_dim % 8 != 0) return PA_ERR_INVALID;
    if (n == 0) return PA_OK;
    if (!k_cache || !v_cache || !copies || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
        !aligned(copies, 4))
        return PA_ERR_INVALID;
    const cudaError_t e = launch_copy_blocks(k_cache, v_cache, copies, n, *desc, (cudaStream_t)stream);
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

static int check_decode_shape(int32_t num_seqs, int32_t max_context_len, const pa_cache_desc* d) {
    int rc = check_desc(d);
    if (rc != PA_OK) return rc;
    if (num_seqs < 0 || num_seqs > 65535 || max_context_len < 0) return PA_ERR_INVALID;
    if (d->head_dim != 64 && d->head_dim != 128) return PA_ERR_UNSUPPORTED;
    if (!supported_block_size(d->block_size)) return PA_ERR_UNSUPPORTED;
    if (d->num_q_heads / d->num_kv_heads > 16) return PA_ERR_UNSUPPORTED;
    if (d->num_kv_heads > 65535) return PA_ERR_UNSUPPORTED;
    return PA_OK;
}

extern "C" size_t pa_decode_workspace_size_ex(int32_t num_seqs, int32_t max_context_len,
                                              const pa_cache_desc* desc,
                                              const pa_decode_options* options) {
    if (check_decode_shape(num_seqs, max_context_len, desc) != PA_OK) return 0;
    DecodePlan plan;
    if (make_decode_plan(num_seqs, max_context_len, *desc, options, &plan) != PA_OK) return 0;
    return plan.bytes;
}

extern "C" size_t pa_decode_workspace_size(int32_t num_seqs, int32_t max_context_len,
                                           const pa_cache_desc* desc) {
    return pa_decode_workspace_size_ex(num_seqs, max_context_len, desc, nullptr);
}

extern "C" int32_t pa_decode_max_splits(int32_t num_seqs, int32_t max_context_len,
                                        const pa_cache_desc* desc,
                                        const pa_decode_options* options) {
    if (check_decode_shape(num_seqs, max_context_len, desc) != PA_OK) return -1;
    DecodePlan plan;
    if (make_decode_plan(num_seqs, max_context_len, *desc, options, &plan) != PA_OK) return -1;
    return plan.max_splits;
}

extern "C" int pa_decode_describe(int32_t num_seqs, int32_t max_context_len, const pa_cache_desc* desc,
                                  const pa_decode_options* options, pa_decode_plan_info* out) {
    if (!out) return PA_ERR_INVALID;
    int rc = check_decode_shape(num_seqs, max_context_len, desc);
    if (rc != PA_OK) return rc;
    DecodePlan plan;
    rc = make_decode_plan(num_seqs, max_context_len, *desc, options, &plan);
    if (rc != PA_OK) return rc;
    out->kernel = plan.kernel == DecodeKernel::kStream  ? PA_KERNEL_TENSOR
                  : plan.kernel == DecodeKernel::kSplit ? PA_KERNEL_TENSOR_SPLIT
                                                        : PA_KERNEL_SIMT;
    out->ctas = plan.kernel == DecodeKernel::kStream ? plan.grid : 0;
    out->split_tokens = plan.kernel == DecodeKernel::kStream
                            ? stream_slab_tokens(options && options->kv_dtype == PA_KV_E4M3, desc->head_dim)
                            : plan.split_tokens;
    out->max_splits = plan.max_splits;
    return PA_OK;
}

// Shared by pa_decode_ex (k_new == v_new == null) and pa_append_decode.
static int decode_call(const pa_bf16* q, const pa_bf16* k_new, const pa_bf16* v_new,
                       const pa_bf16* k_cache, const pa_bf16* v_cache, const int32_t* block_tables,
                       const int32_t* context_lens, int32_t num_seqs, int32_t max_context_len,
                       float scale, pa_bf16* out, void* workspace, size_t workspace_bytes,
                       const pa_cache_desc* desc, const pa_decode_options* options, void* stream) {
    int rc = check_decode_shape(num_seqs, max_context_len, desc);
    if (rc != PA_OK) return rc;
    if (options && (options->max_ctas < 0 || options->kernel < 0 || options->kernel > 3 ||
                    (options->flags & ~(PA_FLAG_CHECK | PA_FLAG_PDL | PA_FLAG_SELFTEST_STALL)) != 0 ||
                    !(options->rope_theta >= 0.f) || !(options->rope_theta < INFINITY) ||
                    (options->kv_dtype != PA_KV_BF16 && options->kv_dtype != PA_KV_E4M3)))
        return PA_ERR_INVALID;
    const float rope_theta = options ? options->rope_theta : 0.f;
    const bool fp8 = options && options->kv_dtype == PA_KV_E4M3;
    if (fp8 && (!(options->k_scale > 0.f) || !(options->k_scale < INFINITY) ||
                !(options->v_scale > 0.f) || !(options->v_scale < INFINITY)))
        return PA_ERR_INVALID;
    if (rope_theta > 0.f && !k_new) return PA_ERR_INVALID;   // RoPE needs the new token (pa_append_decode)
    if (num_seqs == 0) return PA_OK;
    if (!q || !k_cache || !v_cache || !block_tables || !context_lens || !out)
        return PA_ERR_INVALID;
    if (!aligned(q, 16) || !aligned(out, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
        !aligned(block_tables, 4) || !aligned(context_lens, 4))
        return PA_ERR_INVALID;
    DecodePlan plan;
    rc = make_decode_plan(num_seqs, max_context_len, *desc, options, &plan);
    if (rc != PA_OK) return rc;
    const bool stall = options && (options->flags & PA_FLAG_SELFTEST_STALL);
    if (stall && plan.kernel != DecodeKernel::kStream) return PA_ERR_UNSUPPORTED;
    if (!workspace || !aligned(workspace, kWorkspaceAlign) || workspace_bytes < plan.bytes)
        return PA_ERR_WORKSPACE;
    char* ws = static_cast<char*>(workspace);
    DecodeParams p;
    p.grid = plan.grid;
    p.selftest_stall = stall ? 1 : 0;
    p.wait_ns = stall ? kSelftestWaitNs : kDecodeWaitNs;
    p.q = q;
    p.k_cache = k_cache;
    p.v_cache = v_cache;
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    p.k_new = k_new;
    p.v_new = v_new;
    p.out = out;
    p.status = reinterpret_cast<int32_t*>(ws);
    p.work_counter = reinterpret_cast<int32_t*>(ws) + 1;
    p.done_counter = reinterpret_cast<int32_t*>(ws) + 2;
    p.seq_desc = reinterpret_cast<int32_t*>(ws + plan.off_desc);
    p.part_lse = reinterpret_cast<float*>(ws + plan.off_lse);
    p.part_o = reinterpret_cast<float*>(ws + plan.off_o);
    p.num_seqs = num_seqs;
    p.num_blocks = desc->num_blocks;
    p.block_size = desc->block_size;
    p.num_kv_heads = desc->num_kv_heads;
    p.num_q_heads = desc->num_q_heads;
    p.head_dim = desc->head_dim;
    p.group = desc->num_q_heads / desc->num_kv_heads;
    p.max_blocks_per_seq = desc->max_blocks_per_seq;
    p.max_context_len = max_context_len;
    p.split_tokens = plan.split_tokens;
    p.max_splits = plan.max_splits;
    p.scale_log2 = scale * (fp8 ? options->k_scale : 1.f) * 1.4426950408889634f;
    p.kv_fp8 = fp8 ? 1 : 0;
    p.k_inv_scale = fp8 ? 1.f / options->k_scale : 1.f;
    p.v_inv_scale = fp8 ? 1.f / options->v_scale : 1.f;
    p.out_scale = fp8 ? options->v_scale : 1.f;
    p.early = plan.kernel == DecodeKernel::kStream && options && (options->flags & PA_FLAG_PDL) ? 1 : 0;
    p.rope_theta = plan.kernel == DecodeKernel::kStream ? rope_theta : 0.f;
    cudaError_t e;
    const cudaStream_t st = (cudaStream_t)stream;
    if (k_new && plan.kernel != DecodeKernel::kStream) {   // only the stream kernel fuses the append
        if (rope_theta > 0.f) {
            uint16_t* q_rot = reinterpret_cast<uint16_t*>(ws + plan.off_qrot);
            p.rope_theta = rope_theta;
            e = launch_rope_append_at_end(p, q_rot, st);
            p.rope_theta = 0.f;
            p.q = q_rot;
        } else {
            e = launch_append_at_end(p, st);
        }
        if (e != cudaSuccess) return PA_ERR_CUDA;
        p.k_new = p.v_new = nullptr;
    }
    switch (plan.kernel) {
        case DecodeKernel::kStream:
            e = launch_decode_stream(p, plan.grid, p.early != 0, st);
            break;
        case DecodeKernel::kSplit: e = launch_decode_tensor(p, st); break;
        default: e = launch_decode_simt(p, st); break;
    }
    // second pass: merge the pieces of every sequence that was cut
    if (e == cudaSuccess && (plan.kernel == DecodeKernel::kStream || plan.max_splits > 1))
        e = launch_merge(p, plan.kernel == DecodeKernel::kStream,
                         plan.kernel != DecodeKernel::kSimt, st);
    if (e != cudaSuccess) return PA_ERR_CUDA;
    if (options && (options->flags & PA_FLAG_CHECK))
        return pa_decode_status(workspace, workspace_bytes, stream);
    return PA_OK;
}

extern "C" int pa_decode_ex(const pa_bf16* q, const pa_bf16* k_cache, const pa_bf16* v_cache,
                            const int32_t* block_tables, const int32_t* context_lens,
                            int32_t num_seqs, int32_t max_context_len, float scale, pa_bf16* out,
                            void* workspace, size_t workspace_bytes, const pa_cache_desc* desc,
                            const pa_decode_options* options, void* stream) {
    return decode_call(q, nullptr, nullptr, k_cache, v_cache, block_tables, context_lens, num_seqs,
                       max_context_len, scale, out, workspace, workspace_bytes, desc, options, stream);
}

extern "C" int pa_append_decode(const pa_bf16* q, const pa_bf16* k, const pa_bf16* v,
                                pa_bf16* k_cache, pa_bf16* v_cache, const int32_t* block_tables,
                                const int32_t* context_lens, int32_t num_seqs,
                                int32_t max_context_len, float scale, pa_bf16* out,
                                void* workspace, size_t workspace_bytes, const pa_cache_desc* desc,
                                const pa_decode_options* options, void* stream) {
    if (num_seqs > 0 && (!k || !v || ((uintptr_t)k % 16) || ((uintptr_t)v % 16) ||
                         desc == nullptr || desc->head_dim % 8 != 0))
        return PA_ERR_INVALID;
    return decode_call(q, k, v, k_cache, v_cache, block_tables, context_lens, num_seqs,
                       max_context_len, scale, out, workspace, workspace_bytes, desc, options, stream);
}

extern "C" int pa_decode(const pa_bf16* q, const pa_bf16* k_cache, const pa_bf16* v_cache,
                         const int32_t* block_tables, const int32_t* context_lens,
                         int32_t num_seqs, int32_t max_context_len, float scale, pa_bf16* out,
                         void* workspace, size_t workspace_bytes, const pa_cache_desc* desc,
                         void* stream) {
    return pa_decode_ex(q, k_cache, v_cache, block_tables, context_lens, num_seqs,
                        max_context_len, scale, out, workspace, workspace_bytes, desc, nullptr,
                        stream);
}

extern "C" int pa_decode_status(void* workspace, size_t workspace_bytes, void* stream) {
    if (!workspace || workspace_bytes < sizeof(int32_t)) return PA_ERR_WORKSPACE;
    int32_t word = 0;
    cudaStream_t s = (cudaStream_t)stream;
    if (cudaMemcpyAsync(&word, workspace, sizeof word, cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return PA_ERR_CUDA;
    if (cudaMemsetAsync(workspace, 0, sizeof word, s) != cudaSuccess) return PA_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return PA_ERR_CUDA;
    if (word & kStatusBadBlock) return PA_ERR_BAD_BLOCK;
    if (word & kStatusBadLength) return PA_ERR_BAD_LENGTH;
    if (word & kStatusTimeout) return PA_ERR_TIMEOUT;
    if (word & kStatusSmemAlign) return PA_ERR_UNSUPPORTED;
    return PA_OK;
}
