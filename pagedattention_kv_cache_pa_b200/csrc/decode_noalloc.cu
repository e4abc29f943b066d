// pa_decode_noalloc: paged decode attention for callers that cannot allocate
// device memory.
//
// pa_decode needs a scratch workspace (status word, split descriptors and the
// partial states of sequences cut across CTAs) that the caller allocates.
// Some callers cannot: code that runs under a memory planner which owns every
// device allocation up front (inference runtimes that hand plugins only their
// inputs and outputs), code on a path where a cudaMalloc would synchronise the
// device or fail for lack of a free block at the wrong moment (latency-bound
// serving loops, real-time pipelines), or C callers without an allocator of
// their own.  This entry point takes the scratch from a fixed array that lives
// in this library's device image instead.
//
// The array is file-scope `static __device__` storage of kNoAllocScratchBytes:
// every GPU that loads the library holds it until the process exits.  Host code
// cannot use the array's name as a device address (in host code it names a
// host-side stand-in), so on the first call on each device, with that device
// current, its address is looked up once with cudaGetSymbolAddress and cached.
// Calls share the array and it keeps the previous call's contents; the words
// that must start at zero are cleared by a cudaMemsetAsync on the call's stream.
// The address belongs to the device's primary context (the runtime API's
// context); a caller that makes another driver-API context current on the same
// device must not call this entry point from it.
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "pa.h"
#include "pa_internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = PA_NOALLOC_SCRATCH_BYTES;   // 16 MiB

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::atomic<void*> g_scratch_ptr[kMaxDevices];
std::mutex g_setup_mutex;

// Device address of g_noalloc_scratch on the current device (looked up once per device).
int scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PA_ERR_CUDA;
    void* p = g_scratch_ptr[dev].load(std::memory_order_acquire);
    if (!p) {
        std::lock_guard<std::mutex> lock(g_setup_mutex);
        p = g_scratch_ptr[dev].load(std::memory_order_relaxed);
        if (!p) {
            if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return PA_ERR_CUDA;
            g_scratch_ptr[dev].store(p, std::memory_order_release);
        }
    }
    *out = p;
    return PA_OK;
}

}  // namespace

extern "C" int pa_decode_noalloc(const pa_bf16* q, const pa_bf16* k_cache, const pa_bf16* v_cache,
                                 const int32_t* block_tables, const int32_t* context_lens,
                                 int32_t num_seqs, int32_t max_context_len, float scale,
                                 pa_bf16* out, const pa_cache_desc* desc,
                                 const pa_decode_options* options, void* stream) {
    if (num_seqs == 0) return PA_OK;
    const size_t need = pa_decode_workspace_size_ex(num_seqs, max_context_len, desc, options);
    if (need == 0)   // arguments pa_decode_ex refuses: let it name the error (it fails before
                     // touching the workspace, so nothing is launched)
        return pa_decode_ex(q, k_cache, v_cache, block_tables, context_lens, num_seqs,
                            max_context_len, scale, out, nullptr, 0, desc, options, stream);
    if (need > kNoAllocScratchBytes) return PA_ERR_WORKSPACE;   // shape needs more than the array
    void* scratch = nullptr;
    const int rc = scratch_address(&scratch);
    if (rc != PA_OK) return rc;
    // status word and work counters must start at zero; the rest is written before it is read
    if (cudaMemsetAsync(scratch, 0, 256, (cudaStream_t)stream) != cudaSuccess) return PA_ERR_CUDA;
    return pa_decode_ex(q, k_cache, v_cache, block_tables, context_lens, num_seqs, max_context_len,
                        scale, out, scratch, kNoAllocScratchBytes, desc, options, stream);
}
