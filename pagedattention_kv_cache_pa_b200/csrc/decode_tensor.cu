// Paged decode attention with TMA-staged pages and tensor-core q.K / p.V.
// (Placeholder until the kernel lands: reports itself unsupported, so
// pa_decode dispatches to the CUDA-core kernel.)
#include <cuda_runtime.h>

#include "pa_internal.h"

namespace pa {

bool tensor_kernel_supports(const DecodeParams&) { return false; }

cudaError_t launch_decode_tensor(const DecodeParams&, cudaStream_t) {
    return cudaErrorNotSupported;
}

}  // namespace pa
