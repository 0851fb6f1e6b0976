// ssd_chunk.cu -- Mamba2 SSD chunked scan (placeholder until the tcgen05
// kernel lands) and the library's device-side error word.
#include <cuda_runtime.h>

#include "internal.h"

namespace ssm {

__device__ unsigned g_device_error;

size_t ssd_workspace_bytes(int64_t, int64_t, int64_t, int64_t, int64_t, int64_t) { return 0; }

cudaError_t launch_ssd(const SSDArgs &, cudaStream_t) { return cudaErrorNotSupported; }

cudaError_t read_and_clear_device_error(unsigned *value, cudaStream_t stream)
{
    cudaError_t e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess)
        return e;
    e = cudaMemcpyFromSymbol(value, g_device_error, sizeof(unsigned));
    if (e != cudaSuccess)
        return e;
    const unsigned zero = 0;
    return cudaMemcpyToSymbol(g_device_error, &zero, sizeof(unsigned));
}

}  // namespace ssm
