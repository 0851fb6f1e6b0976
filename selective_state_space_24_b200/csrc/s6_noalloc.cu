// s6_noalloc.cu -- ssm_scan_fwd_noalloc: the single-direction S6 scan for
// callers that cannot hand the library a workspace.
//
// Who needs this: code that may not allocate device memory at the moment it
// runs the scan -- for instance a plugin inside an inference engine that is
// given only its tensors and a stream when it is enqueued, or a serving loop
// that forbids allocations after start-up so that its memory footprint stays
// fixed.  ssm_scan_fwd needs caller-provided scratch for long sequences (the
// per-segment carries); this entry point takes that scratch from one array
// that the library itself owns instead.
//
// The scratch is the file-scope device array below.  Every GPU that loads the
// library holds it (SSM_NOALLOC_SCRATCH_BYTES) until the process exits.  Host
// code cannot use the array's name as a device address, so on the first call
// on each device (with that device current) the entry point looks the address
// up with cudaGetSymbolAddress and keeps it; that first call therefore makes a
// CUDA runtime call of its own and should come before any stream capture.
// All calls share the array and it keeps whatever the last call left there:
// nothing in it has to start at zero (every carry it holds is written before
// it is read within the same call), but two calls whose kernels overlap on
// the GPU (different streams, or different host threads) race on it.  This
// entry point allocates nothing and calls no allocating routine.
#include <cuda_runtime.h>
#include <mutex>
#include <stdint.h>
#include <string.h>

#include "../../include/ssm.h"
#include "internal.h"

namespace {

static __device__ __align__(256) unsigned char g_s6_scratch[SSM_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void *g_scratch_ptr[kMaxDevices];
std::mutex g_scratch_mu;

// Device address of g_s6_scratch on the current device (looked up once).
cudaError_t scratch_address(void **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev < 0 || dev >= kMaxDevices)
        return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_s6_scratch);
        if (e != cudaSuccess)
            return e;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" SSM_API ssm_status ssm_scan_fwd_noalloc(const ssm_dims *dims, const void *x, const void *delta,
                                                   const float *delta_bias, int delta_softplus,
                                                   const float *A, const void *B, const void *C,
                                                   const float *D, const void *z, int reverse, void *out,
                                                   float *last_state, void *stream)
{
    // the same argument rules as ssm_scan_fwd
    if (!dims || dims->batch < 0 || dims->seqlen < 0 || dims->dim < 0 || dims->dstate < 0)
        return SSM_ERR_INVALID_ARG;
    if (dims->dtype != SSM_F32 && dims->dtype != SSM_BF16)
        return SSM_ERR_UNSUPPORTED_DTYPE;
    if (dims->dstate < 1 || dims->dstate > 16 || dims->batch > INT32_MAX || dims->seqlen > INT32_MAX ||
        dims->dim > INT32_MAX)
        return SSM_ERR_UNSUPPORTED_SHAPE;
    if (dims->dim % (dims->dtype == SSM_F32 ? 4 : 8) != 0)
        return SSM_ERR_MISALIGNED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (dims->batch == 0 || dims->seqlen == 0 || dims->dim == 0) {
        if (last_state && !aligned16(last_state))
            return SSM_ERR_MISALIGNED;
        const size_t n = (size_t)dims->batch * dims->dim * dims->dstate;
        if (!last_state || n == 0)
            return SSM_OK;
        return cudaMemsetAsync(last_state, 0, n * sizeof(float), st) == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
    }
    if (!x || !delta || !out || !A || !B || !C)
        return SSM_ERR_INVALID_ARG;
    const void *ptrs[] = {x, delta, delta_bias, A, B, C, D, z, out, last_state};
    for (const void *q : ptrs)
        if (q && !aligned16(q))
            return SSM_ERR_MISALIGNED;
    const int dt = dims->dtype == SSM_F32 ? 0 : 1;
    // the kernel ssm_scan_fwd takes for these sizes; the four-threads-per-
    // channel one needs no scratch (one pass, single direction)
    const int split = ssm::split_threads(dims->batch, dims->seqlen, dims->dim, dims->dstate, 1);
    ssm::S6Plan plan = ssm::plan_s6(dims->batch, dims->seqlen, dims->dim, dims->dstate, 1, dt);
    if (split) {
        plan.S = 1;
        plan.T = (int)dims->seqlen;
        plan.workspace_bytes = 0;
    }
    if (plan.workspace_bytes > (size_t)SSM_NOALLOC_SCRATCH_BYTES)
        return SSM_ERR_WORKSPACE_TOO_SMALL;   // more scratch than the built-in array holds

    void *scratch = nullptr;
    if (plan.workspace_bytes > 0 && scratch_address(&scratch) != cudaSuccess)
        return SSM_ERR_CUDA;

    ssm::S6Args a;
    memset(&a, 0, sizeof(a));
    a.Bsz = (int)dims->batch;
    a.L = (int)dims->seqlen;
    a.D = (int)dims->dim;
    a.N = (int)dims->dstate;
    a.S = plan.S;
    a.T = plan.T;
    a.cpl = plan.cpl;
    a.dtype = dt;
    a.softplus = delta_softplus ? 1 : 0;
    a.ndir = 1;
    a.reverse = reverse ? 1 : 0;
    a.x = x;
    a.delta = delta;
    a.dir[0] = ssm::DirArgs{delta_bias, A, B, C, D, z, last_state};
    a.out = out;
    a.split = split;
    if (split == 2)   // the same launch ssm_scan_fwd makes
        a.mix_rows2 = ssm::split_mix_rows(dims->batch, dims->dim, 1);
    if (a.S > 1) {
        char *w = static_cast<char *>(scratch);
        a.carry_h = reinterpret_cast<float *>(w + plan.carry_h_off);
        a.carry_s = reinterpret_cast<float *>(w + plan.carry_s_off);
    }
    return ssm::launch_s6(a, st) == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}
