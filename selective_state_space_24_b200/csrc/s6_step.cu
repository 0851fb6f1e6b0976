// s6_step.cu -- one decode step of the S6 recurrence for every (batch,
// channel), from a stored state that is updated in place: the recurrent
// inference form of the Mamba2 page "手写简化版Mamba2", sec. 5.2 (only the
// previous h is needed, so generation keeps a (D, N) state per sequence and
// advances it one token at a time), with the step of sec. 4.3 - 4.4:
//     dt = softplus(delta + bias),  h = exp(dt A) h + dt B x,
//     y  = (C h + D x) silu(z).
//
// One thread per (b, d) keeps the N <= 16 states of its row in registers.
// The state is the only large operand (B D N float32 read and written once),
// so the kernel is HBM-bound: consecutive threads own consecutive rows, and
// a row is read and written as 16-byte vectors when N is a multiple of 4.
// The transcendentals take the same forms as in the scan kernels
// (s6_math.cuh), with A scaled by log2(e) before the product with dt.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"
#include "s6_math.cuh"

namespace ssm {
namespace {

template <typename T> __device__ __forceinline__ float ldv(const T *p, size_t i);
template <> __device__ __forceinline__ float ldv<float>(const float *p, size_t i) { return __ldg(p + i); }
template <> __device__ __forceinline__ float ldv<__nv_bfloat16>(const __nv_bfloat16 *p, size_t i)
{
    return __bfloat162float(__ldg(p + i));
}
__device__ __forceinline__ void stv(float *p, size_t i, float v) { p[i] = v; }
__device__ __forceinline__ void stv(__nv_bfloat16 *p, size_t i, float v) { p[i] = __float2bfloat16_rn(v); }

template <typename T, int NS, bool VEC>
__global__ void __launch_bounds__(256) s6_step_kernel(const StepArgs a)
{
    const size_t row = (size_t)blockIdx.x * blockDim.x + threadIdx.x;   // b * D + d
    if (row >= (size_t)a.Bsz * a.D)
        return;
    const int N = a.N;
    const int d = (int)(row % a.D);
    const size_t b = row / a.D;
    const T *x = static_cast<const T *>(a.x), *dl = static_cast<const T *>(a.delta);
    const T *Bm = static_cast<const T *>(a.B), *Cm = static_cast<const T *>(a.C);
    const T *z = static_cast<const T *>(a.z);

    const float xv = ldv(x, row);
    float dt = ldv(dl, row) + (a.bias ? a.bias[d] : 0.f);
    if (a.softplus)
        dt = softplus_f(dt);
    const float dtx = dt * xv;

    float h[NS], Av[NS];
    float *st = a.state + row * N;
    const float *Ar = a.A + (size_t)d * N;
    if (VEC) {   // N == NS, a multiple of 4: 16-byte rows
#pragma unroll
        for (int q = 0; q < NS / 4; q++) {
            const float4 hv = reinterpret_cast<const float4 *>(st)[q];
            const float4 av = __ldg(reinterpret_cast<const float4 *>(Ar) + q);
            h[4 * q] = hv.x, h[4 * q + 1] = hv.y, h[4 * q + 2] = hv.z, h[4 * q + 3] = hv.w;
            Av[4 * q] = av.x * kLog2e, Av[4 * q + 1] = av.y * kLog2e;
            Av[4 * q + 2] = av.z * kLog2e, Av[4 * q + 3] = av.w * kLog2e;
        }
    } else {
#pragma unroll
        for (int n = 0; n < NS; n++) {
            h[n] = n < N ? st[n] : 0.f;
            Av[n] = n < N ? Ar[n] * kLog2e : 0.f;
        }
    }
    float y = 0.f;
#pragma unroll
    for (int n = 0; n < NS; n++) {
        if (n < N) {
            const float e = ex2_mufu(dt * Av[n]);
            h[n] = fmaf(e, h[n], dtx * ldv(Bm, b * N + n));
            y = fmaf(ldv(Cm, b * N + n), h[n], y);
        }
    }
    if (VEC) {
#pragma unroll
        for (int q = 0; q < NS / 4; q++)
            reinterpret_cast<float4 *>(st)[q] = make_float4(h[4 * q], h[4 * q + 1], h[4 * q + 2], h[4 * q + 3]);
    } else {
#pragma unroll
        for (int n = 0; n < NS; n++)
            if (n < N)
                st[n] = h[n];
    }
    if (a.Dskip)
        y = fmaf(a.Dskip[d], xv, y);
    if (z)
        y *= silu_f<T>(ldv(z, row));
    stv(static_cast<T *>(a.out), row, y);
}

template <typename T, int NS>
cudaError_t launch_ns(const StepArgs &a, cudaStream_t st)
{
    const size_t rows = (size_t)a.Bsz * a.D;
    const unsigned grid = (unsigned)((rows + 255) / 256);
    if (a.N == NS && NS % 4 == 0)
        s6_step_kernel<T, NS, true><<<grid, 256, 0, st>>>(a);
    else
        s6_step_kernel<T, NS, false><<<grid, 256, 0, st>>>(a);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_typed(const StepArgs &a, cudaStream_t st)
{
    if (a.N <= 4)
        return launch_ns<T, 4>(a, st);
    if (a.N <= 8)
        return launch_ns<T, 8>(a, st);
    return launch_ns<T, 16>(a, st);
}

}  // namespace

cudaError_t launch_step(const StepArgs &a, cudaStream_t st)
{
    if (a.Bsz == 0 || a.D == 0)
        return cudaSuccess;
    return a.dtype == 0 ? launch_typed<float>(a, st) : launch_typed<__nv_bfloat16>(a, st);
}

}  // namespace ssm
