// s6_step.cu -- one decode step of the S6 recurrence for every (batch,
// channel), from a stored state that is updated in place: the recurrent
// inference form of the Mamba2 page "手写简化版Mamba2", sec. 5.2 (only the
// previous h is needed, so generation keeps a (D, N) state per sequence and
// advances it one token at a time), with the step of sec. 4.3 - 4.4:
//     dt = softplus(delta + bias),  h = exp(dt A) h + dt B x,
//     y  = (C h + D x) silu(z).
//
// The state is the only large operand (B D N float32 read and written
// once), so the kernel is HBM-bound; four lanes share one (b, d) row, each
// holding a quarter of its N <= 16 states in registers.
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

// Four lanes share one (b, d) row: lane part p owns states [p K, p K + K),
// K = NS / 4, so a warp's state loads and stores cover 8 whole rows
// (8 x 4 N bytes) contiguously.  The readout is summed over the four lanes
// with two shuffles.
template <typename T, int NS, bool VEC>
__global__ void __launch_bounds__(256) s6_step_kernel(const StepArgs a)
{
    constexpr int K = NS / 4;
    const size_t tid = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    const size_t row = tid >> 2;   // b * D + d
    const int part = (int)(tid & 3);
    const bool live = row < (size_t)a.Bsz * a.D;   // whole groups of 4 agree
    const int N = a.N;
    const int d = live ? (int)(row % a.D) : 0;
    const size_t b = live ? row / a.D : 0;
    const T *x = static_cast<const T *>(a.x), *dl = static_cast<const T *>(a.delta);
    const T *Bm = static_cast<const T *>(a.B), *Cm = static_cast<const T *>(a.C);
    const T *z = static_cast<const T *>(a.z);

    float y = 0.f, xv = 0.f;
    if (live) {
        xv = ldv(x, row);
        float dt = ldv(dl, row) + (a.bias ? a.bias[d] : 0.f);
        if (a.softplus)
            dt = softplus_f(dt);
        const float dtx = dt * xv;
        float h[K], Av[K];
        float *st = a.state + row * N + part * K;
        const float *Ar = a.A + (size_t)d * N + part * K;
        if (VEC) {   // N == NS: this lane's K states are one aligned vector
            if (K == 4) {
                const float4 hv = *reinterpret_cast<const float4 *>(st);
                const float4 av = __ldg(reinterpret_cast<const float4 *>(Ar));
                h[0] = hv.x, h[1] = hv.y, h[2] = hv.z, h[3] = hv.w;
                Av[0] = av.x, Av[1] = av.y, Av[2] = av.z, Av[3] = av.w;
            } else if (K == 2) {
                const float2 hv = *reinterpret_cast<const float2 *>(st);
                const float2 av = __ldg(reinterpret_cast<const float2 *>(Ar));
                h[0] = hv.x, h[1] = hv.y;
                Av[0] = av.x, Av[1] = av.y;
            } else {
                h[0] = st[0];
                Av[0] = __ldg(Ar);
            }
        } else {
#pragma unroll
            for (int k = 0; k < K; k++) {
                const bool in = part * K + k < N;
                h[k] = in ? st[k] : 0.f;
                Av[k] = in ? Ar[k] : 0.f;
            }
        }
        // this lane's B and C values (one 16-byte load each for fp32, N = 16)
        float Bv[K], Cv[K];
        if (VEC && K == 4 && sizeof(T) == 4) {
            const float4 bv = __ldg(reinterpret_cast<const float4 *>(Bm) + (b * N + part * K) / 4);
            const float4 cv = __ldg(reinterpret_cast<const float4 *>(Cm) + (b * N + part * K) / 4);
            Bv[0] = bv.x, Bv[1] = bv.y, Bv[2] = bv.z, Bv[3] = bv.w;
            Cv[0] = cv.x, Cv[1] = cv.y, Cv[2] = cv.z, Cv[3] = cv.w;
        } else {
#pragma unroll
            for (int k = 0; k < K; k++) {
                const int n = part * K + k;
                Bv[k] = (VEC || n < N) ? ldv(Bm, b * N + n) : 0.f;
                Cv[k] = (VEC || n < N) ? ldv(Cm, b * N + n) : 0.f;
            }
        }
#pragma unroll
        for (int k = 0; k < K; k++) {
            const int n = part * K + k;
            if (VEC || n < N) {
                const float e = ex2_mufu(dt * (Av[k] * kLog2e));
                h[k] = fmaf(e, h[k], dtx * Bv[k]);
                y = fmaf(Cv[k], h[k], y);
            }
        }
        if (VEC) {
            if (K == 4)
                *reinterpret_cast<float4 *>(st) = make_float4(h[0], h[1], h[2], h[3]);
            else if (K == 2)
                *reinterpret_cast<float2 *>(st) = make_float2(h[0], h[1]);
            else
                st[0] = h[0];
        } else {
#pragma unroll
            for (int k = 0; k < K; k++)
                if (part * K + k < N)
                    st[k] = h[k];
        }
    }
    y += __shfl_xor_sync(0xffffffffu, y, 1);
    y += __shfl_xor_sync(0xffffffffu, y, 2);
    if (live && part == 0) {
        if (a.Dskip)
            y = fmaf(a.Dskip[d], xv, y);
        if (z)
            y *= silu_f<T>(ldv(z, row));
        stv(static_cast<T *>(a.out), row, y);
    }
}

template <typename T, int NS>
cudaError_t launch_ns(const StepArgs &a, cudaStream_t st)
{
    const size_t threads = (size_t)a.Bsz * a.D * 4;
    const unsigned grid = (unsigned)((threads + 255) / 256);
    if (a.N == NS)
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
