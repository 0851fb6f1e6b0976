// s6_step.cu -- one decode step of the S6 recurrence for every (batch,
// channel), from a stored state that is updated in place: the recurrent
// inference form of the Mamba2 page "手写简化版Mamba2", sec. 5.2 (only the
// previous h is needed, so generation keeps a (D, N) state per sequence and
// advances it one token at a time), with the step of sec. 4.3 - 4.4:
//     dt = softplus(delta + bias),  h = exp(dt A) h + dt B x,
//     y  = (C h + D x) silu(z).
//
// The state is the only large operand (B D N float32 read and written
// once); one or two lanes share one (b, d) row, each holding its share of
// the row's N <= 16 states in registers.
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

// LANES lanes (1, 2 or 4) share one (b, d) row: lane part p owns states
// [p K, p K + K), K = NS / LANES, so a warp covers 32 / LANES consecutive
// rows and each of its state loads spans them contiguously.  All of a
// row's loads are issued before its arithmetic.  The readout is summed over
// a row's lanes with log2(LANES) shuffles.  The per-row scalar work
// (softplus, the gate, the index arithmetic) is done by every lane of the
// row, so fewer lanes per row issue fewer instructions per state; more
// states per lane hold more registers and keep fewer rows in flight.
// Measured on B200 (L2 flushed before each step): N = 16 fp32 (B 512,
// D 1536) 28.7 us with two lanes per row, 32.8 with four, 34.8 with one;
// N = 8 bf16 (B 256, D 1000) 10.7 us with one lane, 12.3 with two or four.
// SSM_STEP_LANES = 0 takes those (two lanes for 16 states, else one).
#ifndef SSM_STEP_LANES
#define SSM_STEP_LANES 0
#endif
template <typename T, int NS, bool VEC, int LANES>
__global__ void __launch_bounds__(256) s6_step_kernel(const StepArgs a)
{
    constexpr int K = NS / LANES;
    static_assert(K >= 1 && NS % LANES == 0, "states split evenly over the lanes");
    const size_t tid = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    const size_t row = tid / LANES;   // b * D + d
    const int part = (int)(tid % LANES);
    const size_t nrows = (size_t)a.Bsz * a.D;
    const bool live = row < nrows;    // whole groups of LANES lanes agree
    const int N = a.N;
    size_t b = 0;
    int d = 0;
    if (live) {
        if (nrows <= 0xffffffffu)
            b = (unsigned)row / (unsigned)a.D;
        else
            b = row / (size_t)a.D;
        d = (int)(row - b * (size_t)a.D);
    }
    const T *x = static_cast<const T *>(a.x), *dl = static_cast<const T *>(a.delta);
    const T *Bm = static_cast<const T *>(a.B), *Cm = static_cast<const T *>(a.C);
    const T *z = static_cast<const T *>(a.z);

    float y = 0.f, xv = 0.f, zv = 0.f, Dk = 0.f;
    if (live) {
        float h[K], Av[K], Bv[K], Cv[K];
        xv = ldv(x, row);
        const float dv = ldv(dl, row);
        if (z)
            zv = ldv(z, row);
        const float bias = a.bias ? a.bias[d] : 0.f;
        Dk = a.Dskip ? a.Dskip[d] : 0.f;   // with the row's other loads, not after the shuffles
        float *st = a.state + row * N + part * K;
        const float *Ar = a.A + (size_t)d * N + part * K;
        if (VEC && K % 4 == 0) {   // N == NS: this lane's K states are K / 4 aligned vectors
#pragma unroll
            for (int v = 0; v < K / 4; v++) {
                const float4 hv = reinterpret_cast<const float4 *>(st)[v];
                const float4 av = __ldg(reinterpret_cast<const float4 *>(Ar) + v);
                h[4 * v] = hv.x, h[4 * v + 1] = hv.y, h[4 * v + 2] = hv.z, h[4 * v + 3] = hv.w;
                Av[4 * v] = av.x, Av[4 * v + 1] = av.y, Av[4 * v + 2] = av.z, Av[4 * v + 3] = av.w;
            }
        } else if (VEC && K == 2) {
            const float2 hv = *reinterpret_cast<const float2 *>(st);
            const float2 av = __ldg(reinterpret_cast<const float2 *>(Ar));
            h[0] = hv.x, h[1] = hv.y;
            Av[0] = av.x, Av[1] = av.y;
        } else {
#pragma unroll
            for (int k = 0; k < K; k++) {
                const bool in = VEC || part * K + k < N;
                h[k] = in ? st[k] : 0.f;
                Av[k] = in ? Ar[k] : 0.f;
            }
        }
        // this lane's B and C values (16-byte loads for fp32 and N = NS)
        if (VEC && K % 4 == 0 && sizeof(T) == 4) {
#pragma unroll
            for (int v = 0; v < K / 4; v++) {
                const float4 bv = __ldg(reinterpret_cast<const float4 *>(Bm) + (b * N + part * K) / 4 + v);
                const float4 cv = __ldg(reinterpret_cast<const float4 *>(Cm) + (b * N + part * K) / 4 + v);
                Bv[4 * v] = bv.x, Bv[4 * v + 1] = bv.y, Bv[4 * v + 2] = bv.z, Bv[4 * v + 3] = bv.w;
                Cv[4 * v] = cv.x, Cv[4 * v + 1] = cv.y, Cv[4 * v + 2] = cv.z, Cv[4 * v + 3] = cv.w;
            }
        } else {
#pragma unroll
            for (int k = 0; k < K; k++) {
                const int n = part * K + k;
                Bv[k] = (VEC || n < N) ? ldv(Bm, b * N + n) : 0.f;
                Cv[k] = (VEC || n < N) ? ldv(Cm, b * N + n) : 0.f;
            }
        }
        float dt = dv + bias;
        if (a.softplus)
            dt = softplus_f(dt);
        const float dtx = dt * xv;
#pragma unroll
        for (int k = 0; k < K; k++) {
            const int n = part * K + k;
            if (VEC || n < N) {
                const float e = ex2_mufu(dt * (Av[k] * kLog2e));
                h[k] = fmaf(e, h[k], dtx * Bv[k]);
                y = fmaf(Cv[k], h[k], y);
            }
        }
        if (VEC && K % 4 == 0) {
#pragma unroll
            for (int v = 0; v < K / 4; v++)
                reinterpret_cast<float4 *>(st)[v] = make_float4(h[4 * v], h[4 * v + 1], h[4 * v + 2], h[4 * v + 3]);
        } else if (VEC && K == 2) {
            *reinterpret_cast<float2 *>(st) = make_float2(h[0], h[1]);
        } else {
#pragma unroll
            for (int k = 0; k < K; k++)
                if (VEC || part * K + k < N)
                    st[k] = h[k];
        }
    }
#pragma unroll
    for (int o = 1; o < LANES; o <<= 1)
        y += __shfl_xor_sync(0xffffffffu, y, o);
    if (live && part == 0) {
        y = fmaf(Dk, xv, y);
        if (z)
            y *= silu_f<T>(zv);
        stv(static_cast<T *>(a.out), row, y);
    }
}

template <typename T, int NS>
cudaError_t launch_ns(const StepArgs &a, cudaStream_t st)
{
    constexpr int LANES = SSM_STEP_LANES == 0 ? (NS == 16 ? 2 : 1)
                                              : (NS >= SSM_STEP_LANES ? SSM_STEP_LANES : NS);
    const size_t threads = (size_t)a.Bsz * a.D * LANES;
    const unsigned grid = (unsigned)((threads + 255) / 256);
    if (a.N == NS)
        s6_step_kernel<T, NS, true, LANES><<<grid, 256, 0, st>>>(a);
    else
        s6_step_kernel<T, NS, false, LANES><<<grid, 256, 0, st>>>(a);
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
