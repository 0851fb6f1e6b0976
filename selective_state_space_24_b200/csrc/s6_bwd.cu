// s6_bwd.cu -- gradients of the single-direction S6 scan (the training use
// of the Mamba2 page "手写简化版Mamba2", sec. 5.1, which backpropagates
// through the scan loop; here the adjoint is written out and run as a
// reverse scan instead of storing every step).
//
// Per (b, d), along the scan order i (t = i, or L-1-i reversed), with
// dt_i = softplus(v_i), v_i = delta_i + bias, a_i[n] = exp(dt_i A[n]),
// h_i = a_i h_{i-1} + dt_i B_i x_i, y_i = C_i . h_i + D x_i, out_i = y_i silu(z_i),
// and the incoming gradient g_i of out_i:
//   dy_i = g_i silu(z_i);   dz_i = g_i y_i silu'(z_i)
//   lam_i[n] = dy_i C_i[n] + a_{i+1}[n] lam_{i+1}[n]     (lam = dL/dh, run backwards)
//   dC_i[n] += dy_i h_i[n];  dB_i[n] += lam_i[n] dt_i x_i  (summed over channels)
//   dx_i = dy_i D + dt_i sum_n lam_i[n] B_i[n]
//   ddt_i = sum_n lam_i[n] (B_i[n] x_i + A[n] a_i[n] h_{i-1}[n])
//   dA[n] += lam_i[n] dt_i a_i[n] h_{i-1}[n];  dD += dy_i x_i
//   ddelta_i = ddt_i softplus'(v_i) = ddt_i sigmoid(v_i);  dbias += ddelta_i
//
// Two kernels.  s6_bwd_ckpt_kernel runs the forward recurrence once and
// stores h entering every chunk of kKc steps.  s6_bwd_kernel walks the
// chunks backwards: it recomputes the chunk's states into shared memory
// from the checkpoint, then sweeps the chunk backwards with lam in
// registers.  One thread per (b, d); a CTA holds 64 channels of one batch
// row, and sums dB, dC over them in shared memory before one atomic add
// per (t, n).  All gradients are float32.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"
#include "s6_math.cuh"

namespace ssm {
namespace {

constexpr int kKc = 8;         // steps per checkpointed chunk
constexpr int kCta = 64;       // channels (threads) per CTA

template <typename T> __device__ __forceinline__ float ldv(const T *p, size_t i);
template <> __device__ __forceinline__ float ldv<float>(const float *p, size_t i) { return __ldg(p + i); }
template <> __device__ __forceinline__ float ldv<__nv_bfloat16>(const __nv_bfloat16 *p, size_t i)
{
    return __bfloat162float(__ldg(p + i));
}

__device__ __forceinline__ float dt_of(float v, int softplus) { return softplus ? softplus_f(v) : v; }
__device__ __forceinline__ float sigmoid_f(float v) { return 1.f / (1.f + ex2_mufu(-v * kLog2e)); }

template <typename T, int NS>
__global__ void __launch_bounds__(kCta) s6_bwd_ckpt_kernel(const BwdArgs a)
{
    const int d = blockIdx.x * kCta + threadIdx.x;
    const int b = blockIdx.y;
    if (d >= a.D)
        return;
    const int N = a.N, L = a.L, nch = (L + kKc - 1) / kKc;
    const T *x = static_cast<const T *>(a.x), *dl = static_cast<const T *>(a.delta);
    const T *Bm = static_cast<const T *>(a.B);
    float Al[NS], h[NS];
#pragma unroll
    for (int n = 0; n < NS; n++) {
        Al[n] = n < N ? a.A[(size_t)d * N + n] * kLog2e : 0.f;
        h[n] = 0.f;
    }
    const float bias = a.bias ? a.bias[d] : 0.f;
    for (int c = 0; c < nch; c++) {
        float *ck = a.ckpt + (((size_t)b * nch + c) * a.D + d) * N;
#pragma unroll
        for (int n = 0; n < NS; n++)
            if (n < N)
                ck[n] = h[n];
        for (int k = 0; k < kKc; k++) {
            const int i = c * kKc + k;
            if (i >= L)
                break;
            const int t = a.reverse ? L - 1 - i : i;
            const size_t row = (size_t)b * L + t;
            const float dt = dt_of(ldv(dl, row * a.D + d) + bias, a.softplus);
            const float dtx = dt * ldv(x, row * a.D + d);
#pragma unroll
            for (int n = 0; n < NS; n++)
                if (n < N)
                    h[n] = fmaf(ex2_mufu(dt * Al[n]), h[n], dtx * ldv(Bm, row * N + n));
        }
    }
}

template <typename T, int NS>
__global__ void __launch_bounds__(kCta) s6_bwd_kernel(const BwdArgs a)
{
    // states of the current chunk: hs[k][n][thread]; channel sums: red[thread][2 NS + 1]
    __shared__ float hs[kKc][NS][kCta];
    __shared__ float red[kCta][2 * NS + 1];
    const int tid = threadIdx.x;
    const int d = blockIdx.x * kCta + tid;
    const int b = blockIdx.y;
    const bool active = d < a.D;
    const int dd = active ? d : 0;
    const int N = a.N, L = a.L, nch = (L + kKc - 1) / kKc;
    const T *x = static_cast<const T *>(a.x), *dl = static_cast<const T *>(a.delta);
    const T *Bm = static_cast<const T *>(a.B), *Cm = static_cast<const T *>(a.C);
    const T *zp = static_cast<const T *>(a.z), *go = static_cast<const T *>(a.dout);
    float A[NS], Al[NS], lam[NS], gA[NS];
#pragma unroll
    for (int n = 0; n < NS; n++) {
        A[n] = (active && n < N) ? a.A[(size_t)dd * N + n] : 0.f;
        Al[n] = A[n] * kLog2e;
        lam[n] = 0.f;   // a_{i+1} lam_{i+1}, carried backwards
        gA[n] = 0.f;
    }
    const float bias = (active && a.bias) ? a.bias[dd] : 0.f;
    const float Dv = (active && a.Dskip) ? a.Dskip[dd] : 0.f;
    float gD = 0.f, gbias = 0.f;

    for (int c = nch - 1; c >= 0; c--) {
        const int i0 = c * kKc, kn = min(kKc, L - i0);
        // recompute the chunk's states from the checkpoint
        float hp[NS];
        const float *ck = a.ckpt + (((size_t)b * nch + c) * a.D + dd) * N;
#pragma unroll
        for (int n = 0; n < NS; n++)
            hp[n] = (active && n < N) ? ck[n] : 0.f;
        {
            float h[NS];
#pragma unroll
            for (int n = 0; n < NS; n++)
                h[n] = hp[n];
            for (int k = 0; k < kn; k++) {
                const int t = a.reverse ? L - 1 - (i0 + k) : i0 + k;
                const size_t row = (size_t)b * L + t;
                float dt = 0.f, dtx = 0.f;
                if (active) {
                    dt = dt_of(ldv(dl, row * a.D + dd) + bias, a.softplus);
                    dtx = dt * ldv(x, row * a.D + dd);
                }
#pragma unroll
                for (int n = 0; n < NS; n++) {
                    if (n < N)
                        h[n] = fmaf(ex2_mufu(dt * Al[n]), h[n], dtx * ldv(Bm, row * N + n));
                    hs[k][n][tid] = h[n];
                }
            }
        }
        // backward sweep over the chunk
        for (int k = kn - 1; k >= 0; k--) {
            const int t = a.reverse ? L - 1 - (i0 + k) : i0 + k;
            const size_t row = (size_t)b * L + t;
            const size_t io = row * a.D + dd;
            float dtx = 0.f, dt = 0.f, xv = 0.f, v = 0.f, dy = 0.f;
            if (active) {
                v = ldv(dl, io) + bias;
                dt = dt_of(v, a.softplus);
                xv = ldv(x, io);
                dtx = dt * xv;
                const float g = ldv(go, io);
                // y_i = C . h_i + D x_i
                float y = Dv * xv;
#pragma unroll
                for (int n = 0; n < NS; n++)
                    if (n < N)
                        y = fmaf(ldv(Cm, row * N + n), hs[k][n][tid], y);
                if (zp) {
                    const float zv = ldv(zp, io);
                    const float s = sigmoid_f(zv);
                    dy = g * zv * s;
                    if (a.dz)
                        a.dz[io] = g * y * s * (1.f + zv * (1.f - s));
                } else {
                    dy = g;
                }
            }
            float ddt = 0.f, dxs = 0.f;
#pragma unroll
            for (int n = 0; n < NS; n++) {
                float gB = 0.f, gC = 0.f;
                if (n < N) {
                    const float Bn = ldv(Bm, row * N + n), Cn = ldv(Cm, row * N + n);
                    const float hprev = k > 0 ? hs[k - 1][n][tid] : hp[n];
                    const float an = ex2_mufu(dt * Al[n]);
                    const float l = fmaf(dy, Cn, lam[n]);        // lam_i[n]
                    gC = dy * hs[k][n][tid];
                    gB = l * dtx;
                    dxs = fmaf(l, Bn, dxs);
                    const float ah = an * hprev;
                    ddt = fmaf(l, fmaf(Bn, xv, A[n] * ah), ddt);
                    gA[n] = fmaf(l * dt, ah, gA[n]);
                    lam[n] = an * l;                              // a_i lam_i for step i - 1
                }
                red[tid][n] = active ? gB : 0.f;
                red[tid][NS + n] = active ? gC : 0.f;
            }
            if (active) {
                a.dx[io] = (a.accumulate ? a.dx[io] : 0.f) + fmaf(dy, Dv, dt * dxs);
                const float dv = a.softplus ? ddt * sigmoid_f(v) : ddt;
                a.ddelta[io] = (a.accumulate ? a.ddelta[io] : 0.f) + dv;
                gbias += dv;
                gD = fmaf(dy, xv, gD);
            }
            __syncthreads();
            // sum dB, dC over the CTA's channels: thread j < 2 NS owns column j
            if (tid < 2 * NS && (tid % NS) < N) {
                float s = 0.f;
#pragma unroll 8
                for (int r = 0; r < kCta; r++)
                    s += red[r][tid];
                float *dst = tid < NS ? a.dB : a.dC;
                atomicAdd(dst + row * N + (tid % NS), s);
            }
            __syncthreads();
        }
    }
    if (active) {
#pragma unroll
        for (int n = 0; n < NS; n++)
            if (n < N)
                atomicAdd(a.dA + (size_t)dd * N + n, gA[n]);
        if (a.dD)
            atomicAdd(a.dD + dd, gD);
        if (a.dbias)
            atomicAdd(a.dbias + dd, gbias);
    }
}

template <typename T, int NS>
cudaError_t launch_ns(const BwdArgs &a, cudaStream_t st)
{
    dim3 g((a.D + kCta - 1) / kCta, a.Bsz);
    s6_bwd_ckpt_kernel<T, NS><<<g, kCta, 0, st>>>(a);
    s6_bwd_kernel<T, NS><<<g, kCta, 0, st>>>(a);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_typed(const BwdArgs &a, cudaStream_t st)
{
    if (a.N <= 4)
        return launch_ns<T, 4>(a, st);
    if (a.N <= 8)
        return launch_ns<T, 8>(a, st);
    return launch_ns<T, 16>(a, st);
}

}  // namespace

size_t bwd_workspace_bytes(int64_t Bsz, int64_t L, int64_t D, int64_t N)
{
    const int64_t nch = (L + kKc - 1) / kKc;
    return (size_t)Bsz * nch * D * N * sizeof(float);
}

cudaError_t launch_bwd(const BwdArgs &a, cudaStream_t st)
{
    if (a.Bsz == 0 || a.L == 0 || a.D == 0)
        return cudaSuccess;
    return a.dtype == 0 ? launch_typed<float>(a, st) : launch_typed<__nv_bfloat16>(a, st);
}

}  // namespace ssm
