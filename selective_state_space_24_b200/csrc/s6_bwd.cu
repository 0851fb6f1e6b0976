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
// row and stages each chunk's B and C rows in shared memory; the per-step
// inputs of a chunk are loaded together before its work.  dB and dC are
// summed over a warp's 32 channels with a butterfly of shuffles, then added
// with one atomic per (warp, t, n).  All gradients are float32.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"
#include "s6_math.cuh"

namespace ssm {
namespace {

constexpr int kKc = 4;         // steps per checkpointed chunk (4: the backward kernel's shared
                               // memory then allows 6 CTAs per SM, one wave for Vim-Small)
constexpr int kCta = 64;       // channels (threads) per CTA

template <typename T> __device__ __forceinline__ float ldv(const T *p, size_t i);
template <> __device__ __forceinline__ float ldv<float>(const float *p, size_t i) { return __ldg(p + i); }
template <> __device__ __forceinline__ float ldv<__nv_bfloat16>(const __nv_bfloat16 *p, size_t i)
{
    return __bfloat162float(__ldg(p + i));
}

__device__ __forceinline__ float dt_of(float v, int softplus) { return softplus ? softplus_f(v) : v; }
__device__ __forceinline__ float sigmoid_f(float v) { return 1.f / (1.f + ex2_mufu(-v * kLog2e)); }

// B (and C) rows of steps [i0, i0 + kKc) in scan order into shared memory:
// bc[k][n] for B, bc[k][NS + n] for C (zero past L or N).  Whole CTA.
template <typename T, int NS, bool WITH_C>
__device__ __forceinline__ void stage_bc(const BwdArgs &a, int b, int i0, float (*bc)[2 * NS])
{
    const T *Bm = static_cast<const T *>(a.B), *Cm = static_cast<const T *>(a.C);
    constexpr int kVals = kKc * (WITH_C ? 2 : 1) * NS;
    for (int j = threadIdx.x; j < kVals; j += kCta) {
        const int k = j / ((WITH_C ? 2 : 1) * NS), r = j % ((WITH_C ? 2 : 1) * NS);
        const int n = r % NS, i = i0 + k;
        float v = 0.f;
        if (i < a.L && n < a.N) {
            const int t = a.reverse ? a.L - 1 - i : i;
            v = ldv(r < NS ? Bm : Cm, ((size_t)b * a.L + t) * a.N + n);
        }
        bc[k][r] = v;
    }
}

// Sum v[0..31] over the 32 lanes of the warp: afterwards lane j holds the
// sum of every lane's v[j] (butterfly: at each stage a lane keeps one half of
// its values -- the upper half if its lane bit is set -- and adds the
// partner's copy of that half).
__device__ __forceinline__ float warp_transpose_sum(float (&v)[32])
{
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        const bool up = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < o; i++) {
            const float send = up ? v[i] : v[i + o];
            const float keep = up ? v[i + o] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
    }
    return v[0];
}

template <typename T, int NS>
__global__ void __launch_bounds__(kCta) s6_bwd_ckpt_kernel(const BwdArgs a)
{
    __shared__ float bc[kKc][2 * NS];
    const int d = blockIdx.x * kCta + threadIdx.x;
    const int b = blockIdx.y;
    const bool active = d < a.D;
    const int dd = active ? d : 0;
    const int N = a.N, L = a.L, nch = (L + kKc - 1) / kKc;
    const T *x = static_cast<const T *>(a.x), *dl = static_cast<const T *>(a.delta);
    float Al[NS], h[NS];
#pragma unroll
    for (int n = 0; n < NS; n++) {
        Al[n] = (active && n < N) ? a.A[(size_t)dd * N + n] * kLog2e : 0.f;
        h[n] = 0.f;
    }
    const float bias = (active && a.bias) ? a.bias[dd] : 0.f;
    for (int c = 0; c < nch; c++) {
        const int i0 = c * kKc;
        if (active) {
            float *ck = a.ckpt + (((size_t)b * nch + c) * a.D + dd) * N;
#pragma unroll
            for (int n = 0; n < NS; n++)
                if (n < N)
                    ck[n] = h[n];
        }
        // this chunk's per-step scalars, all loads issued together
        float dtk[kKc], xk[kKc];
#pragma unroll
        for (int k = 0; k < kKc; k++) {
            const int i = i0 + k;
            dtk[k] = 0.f;
            xk[k] = 0.f;
            if (active && i < L) {
                const int t = a.reverse ? L - 1 - i : i;
                const size_t io = ((size_t)b * L + t) * a.D + dd;
                dtk[k] = ldv(dl, io);
                xk[k] = ldv(x, io);
            }
        }
        __syncthreads();   // the previous chunk is done with bc
        stage_bc<T, NS, false>(a, b, i0, bc);
        __syncthreads();
#pragma unroll
        for (int k = 0; k < kKc; k++) {
            const float dt = (i0 + k < L) ? dt_of(dtk[k] + bias, a.softplus) : 0.f;
            const float dtx = dt * xk[k];
#pragma unroll
            for (int n = 0; n < NS; n++)
                h[n] = fmaf(ex2_mufu(dt * Al[n]), h[n], dtx * bc[k][n]);
        }
    }
}

template <typename T, int NS>
__global__ void __launch_bounds__(kCta) s6_bwd_kernel(const BwdArgs a)
{
    // states of the current chunk: hs[k][n][thread]; the chunk's B and C
    // rows; this thread's per-step scalars sc[k][dt, x, dout, z][thread]
    __shared__ float hs[kKc][NS][kCta];
    __shared__ float bc[kKc][2 * NS];
    __shared__ float sc[kKc][5][kCta];
    const int tid = threadIdx.x, lane = tid & 31;
    const int d = blockIdx.x * kCta + tid;
    const int b = blockIdx.y;
    const bool active = d < a.D;
    const int dd = active ? d : 0;
    const int N = a.N, L = a.L, nch = (L + kKc - 1) / kKc;
    const T *x = static_cast<const T *>(a.x), *dl = static_cast<const T *>(a.delta);
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
        __syncthreads();   // the previous chunk is done with bc, hs and sc
        // this chunk's per-step scalars and the checkpoint, all loads issued together
#pragma unroll
        for (int k = 0; k < kKc; k++) {
            float v = 0.f, xv = 0.f, g = 0.f, zv = 0.f;
            if (active && k < kn) {
                const int t = a.reverse ? L - 1 - (i0 + k) : i0 + k;
                const size_t io = ((size_t)b * L + t) * a.D + dd;
                v = ldv(dl, io) + bias;
                xv = ldv(x, io);
                g = ldv(go, io);
                if (zp)
                    zv = ldv(zp, io);
            }
            sc[k][0][tid] = v;
            sc[k][1][tid] = xv;
            sc[k][2][tid] = g;
            sc[k][3][tid] = zv;
        }
        float hp[NS];
        const float *ck = a.ckpt + (((size_t)b * nch + c) * a.D + dd) * N;
#pragma unroll
        for (int n = 0; n < NS; n++)
            hp[n] = (active && n < N) ? ck[n] : 0.f;
        stage_bc<T, NS, true>(a, b, i0, bc);
        __syncthreads();
        // recompute the chunk's states from the checkpoint
        {
            float h[NS];
#pragma unroll
            for (int n = 0; n < NS; n++)
                h[n] = hp[n];
#pragma unroll
            for (int k = 0; k < kKc; k++) {
                const float dt = (k < kn) ? dt_of(sc[k][0][tid], a.softplus) : 0.f;
                sc[k][4][tid] = dt;
                const float dtx = dt * sc[k][1][tid];
#pragma unroll
                for (int n = 0; n < NS; n++) {
                    h[n] = fmaf(ex2_mufu(dt * Al[n]), h[n], dtx * bc[k][n]);
                    hs[k][n][tid] = h[n];
                }
            }
        }
        // backward sweep over the chunk; hk holds h_k, loaded once per step
        float hk[NS];
#pragma unroll
        for (int n = 0; n < NS; n++)
            hk[n] = hs[kn - 1][n][tid];
#pragma unroll 1
        for (int k = kn - 1; k >= 0; k--) {
            const int t = a.reverse ? L - 1 - (i0 + k) : i0 + k;
            const size_t row = (size_t)b * L + t;
            const size_t io = row * a.D + dd;
            const float dt = sc[k][4][tid], xv = sc[k][1][tid], dtx = dt * xv;
            const float gk = sc[k][2][tid], zk = sc[k][3][tid];
            // y_i = C . h_i + D x_i, then the gate
            float y = Dv * xv;
#pragma unroll
            for (int n = 0; n < NS; n++)
                y = fmaf(bc[k][NS + n], hk[n], y);
            float dy = gk;
            if (zp) {
                const float s = sigmoid_f(zk);
                dy = gk * zk * s;
                if (active && a.dz)
                    a.dz[io] = gk * y * s * (1.f + zk * (1.f - s));
            }
            if (!active)
                dy = 0.f;
            float ddt = 0.f, dxs = 0.f;
            float red[32];
#pragma unroll
            for (int n = 0; n < NS; n++) {
                const float Bn = bc[k][n], Cn = bc[k][NS + n];
                const float hprev = k > 0 ? hs[k - 1 < 0 ? 0 : k - 1][n][tid] : hp[n];
                const float hcur = hk[n];
                hk[n] = hprev;                                  // h_{k-1} for the next step
                const float an = ex2_mufu(dt * Al[n]);
                const float l = fmaf(dy, Cn, lam[n]);        // lam_i[n]
                red[n] = l * dtx;                              // dB contribution
                red[16 + n] = dy * hcur;                       // dC contribution
                dxs = fmaf(l, Bn, dxs);
                const float ah = an * hprev;
                ddt = fmaf(l, fmaf(Bn, xv, A[n] * ah), ddt);
                gA[n] = fmaf(l * dt, ah, gA[n]);
                lam[n] = an * l;                               // a_i lam_i for step i - 1
            }
#pragma unroll
            for (int n = NS; n < 16; n++)
                red[n] = red[16 + n] = 0.f;
            if (active) {
                a.dx[io] = (a.accumulate ? a.dx[io] : 0.f) + fmaf(dy, Dv, dt * dxs);
                const float dv = a.softplus ? ddt * sigmoid_f(sc[k][0][tid]) : ddt;
                a.ddelta[io] = (a.accumulate ? a.ddelta[io] : 0.f) + dv;
                gbias += dv;
                gD = fmaf(dy, xv, gD);
            }
            // dB, dC summed over the warp's 32 channels; lane j holds value j
            const float s = warp_transpose_sum(red);
            const int n = lane & 15;
            if (n < N)
                atomicAdd((lane < 16 ? a.dB : a.dC) + row * N + n, s);
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
