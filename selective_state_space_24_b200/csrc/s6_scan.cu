// s6_scan.cu -- Mamba S6 selective scan and the fused Vision-Mamba
// bidirectional scan for sm_100a.
//
// Operation (Mamba2 page "手写简化版Mamba2", sec. 2.2, 4.3, 4.4; Vim page
// sec. 3.1-3.2): for every (batch b, channel d) and state n
//     dt      = softplus(delta[b,t,d] + bias[d])
//     h[n]    = exp(dt A[d,n]) h[n] + dt B[b,t,n] x[b,t,d]
//     y[b,t,d]= (sum_n C[b,t,n] h[n] + D[d] x[b,t,d]) silu(z[b,t,d])
// and, bidirectionally, the same with the sequence reversed and a second
// parameter set, the two results summed.
//
// Work decomposition
//   * One thread owns one (b, d, direction) column and keeps its N states in
//     fp32 registers; the h sequence never leaves the SM (the fusion rule of
//     the pages: never materialise (B, L, D, N)).
//   * Lanes of a warp own 32 consecutive channels, so every x / delta / z
//     access of a warp is one contiguous row segment.  B[t], C[t] are the
//     same for every lane (broadcast loads).
//   * Bidirectional: a CTA holds warp pairs (forward warp, reversed warp)
//     over the same 32 channels.  The forward warp walks its segment upward
//     while the reversed warp walks it downward; each stashes the first half
//     of its outputs in shared memory, one barrier at the middle, and in the
//     second half each adds the other direction's stashed value and writes
//     the final sum.  out is written exactly once; x and delta are read by
//     both warps of the CTA, the second read served from L1/L2.
//   * Long sequences are cut into S segments (the chunked scan with
//     state hand-off of the Mamba2 page sec. 3.2): a summary kernel computes
//     each segment's local end state and sum of dt, a carry kernel composes
//     them with (a, b) o (a', b') = (a a', a' b + b'), and the main kernel
//     rescans every segment from its true entering state.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"

namespace ssm {
namespace {

constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float ex2_approx(float v)
{
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(v));
    return r;
}

template <typename T> __device__ __forceinline__ float ldf(const T *p, size_t i);
template <> __device__ __forceinline__ float ldf<float>(const float *p, size_t i) { return __ldg(p + i); }
template <> __device__ __forceinline__ float ldf<__nv_bfloat16>(const __nv_bfloat16 *p, size_t i)
{
    return __bfloat162float(__ldg(p + i));
}

template <typename T> __device__ __forceinline__ void stf(T *p, size_t i, float v);
template <> __device__ __forceinline__ void stf<float>(float *p, size_t i, float v) { p[i] = v; }
template <> __device__ __forceinline__ void stf<__nv_bfloat16>(__nv_bfloat16 *p, size_t i, float v)
{
    p[i] = __float2bfloat16_rn(v);
}

// dt' = softplus(v) with the usual threshold (softplus(v) = v above 20).
__device__ __forceinline__ float softplus_f(float v)
{
    return v > 20.f ? v : log1pf(expf(v));
}

__device__ __forceinline__ float silu_f(float z) { return z / (1.f + expf(-z)); }

// Is `seg` the first segment in this direction's scan order (zero entering state)?
__device__ __forceinline__ bool first_in_order(int seg, int S, bool rev) { return rev ? seg == S - 1 : seg == 0; }
// Is `seg` the last segment in scan order (its end state is last_state)?
__device__ __forceinline__ bool last_in_order(int seg, int S, bool rev) { return rev ? seg == 0 : seg == S - 1; }

// ---------------------------------------------------------------- summary
// Per (direction, b, segment, d): local end state from zero and sum of dt
// over the segment.  Only segments whose summary a later one needs.
template <typename T, int NS>
__global__ void __launch_bounds__(128) s6_summary_kernel(const S6Args a)
{
    const int d = blockIdx.x * blockDim.x + threadIdx.x;
    const int seg = blockIdx.y;
    const int dsel = blockIdx.z % a.ndir;
    const int b = blockIdx.z / a.ndir;
    const bool rev = a.ndir == 2 ? dsel == 1 : a.reverse != 0;
    if (d >= a.D || last_in_order(seg, a.S, rev))
        return;
    const DirArgs &P = a.dir[dsel];
    const int N = a.N;
    const int s0 = seg * a.T, s1 = min(a.L, s0 + a.T), Tn = s1 - s0;
    const T *x = static_cast<const T *>(a.x);
    const T *dl = static_cast<const T *>(a.delta);
    const T *Bm = static_cast<const T *>(P.B);
    float Al2[NS], h[NS];
#pragma unroll
    for (int n = 0; n < NS; n++) {
        Al2[n] = n < N ? P.A[(size_t)d * N + n] * kLog2e : 0.f;
        h[n] = 0.f;
    }
    const float bias = P.bias ? P.bias[d] : 0.f;
    float sdt = 0.f;
    for (int i = 0; i < Tn; i++) {
        const int t = rev ? s1 - 1 - i : s0 + i;
        const size_t row = (size_t)b * a.L + t;
        const float xv = ldf(x, row * a.D + d);
        float dt = ldf(dl, row * a.D + d) + bias;
        if (a.softplus)
            dt = softplus_f(dt);
        sdt += dt;
        const float dtx = dt * xv;
#pragma unroll
        for (int n = 0; n < NS; n++) {
            const float bn = n < N ? ldf(Bm, row * N + n) : 0.f;
            h[n] = fmaf(ex2_approx(dt * Al2[n]), h[n], dtx * bn);
        }
    }
    const size_t ci = (((size_t)dsel * a.Bsz + b) * a.S + seg) * a.D + d;
#pragma unroll
    for (int n = 0; n < NS; n++)
        if (n < N)
            a.carry_h[ci * N + n] = h[n];
    a.carry_s[ci] = sdt;
}

// ------------------------------------------------------------------ carry
// Per (direction, b, d, n): walk the segments in scan order, replace each
// summary by the state entering that segment.
__global__ void s6_carry_kernel(const S6Args a)
{
    const size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    const size_t total = (size_t)a.ndir * a.Bsz * a.D * a.N;
    if (idx >= total)
        return;
    const int n = idx % a.N;
    const int d = (idx / a.N) % a.D;
    const int b = (idx / ((size_t)a.N * a.D)) % a.Bsz;
    const int dsel = idx / ((size_t)a.N * a.D * a.Bsz);
    const bool rev = a.ndir == 2 ? dsel == 1 : a.reverse != 0;
    const float Al2 = a.dir[dsel].A[(size_t)d * a.N + n] * kLog2e;
    float hin = 0.f;
    for (int k = 0; k < a.S; k++) {
        const int seg = rev ? a.S - 1 - k : k;
        const size_t ci = (((size_t)dsel * a.Bsz + b) * a.S + seg) * a.D + d;
        if (k == a.S - 1) {
            a.carry_h[ci * a.N + n] = hin;
            break;
        }
        const float hl = a.carry_h[ci * a.N + n];
        const float s = a.carry_s[ci];
        a.carry_h[ci * a.N + n] = hin;
        hin = fmaf(ex2_approx(Al2 * s), hin, hl);
    }
}

// ------------------------------------------------------------------- main
template <typename T, int NS, bool BIDIR>
__global__ void __launch_bounds__(128) s6_main_kernel(const S6Args a)
{
    extern __shared__ float stash[];  // BIDIR: [pair][T][32]
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int dsel = BIDIR ? (warp & 1) : 0;
    const int dbase = BIDIR ? (blockIdx.x * 2 + (warp >> 1)) * 32 : (blockIdx.x * 4 + warp) * 32;
    const int d = dbase + lane;
    const bool active = d < a.D;
    const int seg = blockIdx.y, b = blockIdx.z;
    const int N = a.N;
    const int s0 = seg * a.T, s1 = min(a.L, s0 + a.T), Tn = s1 - s0;
    const bool rev = BIDIR ? dsel == 1 : a.reverse != 0;
    const DirArgs &P = a.dir[dsel];
    const T *x = static_cast<const T *>(a.x);
    const T *dl = static_cast<const T *>(a.delta);
    const T *Bm = static_cast<const T *>(P.B);
    const T *Cm = static_cast<const T *>(P.C);
    const T *zp = static_cast<const T *>(P.z);
    T *out = static_cast<T *>(a.out);

    float Al2[NS], h[NS];
    const bool has_carry = a.S > 1 && !first_in_order(seg, a.S, rev);
    const size_t ci = (((size_t)dsel * a.Bsz + b) * a.S + seg) * a.D + d;
#pragma unroll
    for (int n = 0; n < NS; n++) {
        Al2[n] = (active && n < N) ? P.A[(size_t)d * N + n] * kLog2e : 0.f;
        h[n] = (active && n < N && has_carry) ? a.carry_h[ci * N + n] : 0.f;
    }
    const float bias = (active && P.bias) ? P.bias[d] : 0.f;
    const float Dd = (active && P.D) ? P.D[d] : 0.f;
    const bool gate = zp != nullptr;

    auto step = [&](int t) -> float {
        const size_t row = (size_t)b * a.L + t;
        const size_t io = row * a.D + d;
        const float xv = active ? ldf(x, io) : 0.f;
        float dt = (active ? ldf(dl, io) : 0.f) + bias;
        if (a.softplus)
            dt = softplus_f(dt);
        const float dtx = dt * xv;
        float y = 0.f;
#pragma unroll
        for (int n = 0; n < NS; n++) {
            const float bn = n < N ? ldf(Bm, row * N + n) : 0.f;
            const float cn = n < N ? ldf(Cm, row * N + n) : 0.f;
            h[n] = fmaf(ex2_approx(dt * Al2[n]), h[n], dtx * bn);
            y = fmaf(cn, h[n], y);
        }
        y = fmaf(Dd, xv, y);
        if (gate) {
            const float zv = active ? ldf(zp, io) : 0.f;
            y *= silu_f(zv);
        }
        return y;
    };

    if (!BIDIR) {
        for (int i = 0; i < Tn; i++) {
            const int t = rev ? s1 - 1 - i : s0 + i;
            const float y = step(t);
            if (active)
                stf(out, ((size_t)b * a.L + t) * a.D + d, y);
        }
    } else {
        float *st = stash + (size_t)(warp >> 1) * a.T * 32;
        // forward warp stashes local steps [0, ceil(Tn/2)), reversed warp
        // stashes [ceil(Tn/2), Tn); after the barrier each finishes the other half.
        const int half = rev ? Tn / 2 : (Tn + 1) / 2;
        for (int i = 0; i < half; i++) {
            const int t = rev ? s1 - 1 - i : s0 + i;
            st[(t - s0) * 32 + lane] = step(t);
        }
        __syncthreads();
        for (int i = half; i < Tn; i++) {
            const int t = rev ? s1 - 1 - i : s0 + i;
            const float y = step(t);
            if (active)
                stf(out, ((size_t)b * a.L + t) * a.D + d, y + st[(t - s0) * 32 + lane]);
        }
    }
    if (active && P.last_state && last_in_order(seg, a.S, rev)) {
#pragma unroll
        for (int n = 0; n < NS; n++)
            if (n < N)
                P.last_state[((size_t)b * a.D + d) * N + n] = h[n];
    }
}

template <typename T, int NS>
cudaError_t launch_typed(const S6Args &a, cudaStream_t st)
{
    if (a.S > 1) {
        dim3 g1((a.D + 127) / 128, a.S, a.Bsz * a.ndir);
        s6_summary_kernel<T, NS><<<g1, 128, 0, st>>>(a);
        const size_t tot = (size_t)a.ndir * a.Bsz * a.D * a.N;
        s6_carry_kernel<<<(unsigned)((tot + 255) / 256), 256, 0, st>>>(a);
    }
    if (a.ndir == 2) {
        const size_t smem = (size_t)2 * a.T * 32 * sizeof(float);
        auto k = s6_main_kernel<T, NS, true>;
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess)
            return e;
        dim3 g((a.D + 63) / 64, a.S, a.Bsz);
        k<<<g, 128, smem, st>>>(a);
    } else {
        dim3 g((a.D + 127) / 128, a.S, a.Bsz);
        s6_main_kernel<T, NS, false><<<g, 128, 0, st>>>(a);
    }
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_ns(const S6Args &a, cudaStream_t st)
{
    if (a.N <= 4)
        return launch_typed<T, 4>(a, st);
    if (a.N <= 8)
        return launch_typed<T, 8>(a, st);
    return launch_typed<T, 16>(a, st);
}

}  // namespace

S6Plan plan_s6(int64_t Bsz, int64_t L, int64_t D, int64_t N, int ndir)
{
    S6Plan p{1, (int)L, 0};
    if (L <= 0)
        return p;
    const int64_t kMaxT = 256;            // bidir stash: 2 pairs * T * 32 * 4 B <= 64 KB
    const int64_t kMinT = 16;
    const int64_t kTargetThreads = 148 * 384;
    const int64_t cols = (int64_t)ndir * Bsz * D;
    int64_t S = 1;
    if (cols > 0 && cols < kTargetThreads)
        S = (kTargetThreads + cols - 1) / cols;
    const int64_t smax = (L + kMinT - 1) / kMinT;
    if (S > smax)
        S = smax;
    if (ndir == 2) {
        const int64_t smin = (L + kMaxT - 1) / kMaxT;
        if (S < smin)
            S = smin;
    }
    if (S < 1)
        S = 1;
    int64_t T = (L + S - 1) / S;
    S = (L + T - 1) / T;
    p.S = (int)S;
    p.T = (int)T;
    if (S > 1)
        p.workspace_bytes = (size_t)ndir * Bsz * S * D * (N + 1) * sizeof(float) + 256;
    return p;
}

cudaError_t launch_s6(const S6Args &a, cudaStream_t st)
{
    if (a.dtype == 0)
        return launch_ns<float>(a, st);
    return launch_ns<__nv_bfloat16>(a, st);
}

}  // namespace ssm
