// s6_bwd_split.cu -- gradients of the single-direction S6 scan (N = 16)
// with each channel's 16 states split over four threads, from the state
// entering every 4-step chunk (the checkpoint array the checkpointing
// forward or the recompute pass of s6_bwd.cu writes).  Same operation and
// formulas as s6_bwd.cu (the adjoint of the Mamba2 page "手写简化版Mamba2",
// sec. 5.1, written out and run as a reverse scan):
//   dy_i = g_i silu(z_i),  dz_i = g_i y_i silu'(z_i),
//   lam_i = dy_i C_i + a_{i+1} lam_{i+1},
//   dC_i += dy_i h_i,  dB_i += lam_i dt_i x_i,  dx_i = dy_i D + dt_i lam_i . B_i,
//   ddt_i = lam_i . (B_i x_i + A a_i h_{i-1}),  dA += lam_i dt_i a_i h_{i-1},
//   ddelta_i = ddt_i softplus'(v_i).
//
// Thread (g, q) of a warp (g = lane / 4) owns states [4q, 4q + 4) of
// channel d0 + g of the warp's 8 channels.  A chunk runs
//   A  thread q: the scalars of step q (dt, dt x, dy, the gate) once per
//      channel; shuffles hand them to the channel's other three threads;
//   B  every thread recomputes its 4 states over the chunk from the
//      checkpoint, keeping h and a = exp(dt A) of every step (so the sweep
//      needs no second exp), and its share of C . h per step, summed over
//      the channel's threads so that thread q holds y of step q (for dz);
//   C  the sweep over the chunk's steps backwards: lam and the per-state
//      products; dB / dC of each step summed over the warp's 8 channels by
//      a shuffle butterfly and then over the CTA's 4 warps in shared memory,
//      one atomic per (step, state); dx / ddt summed over the channel's
//      threads so that thread q stores step q's dx, ddelta.
// A CTA is 4 warps (32 channels): the same atomic count per step as the
// one-thread-per-channel kernel, which sums over a warp of 32 channels.
// Each warp streams the chunks' rows (delta, x, dout, z for 8 channels; B,
// C rows) and the chunk's checkpoint through a cp.async ring, chunks in
// descending order.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"
#include "s6_math.cuh"

namespace ssm {
namespace {

constexpr int kQ = 4;          // threads per channel
constexpr int kChW = 32 / kQ;  // channels per warp
constexpr int kWarpsB = 4;     // warps per CTA
constexpr int kKc = 4;         // steps per chunk: thread q owns step q's scalars
constexpr int kStages = 3;     // chunks in the copy ring
static_assert(kKc == kQ, "thread q of a channel takes step q of a chunk");

// Smallest stride >= bytes (16-byte steps) whose word offset mod 32 is an
// odd multiple of w: the 4 threads of a channel reading 4 steps' rows at
// once then hit distinct banks.
constexpr int skew_stride(int bytes, int w)
{
    int s = bytes;
    while (!(((s / 4) % 32) % w == 0 && (((s / 4) % 32) / w) % 2 == 1))
        s += 16;
    return s;
}

template <typename T, bool GATE> struct BSlot {
    static constexpr int kRow = kChW * (int)sizeof(T);   // 8 channels of delta, x, dout or z
    static constexpr int kBC = 16 * (int)sizeof(T);
    static constexpr int kDl = 0, kX = kRow, kG = 2 * kRow, kZ = 3 * kRow;
    static constexpr int kB = (GATE ? 4 : 3) * kRow, kC = kB + kBC;
    static constexpr int kStepBytes = kC + kBC;
    static constexpr int kStepPieces = kStepBytes / 16;
    static constexpr int kStride = skew_stride(kStepBytes, kRow / 4);
    static constexpr int kCk = kKc * kStride;                   // the chunk's checkpoint: 8 x 16 floats
    static constexpr int kChunkBytes = kCk + kChW * 16 * 4;
    static constexpr int kPieces = kKc * kStepPieces + kChW * 16 * 4 / 16;
    static constexpr int kPerLane = (kPieces + 31) / 32;
    static_assert(kStepBytes % 16 == 0 && kRow % 16 == 0 && kB % 16 == 0, "16-byte pieces");
};

__device__ __forceinline__ void cp16(uint32_t dst, const char *src, int n)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int K> __device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(K) : "memory"); }

template <typename T> __device__ __forceinline__ float lds1(const char *p);
template <> __device__ __forceinline__ float lds1<float>(const char *p) { return *reinterpret_cast<const float *>(p); }
template <> __device__ __forceinline__ float lds1<__nv_bfloat16>(const char *p)
{
    return __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(p));
}
template <typename T> __device__ __forceinline__ float4 lds4(const char *p);
template <> __device__ __forceinline__ float4 lds4<float>(const char *p) { return *reinterpret_cast<const float4 *>(p); }
template <> __device__ __forceinline__ float4 lds4<__nv_bfloat16>(const char *p)
{
    const uint2 u = *reinterpret_cast<const uint2 *>(p);
    return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u), __uint_as_float(u.y << 16),
                       __uint_as_float(u.y & 0xffff0000u));
}

__device__ __forceinline__ float sigmoid_f(float v) { return 1.f / (1.f + ex2_mufu(-v * kLog2e)); }

template <typename T, bool GATE> struct BwdSplitSmem {
    __align__(16) char ring[kWarpsB][kStages][BSlot<T, GATE>::kChunkBytes];
    float red[2][kKc][kWarpsB][32];   // per chunk parity: each warp's channel-summed dB / dC by step
};

#ifndef SSM_BWD_SPLIT_MINB
#define SSM_BWD_SPLIT_MINB 4
#endif
#ifndef SSM_BWD_SPLIT_KEEP_A
#define SSM_BWD_SPLIT_KEEP_A 1
#endif
template <typename T, bool GATE>
__global__ void __launch_bounds__(32 * kWarpsB, SSM_BWD_SPLIT_MINB) s6_bwd_split_kernel(const BwdArgs a)
{
    using S = BSlot<T, GATE>;
    __shared__ BwdSplitSmem<T, GATE> sm;
    constexpr float kLn2 = 0.693147180559945309f;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, q = lane & 3;
    const int d0w = blockIdx.x * (kChW * kWarpsB) + warp * kChW;   // the warp's first channel
    const int d = d0w + g;
    const int b = blockIdx.y;
    const int L = a.L, D = a.D, nch = (L + kKc - 1) / kKc;
    const bool active = d < D;
    const bool rev = a.reverse != 0;

    // this thread's states [4q, 4q + 4), A scaled by log2(e)
    float4 A4 = make_float4(0.f, 0.f, 0.f, 0.f);
    if (active)
        A4 = *reinterpret_cast<const float4 *>(a.A + (size_t)d * 16 + 4 * q);
    const float2 Al[2] = {make_float2(A4.x * kLog2e, A4.y * kLog2e), make_float2(A4.z * kLog2e, A4.w * kLog2e)};
    const float bias = (active && a.bias) ? a.bias[d] : 0.f;
    const float Dv = (active && a.Dskip) ? a.Dskip[d] : 0.f;
    float2 lam[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};   // a_{i+1} lam_{i+1}, carried backwards
    float2 gA[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};    // dA
    float gD = 0.f, gbias = 0.f;

    // --- copies: this lane's pieces of a chunk (piece p = lane + 32 j)
    const uint32_t ring_s = (uint32_t)__cvta_generic_to_shared(&sm.ring[warp][0][0]);
    const char *safe = static_cast<const char *>(a.x);
    const char *cur[S::kPerLane];
    int cstep[S::kPerLane];         // bytes from one chunk's source to the previous chunk's
    uint32_t dst[S::kPerLane];
    bool pok[S::kPerLane];
    const int c0 = nch - 1;         // the first chunk processed
#pragma unroll
    for (int j = 0; j < S::kPerLane; j++) {
        const int p = lane + 32 * j;
        const bool exists = p < S::kPieces;
        const int pp = exists ? p : 0;
        bool ok = exists;
        const char *base;
        long long step;
        if (pp < kKc * S::kStepPieces) {
            const int s = pp / S::kStepPieces, off = (pp % S::kStepPieces) * 16;
            dst[j] = (uint32_t)(s * S::kStride + off);
            const int i0 = c0 * kKc + s;
            const long long t0 = rev ? (long long)L - 1 - i0 : i0;   // may lie outside [0, L) only for a
                                                                     // step past L (never read)
            long long row;
            if (off < S::kB) {
                const int arr = off / S::kRow, jb = off % S::kRow;
                const void *src = arr == 0 ? a.delta : arr == 1 ? a.x : arr == 2 ? a.dout : a.z;
                ok = ok && d0w + jb / (int)sizeof(T) < D;
                row = (long long)D * sizeof(T);
                base = reinterpret_cast<const char *>(src) + ((long long)b * L + t0) * row +
                       (long long)d0w * sizeof(T) + jb;
            } else {
                const int o2 = off - S::kB;
                row = 16 * (long long)sizeof(T);
                base = reinterpret_cast<const char *>(o2 < S::kBC ? a.B : a.C) + ((long long)b * L + t0) * row +
                       o2 % S::kBC;
            }
            step = (rev ? 1 : -1) * (long long)kKc * row;   // chunks descend: t descends (ascends reversed)
        } else {
            const int cp = pp - kKc * S::kStepPieces;   // 16 bytes of the checkpoint rows
            dst[j] = (uint32_t)(S::kCk + cp * 16);
            ok = ok && d0w + cp / 4 < D;
            base = reinterpret_cast<const char *>(a.ckpt) + (((long long)b * nch + c0) * D + d0w) * 64 + cp * 16;
            step = -(long long)D * 64;
        }
        pok[j] = ok;
        cur[j] = ok ? base : safe;
        cstep[j] = ok ? (int)step : 0;
    }
    auto issue = [&](int jj) {   // processed index jj: chunk nch - 1 - jj
        if (jj < nch) {
            const int c = nch - 1 - jj;
            const uint32_t sb = ring_s + (uint32_t)((jj % kStages) * S::kChunkBytes);
            if ((c + 1) * kKc <= L) {
#pragma unroll
                for (int j = 0; j < S::kPerLane; j++)
                    if (lane + 32 * j < S::kPieces)
                        cp16(sb + dst[j], cur[j], pok[j] ? 16 : 0);
            } else {   // the short last chunk: steps past L are zero-filled, not read
#pragma unroll
                for (int j = 0; j < S::kPerLane; j++) {
                    const int p = lane + 32 * j;
                    if (p < S::kPieces) {
                        const bool ck = p >= kKc * S::kStepPieces;
                        const bool in = pok[j] && (ck || c * kKc + p / S::kStepPieces < L);
                        cp16(sb + dst[j], in ? cur[j] : safe, in ? 16 : 0);
                    }
                }
            }
#pragma unroll
            for (int j = 0; j < S::kPerLane; j++)
                cur[j] += cstep[j];
        }
        cp_commit();
    };
#pragma unroll
    for (int k = 0; k < kStages - 1; k++)
        issue(k);

    const bool acc = a.accumulate != 0;
    const int base_sh = lane & ~3;
    for (int jj = 0; jj < nch; jj++) {
        const int c = nch - 1 - jj;
        issue(jj + kStages - 1);
        cp_wait<kStages - 1>();
        __syncwarp();
        const char *cs = &sm.ring[warp][jj % kStages][0];
        const int i0 = c * kKc;
        // A: step q's scalars
        const int iq = i0 + q;
        const bool vq = iq < L;
        const char *sq = cs + q * S::kStride + g * (int)sizeof(T);
        const float vraw = lds1<T>(sq + S::kDl) + bias;
        const float xq = lds1<T>(sq + S::kX);
        const float gq = lds1<T>(sq + S::kG);
        float dtq = a.softplus ? softplus_f(vraw) : vraw;
        dtq = vq ? dtq : 0.f;
        const float dtxq = dtq * xq;
        float zq = 0.f, sgq = 0.f, dyq = gq;
        if (GATE) {
            zq = lds1<T>(sq + S::kZ);
            sgq = sigmoid_f(zq);
            dyq = gq * zq * sgq;
        }
        dyq = (vq && active) ? dyq : 0.f;
        const size_t rowq = (size_t)b * L + (rev ? L - 1 - iq : iq);
        const size_t ioq = rowq * D + (active ? d : 0);
        float old_dx = 0.f, old_dd = 0.f;
        if (acc && vq && active) {
            old_dx = a.dx[ioq];
            old_dd = a.ddelta[ioq];
        }
        float dt[kKc], dtx[kKc], dy[kKc];
#pragma unroll
        for (int k = 0; k < kKc; k++) {
            dt[k] = __shfl_sync(0xffffffffu, dtq, base_sh | k);
            dtx[k] = __shfl_sync(0xffffffffu, dtxq, base_sh | k);
            dy[k] = __shfl_sync(0xffffffffu, dyq, base_sh | k);
        }
        // B: recompute the chunk's states from the checkpoint, keeping h and a
        float2 h[kKc + 1][2], an[kKc][2];
        {
            const float4 c4 = *reinterpret_cast<const float4 *>(cs + S::kCk + g * 64 + q * 16);
            h[0][0] = make_float2(c4.x, c4.y);
            h[0][1] = make_float2(c4.z, c4.w);
        }
        float yp[kKc];
#pragma unroll
        for (int k = 0; k < kKc; k++) {
            const char *sk = cs + k * S::kStride + q * 4 * (int)sizeof(T);
            const float4 B4 = lds4<T>(sk + S::kB), C4 = lds4<T>(sk + S::kC);
            const float2 dt2 = make_float2(dt[k], dt[k]), dtx2 = make_float2(dtx[k], dtx[k]);
#pragma unroll
            for (int e = 0; e < 2; e++) {
                const float2 w = __fmul2_rn(dt2, Al[e]);
                an[k][e] = make_float2(ex2_mufu(w.x), ex2_mufu(w.y));
                h[k + 1][e] = __ffma2_rn(an[k][e], h[k][e],
                                         __fmul2_rn(dtx2, e ? make_float2(B4.z, B4.w) : make_float2(B4.x, B4.y)));
            }
            float2 y2 = __fmul2_rn(make_float2(C4.x, C4.y), h[k + 1][0]);
            y2 = __ffma2_rn(make_float2(C4.z, C4.w), h[k + 1][1], y2);
            yp[k] = y2.x + y2.y;
        }
        // y of step q, summed over the channel's four threads, then dz
        {
            const bool hi1 = (q & 2) != 0, hi0 = (q & 1) != 0;
            float ka = hi1 ? yp[2] : yp[0], kb = hi1 ? yp[3] : yp[1];
            ka += __shfl_xor_sync(0xffffffffu, hi1 ? yp[0] : yp[2], 2);
            kb += __shfl_xor_sync(0xffffffffu, hi1 ? yp[1] : yp[3], 2);
            const float ys = (hi0 ? kb : ka) + __shfl_xor_sync(0xffffffffu, hi0 ? ka : kb, 1);
            if (GATE && a.dz && vq && active)
                a.dz[ioq] = gq * fmaf(Dv, xq, ys) * sgq * (1.f + zq * (1.f - sgq));
        }
        // C: the sweep, steps descending (a = exp(dt A) kept from the
        // recompute, or recomputed here when registers are short)
        float dxs[kKc], dta[kKc];
        float (*red)[kWarpsB][32] = sm.red[jj & 1];
#pragma unroll
        for (int k = kKc - 1; k >= 0; k--) {
            const char *sk = cs + k * S::kStride + q * 4 * (int)sizeof(T);
            const float4 B4 = lds4<T>(sk + S::kB), C4 = lds4<T>(sk + S::kC);
            const float2 dy2 = make_float2(dy[k], dy[k]), dtx2 = make_float2(dtx[k], dtx[k]),
                         dt2 = make_float2(dt[k], dt[k]);
            float2 dxs2 = make_float2(0.f, 0.f), dta2 = make_float2(0.f, 0.f);
            float v[8];   // dB of states 4q..4q+3, then dC
#pragma unroll
            for (int e = 0; e < 2; e++) {
                const float2 Bn = e ? make_float2(B4.z, B4.w) : make_float2(B4.x, B4.y);
                const float2 Cn = e ? make_float2(C4.z, C4.w) : make_float2(C4.x, C4.y);
                const float2 l = __ffma2_rn(dy2, Cn, lam[e]);                  // lam_i
                const float2 rb = __fmul2_rn(l, dtx2);
                const float2 rc = __fmul2_rn(dy2, h[k + 1][e]);
                v[2 * e] = rb.x;
                v[2 * e + 1] = rb.y;
                v[4 + 2 * e] = rc.x;
                v[4 + 2 * e + 1] = rc.y;
                dxs2 = __ffma2_rn(l, Bn, dxs2);
                float2 ak;
                if (SSM_BWD_SPLIT_KEEP_A) {
                    ak = an[k][e];
                } else {
                    const float2 w = __fmul2_rn(dt2, Al[e]);
                    ak = make_float2(ex2_mufu(w.x), ex2_mufu(w.y));
                }
                const float2 lah = __fmul2_rn(l, __fmul2_rn(ak, h[k][e]));   // lam_i a_i h_{i-1}
                dta2 = __ffma2_rn(lah, Al[e], dta2);
                gA[e] = __ffma2_rn(dt2, lah, gA[e]);
                lam[e] = __fmul2_rn(ak, l);
            }
            dxs[k] = dxs2.x + dxs2.y;
            dta[k] = dta2.x + dta2.y;
            // sum the 8 values over the warp's 8 channels (lanes g = 0..7 with
            // this q): afterwards lane (g, q) holds value g
#pragma unroll
            for (int o = 4; o >= 1; o >>= 1) {
                const bool up = (g & o) != 0;
#pragma unroll
                for (int i = 0; i < o; i++) {
                    const float send = up ? v[i] : v[i + o];
                    const float keep = up ? v[i + o] : v[i];
                    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 4 * o);
                }
            }
            red[k][warp][lane] = v[0];
        }
        // dx, ddt of step q: the channel's four threads' sums
        {
            const bool hi1 = (q & 2) != 0, hi0 = (q & 1) != 0;
            float xa = hi1 ? dxs[2] : dxs[0], xb = hi1 ? dxs[3] : dxs[1];
            float ta = hi1 ? dta[2] : dta[0], tb = hi1 ? dta[3] : dta[1];
            xa += __shfl_xor_sync(0xffffffffu, hi1 ? dxs[0] : dxs[2], 2);
            xb += __shfl_xor_sync(0xffffffffu, hi1 ? dxs[1] : dxs[3], 2);
            ta += __shfl_xor_sync(0xffffffffu, hi1 ? dta[0] : dta[2], 2);
            tb += __shfl_xor_sync(0xffffffffu, hi1 ? dta[1] : dta[3], 2);
            const float dxsum = (hi0 ? xb : xa) + __shfl_xor_sync(0xffffffffu, hi0 ? xa : xb, 1);
            const float dtsum = (hi0 ? tb : ta) + __shfl_xor_sync(0xffffffffu, hi0 ? ta : tb, 1);
            if (vq && active) {
                const float ddt = fmaf(xq, dxsum, kLn2 * dtsum);
                a.dx[ioq] = old_dx + fmaf(dyq, Dv, dtq * dxsum);
                const float dv = a.softplus ? ddt * sigmoid_f(vraw) : ddt;
                a.ddelta[ioq] = old_dd + dv;
                gbias += dv;
                gD = fmaf(dyq, xq, gD);
            }
        }
        // dB / dC of the chunk's steps, summed over the CTA's 4 warps: one
        // atomic per (step, state); the other parity's buffer is free for the
        // next chunk
        __syncthreads();
        {
            const int k = threadIdx.x >> 5, l = threadIdx.x & 31;   // 128 threads: 4 steps x 32 values
            const int i = i0 + k;
            const int gg = l >> 2, qq = l & 3;
            const int n = 4 * qq + (gg & 3);
            if (i < L) {
                const float s = red[k][0][l] + red[k][1][l] + red[k][2][l] + red[k][3][l];
                const size_t row = (size_t)b * L + (rev ? L - 1 - i : i);
                atomicAdd((gg < 4 ? a.dB : a.dC) + row * 16 + n, s);
            }
        }
        __syncwarp();   // every thread of the warp is done with this chunk's slots
    }
    cp_wait<0>();

    // dA, dD, dbias: per channel
    if (active) {
        float *dA = a.dA + (size_t)d * 16 + 4 * q;
        atomicAdd(dA, gA[0].x);
        atomicAdd(dA + 1, gA[0].y);
        atomicAdd(dA + 2, gA[1].x);
        atomicAdd(dA + 3, gA[1].y);
    }
    gD += __shfl_xor_sync(0xffffffffu, gD, 1);
    gD += __shfl_xor_sync(0xffffffffu, gD, 2);
    gbias += __shfl_xor_sync(0xffffffffu, gbias, 1);
    gbias += __shfl_xor_sync(0xffffffffu, gbias, 2);
    if (active && q == 0) {
        if (a.dD)
            atomicAdd(a.dD + d, gD);
        if (a.dbias)
            atomicAdd(a.dbias + d, gbias);
    }
}

template <typename T>
cudaError_t launch_typed(const BwdArgs &a, cudaStream_t st)
{
    const dim3 grid((unsigned)((a.D + kChW * kWarpsB - 1) / (kChW * kWarpsB)), (unsigned)a.Bsz);
    if (a.z)
        s6_bwd_split_kernel<T, true><<<grid, 32 * kWarpsB, 0, st>>>(a);
    else
        s6_bwd_split_kernel<T, false><<<grid, 32 * kWarpsB, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd_split(const BwdArgs &a, cudaStream_t st)
{
    return a.dtype == 0 ? launch_typed<float>(a, st) : launch_typed<__nv_bfloat16>(a, st);
}

}  // namespace ssm
