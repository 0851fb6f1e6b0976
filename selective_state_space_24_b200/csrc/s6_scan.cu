// s6_scan.cu -- Mamba S6 selective scan and the fused Vision-Mamba
// bidirectional scan for sm_100a.
//
// Operation (Mamba2 page "手写简化版Mamba2", sec. 2.2, 4.3, 4.4; Vim page
// sec. 3.1-3.2): for every (batch b, channel d) and state n
//     dt       = softplus(delta[b,t,d] + bias[d])
//     h[n]     = exp(dt A[d,n]) h[n] + dt B[b,t,n] x[b,t,d]
//     y[b,t,d] = (sum_n C[b,t,n] h[n] + D[d] x[b,t,d]) silu(z[b,t,d])
// and, bidirectionally, the same with the sequence reversed and a second
// parameter set, the two results summed.
//
// Work decomposition
//   * One thread owns one (b, d, direction) column and keeps its N states in
//     fp32 registers; the h sequence never leaves the SM (the pages' fusion
//     rule: never materialise (B, L, D, N)).
//   * Lanes of a warp own 32 consecutive channels, so every x / delta / z
//     access of a warp is one contiguous row segment, prefetched one step
//     ahead.  B[t] and C[t] are the same for every lane: each warp stages
//     them for 16 steps at a time in shared memory as fp32 (zero-padded to
//     the template state count) and reads them back as broadcast 16-byte
//     loads.
//   * Bidirectional: a CTA is a warp pair over the same 32 channels, the
//     forward warp walking its segment upward, the reversed warp downward.
//     Each parks the first half of its outputs in an fp32 stash (the output
//     itself for fp32, the workspace for bf16), the pair meets at one named
//     barrier, and in the second half each adds the other direction's parked
//     value and writes the final sum.  x and delta are read by both warps;
//     the second read is served by L1/L2.
//   * Long sequences are cut into S segments (the chunked scan with
//     state hand-off of the Mamba2 page sec. 3.2): a summary kernel computes
//     each segment's local end state and sum of dt, a carry kernel composes
//     them with (a, b) o (a', b') = (a a', a' b + b'), and the main kernel
//     rescans every segment from its true entering state.
//   * exp(dt A) is 2^(dt A log2 e).  The first NS - NPOLY states use the MUFU
//     ex2.approx instruction, the last NPOLY states a degree-5 polynomial on
//     the FMA pipe (Cody-Waite style split into integer and fraction,
//     minimax coefficients fitted by fit_exp2_poly.py), so that the MUFU and
//     FMA pipes share the work.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"

namespace ssm {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr int kTC = 16;        // steps per B/C staging chunk
constexpr int kWarps = 2;      // warps per CTA

__device__ __forceinline__ float ex2_mufu(float v)
{
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(v));
    return r;
}

__device__ __forceinline__ float lg2_mufu(float v)
{
    float r;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(v));
    return r;
}

__device__ __forceinline__ float rcp_mufu(float v)
{
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(v));
    return r;
}

// 2^v on the FMA pipe: v = j + f with j = rint(v), |f| <= 1/2; 2^f by a
// degree-5 minimax polynomial (relative error 2.1e-7 in fp32); 2^j added to
// the exponent field.  v is clamped to [-126, 127] so the exponent stays in
// range.
__device__ __forceinline__ float ex2_poly(float v)
{
    v = fminf(fmaxf(v, -126.f), 127.f);
    const float kMagic = 12582912.f;  // 1.5 * 2^23: v + kMagic rounds v to an integer
    const float t = v + kMagic;
    const float f = v - (t - kMagic);
    float p = 1.327647245e-03f;
    p = fmaf(p, f, 9.675540961e-03f);
    p = fmaf(p, f, 5.550713092e-02f);
    p = fmaf(p, f, 2.402212024e-01f);
    p = fmaf(p, f, 6.931469440e-01f);
    p = fmaf(p, f, 1.000000119e+00f);
    return __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
}

// softplus(v) = max(v, 0) + log1p(e), e = exp(-|v|) in (0, 1].  log1p(e) is
// a 6-term series for e < 1/16 (truncation < 1e-8 relative) and
// lg2(1 + e) ln 2 otherwise.
__device__ __forceinline__ float softplus_f(float v)
{
    const float e = ex2_mufu(-fabsf(v) * kLog2e);
    const float s = e * fmaf(e, fmaf(e, fmaf(e, fmaf(e, fmaf(e, -1.f / 6.f, 0.2f), -0.25f),
                                              1.f / 3.f), -0.5f), 1.f);
    const float g = lg2_mufu(1.f + e) * kLn2;
    return fmaxf(v, 0.f) + (e < 0.0625f ? s : g);
}

__device__ __forceinline__ float silu_f(float z) { return z * rcp_mufu(1.f + ex2_mufu(-z * kLog2e)); }

template <typename T> struct IO;
template <> struct IO<float> {
    static __device__ __forceinline__ float ld(const float *p, size_t i) { return __ldg(p + i); }
    static __device__ __forceinline__ void st(float *p, size_t i, float v) { p[i] = v; }
};
template <> struct IO<__nv_bfloat16> {
    static __device__ __forceinline__ float ld(const __nv_bfloat16 *p, size_t i)
    {
        return __bfloat162float(__ldg(p + i));
    }
    static __device__ __forceinline__ void st(__nv_bfloat16 *p, size_t i, float v)
    {
        p[i] = __float2bfloat16_rn(v);
    }
};

__device__ __forceinline__ bool first_in_order(int seg, int S, bool rev) { return rev ? seg == S - 1 : seg == 0; }
__device__ __forceinline__ bool last_in_order(int seg, int S, bool rev) { return rev ? seg == 0 : seg == S - 1; }

__device__ __forceinline__ void pair_barrier() { asm volatile("bar.sync 1, 64;" ::: "memory"); }

// Per-warp staging of B[t], C[t] for kTC steps.  Row i of a chunk holds
// B (NS floats) then C (NS floats) of time t(i); lane l fills half l & 1
// (B or C) of row l >> 1.  Rows past the segment and states past N are 0.
template <typename T, int NS>
struct BCStage {
    float v[NS];

    __device__ __forceinline__ void load(const T *Bm, const T *Cm, int N, size_t rowbase, int s0,
                                         int s1, bool rev, int i0, int lane)
    {
        const int i = i0 + (lane >> 1);
        const int Tn = s1 - s0;
        const T *src = (lane & 1) ? Cm : Bm;
#pragma unroll
        for (int n = 0; n < NS; n++)
            v[n] = 0.f;
        if (i < Tn) {
            const int t = rev ? s1 - 1 - i : s0 + i;
            const T *row = src + (rowbase + t) * N;
            if (N == NS && sizeof(T) == 4 && NS % 4 == 0) {
#pragma unroll
                for (int q = 0; q < NS / 4; q++) {
                    const float4 w = __ldg(reinterpret_cast<const float4 *>(row) + q);
                    v[4 * q] = w.x;
                    v[4 * q + 1] = w.y;
                    v[4 * q + 2] = w.z;
                    v[4 * q + 3] = w.w;
                }
            } else if (N == NS && sizeof(T) == 2 && NS % 8 == 0) {
#pragma unroll
                for (int q = 0; q < NS / 8; q++) {
                    const uint4 w = __ldg(reinterpret_cast<const uint4 *>(row) + q);
                    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                    for (int k = 0; k < 4; k++) {
                        v[8 * q + 2 * k] = __uint_as_float(u[k] << 16);
                        v[8 * q + 2 * k + 1] = __uint_as_float(u[k] & 0xffff0000u);
                    }
                }
            } else {
#pragma unroll
                for (int n = 0; n < NS; n++)
                    if (n < N)
                        v[n] = IO<T>::ld(row, n);
            }
        }
    }

    __device__ __forceinline__ void store(float *buf, int lane) const
    {
        float4 *dst = reinterpret_cast<float4 *>(buf + (lane >> 1) * 2 * NS + (lane & 1) * NS);
#pragma unroll
        for (int q = 0; q < NS / 4; q++)
            dst[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    }
};

__device__ __forceinline__ void cp_async4(void *smem, const void *gmem)
{
    const unsigned sa = (unsigned)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(sa), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int K> __device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(K) : "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

__device__ __forceinline__ float bf16_bits_to_f(unsigned short u) { return __uint_as_float((unsigned)u << 16); }

// Per-warp ring of kStages stages x kSub steps; each step slot holds four
// 128-byte rows: x, delta, z (the warp's 32 channels in the storage dtype)
// and the fp32 stash row.  Rows arrive by cp.async, kStages - 1 stages
// (12 steps) ahead of use.
constexpr int kSub = 4;
constexpr int kStages = 4;
constexpr int kRowB = 128;
constexpr int kSlotB = 4 * kRowB;
constexpr int kRingB = kStages * kSub * kSlotB;

// One warp's scan over one segment of one column per lane.
//   SUMMARY: local end state from the given h, plus the sum of dt; no output.
//   otherwise: outputs; BIDIR adds the midpoint exchange with the partner warp.
template <typename T, int NS, int NPOLY, bool SUMMARY, bool BIDIR>
__device__ __forceinline__ void scan_segment(const S6Args &a, const DirArgs &P, float *sbc,
                                             char *ring, int b, int dbase, bool active, int s0,
                                             int s1, bool rev, float (&h)[NS], float &sdt)
{
    const int lane = threadIdx.x & 31;
    const int d = dbase + lane;
    const int N = a.N;
    const int Tn = s1 - s0;
    const size_t rowbase = (size_t)b * a.L;
    const T *x = static_cast<const T *>(a.x);
    const T *dl = static_cast<const T *>(a.delta);
    const T *zp = static_cast<const T *>(P.z);
    T *out = static_cast<T *>(a.out);
    float *stash = a.stash;
    const bool gate = zp != nullptr;
    constexpr bool kF32 = sizeof(T) == 4;

    float Al2[NS];
#pragma unroll
    for (int n = 0; n < NS; n++)
        Al2[n] = (active && n < N) ? P.A[(size_t)d * N + n] * kLog2e : 0.f;
    const float bias = (active && P.bias) ? P.bias[d] : 0.f;
    const float Dd = (active && P.D) ? P.D[d] : 0.f;

    // midpoint of the pair exchange (see file comment)
    const int M = rev ? Tn / 2 : (Tn + 1) / 2;
    auto tpos = [&](int i) { return rev ? s1 - 1 - i : s0 + i; };
    const int w = lane & 15;                    // bf16 rows: 16 words of 2 channels
    const bool wok = 2 * w < a.D - dbase;

    // copy x / delta / z (and the stash when allowed) of step i into its slot
    auto issue_step = [&](int i, bool with_stash) {
        const int t = tpos(i);
        char *slot = ring + ((i / kSub) % kStages) * kSub * kSlotB + (i % kSub) * kSlotB;
        const size_t ro = (rowbase + t) * a.D + dbase;
        if (kF32) {
            if (active) {
                cp_async4(slot + lane * 4, x + ro + lane);
                cp_async4(slot + kRowB + lane * 4, dl + ro + lane);
                if (!SUMMARY && gate)
                    cp_async4(slot + 2 * kRowB + lane * 4, zp + ro + lane);
            }
        } else if (wok) {
            cp_async4(slot + (lane >> 4) * kRowB + w * 4, (lane < 16 ? x : dl) + ro + 2 * w);
            if (!SUMMARY && gate && lane < 16)
                cp_async4(slot + 2 * kRowB + w * 4, zp + ro + 2 * w);
        }
        if (BIDIR && with_stash && i >= M && active)
            cp_async4(slot + 3 * kRowB + lane * 4, stash + ro + lane);
    };
    auto issue_chunk = [&](int c, bool with_stash) {
#pragma unroll
        for (int j = 0; j < kSub; j++) {
            const int i = c * kSub + j;
            if (i < Tn)
                issue_step(i, with_stash);
        }
        cp_async_commit();
    };

    BCStage<T, NS> stg;
    stg.load(static_cast<const T *>(P.B), static_cast<const T *>(P.C), N, rowbase, s0, s1, rev, 0,
             lane);
    stg.store(sbc, lane);
    constexpr int kSubPerTC = kTC / kSub;
    const int nbc = (Tn + kTC - 1) / kTC;
    const int nchunks = (Tn + kSub - 1) / kSub;
    bool stash_ok = false;
#pragma unroll
    for (int c = 0; c < kStages - 1; c++)
        issue_chunk(c, false);
    __syncwarp();

    for (int c = 0; c < nchunks; c++) {
        issue_chunk(c + kStages - 1, stash_ok);
        cp_async_wait<kStages - 1>();
        __syncwarp();
        const int kb = c / kSubPerTC;
        if (c % kSubPerTC == 0 && kb + 1 < nbc)
            stg.load(static_cast<const T *>(P.B), static_cast<const T *>(P.C), N, rowbase, s0, s1,
                     rev, (kb + 1) * kTC, lane);
        const float *cur = sbc + (kb & 1) * kTC * 2 * NS + (c % kSubPerTC) * kSub * 2 * NS;
        const char *stage = ring + (c % kStages) * kSub * kSlotB;
#pragma unroll
        for (int j = 0; j < kSub; j++) {
            const int i = c * kSub + j;
            if (i >= Tn)
                break;
            if (BIDIR && i == M) {
                pair_barrier();
                stash_ok = true;
                // steps already in flight were issued without their stash rows
                const int fr = min(Tn, (c + kStages) * kSub);
                for (int ii = M; ii < fr; ii++) {
                    char *slot = ring + ((ii / kSub) % kStages) * kSub * kSlotB + (ii % kSub) * kSlotB;
                    if (active)
                        cp_async4(slot + 3 * kRowB + lane * 4,
                                  stash + (rowbase + tpos(ii)) * a.D + d);
                }
                cp_async_wait_all();
                __syncwarp();
            }
            const char *slot = stage + j * kSlotB;
            float xv, dv, zv = 0.f;
            if (kF32) {
                xv = *reinterpret_cast<const float *>(slot + lane * 4);
                dv = *reinterpret_cast<const float *>(slot + kRowB + lane * 4);
                if (!SUMMARY && gate)
                    zv = *reinterpret_cast<const float *>(slot + 2 * kRowB + lane * 4);
            } else {
                xv = bf16_bits_to_f(*reinterpret_cast<const unsigned short *>(slot + lane * 2));
                dv = bf16_bits_to_f(*reinterpret_cast<const unsigned short *>(slot + kRowB + lane * 2));
                if (!SUMMARY && gate)
                    zv = bf16_bits_to_f(
                        *reinterpret_cast<const unsigned short *>(slot + 2 * kRowB + lane * 2));
            }
            float dt = dv + bias;
            if (a.softplus)
                dt = softplus_f(dt);
            const float dtx = dt * xv;
            const float4 *row = reinterpret_cast<const float4 *>(cur + j * 2 * NS);
            if (SUMMARY) {
                sdt += dt;
#pragma unroll
                for (int q = 0; q < NS / 4; q++) {
                    const float4 bq = row[q];
                    const float bb[4] = {bq.x, bq.y, bq.z, bq.w};
#pragma unroll
                    for (int r = 0; r < 4; r++) {
                        const int n = 4 * q + r;
                        const float e = n < NS - NPOLY ? ex2_mufu(dt * Al2[n]) : ex2_poly(dt * Al2[n]);
                        h[n] = fmaf(e, h[n], dtx * bb[r]);
                    }
                }
            } else {
                float y0 = 0.f, y1 = 0.f;
#pragma unroll
                for (int q = 0; q < NS / 4; q++) {
                    const float4 bq = row[q];
                    const float4 cq = row[NS / 4 + q];
                    const float bb[4] = {bq.x, bq.y, bq.z, bq.w};
                    const float cc[4] = {cq.x, cq.y, cq.z, cq.w};
#pragma unroll
                    for (int r = 0; r < 4; r++) {
                        const int n = 4 * q + r;
                        const float e = n < NS - NPOLY ? ex2_mufu(dt * Al2[n]) : ex2_poly(dt * Al2[n]);
                        h[n] = fmaf(e, h[n], dtx * bb[r]);
                        if (r & 1)
                            y1 = fmaf(cc[r], h[n], y1);
                        else
                            y0 = fmaf(cc[r], h[n], y0);
                    }
                }
                float y = fmaf(Dd, xv, y0 + y1);
                if (gate)
                    y *= silu_f(zv);
                if (active) {
                    const size_t io = (rowbase + tpos(i)) * a.D + d;
                    if (!BIDIR)
                        IO<T>::st(out, io, y);
                    else if (i < M)
                        stash[io] = y;
                    else
                        IO<T>::st(out, io, y + *reinterpret_cast<const float *>(slot + 3 * kRowB + lane * 4));
                }
            }
        }
        __syncwarp();
        if (c % kSubPerTC == kSubPerTC - 1 && kb + 1 < nbc) {
            stg.store(sbc + ((kb + 1) & 1) * kTC * 2 * NS, lane);
            __syncwarp();
        }
    }
    cp_async_wait_all();
    if (BIDIR && M == Tn)
        pair_barrier();
}

// ---------------------------------------------------------------- summary
template <typename T, int NS, int NPOLY>
__global__ void __launch_bounds__(64, 8) s6_summary_kernel(const S6Args a)
{
    __shared__ __align__(16) float sbc[kWarps][2 * kTC * 2 * NS];
    __shared__ __align__(16) char ring[kWarps][kRingB];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int dbase = (blockIdx.x * kWarps + warp) * 32;
    const int d = dbase + lane;
    const int seg = blockIdx.y;
    const int dsel = blockIdx.z % a.ndir;
    const int b = blockIdx.z / a.ndir;
    const bool rev = a.ndir == 2 ? dsel == 1 : a.reverse != 0;
    if (last_in_order(seg, a.S, rev) || (blockIdx.x * kWarps + warp) * 32 >= a.D)
        return;
    const bool active = d < a.D;
    const int s0 = seg * a.T, s1 = min(a.L, s0 + a.T);
    float h[NS];
#pragma unroll
    for (int n = 0; n < NS; n++)
        h[n] = 0.f;
    float sdt = 0.f;
    scan_segment<T, NS, NPOLY, true, false>(a, a.dir[dsel], sbc[warp], ring[warp], b, dbase,
                                            active, s0, s1, rev, h, sdt);
    if (!active)
        return;
    const size_t ci = (((size_t)dsel * a.Bsz + b) * a.S + seg) * a.D + d;
#pragma unroll
    for (int n = 0; n < NS; n++)
        if (n < a.N)
            a.carry_h[ci * a.N + n] = h[n];
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
        hin = fmaf(ex2_mufu(Al2 * s), hin, hl);
    }
}

// ------------------------------------------------------------------- main
template <typename T, int NS, int NPOLY, bool BIDIR>
__global__ void __launch_bounds__(64, 8) s6_main_kernel(const S6Args a)
{
    __shared__ __align__(16) float sbc[kWarps][2 * kTC * 2 * NS];
    __shared__ __align__(16) char ring[kWarps][kRingB];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int dsel = BIDIR ? warp : 0;
    const int dbase = BIDIR ? blockIdx.x * 32 : (blockIdx.x * kWarps + warp) * 32;
    const int d = dbase + lane;
    const bool active = d < a.D;
    const int seg = blockIdx.y, b = blockIdx.z;
    const int s0 = seg * a.T, s1 = min(a.L, s0 + a.T);
    const bool rev = BIDIR ? dsel == 1 : a.reverse != 0;
    const DirArgs &P = a.dir[dsel];
    if (!BIDIR && (blockIdx.x * kWarps + warp) * 32 >= a.D)
        return;   // whole warp past the channels (never with a barrier partner)
    float h[NS];
    const bool has_carry = a.S > 1 && !first_in_order(seg, a.S, rev);
    const size_t ci = (((size_t)dsel * a.Bsz + b) * a.S + seg) * a.D + d;
#pragma unroll
    for (int n = 0; n < NS; n++)
        h[n] = (active && n < a.N && has_carry) ? a.carry_h[ci * a.N + n] : 0.f;
    float sdt = 0.f;
    scan_segment<T, NS, NPOLY, false, BIDIR>(a, P, sbc[warp], ring[warp], b, dbase, active, s0, s1,
                                             rev, h, sdt);
    if (active && P.last_state && last_in_order(seg, a.S, rev)) {
#pragma unroll
        for (int n = 0; n < NS; n++)
            if (n < a.N)
                P.last_state[((size_t)b * a.D + d) * a.N + n] = h[n];
    }
}

template <typename T, int NS, int NPOLY>
cudaError_t launch_typed(const S6Args &a, cudaStream_t st)
{
    if (a.S > 1) {
        dim3 g1((a.D + 63) / 64, a.S, a.Bsz * a.ndir);
        s6_summary_kernel<T, NS, NPOLY><<<g1, 64, 0, st>>>(a);
        const size_t tot = (size_t)a.ndir * a.Bsz * a.D * a.N;
        s6_carry_kernel<<<(unsigned)((tot + 255) / 256), 256, 0, st>>>(a);
    }
    if (a.ndir == 2) {
        dim3 g((a.D + 31) / 32, a.S, a.Bsz);
        s6_main_kernel<T, NS, NPOLY, true><<<g, 64, 0, st>>>(a);
    } else {
        dim3 g((a.D + 63) / 64, a.S, a.Bsz);
        s6_main_kernel<T, NS, NPOLY, false><<<g, 64, 0, st>>>(a);
    }
    return cudaGetLastError();
}

#ifndef SSM_S6_NPOLY
#define SSM_S6_NPOLY 0
#endif

template <typename T>
cudaError_t launch_ns(const S6Args &a, cudaStream_t st)
{
    if (a.N <= 4)
        return launch_typed<T, 4, 0>(a, st);
    if (a.N <= 8)
        return launch_typed<T, 8, 0>(a, st);
    return launch_typed<T, 16, SSM_S6_NPOLY>(a, st);
}

}  // namespace

S6Plan plan_s6(int64_t Bsz, int64_t L, int64_t D, int64_t N, int ndir, int dtype)
{
    S6Plan p{1, (int)L, 0, 0};
    if (L <= 0)
        return p;
    const int64_t kMinT = 16;
    const int64_t kTargetThreads = 148 * 512;
    const int64_t cols = (int64_t)ndir * Bsz * D;
    int64_t S = 1;
    if (cols > 0 && cols < kTargetThreads)
        S = (kTargetThreads + cols - 1) / cols;
    const int64_t smax = (L + kMinT - 1) / kMinT;
    if (S > smax)
        S = smax;
    if (S < 1)
        S = 1;
    int64_t T = (L + S - 1) / S;
    S = (L + T - 1) / T;
    p.S = (int)S;
    p.T = (int)T;
    size_t off = 0;
    if (S > 1) {
        p.carry_h_off = 0;
        off = (size_t)ndir * Bsz * S * D * N * sizeof(float);
        off = (off + 255) / 256 * 256;
        p.carry_s_off = off;
        off += (size_t)ndir * Bsz * S * D * sizeof(float);
        off = (off + 255) / 256 * 256;
    }
    if (ndir == 2 && dtype != 0) {
        p.stash_off = off;
        off += (size_t)Bsz * L * D * sizeof(float);
    }
    p.workspace_bytes = off;
    return p;
}

cudaError_t launch_s6(const S6Args &a, cudaStream_t st)
{
    if (a.dtype == 0)
        return launch_ns<float>(a, st);
    return launch_ns<__nv_bfloat16>(a, st);
}

}  // namespace ssm
