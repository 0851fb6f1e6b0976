// s6_scan_impl.cuh -- Mamba S6 selective scan and the fused Vision-Mamba
// bidirectional scan for sm_100a: the kernels.  Each s6_part_*.cu file
// instantiates one element type and kernel variant (so the parts compile in
// parallel); s6_scan.cu holds the plan and the dispatch.
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
//   * One thread owns one or two adjacent channels (CPL) of one (b,
//     direction) and keeps their CPL x N states in fp32 registers; the h
//     sequence never leaves the SM (the pages' fusion rule: never
//     materialise (B, L, D, N)).  The state update runs on packed f32x2
//     FMA/MUL instructions (two states per instruction).  Two channels per
//     lane give each thread more independent work; one channel per lane
//     gives twice the threads when the problem is small.
//   * A warp owns 32 CPL consecutive channels, so every x / delta / z access
//     of a warp is one contiguous row segment.  Those rows arrive by 16-byte
//     cp.async copies in a per-warp shared-memory ring 4 to 8 steps ahead of
//     use.  B[t] and C[t]
//     are the same for every lane: each warp stages them 16 steps at a time
//     in shared memory as fp32 (zero-padded to the template state count) and
//     reads them back as broadcast 16-byte loads.
//   * Bidirectional: a CTA is a warp pair over the same channels, the
//     forward warp walking its segment upward, the reversed warp downward.
//     Each parks the first half of its outputs in an fp32 stash (the output
//     itself for fp32, the workspace for bf16), the pair meets at one named
//     barrier, and in the second half each adds the other direction's parked
//     value and writes the final sum, so out is written once.
//   * Long sequences are cut into S segments (the chunked scan with
//     state hand-off of the Mamba2 page sec. 3.2): a summary kernel computes
//     each segment's local end state and sum of dt, a carry kernel composes
//     them with (a, b) o (a', b') = (a a', a' b + b'), and the main kernel
//     rescans every segment from its true entering state.
//   * exp(dt A) is 2^(dt A log2 e).  The first NS - NPOLY states use the MUFU
//     ex2.approx instruction, the last NPOLY states a degree-5 polynomial on
//     the FMA pipe (integer / fraction split of the exponent, minimax
//     coefficients fitted by fit_polys.py), so that the MUFU and FMA
//     pipes share the work.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#pragma once
#include <stdint.h>

#include "internal.h"
#include "s6_math.cuh"

namespace ssm {
namespace {

// Set when a scan order holds an index outside [0, L) (the entry is then
// treated as its own scan index, so nothing is accessed out of bounds).
// One per translation unit; s6_part_error() reads and clears this one.
__device__ unsigned g_s6_error;

constexpr int kWarps = 2;   // warps per CTA
constexpr int kTC = 16;     // steps per B/C staging chunk
// cp.async ring: steps per group and groups in flight, by channels per lane
// (two channels per lane hold more registers, so shorter groups).
#ifndef SSM_S6_KSUB2
#define SSM_S6_KSUB2 2
#endif
#ifndef SSM_S6_KSTAGES2
#define SSM_S6_KSTAGES2 4
#endif
#ifndef SSM_S6_KSUB1
#define SSM_S6_KSUB1 4
#endif
#ifndef SSM_S6_KSTAGES1
#define SSM_S6_KSTAGES1 2
#endif
template <int CPL> struct Ring {
    static constexpr int kSub = CPL == 2 ? SSM_S6_KSUB2 : SSM_S6_KSUB1;        // steps per group
    static constexpr int kStages = CPL == 2 ? SSM_S6_KSTAGES2 : SSM_S6_KSTAGES1;  // groups in the ring
    static constexpr int kSlots = kSub * kStages;
    static_assert(kTC % kSub == 0, "B/C staging rotates on group boundaries");
};
#ifndef SSM_S6_MINB
#define SSM_S6_MINB 6
#endif
#ifndef SSM_S6_MINB1
#define SSM_S6_MINB1 8
#endif
// Tuning knobs (compile-time): channels per lane (0 = by problem size), the
// thread count below which one channel per lane is used, the waves of
// resident CTAs the segments fill (0: use the target thread counts instead),
// and how many state pairs the summary pass evaluates on the FMA pipe.
#ifndef SSM_S6_CPL
#define SSM_S6_CPL 0
#endif
#ifndef SSM_S6_CPL1_BELOW
#define SSM_S6_CPL1_BELOW (148 * 128)
#endif
#ifndef SSM_S6_WAVES
#define SSM_S6_WAVES 1
#endif
#ifndef SSM_S6_TARGET1
#define SSM_S6_TARGET1 (148 * 640)
#endif
#ifndef SSM_S6_TARGET2
#define SSM_S6_TARGET2 (148 * 320)
#endif
#ifndef SSM_S6_SUM_NPOLY_N
#define SSM_S6_SUM_NPOLY_N 0
#endif
#define SSM_S6_SUM_NPOLY(NS) ((NS) == 16 ? SSM_S6_SUM_NPOLY_N : 0)

// CTAs per SM the register budget is sized for, by channels per lane
template <int CPL> constexpr int min_blocks() { return CPL == 2 ? SSM_S6_MINB : SSM_S6_MINB1; }

// ------------------------------------------------------------ math helpers

// Pairwise multiply / fused multiply-add on two states at once: the packed
// f32x2 instructions of sm_100, or two scalar instructions (SSM_S6_SCALAR).
#ifndef SSM_S6_SCALAR
#define SSM_S6_SCALAR 0
#endif
__device__ __forceinline__ float2 mul2(float2 a, float2 b)
{
    if (SSM_S6_SCALAR)
        return make_float2(a.x * b.x, a.y * b.y);
    return __fmul2_rn(a, b);
}
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c)
{
    if (SSM_S6_SCALAR)
        return make_float2(fmaf(a.x, b.x, c.x), fmaf(a.y, b.y, c.y));
    return __ffma2_rn(a, b, c);
}
__device__ __forceinline__ float2 add2(float2 a, float2 b)
{
    if (SSM_S6_SCALAR)
        return make_float2(a.x + b.x, a.y + b.y);
    return __fadd2_rn(a, b);
}

// 2^v for two values on the FMA pipe: v = j + f with j = rint(v), |f| <= 1/2;
// 2^f by a degree-5 minimax polynomial (relative error 2.1e-7 in fp32); 2^j
// added to the exponent field.  v is clamped to [-126, 127] so the exponent
// stays in range.
__device__ __forceinline__ float2 ex2_poly2(float2 v)
{
    const float kMagic = 12582912.f;  // 1.5 * 2^23: v + kMagic rounds v to an integer
    v.x = fminf(fmaxf(v.x, -126.f), 127.f);
    v.y = fminf(fmaxf(v.y, -126.f), 127.f);
    const float2 t = __fadd2_rn(v, make_float2(kMagic, kMagic));
    const float2 j = __fadd2_rn(t, make_float2(-kMagic, -kMagic));
    const float2 f = __fadd2_rn(v, make_float2(-j.x, -j.y));
    float2 p = make_float2(1.327647245e-03f, 1.327647245e-03f);
    p = __ffma2_rn(p, f, make_float2(9.675540961e-03f, 9.675540961e-03f));
    p = __ffma2_rn(p, f, make_float2(5.550713092e-02f, 5.550713092e-02f));
    p = __ffma2_rn(p, f, make_float2(2.402212024e-01f, 2.402212024e-01f));
    p = __ffma2_rn(p, f, make_float2(6.931469440e-01f, 6.931469440e-01f));
    p = __ffma2_rn(p, f, make_float2(1.000000119e+00f, 1.000000119e+00f));
    return make_float2(__int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23)),
                       __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23)));
}

// ----------------------------------------------------- storage-type helpers

// CPL adjacent channels of one lane: loads from the staging ring (shared
// memory) and stores to the output.
template <typename T, int CPL> struct IO;
template <> struct IO<float, 2> {
    static __device__ __forceinline__ void ld(const void *p, float (&v)[2])
    {
        const float2 u = *reinterpret_cast<const float2 *>(p);
        v[0] = u.x;
        v[1] = u.y;
    }
    static __device__ __forceinline__ void st(float *p, const float (&v)[2])
    {
        *reinterpret_cast<float2 *>(p) = make_float2(v[0], v[1]);
    }
};
template <> struct IO<float, 1> {
    static __device__ __forceinline__ void ld(const void *p, float (&v)[1])
    {
        v[0] = *reinterpret_cast<const float *>(p);
    }
    static __device__ __forceinline__ void st(float *p, const float (&v)[1]) { *p = v[0]; }
};
template <> struct IO<__nv_bfloat16, 2> {
    static __device__ __forceinline__ void ld(const void *p, float (&v)[2])
    {
        const uint32_t u = *reinterpret_cast<const uint32_t *>(p);
        v[0] = __uint_as_float(u << 16);
        v[1] = __uint_as_float(u & 0xffff0000u);
    }
    static __device__ __forceinline__ void st(__nv_bfloat16 *p, const float (&v)[2])
    {
        *reinterpret_cast<__nv_bfloat162 *>(p) = __floats2bfloat162_rn(v[0], v[1]);
    }
};
template <> struct IO<__nv_bfloat16, 1> {
    static __device__ __forceinline__ void ld(const void *p, float (&v)[1])
    {
        v[0] = __uint_as_float((uint32_t)*reinterpret_cast<const unsigned short *>(p) << 16);
    }
    static __device__ __forceinline__ void st(__nv_bfloat16 *p, const float (&v)[1])
    {
        *p = __float2bfloat16_rn(v[0]);
    }
};

template <typename T>
__device__ __forceinline__ float ld1(const T *p, size_t i);
template <> __device__ __forceinline__ float ld1<float>(const float *p, size_t i) { return __ldg(p + i); }
template <> __device__ __forceinline__ float ld1<__nv_bfloat16>(const __nv_bfloat16 *p, size_t i)
{
    return __bfloat162float(__ldg(p + i));
}

__device__ __forceinline__ bool first_in_order(int seg, int S, bool rev) { return rev ? seg == S - 1 : seg == 0; }

// Position visited at scan index t: order[t], or t itself without an order.
__device__ __forceinline__ int position(int t, const int *order, int L)
{
    if (!order)
        return t;
    const int p = __ldg(order + t);
    if ((unsigned)p < (unsigned)L)
        return p;
    atomicOr(&g_s6_error, 1u);
    return t;
}
__device__ __forceinline__ bool last_in_order(int seg, int S, bool rev) { return rev ? seg == 0 : seg == S - 1; }

__device__ __forceinline__ void pair_barrier() { asm volatile("bar.sync 1, 64;" ::: "memory"); }

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem)
{
    const unsigned sa = (unsigned)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.ca.shared.global [%0], [%1], 16;" ::"r"(sa), "l"(gmem) : "memory");
}
// L2 eviction priorities for the bidirectional pass.  x and delta are read
// by both warps of a pair, the first reader in the first half of its scan
// and the second in the second half: the first read marks the line
// evict-last (the 77 MB of x and delta of Vim-Small then stay in the 126 MB
// L2 until the partner reads them), the second read and the read-once
// streams (z, the final output) evict-first.  The parked half-outputs are
// written evict-last and read back evict-first.
#ifndef SSM_S6_L2HINT
#define SSM_S6_L2HINT 1
#endif
__device__ __forceinline__ uint64_t l2_evict_last()
{
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t l2_evict_first()
{
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ void cp_async16(void *smem, const void *gmem, uint64_t pol)
{
    const unsigned sa = (unsigned)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.ca.shared.global.L2::cache_hint [%0], [%1], 16, %2;" ::"r"(sa), "l"(gmem), "l"(pol)
                 : "memory");
}
__device__ __forceinline__ void st_hint(float *p, const float (&v)[2], uint64_t pol)
{
    asm volatile("st.global.L2::cache_hint.v2.f32 [%0], {%1, %2}, %3;" ::"l"(p), "f"(v[0]), "f"(v[1]), "l"(pol)
                 : "memory");
}
__device__ __forceinline__ void st_hint(float *p, const float (&v)[1], uint64_t pol)
{
    asm volatile("st.global.L2::cache_hint.f32 [%0], %1, %2;" ::"l"(p), "f"(v[0]), "l"(pol) : "memory");
}
__device__ __forceinline__ void st_hint(__nv_bfloat16 *p, const float (&v)[2], uint64_t pol)
{
    const __nv_bfloat162 h = __floats2bfloat162_rn(v[0], v[1]);
    const uint32_t u = *reinterpret_cast<const uint32_t *>(&h);
    asm volatile("st.global.L2::cache_hint.b32 [%0], %1, %2;" ::"l"(p), "r"(u), "l"(pol) : "memory");
}
__device__ __forceinline__ void st_hint(__nv_bfloat16 *p, const float (&v)[1], uint64_t pol)
{
    const __nv_bfloat16 h = __float2bfloat16_rn(v[0]);
    const unsigned short u = *reinterpret_cast<const unsigned short *>(&h);
    asm volatile("st.global.L2::cache_hint.b16 [%0], %1, %2;" ::"l"(p), "h"(u), "l"(pol) : "memory");
}
// 16-byte store of two state pairs with an L2 eviction policy
__device__ __forceinline__ void st4_hint(float *p, float2 a, float2 b, uint64_t pol)
{
    asm volatile("st.global.L2::cache_hint.v4.f32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(p), "f"(a.x), "f"(a.y),
                 "f"(b.x), "f"(b.y), "l"(pol)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int K> __device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(K) : "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Per-warp staging of B[t], C[t] for kTC steps.  Row i of a chunk holds
// B (NS floats) then C (NS floats) of time t(i); lane l fills half l & 1
// (B or C) of row l >> 1.  Rows past the segment and states past N are 0.
template <typename T, int NS>
struct BCStage {
    float v[NS];

    __device__ __forceinline__ void load(const T *Bm, const T *Cm, int N, size_t rowbase, int s0,
                                         int s1, bool rev, int i0, int lane, const int *order, int L)
    {
        const int i = i0 + (lane >> 1);
        const int Tn = s1 - s0;
        const T *src = (lane & 1) ? Cm : Bm;
#pragma unroll
        for (int n = 0; n < NS; n++)
            v[n] = 0.f;
        if (i < Tn) {
            const int t = position(rev ? s1 - 1 - i : s0 + i, order, L);
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
                        v[n] = ld1<T>(row, n);
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

template <bool V> struct PhaseTag {
    static constexpr bool value = V;
};

// Shared memory of one warp: the x / delta / z / stash ring and the B/C rows.
// A warp owns 32 * CPL consecutive channels; one ring slot holds one step.
template <typename T, int NS, int CPL>
struct WarpSmem {
    static constexpr int kCh = 32 * CPL;                  // channels per warp
    static constexpr int kRowB = kCh * (int)sizeof(T);   // one x, delta or z row
    static constexpr int kStashB = kCh * 4;              // one fp32 stash row
    static constexpr int kSlotB = 3 * kRowB + kStashB;
    char ring[Ring<CPL>::kSlots * kSlotB];
    float bc[2 * kTC * 2 * NS];
};

// Copies of whole rows into the ring, 16 bytes per lane: ROWB / 16 lanes
// cover one step's row, so one pass of the warp moves 512 / ROWB steps.
// Every 16-byte piece lies entirely inside or entirely past the channel
// range (D is a multiple of 16 / sizeof(element), the warp's first channel
// a multiple of 32).
template <int ROWB>
struct RowCopy {
    static constexpr int kLanesPerRow = ROWB / 16;
    static constexpr int kRowsPerPass = 32 / kLanesPerRow;
    static_assert(ROWB % 16 == 0 && kLanesPerRow <= 32, "row must be whole 16-byte pieces");
};

// One warp's scan over one segment, CPL adjacent channels per lane.
//   SUMMARY: local end state from the given h, plus the sum of dt; no output.
//   otherwise: outputs; BIDIR adds the midpoint exchange with the partner warp.
template <typename T, int NS, int CPL, int NPOLY, bool SUMMARY, bool BIDIR, bool GATE, bool SOFTPLUS,
          bool ORD, bool CONV, bool CKPT = false>
__device__ __forceinline__ void scan_segment(const S6Args &a, const DirArgs &P,
                                             WarpSmem<T, NS, CPL> &sm, int b, int dbase, bool active,
                                             int s0, int s1, bool rev, float2 (&h)[CPL][NS / 2],
                                             float (&sdt)[CPL], char *ck_tile = nullptr)
{
    using WS = WarpSmem<T, NS, CPL>;
    using RC = RowCopy<WS::kRowB>;
    using RS = RowCopy<WS::kStashB>;
    constexpr int kSub = Ring<CPL>::kSub, kStages = Ring<CPL>::kStages, kSlots = Ring<CPL>::kSlots;
    static_assert(NPOLY % 2 == 0 && NPOLY <= NS, "NPOLY counts state pairs");
    const int lane = threadIdx.x & 31;
    const int d = dbase + CPL * lane;
    const int N = a.N;
    const int Tn = s1 - s0;
    const size_t rowbase = (size_t)b * a.L;
    const T *x = static_cast<const T *>(a.x);
    const T *dl = static_cast<const T *>(a.delta);
    const T *zp = static_cast<const T *>(P.z);
    T *out = static_cast<T *>(a.out);
    float *stash = a.stash;

    // A log2(e) per channel, as pairs of states
    float2 Ap[CPL][NS / 2];
    float bias[CPL], Dd[CPL];
#pragma unroll
    for (int c = 0; c < CPL; c++) {
        const float *Ar = P.A + (size_t)(d + c) * N;
#pragma unroll
        for (int k = 0; k < NS / 2; k++) {
            const int n = 2 * k;
            Ap[c][k] = make_float2((active && n < N) ? Ar[n] * kLog2e : 0.f,
                                   (active && n + 1 < N) ? Ar[n + 1] * kLog2e : 0.f);
        }
        bias[c] = (active && P.bias) ? P.bias[d + c] : 0.f;
        Dd[c] = (active && P.D) ? P.D[d + c] : 0.f;
    }

    // CONV: x holds the conv input x_in; u = act(bias + sum_k w[k] x_in) over
    // this and the previous 3 steps in scan order (weights right-aligned in
    // cw, zero beyond the conv width).  xh[c][j] is x_in at scan offset
    // -(3 - j); the window is preloaded from the steps before the segment.
    float cw[CPL][4], cb[CPL], xh[CPL][3];
    if (CONV) {
        const int K = P.conv_k;
#pragma unroll
        for (int c = 0; c < CPL; c++) {
#pragma unroll
            for (int j = 0; j < 4; j++) {
                const int k = K - 4 + j;   // weight index for scan offset -(3 - j)
                cw[c][j] = (active && k >= 0) ? P.conv_w[(size_t)(d + c) * K + k] : 0.f;
            }
            cb[c] = (active && P.conv_b) ? P.conv_b[d + c] : 0.f;
#pragma unroll
            for (int j = 0; j < 3; j++) {
                const int off = 3 - j;   // steps before the segment's first
                const int t = rev ? s1 - 1 + off : s0 - off;
                xh[c][j] = (active && t >= 0 && t < a.L) ? ld1<T>(x, (rowbase + t) * a.D + d + c) : 0.f;
            }
        }
    }

    // midpoint of the pair exchange (see file comment)
    const int M = BIDIR ? (rev ? Tn / 2 : (Tn + 1) / 2) : Tn;
    // position of step i (the scan index, mapped through the order if any)
    // (ORD: the kernel was launched with an order and / or a token mask)
    const int *order = ORD ? a.order : nullptr;
    const unsigned char *tmask = ORD ? a.mask : nullptr;
    auto tpos = [&](int i) { return position(rev ? s1 - 1 - i : s0 + i, order, a.L); };
    auto slot_of = [&](int i) { return sm.ring + (i % kSlots) * WS::kSlotB; };

    // this lane's 16-byte piece of a row and of a stash row
    const int pc = lane % RC::kLanesPerRow, pr = lane / RC::kLanesPerRow;
    const int spc = lane % RS::kLanesPerRow, spr = lane / RS::kLanesPerRow;
    const bool pc_on = dbase + pc * (16 / (int)sizeof(T)) < a.D;
    const bool spc_on = dbase + spc * 4 < a.D;
    // stash rows of steps [i0, i1)
    constexpr bool kHint = SSM_S6_L2HINT && BIDIR && !SUMMARY;
    const uint64_t pol_last = kHint ? l2_evict_last() : 0, pol_first = kHint ? l2_evict_first() : 0;
    auto issue_stash = [&](int i0, int i1) {
        for (int i = i0 + spr; i < i1; i += RS::kRowsPerPass)
            if (spc_on) {
                char *dst = slot_of(i) + 3 * WS::kRowB + spc * 16;
                const float *src = stash + (rowbase + tpos(i)) * a.D + dbase + spc * 4;
                if (kHint)
                    cp_async16(dst, src, pol_first);
                else
                    cp_async16(dst, src);
            }
    };
    // x / delta / z (and stash when allowed) rows of group c
    auto issue_chunk = [&](int c, bool with_stash) {
        const int i0 = c * kSub, i1 = min(Tn, i0 + kSub);
#pragma unroll
        for (int p = 0; p < (kSub + RC::kRowsPerPass - 1) / RC::kRowsPerPass; p++) {
            const int i = i0 + p * RC::kRowsPerPass + pr;
            if (i < i1 && pc_on) {
                char *slot = slot_of(i) + pc * 16;
                const size_t ro = (rowbase + tpos(i)) * a.D + dbase + pc * (16 / (int)sizeof(T));
                if (kHint) {
                    const uint64_t pxd = i < M ? pol_last : pol_first;
                    cp_async16(slot, x + ro, pxd);
                    cp_async16(slot + WS::kRowB, dl + ro, pxd);
                    if (GATE)
                        cp_async16(slot + 2 * WS::kRowB, zp + ro, pol_first);
                } else {
                    cp_async16(slot, x + ro);
                    cp_async16(slot + WS::kRowB, dl + ro);
                    if (!SUMMARY && GATE)
                        cp_async16(slot + 2 * WS::kRowB, zp + ro);
                }
            }
        }
        if (BIDIR && with_stash)
            issue_stash(i0, i1);
        cp_async_commit();
    };

    BCStage<T, NS> stg;
    const T *Bm = static_cast<const T *>(P.B);
    const T *Cm = static_cast<const T *>(P.C);
    stg.load(Bm, Cm, N, rowbase, s0, s1, rev, 0, lane, order, a.L);
    stg.store(sm.bc, lane);
    stg.load(Bm, Cm, N, rowbase, s0, s1, rev, kTC, lane, order, a.L);
#pragma unroll
    for (int c = 0; c < kStages - 1; c++)
        issue_chunk(c, false);
    __syncwarp();

    bool with_stash = false;
    // chunk management at a group-aligned step: refill the stage consumed
    // last, wait for the one holding step i, rotate the B/C staging
    auto chunk_mgmt = [&](int i) {
        __syncwarp();
        issue_chunk(i / kSub + kStages - 1, with_stash);
        cp_async_wait<kStages - 1>();
        if ((i & (kTC - 1)) == 0 && i > 0) {
            stg.store(sm.bc + ((i / kTC) & 1) * kTC * 2 * NS, lane);
            stg.load(Bm, Cm, N, rowbase, s0, s1, rev, i + kTC, lane, order, a.L);
        }
        __syncwarp();
    };
    // Step stages.  load_dt: operands from the ring and dt (independent of h);
    // recur: the state update and readout (the only part that depends on the
    // previous step); finish: skip term, gate, store.
    struct StepIn {
        float xv[CPL], zv[CPL], dt[CPL];
        bool keep;   // false: the token is masked (bypassed)
    };
    auto load_dt = [&](int i) {
        const char *slot = slot_of(i) + lane * CPL * (int)sizeof(T);
        StepIn o;
        o.keep = !ORD || !tmask || tmask[rowbase + tpos(i)] != 0;
        float dv[CPL];
        IO<T, CPL>::ld(slot, o.xv);
        if (CONV) {
#pragma unroll
            for (int c = 0; c < CPL; c++) {
                float u = fmaf(cw[c][3], o.xv[c], cb[c]);
#pragma unroll
                for (int j = 0; j < 3; j++)
                    u = fmaf(cw[c][j], xh[c][j], u);
                xh[c][0] = xh[c][1];
                xh[c][1] = xh[c][2];
                xh[c][2] = o.xv[c];
                o.xv[c] = P.conv_silu ? silu_f<T>(u) : u;
            }
        }
        IO<T, CPL>::ld(slot + WS::kRowB, dv);
        if (!SUMMARY && GATE)
            IO<T, CPL>::ld(slot + 2 * WS::kRowB, o.zv);
#pragma unroll
        for (int c = 0; c < CPL; c++) {
            o.dt[c] = dv[c] + bias[c];
            if (SOFTPLUS)
                o.dt[c] = softplus_f(o.dt[c]);
            if (ORD && !o.keep)
                o.dt[c] = 0.f;   // exp(0 A) = 1 and dt B x = 0: the state passes through
            o.zv[c] = (!SUMMARY && GATE) ? silu_f<T>(o.zv[c]) : 0.f;   // zv now holds the gate
        }
        return o;
    };
    struct StepOut {
        float y[CPL];
    };
    // CKPT: the state entering every 4-step chunk of the direction's scan
    // order (global scan index g of local step i), stored before step i.  The
    // warp's channels are consecutive, so its checkpoint is one contiguous
    // tile of 32 CPL x NS floats; the lanes first put their rows into a
    // shared tile (16-byte pieces, XOR-swizzled within each 128-byte line so
    // that neither the row writes nor the contiguous reads conflict) and
    // then store it as whole 512-byte warp rows, evict-first in L2 (nothing
    // in this scan reads them again, and they must not push out the x / delta
    // lines the partner warp re-reads).
    const int nck = (a.L + 3) / 4;
    const uint64_t pol_ck = CKPT ? l2_evict_first() : 0;
    constexpr int kCkPieces = 32 * CPL * NS / 4;   // 16-byte pieces of the warp's tile
    auto ck_slot = [](int piece) {                  // byte offset of a piece in the swizzled tile
        const int line = piece >> 3;
        return line * 128 + (((piece & 7) ^ (line & 7)) << 4);
    };
    auto recur = [&](int i, const StepIn &in) {
        if (CKPT && !SUMMARY) {
            const int g = rev ? a.L - s1 + i : s0 + i;
            if ((g & 3) == 0) {
#pragma unroll
                for (int c = 0; c < CPL; c++)
#pragma unroll
                    for (int q = 0; q < NS / 4; q++) {
                        const int piece = (lane * CPL + c) * (NS / 4) + q;
                        *reinterpret_cast<float4 *>(ck_tile + ck_slot(piece)) =
                            make_float4(h[c][2 * q].x, h[c][2 * q].y, h[c][2 * q + 1].x, h[c][2 * q + 1].y);
                    }
                __syncwarp();
                float *ck = P.ckpt + (((size_t)b * nck + (g >> 2)) * a.D + dbase) * NS;
#pragma unroll
                for (int k = 0; k < kCkPieces / 32; k++) {
                    const int piece = k * 32 + lane;
                    const float4 v = *reinterpret_cast<const float4 *>(ck_tile + ck_slot(piece));
                    if (dbase + piece / (NS / 4) < a.D)
                        st4_hint(ck + 4 * piece, make_float2(v.x, v.y), make_float2(v.z, v.w), pol_ck);
                }
                __syncwarp();
            }
        }
        float2 dtc[CPL], dtx[CPL];
#pragma unroll
        for (int c = 0; c < CPL; c++) {
            dtc[c] = make_float2(in.dt[c], in.dt[c]);
            const float u = in.dt[c] * in.xv[c];
            dtx[c] = make_float2(u, u);
        }
        const float4 *row = reinterpret_cast<const float4 *>(sm.bc + (i & (2 * kTC - 1)) * 2 * NS);
        float2 ya[CPL], yb[CPL];
#pragma unroll
        for (int c = 0; c < CPL; c++) {
            ya[c] = make_float2(0.f, 0.f);
            yb[c] = make_float2(0.f, 0.f);
            if (SUMMARY)
                sdt[c] += in.dt[c];
        }
#pragma unroll
        for (int q = 0; q < NS / 4; q++) {
            const float4 bq = row[q];
            float4 cq = make_float4(0.f, 0.f, 0.f, 0.f);
            if (!SUMMARY)
                cq = row[NS / 4 + q];
            const float2 bp[2] = {make_float2(bq.x, bq.y), make_float2(bq.z, bq.w)};
            const float2 cp[2] = {make_float2(cq.x, cq.y), make_float2(cq.z, cq.w)};
#pragma unroll
            for (int r = 0; r < 2; r++) {
                const int k = 2 * q + r;   // state pair index
#pragma unroll
                for (int c = 0; c < CPL; c++) {
                    const float2 v = mul2(dtc[c], Ap[c][k]);
                    float2 e;
                    if (2 * k < NS - NPOLY) {
                        e.x = ex2_mufu(v.x);
                        e.y = ex2_mufu(v.y);
                    } else {
                        e = ex2_poly2(v);
                    }
                    h[c][k] = fma2(e, h[c][k], mul2(dtx[c], bp[r]));
                    if (!SUMMARY) {
                        if (r == 0)
                            ya[c] = fma2(cp[r], h[c][k], ya[c]);
                        else
                            yb[c] = fma2(cp[r], h[c][k], yb[c]);
                    }
                }
            }
        }
        StepOut o;
#pragma unroll
        for (int c = 0; c < CPL; c++) {
            const float2 sv = add2(ya[c], yb[c]);
            o.y[c] = sv.x + sv.y;
        }
        return o;
    };
    auto finish = [&](int i, const StepIn &in, const StepOut &ys, auto phase2_tag) {
        constexpr bool kPhase2 = decltype(phase2_tag)::value;
        float y[CPL];
#pragma unroll
        for (int c = 0; c < CPL; c++) {
            y[c] = fmaf(Dd[c], in.xv[c], ys.y[c]);
            if (GATE)
                y[c] *= in.zv[c];
            if (ORD && !in.keep)
                y[c] = 0.f;
        }
        if (!SUMMARY && active) {
            const size_t io = (rowbase + tpos(i)) * a.D + d;
            if (!BIDIR) {
                IO<T, CPL>::st(out + io, y);
            } else if (!kPhase2) {
                if (kHint)
                    st_hint(stash + io, y, pol_last);
                else
                    IO<float, CPL>::st(stash + io, y);
            } else {
                float o[CPL];
                IO<float, CPL>::ld(slot_of(i) + 3 * WS::kRowB + lane * CPL * 4, o);
#pragma unroll
                for (int c = 0; c < CPL; c++)
                    y[c] += o[c];
                if (kHint)
                    st_hint(out + io, y, pol_first);
                else
                    IO<T, CPL>::st(out + io, y);
            }
        }
    };
    auto step = [&](int i, auto phase2_tag) {
        const StepIn in = load_dt(i);
        finish(i, in, recur(i, in), phase2_tag);
    };
    // a full group of kSub steps: all operands and dt first, then the
    // recurrences back to back, then the epilogues
    auto group = [&](int i, auto phase2_tag) {
        StepIn in[kSub];
        StepOut ys[kSub];
#pragma unroll
        for (int j = 0; j < kSub; j++)
            in[j] = load_dt(i + j);
#pragma unroll
        for (int j = 0; j < kSub; j++)
            ys[j] = recur(i + j, in[j]);
#pragma unroll
        for (int j = 0; j < kSub; j++)
            finish(i + j, in[j], ys[j], phase2_tag);
    };
    // steps [i0, i1): unaligned head one by one, then straight-line groups of
    // kSub steps (so consecutive steps' independent work can interleave),
    // then the tail
    auto run = [&](int i0, int i1, auto phase2_tag) {
        int i = i0;
        for (; i < i1 && (i & (kSub - 1)) != 0; i++)
            step(i, phase2_tag);
        for (; i + kSub <= i1; i += kSub) {
            chunk_mgmt(i);
            group(i, phase2_tag);
        }
        if (i < i1) {
            chunk_mgmt(i);
            for (; i < i1; i++)
                step(i, phase2_tag);
        }
    };

    run(0, M, PhaseTag<false>{});
    if (BIDIR) {
        pair_barrier();
        with_stash = true;
        // steps already in flight were issued without their stash rows
        const int issued = min(Tn, ((M + kSub - 1) / kSub + kStages - 1) * kSub);
        issue_stash(M, issued);
        cp_async_wait_all();
        __syncwarp();
        run(M, Tn, PhaseTag<true>{});
    }
    cp_async_wait_all();
}

template <typename T, int NS, int CPL>
constexpr int smem_bytes() { return kWarps * (int)sizeof(WarpSmem<T, NS, CPL>); }
// the checkpointing variant also stages each warp's checkpoint tile
template <int NS, int CPL>
constexpr int ck_tile_bytes() { return 32 * CPL * NS * 4; }

// ---------------------------------------------------------------- summary
template <typename T, int NS, int CPL, int NPOLY, bool SOFTPLUS, bool ORD, bool CONV>
__global__ void __launch_bounds__(64, min_blocks<CPL>()) s6_summary_kernel(const S6Args a)
{
    extern __shared__ __align__(16) char smem_raw[];
    WarpSmem<T, NS, CPL> *sm = reinterpret_cast<WarpSmem<T, NS, CPL> *>(smem_raw);
    constexpr int kCh = 32 * CPL;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int dbase = (blockIdx.x * kWarps + warp) * kCh;
    const int d = dbase + CPL * lane;
    const int seg = blockIdx.y;
    const int dsel = blockIdx.z % a.ndir;
    const int b = blockIdx.z / a.ndir;
    const bool rev = a.ndir == 2 ? dsel == 1 : a.reverse != 0;
    if (last_in_order(seg, a.S, rev) || dbase >= a.D)
        return;
    const bool active = d < a.D;
    const int s0 = seg * a.T, s1 = min(a.L, s0 + a.T);
    float2 h[CPL][NS / 2];
    float sdt[CPL];
#pragma unroll
    for (int c = 0; c < CPL; c++) {
        sdt[c] = 0.f;
#pragma unroll
        for (int k = 0; k < NS / 2; k++)
            h[c][k] = make_float2(0.f, 0.f);
    }
    scan_segment<T, NS, CPL, NPOLY, true, false, false, SOFTPLUS, ORD, CONV>(a, a.dir[dsel], sm[warp], b,
                                                                             dbase, active, s0, s1, rev, h,
                                                                             sdt);
    if (!active)
        return;
#pragma unroll
    for (int c = 0; c < CPL; c++) {
        const size_t ci = (((size_t)dsel * a.Bsz + b) * a.S + seg) * a.D + d + c;
#pragma unroll
        for (int k = 0; k < NS / 2; k++) {
            if (2 * k < a.N)
                a.carry_h[ci * a.N + 2 * k] = h[c][k].x;
            if (2 * k + 1 < a.N)
                a.carry_h[ci * a.N + 2 * k + 1] = h[c][k].y;
        }
        a.carry_s[ci] = sdt[c];
    }
}

// ------------------------------------------------------------------ carry
// Per (direction, b, d, n): walk the segments in scan order from the initial
// state (or zero), replace each
// summary by the state entering that segment.  Summaries are fetched 16
// segments at a time ahead of the dependent chain.
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
    const size_t cbase = ((size_t)dsel * a.Bsz + b) * a.S;   // segment index base
    constexpr int kBatch = 16;
    const float *init = a.dir[dsel].init;
    float hin = init ? init[((size_t)b * a.D + d) * a.N + n] : 0.f;
    for (int k0 = 0; k0 < a.S; k0 += kBatch) {
        float hl[kBatch], sd[kBatch];
#pragma unroll
        for (int j = 0; j < kBatch; j++) {
            const int k = k0 + j;
            hl[j] = 0.f;
            sd[j] = 0.f;
            if (k < a.S - 1) {   // the last segment in scan order has no summary
                const int seg = rev ? a.S - 1 - k : k;
                const size_t ci = (cbase + seg) * a.D + d;
                hl[j] = a.carry_h[ci * a.N + n];
                sd[j] = a.carry_s[ci];
            }
        }
#pragma unroll
        for (int j = 0; j < kBatch; j++) {
            const int k = k0 + j;
            if (k < a.S) {
                const int seg = rev ? a.S - 1 - k : k;
                a.carry_h[((cbase + seg) * a.D + d) * a.N + n] = hin;
                hin = fmaf(ex2_mufu(Al2 * sd[j]), hin, hl[j]);
            }
        }
    }
}

// ------------------------------------------------------------------- main
template <typename T, int NS, int CPL, int NPOLY, bool BIDIR, bool GATE, bool SOFTPLUS, bool ORD, bool CONV,
          bool CKPT>
__global__ void __launch_bounds__(64, min_blocks<CPL>()) s6_main_kernel(const S6Args a)
{
    extern __shared__ __align__(16) char smem_raw[];
    WarpSmem<T, NS, CPL> *sm = reinterpret_cast<WarpSmem<T, NS, CPL> *>(smem_raw);
    constexpr int kCh = 32 * CPL;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int dsel = BIDIR ? warp : 0;
    const int dbase = BIDIR ? blockIdx.x * kCh : (blockIdx.x * kWarps + warp) * kCh;
    const int d = dbase + CPL * lane;
    const bool active = d < a.D;
    const int seg = blockIdx.y, b = blockIdx.z;
    const int s0 = seg * a.T, s1 = min(a.L, s0 + a.T);
    const bool rev = BIDIR ? dsel == 1 : a.reverse != 0;
    const DirArgs &P = a.dir[dsel];
    if (!BIDIR && dbase >= a.D)
        return;   // whole warp past the channels (never with a barrier partner)
    float2 h[CPL][NS / 2];
    float sdt[CPL];
    // the entering state: with segments, the carry pass wrote it for every
    // segment (the first one's is the initial state); otherwise the initial
    // state itself, or zero
    const bool has_carry = a.S > 1;
    const float *init = P.init;
#pragma unroll
    for (int c = 0; c < CPL; c++) {
        sdt[c] = 0.f;
        const size_t ci = (((size_t)dsel * a.Bsz + b) * a.S + seg) * a.D + d + c;
#pragma unroll
        for (int k = 0; k < NS / 2; k++) {
            const float *src = has_carry ? a.carry_h + ci * a.N
                                         : (init ? init + ((size_t)b * a.D + d + c) * a.N : nullptr);
            h[c][k].x = (active && src && 2 * k < a.N) ? src[2 * k] : 0.f;
            h[c][k].y = (active && src && 2 * k + 1 < a.N) ? src[2 * k + 1] : 0.f;
        }
    }
    char *ck_tile = CKPT ? smem_raw + smem_bytes<T, NS, CPL>() + warp * ck_tile_bytes<NS, CPL>() : nullptr;
    scan_segment<T, NS, CPL, NPOLY, false, BIDIR, GATE, SOFTPLUS, ORD, CONV, CKPT>(a, P, sm[warp], b, dbase,
                                                                                   active, s0, s1, rev, h, sdt,
                                                                                   ck_tile);
    if (active && P.last_state && last_in_order(seg, a.S, rev)) {
#pragma unroll
        for (int c = 0; c < CPL; c++) {
            float *ls = P.last_state + ((size_t)b * a.D + d + c) * a.N;
#pragma unroll
            for (int k = 0; k < NS / 2; k++) {
                if (2 * k < a.N)
                    ls[2 * k] = h[c][k].x;
                if (2 * k + 1 < a.N)
                    ls[2 * k + 1] = h[c][k].y;
            }
        }
    }
}

template <typename KernelT>
cudaError_t set_smem(KernelT k, int bytes)
{
    return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

template <typename T, int NS, int CPL, int NPOLY, bool GATE, bool SOFTPLUS, bool ORD, bool CONV, bool CKPT>
cudaError_t launch_typed(const S6Args &a, cudaStream_t st)
{
    constexpr int smem = smem_bytes<T, NS, CPL>();
    constexpr int smem_main = smem + (CKPT ? kWarps * ck_tile_bytes<NS, CPL>() : 0);
    constexpr int kCh = 32 * CPL;
    cudaError_t e;
    if (a.S > 1) {
        auto ks = s6_summary_kernel<T, NS, CPL, SSM_S6_SUM_NPOLY(NS), SOFTPLUS, ORD, CONV>;
        if ((e = set_smem(ks, smem)) != cudaSuccess)
            return e;
        dim3 g1((a.D + kWarps * kCh - 1) / (kWarps * kCh), a.S, a.Bsz * a.ndir);
        ks<<<g1, 64, smem, st>>>(a);
        const size_t tot = (size_t)a.ndir * a.Bsz * a.D * a.N;
        s6_carry_kernel<<<(unsigned)((tot + 255) / 256), 256, 0, st>>>(a);
    }
    if (a.ndir == 2) {
        auto km = s6_main_kernel<T, NS, CPL, NPOLY, true, GATE, SOFTPLUS, ORD, CONV, CKPT>;
        if ((e = set_smem(km, smem_main)) != cudaSuccess)
            return e;
        dim3 g((a.D + kCh - 1) / kCh, a.S, a.Bsz);
        km<<<g, 64, smem_main, st>>>(a);
    } else {
        auto km = s6_main_kernel<T, NS, CPL, NPOLY, false, GATE, SOFTPLUS, ORD, CONV, CKPT>;
        if ((e = set_smem(km, smem_main)) != cudaSuccess)
            return e;
        dim3 g((a.D + kWarps * kCh - 1) / (kWarps * kCh), a.S, a.Bsz);
        km<<<g, 64, smem_main, st>>>(a);
    }
    return cudaGetLastError();
}

// VAR: 0 plain, 1 ordered / masked, 2 conv input, 3 plain with checkpoints
// (each a kernel variant)
template <typename T, int NS, int NPOLY, bool GATE, bool SOFTPLUS, int VAR>
cudaError_t launch_cpl(const S6Args &a, cudaStream_t st)
{
    return a.cpl == 1 ? launch_typed<T, NS, 1, NPOLY, GATE, SOFTPLUS, VAR == 1, VAR == 2, VAR == 3>(a, st)
                      : launch_typed<T, NS, 2, NPOLY, GATE, SOFTPLUS, VAR == 1, VAR == 2, VAR == 3>(a, st);
}

#ifndef SSM_S6_NPOLY
#define SSM_S6_NPOLY 0
#endif

template <typename T, int NS, int NPOLY, int VAR>
cudaError_t launch_flags(const S6Args &a, cudaStream_t st)
{
    const bool gate = a.dir[0].z != nullptr;
    if (gate)
        return a.softplus ? launch_cpl<T, NS, NPOLY, true, true, VAR>(a, st)
                          : launch_cpl<T, NS, NPOLY, true, false, VAR>(a, st);
    return a.softplus ? launch_cpl<T, NS, NPOLY, false, true, VAR>(a, st)
                      : launch_cpl<T, NS, NPOLY, false, false, VAR>(a, st);
}

template <typename T, int VAR>
cudaError_t launch_ns(const S6Args &a, cudaStream_t st)
{
    if (a.N <= 4)
        return launch_flags<T, 4, 0, VAR>(a, st);
    if (a.N <= 8)
        return launch_flags<T, 8, 0, VAR>(a, st);
    return launch_flags<T, 16, SSM_S6_NPOLY, VAR>(a, st);
}

// This translation unit's error word: read it and, if clear, reset it.
cudaError_t s6_part_error(unsigned *value, bool clear)
{
    cudaError_t e = cudaMemcpyFromSymbol(value, g_s6_error, sizeof(unsigned));
    if (e != cudaSuccess || !clear)
        return e;
    const unsigned zero = 0;
    return cudaMemcpyToSymbol(g_s6_error, &zero, sizeof(unsigned));
}

}  // namespace
}  // namespace ssm

// One instantiation part: SSM_S6_PART(name, element type, variant) defines
// ssm::launch_s6_<name> and ssm::s6_error_<name>.
#define SSM_S6_PART(NAME, TYPE, VAR)                                                              \
    namespace ssm {                                                                               \
    cudaError_t launch_s6_##NAME(const S6Args &a, cudaStream_t st) { return launch_ns<TYPE, VAR>(a, st); } \
    cudaError_t s6_error_##NAME(unsigned *v, bool clear) { return s6_part_error(v, clear); }      \
    }
