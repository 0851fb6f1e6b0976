// s6_split.cu -- the S6 scan (single direction, or the Vision-Mamba pair of
// directions of "复现Vision Mamba", sec. 3.1 - 3.2) with each channel's 16
// states split over Q = 4 threads (described below) or Q = 2 threads (8
// channels a warp becomes 16, 8 states a thread; thread q then does the
// scalar work of steps q and q + 2).  The plan (split_threads) picks Q or
// the one-or-two-channels-per-thread kernels by size; with Q = 2 the last
// batch rows may run with Q = 4 in the same launch (split_mix_rows), which
// evens out the launch's last round of warps.  The same kernel body also
// serves the checkpointing forwards, the backward's checkpoint pass (no
// outputs) and the exact zero-order-hold scans.
//
// Step (Mamba2 page "手写简化版Mamba2", sec. 4.3 - 4.4), per (b, d):
//     dt = softplus(delta + bias),  h[n] = exp(dt A[n]) h[n] + dt B[n] x,
//     y  = (C . h + D x) silu(z).
// Thread (g, q) of a warp -- g = lane / 4 picks one of the warp's 8
// consecutive channels, q = lane % 4 -- owns states [4q, 4q + 4) of that
// channel.  Steps go in groups of four, and the per-channel scalar work of
// a group (softplus, the gate, the skip term, the output store) is spread
// over the channel's four threads: thread q does it for step q of the
// group.  A group runs
//   A  thread q: x, delta, z of step q -> dt, dt x, gate, D x;
//   B  every thread, steps 0..3 in order: step s's dt and dt x from thread
//      s of the channel (shuffles), its 4 states' update and their share of
//      C . h (packed f32x2 multiply / FMA, MUFU exp);
//   C  the four shares of each step are summed with shuffles so that thread
//      q ends with y of step q, and stores its output.
// Each warp streams its rows (x, delta, z: 8 channels; B, C: the whole row
// of 16) through a cp.async ring of kStages groups, so the copies of the
// next three groups are in flight during the current one.
//
// Bidirectional: a CTA is a pair of warps over the same 8 channels, warp 0
// scanning t ascending and warp 1 descending.  Each parks the first half of
// its outputs (in its own scan order) in `stash`, the pair meets at a named
// barrier, and each then adds the partner's parked value to the second half
// of its outputs: out is written once and no step is computed twice.  x
// and delta are read by both warps (and stay in L2 for the partner: the
// problems these layouts take fit in it).
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <type_traits>

#include "internal.h"
#include "s6_math.cuh"

namespace ssm {
namespace {

constexpr int kG = 4;                  // steps per group
constexpr int kStages = 4;             // groups in the copy ring (a power of two)
// CTAs (warp pairs) per SM the registers are sized for, and whether the
// copies and stores carry L2 eviction priorities.  Measured with this
// layout forced (one B200, µs): 12 CTAs (80 registers) without priorities
// -- bidirectional B 8, L 1024, D 768 bf16 135, B 32 / 64, L 197 fp32 90 /
// 164 -- against 16 CTAs (64 registers, spilling in the bidirectional
// variants) with them 164 / 96 / 168; the problems this layout takes fit
// in L2, so the priorities only cost registers.
#ifndef SSM_S6_SPLIT_MINB
#define SSM_S6_SPLIT_MINB 12
#endif
#ifndef SSM_S6_SPLIT_HINTS
#define SSM_S6_SPLIT_HINTS 0
#endif
#ifndef SSM_S6_SPLIT_MINB2
#define SSM_S6_SPLIT_MINB2 10
#endif
#ifndef SSM_S6_SPLIT_MINB2_PAIR
#define SSM_S6_SPLIT_MINB2_PAIR 8
#endif
#ifndef SSM_S6_SPLIT_MINB_PAIR
#define SSM_S6_SPLIT_MINB_PAIR 8
#endif
// CTAs per SM by threads per channel and direction.  Two threads per
// channel hold 8 states each and need more registers: a single direction
// at 10 CTAs (96 registers); the pair's exchange adds more, and its 8 CTAs
// of up to 128 registers measured 3-9% faster -- Vim-Small 131.1 -> 125.0
// us, its checkpointing forward 149.6 -> 136.3, B 48 bf16 107.5 -> 102.4 --
// while a single direction at 8 lost 2%.  Four threads per channel: a
// single direction at 12 (80 registers; 8 lost 7%), the pair at 8 (B 8,
// L 1024, D 768 bf16 144 -> 133 us; B 4, L 512 fp32 61.4 -> 55.3).  The
// zero-order-hold variants keep 1 / A of their states as well.
template <int Q, bool ZOH = false, bool BIDIR = false> constexpr int min_blocks()
{
    return ZOH ? (Q == 2 || BIDIR ? 8 : 10)
               : (Q == 2 ? (BIDIR ? SSM_S6_SPLIT_MINB2_PAIR : SSM_S6_SPLIT_MINB2)
                         : (BIDIR ? SSM_S6_SPLIT_MINB_PAIR : SSM_S6_SPLIT_MINB));
}
static_assert((kStages & (kStages - 1)) == 0, "ring index by mask");
// Which layout the plain calls take (split_threads).  The one-thread-per-
// channel kernels give a warp 64 channels (two a thread); with fewer than
// SSM_S6_SPLIT_MAX_WARPS1 warps (under two per SM sub-partition) they are
// latency-bound, or cut the sequence into segments and scan it twice.  Two
// threads per channel (8 states each) issue fewer instructions per element
// than four and run 4x the warps of the one-channel kernel: measured on
// B200 it is the fastest layout for every problem that gives the
// one-channel kernel at least that many warps (Vim-Small bidirectional
// fp32: 134 against 140 us; B 128: 239 against 261).  Below it a cost model
// fitted to the timings of all three layouts over 62 sizes (batch 1 - 256,
// L 196 - 16384, D 192 - 1536, both dtypes, one and two directions; it
// picks the fastest in 61, the miss costs 1.9%) decides, in microseconds,
// with E = elements B L D N x directions and (single direction / pair):
//   q threads per channel   max(Tl, Tt) + 0.3 min(Tl, Tt) + c,
//        q = 4: Tl = L x 0.067 / 0.082, Tt = E / 2.15e6 / 1.9e6, c = 6 / 9;
//        q = 2: Tl = L x 0.087 / 0.105, Tt = E / 2.9e6 / 2.65e6, c = 11 / 12;
//   the one-channel kernels 22 + 0.01 L + E / 1.333e6.
#ifndef SSM_S6_SPLIT_MAX_WARPS1
#define SSM_S6_SPLIT_MAX_WARPS1 1024
#endif
#ifndef SSM_BWD_SPLIT
#define SSM_BWD_SPLIT 1
#endif

#ifndef SSM_S6_SPLIT_SKEW
#define SSM_S6_SPLIT_SKEW 1
#endif
// Smallest stride >= bytes (16-byte steps) whose word offset mod 32 is an
// odd multiple of w (w = 4, 8 or 16 words).
constexpr int skew_stride(int bytes, int w)
{
    int s = bytes;
    while (!(((s / 4) % 32) % w == 0 && (((s / 4) % 32) / w) % 2 == 1))
        s += 16;
    return s;
}

// One step's slot in the ring: x, delta, (z) for the warp's 8 channels,
// then the B and C rows, then (bidirectional) the partner's 8 parked fp32
// outputs of that step, which are copied only once the pair has met.
template <typename T, bool GATE, bool BIDIR, int Q> struct Slot {
    static constexpr int kChW = 32 / Q;                     // channels per warp
    static constexpr int kRow = kChW * (int)sizeof(T);
    static constexpr int kBC = 16 * (int)sizeof(T);
    static constexpr int kX = 0, kDl = kRow, kZ = 2 * kRow;
    static constexpr int kB = (GATE ? 3 : 2) * kRow, kC = kB + kBC;
    static constexpr int kPk = kC + kBC;                    // parked row (bidirectional)
    static constexpr int kBytes = kPk + (BIDIR ? kChW * 4 : 0);
    static constexpr int kPieces = kBytes / 16;             // 16-byte copies per step
    static constexpr int kGroupPieces = kG * kPieces;
    static constexpr int kPerLane = (kGroupPieces + 31) / 32;
    // Step slots are kStride bytes apart: the Q threads of a channel read
    // the x, delta, z (and parked) values of Q consecutive steps at once, so
    // consecutive slots are skewed by an odd multiple of one step's widest
    // channel block in banks (kRow / 4 words, or kChW for the fp32 parked
    // row) -- a stride that is a multiple of 128 bytes would put every one
    // of those steps on the same banks.
    static constexpr int kStride = SSM_S6_SPLIT_SKEW ? skew_stride(kBytes, BIDIR ? kChW : kRow / 4) : kBytes;
    static constexpr int kGroupBytes = kG * kStride;
    static_assert(kBytes % 16 == 0 && kB % 16 == 0 && kRow % 16 == 0, "16-byte pieces");
};

template <typename T, bool GATE, bool BIDIR, int Q> struct WarpSmem {
    __align__(16) char ring[kStages][Slot<T, GATE, BIDIR, Q>::kGroupBytes];
};

__device__ __forceinline__ uint64_t policy_evict_last()
{
    if (!SSM_S6_SPLIT_HINTS)
        return 0;
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t policy_evict_first()
{
    if (!SSM_S6_SPLIT_HINTS)
        return 0;
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t policy_evict_normal()
{
    if (!SSM_S6_SPLIT_HINTS)
        return 0;
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
    return p;
}
// 16-byte cp.async with an L2 policy; n = 16 copies, n = 0 writes zeros
// without reading (src is a valid address all the same)
__device__ __forceinline__ void cp16(uint32_t dst, const char *src, int n, uint64_t pol)
{
    if (!SSM_S6_SPLIT_HINTS) {
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
        return;
    }
    asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2, %3;" ::"r"(dst), "l"(src), "r"(n),
                 "l"(pol)
                 : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int K> __device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(K) : "memory"); }
__device__ __forceinline__ void pair_barrier() { asm volatile("bar.sync 1, 64;" ::: "memory"); }

__device__ __forceinline__ void st_pol(float *p, float v, uint64_t pol)
{
    if (!SSM_S6_SPLIT_HINTS) {
        *p = v;
        return;
    }
    asm volatile("st.global.L2::cache_hint.f32 [%0], %1, %2;" ::"l"(p), "f"(v), "l"(pol) : "memory");
}
__device__ __forceinline__ void st_pol(__nv_bfloat16 *p, float v, uint64_t pol)
{
    if (!SSM_S6_SPLIT_HINTS) {
        *p = __float2bfloat16_rn(v);
        return;
    }
    const unsigned short u = __bfloat16_as_ushort(__float2bfloat16_rn(v));
    asm volatile("st.global.L2::cache_hint.b16 [%0], %1, %2;" ::"l"(p), "h"(u), "l"(pol) : "memory");
}

template <typename T> __device__ __forceinline__ float lds1(const char *p);
template <> __device__ __forceinline__ float lds1<float>(const char *p) { return *reinterpret_cast<const float *>(p); }
template <> __device__ __forceinline__ float lds1<__nv_bfloat16>(const char *p)
{
    return __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(p));
}
// four consecutive elements (this thread's quarter of a B or C row) as floats
template <typename T> __device__ __forceinline__ float4 lds4(const char *p);
template <> __device__ __forceinline__ float4 lds4<float>(const char *p) { return *reinterpret_cast<const float4 *>(p); }
template <> __device__ __forceinline__ float4 lds4<__nv_bfloat16>(const char *p)
{
    const uint2 u = *reinterpret_cast<const uint2 *>(p);
    return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u), __uint_as_float(u.y << 16),
                       __uint_as_float(u.y & 0xffff0000u));
}

// What a group does with its outputs: store them (one direction); park them
// (first half of a bidirectional pair); park the steps before the exchange
// point, meet the partner, then add to the rest (the group holding the
// exchange point); add the partner's parked values (second half).
enum Mode { kPlain, kPark, kMixed, kAdd };

// The factor of B in a state pair's update: dt x (Bbar = dt B), or for the
// exact zero-order hold (xv = x) x (e - 1) / a, with e = exp(dt a) and
// w = dt a log2(e), taken as x dt (1 + u / 2 + u^2 / 6 + u^3 / 24) with
// u = dt a where |u| < 1/16
template <bool ZOH>
__device__ __forceinline__ float2 in_coef(float2 dt2, float2 xv2, float2 w, float2 e, float2 iA)
{
    if (!ZOH)
        return xv2;   // dt x
    constexpr float kLn2 = 0.693147180559945309f;
    constexpr float c1 = kLn2 / 2.f, c2 = kLn2 * kLn2 / 6.f, c3 = kLn2 * kLn2 * kLn2 / 24.f;
    constexpr float kSeries = 0.0625f / kLn2;   // |u| < 1/16 in units of w
    float2 p = __ffma2_rn(w, make_float2(c3, c3), make_float2(c2, c2));
    p = __ffma2_rn(w, p, make_float2(c1, c1));
    p = __ffma2_rn(w, p, make_float2(1.f, 1.f));
    const float2 series = __fmul2_rn(dt2, p);
    const float2 direct = __fmul2_rn(__fadd2_rn(e, make_float2(-1.f, -1.f)), iA);
    const float2 c = make_float2(fabsf(w.x) < kSeries ? series.x : direct.x, fabsf(w.y) < kSeries ? series.y : direct.y);
    return __fmul2_rn(c, xv2);
}
template <Mode M> using ModeTag = std::integral_constant<Mode, M>;

// OUT = false: the checkpoint pass of the backward (single direction, no
// gate): only the states entering each 4-step group are stored.
// ZOH: the exact zero-order-hold input coefficient of the Mamba2 page,
// sec. 2.2 -- Bbar = (dt A)^-1 (exp(dt A) - I) dt B, per state
// (exp(dt a) - 1) / a -- instead of dt B.  e - 1 from the exponential the
// step computes anyway would lose its leading digits for small dt a, so
// there (|dt a| < 1/16) the coefficient is dt (1 + w / 2 + w^2 / 6 +
// w^3 / 24), w = dt a, whose truncation error is below 1.3e-7 relative.
// The body of one CTA: channel block bx (its warp pair's channels) of
// batch row b.
template <typename T, int Q, bool BIDIR, bool GATE, bool SOFTPLUS, bool OUT, bool ZOH>
__device__ __forceinline__ void split_body(const S6Args &a, WarpSmem<T, GATE, BIDIR, Q> *smem, int bx, int b)
{
    static_assert(Q == 2 || Q == 4, "two or four threads per channel");
    using S = Slot<T, GATE, BIDIR, Q>;
    constexpr int kChW = S::kChW;
    constexpr int NQ = 16 / Q;          // states per thread
    constexpr int NP = NQ / 2;          // state pairs per thread
    constexpr int SPL = kG / Q;         // steps of a group whose scalars a thread computes
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    WarpSmem<T, GATE, BIDIR, Q> &sm = smem[warp];
    const int g = lane / Q, q = lane % Q;
    const int dsel = BIDIR ? warp : 0;
    const int d0 = (BIDIR ? bx : bx * 2 + warp) * kChW;   // the warp's first channel
    const int L = a.L, D = a.D;
    if (!BIDIR && d0 >= D)
        return;   // whole warp past the channels (no barrier partner in this mode)
    const int d = d0 + g;
    const bool active = d < D;
    const bool rev = BIDIR ? dsel == 1 : a.reverse != 0;
    const DirArgs &P = a.dir[dsel];

    // this thread's states [NQ q, NQ q + NQ) as pairs, A scaled by log2(e)
    float2 A2[NP], h2[NP];
    float2 iA2[ZOH ? NP : 1] = {};   // zero-order hold: 1 / A (natural units)
#pragma unroll
    for (int v = 0; v < NQ / 4; v++) {
        float4 av = make_float4(0.f, 0.f, 0.f, 0.f), hv = av;
        if (active) {
            av = *reinterpret_cast<const float4 *>(P.A + (size_t)d * 16 + NQ * q + 4 * v);
            if (P.init)
                hv = *reinterpret_cast<const float4 *>(P.init + ((size_t)b * D + d) * 16 + NQ * q + 4 * v);
        }
        A2[2 * v] = make_float2(av.x * kLog2e, av.y * kLog2e);
        A2[2 * v + 1] = make_float2(av.z * kLog2e, av.w * kLog2e);
        if (ZOH) {   // (a = 0 only ever takes the series branch)
            iA2[2 * v] = make_float2(1.f / av.x, 1.f / av.y);
            iA2[2 * v + 1] = make_float2(1.f / av.z, 1.f / av.w);
        }
        h2[2 * v] = make_float2(hv.x, hv.y);
        h2[2 * v + 1] = make_float2(hv.z, hv.w);
    }
    const float bias = (active && P.bias) ? P.bias[d] : 0.f;
    const float Dd = (active && P.D) ? P.D[d] : 0.f;

    // steps before the exchange (bidirectional), in this warp's scan order
    const int M = BIDIR ? (rev ? L / 2 : (L + 1) / 2) : L;
    const int G = (L + kG - 1) / kG;

    // --- copies: this lane's 16-byte pieces of a group (piece p = lane + 32 j)
    const uint64_t pol_last = policy_evict_last(), pol_first = policy_evict_first();
    const uint64_t pol_normal = policy_evict_normal();
    const T *x = static_cast<const T *>(a.x), *dl = static_cast<const T *>(a.delta);
    const T *zp = static_cast<const T *>(P.z);
    const T *Bm = static_cast<const T *>(P.B), *Cm = static_cast<const T *>(P.C);
    const uint32_t ring_s = (uint32_t)__cvta_generic_to_shared(&sm.ring[0][0]);
    const char *safe = static_cast<const char *>(a.x);
    // (piece p of a group is byte 16 (p % kPieces) of step p / kPieces's slot)
    const char *cur[S::kPerLane];     // source row of the next group to issue
    uint32_t dst[S::kPerLane];        // its offset in a group's slots
    int gstep[S::kPerLane];           // bytes from one group's rows to the next's
    bool pok[S::kPerLane];            // the piece holds channels below D
    bool xd[S::kPerLane];             // an x / delta piece: L2 policy by half
    bool pk[S::kPerLane];             // a piece of the partner's parked row
    bool use[S::kPerLane];            // copied at all (no C rows without outputs)
    uint64_t pfix[S::kPerLane];       // the policy of the other pieces
#pragma unroll
    for (int j = 0; j < S::kPerLane; j++) {
        const int p = lane + 32 * j;
        const bool exists = p < S::kGroupPieces;
        const int pp = exists ? p : 0;
        const int s = pp / S::kPieces, off = (pp % S::kPieces) * 16;
        const int t0 = rev ? L - 1 - s : s;
        dst[j] = (uint32_t)(s * S::kStride + off);
        const char *base;
        long long row;
        bool ok = exists;
        pk[j] = false;
        use[j] = exists;
        if (off >= S::kPk) {   // 4 of the partner's parked fp32 outputs (bidirectional)
            const int jb = off - S::kPk;
            xd[j] = false;
            pk[j] = true;
            pfix[j] = pol_first;
            ok = ok && d0 + jb / 4 < D;
            row = (long long)D * 4;
            base = reinterpret_cast<const char *>(a.stash) + ((long long)b * L + t0) * row + (long long)d0 * 4 + jb;
        } else if (off < S::kB) {   // x, delta or z of 16 bytes' worth of the warp's channels
            const int arr = off / S::kRow, jb = off % S::kRow;
            const T *src = arr == 0 ? x : arr == 1 ? dl : zp;
            xd[j] = arr < 2;
            pfix[j] = pol_first;
            ok = ok && d0 + jb / (int)sizeof(T) < D;
            row = (long long)D * sizeof(T);
            base = reinterpret_cast<const char *>(src) + ((long long)b * L + t0) * row + (long long)d0 * sizeof(T) + jb;
        } else {             // 16 bytes of the B or C row (read by every warp of this batch row)
            const int o2 = off - S::kB;
            const T *src = o2 < S::kBC ? Bm : Cm;
            use[j] = exists && (OUT || o2 < S::kBC);
            xd[j] = false;
            pfix[j] = pol_normal;
            row = 16 * (long long)sizeof(T);
            base = reinterpret_cast<const char *>(src) + ((long long)b * L + t0) * row + o2 % S::kBC;
        }
        pok[j] = ok;
        cur[j] = ok ? base : safe;
        gstep[j] = ok ? (rev ? -1 : 1) * kG * (int)row : 0;
    }
    // parked rows are copied only after the pair has met (parked_live), for
    // the groups wholly after the exchange point
    bool parked_live = false;
    int next_gi = 0;   // groups [0, next_gi) have been copied (next_gi <= G)
    auto issue = [&](int gi) {
        if (gi < G) {
            const uint32_t sb = ring_s + (uint32_t)((gi & (kStages - 1)) * S::kGroupBytes);
            const uint64_t pxd = (BIDIR && gi * kG < M) ? pol_last : pol_first;
            if ((gi + 1) * kG <= L) {
#pragma unroll
                for (int j = 0; j < S::kPerLane; j++)
                    if ((OUT ? lane + 32 * j < S::kGroupPieces : use[j]) && (!BIDIR || !pk[j] || parked_live))
                        cp16(sb + dst[j], cur[j], pok[j] ? 16 : 0, xd[j] ? pxd : pfix[j]);
            } else {   // the last group is short: steps past L are zero-filled, not read
#pragma unroll
                for (int j = 0; j < S::kPerLane; j++)
                    if ((OUT ? lane + 32 * j < S::kGroupPieces : use[j]) && (!BIDIR || !pk[j] || parked_live)) {
                        const bool in = pok[j] && gi * kG + (lane + 32 * j) / S::kPieces < L;
                        cp16(sb + dst[j], in ? cur[j] : safe, in ? 16 : 0, xd[j] ? pxd : pfix[j]);
                    }
            }
#pragma unroll
            for (int j = 0; j < S::kPerLane; j++)
                cur[j] += gstep[j];
            next_gi = gi + 1;   // cur[] now points at group next_gi's rows
        }
        cp_commit();
    };
    // after the pair has met: the parked rows of the groups from g0 on that
    // were copied before it, then every copy in flight drained (so the
    // group counting of the waits stays exact)
    auto catch_up = [&](int g0) {
        for (int gj = g0; gj < next_gi && gj < G; gj++) {
            const uint32_t sb = ring_s + (uint32_t)((gj & (kStages - 1)) * S::kGroupBytes);
#pragma unroll
            for (int j = 0; j < S::kPerLane; j++)
                if (lane + 32 * j < S::kGroupPieces && pk[j]) {
                    const bool in = pok[j] && gj * kG + (lane + 32 * j) / S::kPieces < L;
                    const char *src = cur[j] - (long long)(next_gi - gj) * gstep[j];
                    cp16(sb + dst[j], in ? src : safe, in ? 16 : 0, pfix[j]);
                }
        }
        cp_commit();
        cp_wait<0>();
        __syncwarp();
    };

    // --- outputs: element index of this thread's first step (q) of the
    // current group; its step q + Q r is r Q rows further in scan order
    T *out = static_cast<T *>(a.out);
    float *stash = a.stash;
    long long oi = ((long long)b * L + (rev ? L - 1 - q : q)) * D + d;
    const int ostep = (rev ? -1 : 1) * kG * D;
    const int rstep = (rev ? -1 : 1) * Q * D;

    auto group = [&](int gi, auto mode_tag) {
        constexpr Mode MODE = decltype(mode_tag)::value;
        issue(gi + kStages - 1);
        cp_wait<kStages - 1>();
        __syncwarp();
        const char *gs = &sm.ring[gi & (kStages - 1)][0];
        // A: the scalars of this thread's steps q + Q r of the group
        float dt[SPL], dtx[SPL], gate[SPL], dxv[SPL];
        bool valid[SPL];
#pragma unroll
        for (int r = 0; r < SPL; r++) {
            const int i = gi * kG + q + Q * r;
            valid[r] = i < L;
            const char *sq = gs + (q + Q * r) * S::kStride + g * (int)sizeof(T);
            const float xv = lds1<T>(sq + S::kX);
            float t = lds1<T>(sq + S::kDl) + bias;
            if (SOFTPLUS)
                t = softplus_f(t);
            dt[r] = valid[r] ? t : 0.f;   // past L: exp(0) = 1 and no input, the state passes through
            dtx[r] = ZOH ? xv : dt[r] * xv;   // zero-order hold: x (its coefficient carries dt)
            gate[r] = GATE ? silu_f<T>(lds1<T>(sq + S::kZ)) : 1.f;
            dxv[r] = Dd * xv;
        }
        // checkpointing calls: the state entering this group is the
        // checkpoint of 4-step chunk gi of the scan order; each thread's
        // share of its channel's 16 states is contiguous, so the warp's
        // stores cover its channels' rows in one run
        if (P.ckpt && active) {
            float4 *ck = reinterpret_cast<float4 *>(P.ckpt + (((size_t)b * G + gi) * D + d) * 16 + NQ * q);
#pragma unroll
            for (int v = 0; v < NQ / 4; v++)
                ck[v] = make_float4(h2[2 * v].x, h2[2 * v].y, h2[2 * v + 1].x, h2[2 * v + 1].y);
        }
        // B: the four steps' state updates and shares of C . h (step s's dt
        // and dt x come from thread s % Q of the channel)
        float part[kG];
#pragma unroll
        for (int s = 0; s < kG; s++) {
            const int src = (lane & ~(Q - 1)) | (s % Q);
            const float dts = __shfl_sync(0xffffffffu, dt[s / Q], src);
            const float dtxs = __shfl_sync(0xffffffffu, dtx[s / Q], src);
            const char *ss = gs + s * S::kStride + q * NQ * (int)sizeof(T);
            const float2 dt2 = make_float2(dts, dts), dtx2 = make_float2(dtxs, dtxs);
            float2 y2 = make_float2(0.f, 0.f);
#pragma unroll
            for (int v = 0; v < NQ / 4; v++) {
                const float4 B4 = lds4<T>(ss + S::kB + 4 * v * (int)sizeof(T));
                float2 w = __fmul2_rn(dt2, A2[2 * v]);
                float2 e = make_float2(ex2_mufu(w.x), ex2_mufu(w.y));
                h2[2 * v] = __ffma2_rn(e, h2[2 * v], __fmul2_rn(in_coef<ZOH>(dt2, dtx2, w, e, iA2[ZOH ? 2 * v : 0]),
                                                                make_float2(B4.x, B4.y)));
                w = __fmul2_rn(dt2, A2[2 * v + 1]);
                e = make_float2(ex2_mufu(w.x), ex2_mufu(w.y));
                h2[2 * v + 1] = __ffma2_rn(
                    e, h2[2 * v + 1],
                    __fmul2_rn(in_coef<ZOH>(dt2, dtx2, w, e, iA2[ZOH ? 2 * v + 1 : 0]), make_float2(B4.z, B4.w)));
                if (OUT) {
                    const float4 C4 = lds4<T>(ss + S::kC + 4 * v * (int)sizeof(T));
                    y2 = __ffma2_rn(make_float2(C4.x, C4.y), h2[2 * v], y2);
                    y2 = __ffma2_rn(make_float2(C4.z, C4.w), h2[2 * v + 1], y2);
                }
            }
            part[s] = y2.x + y2.y;
        }
        if (!OUT) {   // checkpoint pass: nothing else to write
            __syncwarp();
            return;
        }
        // C: sum the channel's Q shares of each step so that thread q holds
        // those of its steps q + Q r
        float ysum[SPL];
        if (Q == 4) {
            // exchange halves across q bit 1 (steps {0, 1} vs {2, 3}), then
            // across q bit 0
            const bool hi1 = (q & 2) != 0, hi0 = (q & 1) != 0;
            float ka = hi1 ? part[2] : part[0], kb = hi1 ? part[3] : part[1];
            ka += __shfl_xor_sync(0xffffffffu, hi1 ? part[0] : part[2], 2);
            kb += __shfl_xor_sync(0xffffffffu, hi1 ? part[1] : part[3], 2);
            ysum[0] = (hi0 ? kb : ka) + __shfl_xor_sync(0xffffffffu, hi0 ? ka : kb, 1);
        } else {
            // thread q keeps steps q and q + 2 and sends the other two
            const bool hi = q != 0;
#pragma unroll
            for (int r = 0; r < SPL; r++)
                ysum[r] = (hi ? part[2 * r + 1] : part[2 * r]) +
                          __shfl_xor_sync(0xffffffffu, hi ? part[2 * r] : part[2 * r + 1], 1);
        }
        float y[SPL];
        bool st[SPL];
#pragma unroll
        for (int r = 0; r < SPL; r++) {
            y[r] = (ysum[r] + dxv[r]) * gate[r];
            st[r] = active && valid[r];
        }
        if (MODE == kPlain) {
#pragma unroll
            for (int r = 0; r < SPL; r++)
                if (st[r])
                    st_pol(out + oi + r * rstep, y[r], pol_first);
        } else if (MODE == kPark) {
#pragma unroll
            for (int r = 0; r < SPL; r++)
                if (st[r])
                    st_pol(stash + oi + r * rstep, y[r], pol_last);
        } else if (MODE == kMixed) {
#pragma unroll
            for (int r = 0; r < SPL; r++)
                if (st[r] && gi * kG + q + Q * r < M)
                    st_pol(stash + oi + r * rstep, y[r], pol_last);
            pair_barrier();   // both warps' parked halves are written
#pragma unroll
            for (int r = 0; r < SPL; r++)
                if (st[r] && gi * kG + q + Q * r >= M)
                    st_pol(out + oi + r * rstep, y[r] + __ldcg(stash + oi + r * rstep), pol_first);
        } else {
#pragma unroll
            for (int r = 0; r < SPL; r++)
                if (st[r])   // the partner's parked value, copied with this group's rows
                    st_pol(out + oi + r * rstep,
                           y[r] + *reinterpret_cast<const float *>(gs + (q + Q * r) * S::kStride + S::kPk + 4 * g),
                           pol_first);
        }
        oi += ostep;
        __syncwarp();   // every thread is done with this group's slots and tables
    };

#pragma unroll
    for (int k = 0; k < kStages - 1; k++)
        issue(k);
    if (!BIDIR) {
        for (int gi = 0; gi < G; gi++)
            group(gi, ModeTag<kPlain>{});
    } else {
        // groups [0, g1) lie wholly before the exchange point, [g2, G) wholly after
        const int g1 = M / kG, g2 = (M + kG - 1) / kG;
        for (int gi = 0; gi < g1; gi++)
            group(gi, ModeTag<kPark>{});
        if (g1 < g2)
            group(g1, ModeTag<kMixed>{});
        else
            pair_barrier();
        parked_live = true;
        catch_up(g2);
        for (int gi = g2; gi < G; gi++)
            group(gi, ModeTag<kAdd>{});
    }
    cp_wait<0>();

    if (OUT && active && P.last_state) {
#pragma unroll
        for (int v = 0; v < NQ / 4; v++)
            *reinterpret_cast<float4 *>(P.last_state + ((size_t)b * D + d) * 16 + NQ * q + 4 * v) =
                make_float4(h2[2 * v].x, h2[2 * v].y, h2[2 * v + 1].x, h2[2 * v + 1].y);
    }
}

template <typename T, int Q, bool BIDIR, bool GATE, bool SOFTPLUS, bool OUT = true, bool ZOH = false>
__global__ void __launch_bounds__(64, min_blocks<Q, ZOH, BIDIR>()) s6_split_kernel(const S6Args a)
{
    __shared__ WarpSmem<T, GATE, BIDIR, Q> smem[2];
    split_body<T, Q, BIDIR, GATE, SOFTPLUS, OUT, ZOH>(a, smem, (int)blockIdx.x, (int)blockIdx.y);
}

// Two threads per channel for batch rows [0, a.mix_rows2), four for the
// rest, in one launch (1-D grid, the two-thread CTAs first): the
// half-width four-thread CTAs dispatched last even out the work left on
// the SM sub-partitions at the end of the launch.
template <typename T, bool BIDIR, bool GATE, bool SOFTPLUS, bool OUT = true>
__global__ void __launch_bounds__(64, min_blocks<2, false, BIDIR>()) s6_split_mixed_kernel(const S6Args a)
{
    using W2 = WarpSmem<T, GATE, BIDIR, 2>;
    using W4 = WarpSmem<T, GATE, BIDIR, 4>;
    __shared__ __align__(16) char smem[sizeof(W2) > sizeof(W4) ? 2 * sizeof(W2) : 2 * sizeof(W4)];
    const int nx2 = BIDIR ? (a.D + 15) / 16 : (a.D + 31) / 32, nx4 = BIDIR ? (a.D + 7) / 8 : (a.D + 15) / 16;
    const long long n2 = (long long)a.mix_rows2 * nx2, bid = blockIdx.x;
    if (bid < n2) {
        split_body<T, 2, BIDIR, GATE, SOFTPLUS, OUT, false>(a, reinterpret_cast<W2 *>(smem), (int)(bid % nx2),
                                                          (int)(bid / nx2));
    } else {
        const long long r = bid - n2;
        split_body<T, 4, BIDIR, GATE, SOFTPLUS, OUT, false>(a, reinterpret_cast<W4 *>(smem), (int)(r % nx4),
                                                          a.mix_rows2 + (int)(r / nx4));
    }
}

template <typename T, int Q, bool GATE, bool SOFTPLUS, bool ZOH>
cudaError_t launch_q(const S6Args &a, cudaStream_t st)
{
    constexpr int kChW = 32 / Q;
    if (a.ndir == 2) {
        const dim3 grid((unsigned)((a.D + kChW - 1) / kChW), (unsigned)a.Bsz);
        s6_split_kernel<T, Q, true, GATE, SOFTPLUS, true, ZOH><<<grid, 64, 0, st>>>(a);
    } else {
        const dim3 grid((unsigned)((a.D + 2 * kChW - 1) / (2 * kChW)), (unsigned)a.Bsz);
        s6_split_kernel<T, Q, false, GATE, SOFTPLUS, true, ZOH><<<grid, 64, 0, st>>>(a);
    }
    return cudaGetLastError();
}

template <typename T, bool GATE, bool SOFTPLUS, bool ZOH>
cudaError_t launch_t(const S6Args &a, cudaStream_t st)
{
    if (!ZOH && a.split == 2 && a.mix_rows2 > 0 && a.mix_rows2 < a.Bsz) {
        const bool bidir = a.ndir == 2;
        const long long nx2 = bidir ? (a.D + 15) / 16 : (a.D + 31) / 32, nx4 = bidir ? (a.D + 7) / 8 : (a.D + 15) / 16;
        const unsigned grid = (unsigned)(a.mix_rows2 * nx2 + (long long)(a.Bsz - a.mix_rows2) * nx4);
        if (bidir)
            s6_split_mixed_kernel<T, true, GATE, SOFTPLUS><<<grid, 64, 0, st>>>(a);
        else
            s6_split_mixed_kernel<T, false, GATE, SOFTPLUS><<<grid, 64, 0, st>>>(a);
        return cudaGetLastError();
    }
    return a.split == 2 ? launch_q<T, 2, GATE, SOFTPLUS, ZOH>(a, st) : launch_q<T, 4, GATE, SOFTPLUS, ZOH>(a, st);
}

// the backward's checkpoint pass: one direction, no gate, no outputs
template <typename T, int Q, bool SOFTPLUS>
cudaError_t launch_ckpt_q(const S6Args &a, cudaStream_t st)
{
    constexpr int kChW = 32 / Q;
    const dim3 grid((unsigned)((a.D + 2 * kChW - 1) / (2 * kChW)), (unsigned)a.Bsz);
    s6_split_kernel<T, Q, false, false, SOFTPLUS, false><<<grid, 64, 0, st>>>(a);
    return cudaGetLastError();
}
template <typename T>
cudaError_t launch_ckpt_t(const S6Args &a, cudaStream_t st)
{
    if (a.split == 2 && a.mix_rows2 > 0 && a.mix_rows2 < a.Bsz) {   // the mixed launch, as for the scans
        const unsigned grid = (unsigned)((long long)a.mix_rows2 * ((a.D + 31) / 32) +
                                         (long long)(a.Bsz - a.mix_rows2) * ((a.D + 15) / 16));
        if (a.softplus)
            s6_split_mixed_kernel<T, false, false, true, false><<<grid, 64, 0, st>>>(a);
        else
            s6_split_mixed_kernel<T, false, false, false, false><<<grid, 64, 0, st>>>(a);
        return cudaGetLastError();
    }
    if (a.split == 2)
        return a.softplus ? launch_ckpt_q<T, 2, true>(a, st) : launch_ckpt_q<T, 2, false>(a, st);
    return a.softplus ? launch_ckpt_q<T, 4, true>(a, st) : launch_ckpt_q<T, 4, false>(a, st);
}

template <typename T, bool ZOH>
cudaError_t launch_flags(const S6Args &a, cudaStream_t st)
{
    const bool gate = a.dir[0].z != nullptr;
    if (gate)
        return a.softplus ? launch_t<T, true, true, ZOH>(a, st) : launch_t<T, true, false, ZOH>(a, st);
    return a.softplus ? launch_t<T, false, true, ZOH>(a, st) : launch_t<T, false, false, ZOH>(a, st);
}

}  // namespace

// 0 cost model, 1 never these layouts, 2 four threads per channel whenever
// supported, 3 two threads per channel whenever supported
std::atomic<int> g_split_mode{0};

int split_threads(int64_t Bsz, int64_t L, int64_t D, int64_t N, int ndir)
{
    if (N != 16 || L <= 0 || Bsz <= 0 || D <= 0 || Bsz > 65535)
        return 0;
    const int mode = g_split_mode.load(std::memory_order_relaxed);
    if (mode != 0)
        return mode == 2 ? 4 : mode == 3 ? 2 : 0;
    const int64_t warps1 = (int64_t)ndir * Bsz * ((D + 63) / 64);   // one thread, two channels
    if (warps1 >= SSM_S6_SPLIT_MAX_WARPS1)
        return 2;
    const bool pair = ndir == 2;
    const double E = (double)ndir * Bsz * L * D * 16;
    auto t_split = [&](double lat, double thr, double c) {
        const double tl = (double)L * lat, tt = E / thr;
        return (tl > tt ? tl + 0.3 * tt : tt + 0.3 * tl) + c;
    };
    const double t4 = t_split(pair ? 0.082 : 0.067, pair ? 1.9e6 : 2.15e6, pair ? 9.0 : 6.0);
    const double t2 = t_split(pair ? 0.105 : 0.087, pair ? 2.65e6 : 2.9e6, pair ? 12.0 : 11.0);
    const double t1 = 22.0 + 0.01 * (double)L + E / 1.333e6;
    if (t1 <= t4 && t1 <= t2)
        return 0;
    return t2 < t4 ? 2 : 4;
}

#ifndef SSM_S6_SPLIT_MIX
#define SSM_S6_SPLIT_MIX 1
#endif
int split_mix_rows(int64_t Bsz, int64_t D, int ndir)
{
    if (!SSM_S6_SPLIT_MIX)
        return 0;
    // The launch takes about as long as its busiest SM sub-partition's
    // warps (each CTA is 2 warps): ceil(warps / 592) of them.  Rows moved
    // to four threads per channel become twice the warps at about 0.57 of
    // the cost each, and being dispatched last they fill the sub-partitions
    // left short; mix only when the mean load then ends well below that
    // ceiling.
    constexpr int64_t kSubPartitions = 148 * 4;
    constexpr double kQ4Warp = 0.57, kSlack = 0.3;
    const int64_t nx2 = ndir == 2 ? (D + 15) / 16 : (D + 31) / 32;   // CTAs (2 warps each) per batch row
    const int64_t nx4 = ndir == 2 ? (D + 7) / 8 : (D + 15) / 16;
    const int64_t warps = 2 * Bsz * nx2, levels = warps / kSubPartitions;
    if (levels == 0 || warps % kSubPartitions == 0)
        return 0;
    const int64_t rows2 = levels * kSubPartitions / (2 * nx2);   // these fill `levels` exactly or less
    if (rows2 <= 0 || rows2 >= Bsz || rows2 * nx2 + (Bsz - rows2) * nx4 > 0x7fffffff)
        return 0;   // (the mixed launch's grid is one-dimensional)
    const double mean = (2.0 * rows2 * nx2 + kQ4Warp * 2.0 * (Bsz - rows2) * nx4) / kSubPartitions;
    return mean + kSlack < (double)(levels + 1) ? (int)rows2 : 0;
}

void split_mode_set(int mode) { g_split_mode.store(mode, std::memory_order_relaxed); }

bool bwd_split_enabled() { return SSM_BWD_SPLIT && g_split_mode.load(std::memory_order_relaxed) != 1; }

cudaError_t launch_s6_split_ckpt_only(const S6Args &a, cudaStream_t st)
{
    return a.dtype == 0 ? launch_ckpt_t<float>(a, st) : launch_ckpt_t<__nv_bfloat16>(a, st);
}

cudaError_t launch_s6_split(const S6Args &a, cudaStream_t st)
{
    if (a.zoh)
        return a.dtype == 0 ? launch_flags<float, true>(a, st) : launch_flags<__nv_bfloat16, true>(a, st);
    return a.dtype == 0 ? launch_flags<float, false>(a, st) : launch_flags<__nv_bfloat16, false>(a, st);
}

}  // namespace ssm
