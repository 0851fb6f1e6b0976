// ssd_chunk.cu -- Mamba2 SSD chunked scan for sm_100a (tcgen05 tensor cores,
// TMA, TMEM accumulators), plus the library's device-side error word.
//
// Operation (Mamba2 page "手写简化版Mamba2", sec. 3.1-3.2): the S6
// recurrence with a scalar A per head, computed chunk by chunk.  For head h
// of batch b and a chunk of Q = 64 steps starting at t0, with
//   dt_t = softplus(delta[b,t,h] + bias[h]),  a_t = dt_t A[h],
//   cs_i = a_{t0} + ... + a_{t0+i}            (inclusive, inside the chunk)
// the chunk computes
//   G      = C B^T                              (64 x 64,  K = N = 128)
//   M[i,j] = G[i,j] exp(cs_i - cs_j) dt_j  (j <= i, else 0)
//   Yd     = M X                                (64 x 64,  K = 64)
//   Yo     = C S_in                             (64 x 64,  K = 128)
//   W[j,:] = exp(cs_end - cs_j) dt_j X[j,:]
//   dS     = B^T W                              (128 x 64, K = 64)
//   y      = (Yd + exp(cs_i) Yo + D x) silu(z)
//   S_out  = exp(cs_end) S_in + dS              (the state handed to the next chunk)
// The four products run on tcgen05.mma (bf16 operands in shared memory,
// fp32 accumulators in tensor memory); the state S stays in fp32 registers
// (one row n of S per thread).  The operands computed in the kernel (M, W
// and the copy of S_in) are each stored as a bf16 pair hi + lo with
// lo = bf16(v - hi), and each of their products is issued twice (hi, then
// lo accumulated), so they carry about 16 mantissa bits instead of 8; the
// loaded operands X, B, C are exact in bf16.
//
// One CTA owns one (b, h) and walks its chunks in order.  It has four
// warpgroups of math threads -- warpgroup g owns columns [16 g, 16 g + 16) of
// every 64-wide row --, one warp whose lane 0 issues the tensor-core MMAs
// when the math threads signal (mbarriers) that the operands are written, and
// one warp that issues the TMA loads and computes dt and its cumulative sum
// up to three chunks ahead.  Per chunk c the math threads build the decay
// matrix M(c) as soon as G(c) is done (G has its own commit), then the next
// chunk's W(c + 1) while the tensor core finishes Yo(c), dS(c) and Yd(c),
// then update the state and write S_in(c + 1), then chunk c's outputs; the
// MMA warp issues Yd(c) once M(c) is written and chunk c + 1's G, Yo and dS
// once W(c + 1) and S_in(c + 1) are (W and the Yo accumulator are
// double-buffered by chunk parity, dt / cs triple-buffered).  The hi and lo
// halves of S_in and of W sit side by side as one N = 128 operand, so each
// of those products is one MMA per K-step.  TMA brings each chunk's X, Z
// (64 x 64 bf16) and B, C (64 x 128) tiles into a three-stage shared-memory
// ring with the 128-byte swizzle, which is directly the layout the tensor
// core reads (C and B as K-major operands of C B^T, B as an MN-major operand
// of B^T W, X as an MN-major operand of M X).  Every mbarrier wait is bounded
// and sets the library's error word if it gives up.
#include <atomic>

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include "internal.h"

namespace ssm {

__device__ unsigned g_device_error;

namespace {

constexpr int kQ = 64;          // chunk length
constexpr int kP = 64;          // head dim
constexpr int kN = 128;         // state size
constexpr int kMath = 512;      // four warpgroups; warpgroup g owns columns [16 g, 16 g + 16)
constexpr int kThreads = kMath + 64;   // + one warp that issues the MMAs, one that computes dt
constexpr int kMmaWarp = kMath / 32, kDtWarp = kMath / 32 + 1;
constexpr int kDtBufs = 3;             // dt / cs buffers, one per TMA stage
static_assert(kDtBufs == 3, "the dt buffers are recycled with the TMA stages");
constexpr float kLog2e = 1.4426950408889634f;

// shared-memory plan (byte offsets from a 1024-aligned base)
constexpr int kTileX = kQ * kP * 2;            // 8 KB  (64 rows x 128 B)
constexpr int kTileBC = kQ * 64 * 2;           // 8 KB  (one 64-wide half of B or C)
constexpr int kStageX = 0;
constexpr int kStageZ = kTileX;
constexpr int kStageB = 2 * kTileX;            // two halves (n 0..63, 64..127)
constexpr int kStageC = 2 * kTileX + 2 * kTileBC;
constexpr int kStageBytes = 2 * kTileX + 4 * kTileBC;   // 48 KB
constexpr int kStages = 3;                              // TMA ring depth
constexpr int kOffW = kStages * kStageBytes;            // W [buffer][hi, lo]: 4 x 8 KB, rows j, MN-major
constexpr int kOffM = kOffW + 4 * kTileX;               // M [hi, lo]: 2 x 8 KB, rows i, K-major
constexpr int kSBytes = kN * 128;
constexpr int kOffS = kOffM + 2 * kTileX;               // S_in [hi, lo]: 2 x 16 KB, rows n, MN-major
constexpr int kOffVec = kOffS + 2 * kSBytes;            // cs[kDtBufs][64], dt[kDtBufs][64]
constexpr int kSmemBytes = kOffVec + 2 * kDtBufs * 64 * 4 + 1024; // + alignment slack

// TMEM columns.  dS and Yo hold the hi and lo halves side by side
// (N = 128: columns [0, 64) from the hi operand, [64, 128) from lo); Yo is
// double-buffered by chunk parity because chunk c's outputs read it after
// chunk c + 1's first products were issued.
constexpr uint32_t kColG = 0, kColDS = 64, kColYo = 192, kColYd = 448, kTmemCols = 512;

constexpr long kWaitLimit = 1l << 20;    // default poll limit of a pipeline wait
constexpr long kDrainLimit = 1l << 22;   // poll limit of the teardown waits for in-flight copies / MMAs

__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

// byte offset of 16-byte chunk q of row r inside a [rows x 128 B] block with
// the 128-byte swizzle (chunk index XOR row mod 8)
__device__ __forceinline__ uint32_t sw_chunk(int r, int q) { return r * 128 + ((q ^ (r & 7)) << 4); }

__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo)
{
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);
    d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFF) << 32;
    d |= (uint64_t)1 << 46;   // descriptor version for sm_100
    d |= (uint64_t)2 << 61;   // 128-byte swizzle
    return d;
}

// kind::f16 instruction descriptor: bf16 A and B, fp32 D
constexpr uint32_t idesc_bf16(int M, int N, int a_mn_major, int b_mn_major)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn_major << 15) |
           ((uint32_t)b_mn_major << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void umma(uint32_t d, uint64_t a, uint64_t b, uint32_t id, uint32_t acc)
{
    asm volatile("{.reg .pred p; setp.ne.b32 p, %4, 0; tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;}" ::"r"(d),
                 "l"(a), "l"(b), "r"(id), "r"(acc)
                 : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t *bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// Bounded wait on an mbarrier phase (with SSM_SSD_SUSPEND_NS > 0 each
// try_wait may suspend the thread for up to that long; it resumes when the
// phase completes).  On giving up after `limit` polls, a thread flags the
// library's error word and its CTA's abort word and returns false; every
// later wait in the CTA then gives up at once.  After a failed wait a role
// issues no further copies or MMAs and signals no further barriers, so the
// only asynchronous work left is what was issued before; the teardown waits
// for it (drain_wait) before TMEM is freed and the CTA exits.  The kernel
// then ends promptly with wrong values, reported by ssm_check_device.
#ifndef SSM_SSD_SUSPEND_NS
#define SSM_SSD_SUSPEND_NS 0
#endif
constexpr uint32_t kSuspendNs = SSM_SSD_SUSPEND_NS;
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, volatile int *abort, long limit)
{
    const uint32_t a = smem_u32(bar);
    for (long it = 0; it < limit; it++) {
        uint32_t ok;
        if (kSuspendNs)
            asm volatile("{.reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3; selp.u32 %0, 1, 0, p;}"
                         : "=r"(ok)
                         : "r"(a), "r"(parity), "r"(kSuspendNs)
                         : "memory");
        else
            asm volatile("{.reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p;}"
                         : "=r"(ok)
                         : "r"(a), "r"(parity)
                         : "memory");
        if (ok)
            return true;
        if ((it & 255) == 255 && *abort)
            return false;
    }
    *abort = 1;
    atomicExch(&g_device_error, 1u);
    return false;
}

// Teardown wait for asynchronous work this CTA issued itself (a TMA load
// landing, a tcgen05.commit arriving): it completes on its own, so the wait
// ignores the abort word; it is still bounded, and flags the error word if
// it gives up.
__device__ __forceinline__ void drain_wait(uint64_t *bar, uint32_t parity)
{
    const uint32_t a = smem_u32(bar);
    for (long it = 0; it < kDrainLimit; it++) {
        uint32_t ok;
        asm volatile("{.reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p;}"
                     : "=r"(ok)
                     : "r"(a), "r"(parity)
                     : "memory");
        if (ok)
            return;
    }
    atomicExch(&g_device_error, 1u);
}

__device__ __forceinline__ void tma_load_4d(void *dst, const CUtensorMap *map, int c0, int c1, int c2, int c3,
                                            uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(
            smem_u32(dst)),
        "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, int c0, int c1, int c2, uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(
            smem_u32(dst)),
        "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
        : "memory");
}


// TMEM loads.  They are asynchronous: the registers are valid only after
// tmem_wait_ld(), so several loads can be in flight behind one wait.
//
// 8 columns of one M = 64 accumulator row: threads t < 16 of warp w get row
// 16 (w mod 4) + t, columns [col, col + 8); threads t >= 16 the same row,
// columns [col + 8, col + 16).
__device__ __forceinline__ void tmem_ld_eighth_row(uint32_t taddr, uint32_t (&r)[8])
{
    asm volatile("tcgen05.ld.sync.aligned.16x32bx2.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8], 8;"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
}

// 16 consecutive columns of this thread's lane (an M = 128 accumulator row)
__device__ __forceinline__ void tmem_ld_row16(uint32_t taddr, uint32_t (&r)[16])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

// Wait for this thread's TMEM loads.  The registers pass through an empty
// asm so that no use of them is scheduled above the wait.
template <int K>
__device__ __forceinline__ void tmem_wait_ld(uint32_t (&r)[K])
{
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int k = 0; k < K; k++)
        asm volatile("" : "+r"(r[k]));
}


__device__ __forceinline__ float ex2f(float v)
{
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(v));
    return r;
}

__device__ __forceinline__ float softplus_f(float v)
{
    // max(v, 0) + log1p(exp(-|v|)) with log1p by series below 1/16
    const float e = ex2f(-fabsf(v) * kLog2e);
    float lg;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(lg) : "f"(1.f + e));
    const float s = e * fmaf(e, fmaf(e, fmaf(e, fmaf(e, fmaf(e, -1.f / 6.f, 0.2f), -0.25f), 1.f / 3.f), -0.5f), 1.f);
    return fmaxf(v, 0.f) + (e < 0.0625f ? s : lg * 0.6931471805599453f);
}

// silu(z) = z sigmoid(z) = h (1 + tanh h) with h = z / 2 is evaluated inline
// in the epilogue with tanh.approx (relative error 2^-11, far below the bf16
// output rounding of this path).

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// v = hi + lo with hi = bf16(v) and lo = bf16(v - hi), for two values
__device__ __forceinline__ void split_bf16(float a, float b, uint32_t &hi, uint32_t &lo)
{
    hi = pack_bf16(a, b);
    const float2 r = __fadd2_rn(make_float2(a, b),
                                make_float2(-__uint_as_float(hi << 16), -__uint_as_float(hi & 0xffff0000u)));
    lo = pack_bf16(r.x, r.y);
}

__device__ __forceinline__ float2 unpack_bf16(uint32_t u)
{
    return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

struct SSDKernelArgs {
    int Bsz, L, H, nchunks;
    int softplus;
    const __nv_bfloat16 *delta;
    const float *bias, *A, *D;
    __nv_bfloat16 *out;
    float *last_state;
    int has_z;
    long wait_limit;      // polls before a pipeline wait gives up
    int withhold_chunk;   // >= 0: the dt warp never signals that chunk's dt (device-timeout test)
};

__global__ void __launch_bounds__(kThreads, 1)
    ssd_chunk_kernel(const __grid_constant__ CUtensorMap mapX, const __grid_constant__ CUtensorMap mapZ,
                     const __grid_constant__ CUtensorMap mapB, const __grid_constant__ CUtensorMap mapC,
                     const SSDKernelArgs args)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ __align__(8) uint64_t bar_tma[kStages];
    __shared__ __align__(8) uint64_t bar_g;       // tensor core: G(c) done
    __shared__ __align__(8) uint64_t bar_ds;      // tensor core: dS(c) done (and Yo(c) before it)
    __shared__ __align__(8) uint64_t bar_mma2;    // tensor core: Yd(c) done
    __shared__ __align__(8) uint64_t bar_mready;  // math threads: M(c) written, G(c) read
    __shared__ __align__(8) uint64_t bar_sready;  // math threads: W(c + 1), S_in(c + 1) written, dS(c) read
    __shared__ volatile int abort_sh;
    __shared__ __align__(8) uint64_t bar_dt_full[kDtBufs];    // dt warp: dt / cs of a chunk written
    __shared__ __align__(8) uint64_t bar_free[kDtBufs];       // math threads: done with a chunk's stage and dt
    __shared__ uint32_t tmem_base_sh;
    __shared__ __align__(8) uint64_t bar_drain;   // tensor core: every MMA this CTA issued is done
    __shared__ float dec_s[kDtBufs];              // per chunk: 2^cs_end, the state's decay over the chunk

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wq = warp & 3;      // TMEM lane quadrant of this warp
    const int g = warp >> 2;      // warpgroup: column quarter
    const int bh = blockIdx.x;
    const int b = bh / args.H, h = bh % args.H;
    const int L = args.L;
    const int nch = args.nchunks;
    float *cs_s = reinterpret_cast<float *>(sm + kOffVec);   // [kDtBufs][64], buffer c % kDtBufs
    float *dt_s = cs_s + kDtBufs * 64;                        // [kDtBufs][64]

    const float bias = args.bias ? args.bias[h] : 0.f;
    const float Ah = args.A[h] * kLog2e;   // exponents are taken base 2
    const float Dh = args.D ? args.D[h] : 0.f;

    if (tid == 0) {
        for (int k = 0; k < kStages; k++)
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&bar_tma[k])));
        abort_sh = 0;
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&bar_g)));
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&bar_ds)));
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&bar_mma2)));
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&bar_drain)));
        asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(&bar_mready)), "r"(kMath));
        asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(&bar_sready)), "r"(kMath));
        for (int k = 0; k < kDtBufs; k++) {
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 32;" ::"r"(smem_u32(&bar_dt_full[k])));
            asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(&bar_free[k])), "r"(kMath));
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base_sh)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    // zero S_in (hi and lo): the state entering chunk 0
    for (int k = tid; k < 2 * kSBytes / 16; k += kThreads)
        reinterpret_cast<uint4 *>(sm + kOffS)[k] = make_uint4(0, 0, 0, 0);
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tb = tmem_base_sh;
    const uint32_t tw = tb + ((uint32_t)(wq * 32) << 16);   // this warp's TMEM lanes
    volatile int *abort = &abort_sh;
    const long limit = args.wait_limit;
    // every lane of the calling warp waits; the result is the same for the
    // whole warp (so .sync.aligned instructions after it stay converged)
    auto wait = [&](uint64_t *bar, uint32_t parity) {
        return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort, limit));
    };

    auto issue_tma = [&](int c) {
        uint8_t *st = sm + (c % kStages) * kStageBytes;
        uint64_t *bar = &bar_tma[c % kStages];
        const uint32_t bytes = args.has_z ? kStageBytes : kStageBytes - kTileX;
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                     : "memory");
        const int t0 = c * kQ;
        tma_load_4d(st + kStageX, &mapX, 0, h, t0, b, bar);
        if (args.has_z)
            tma_load_4d(st + kStageZ, &mapZ, 0, h, t0, b, bar);
        tma_load_3d(st + kStageB, &mapB, 0, t0, b, bar);
        tma_load_3d(st + kStageB + kTileBC, &mapB, 64, t0, b, bar);
        tma_load_3d(st + kStageC, &mapC, 0, t0, b, bar);
        tma_load_3d(st + kStageC + kTileBC, &mapC, 64, t0, b, bar);
    };

    // raw delta of steps 2 lane, 2 lane + 1 of chunk c (dt warp)
    auto load_delta2 = [&](int c) {
        const int t = c * kQ + 2 * lane;
        float2 d = make_float2(0.f, 0.f);
        if (c < nch && t < L)
            d.x = __bfloat162float(args.delta[((size_t)b * L + t) * args.H + h]);
        if (c < nch && t + 1 < L)
            d.y = __bfloat162float(args.delta[((size_t)b * L + t + 1) * args.H + h]);
        return d;
    };
    // dt and the inclusive cumulative sum of dt A (base-2 units) of chunk c
    // into buffer c % kDtBufs; one warp, two steps per lane
    auto chunk_dt = [&](int c, float2 draw) {
        const int t = c * kQ + 2 * lane;
        float d0 = 0.f, d1 = 0.f;
        if (t < L) {
            d0 = draw.x + bias;
            if (args.softplus)
                d0 = softplus_f(d0);
        }
        if (t + 1 < L) {
            d1 = draw.y + bias;
            if (args.softplus)
                d1 = softplus_f(d1);
        }
        const float a0 = d0 * Ah, a1 = d1 * Ah;
        float incl = a0 + a1;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o)
                incl += v;
        }
        const float c0 = incl - a1, c1 = incl;
        float *cs = cs_s + (c % kDtBufs) * 64, *dtv = dt_s + (c % kDtBufs) * 64;
        *reinterpret_cast<float2 *>(cs + 2 * lane) = make_float2(c0, c1);
        *reinterpret_cast<float2 *>(dtv + 2 * lane) = make_float2(d0, d1);
        if (lane == 31)   // lane 31 holds cs_end: the chunk's decay, once for every thread
            dec_s[c % kDtBufs] = ex2f(c1);
    };

    // W(c) = exp(cs_end - cs_j) dt_j X[j, :] as bf16 hi + lo, rows j, X's
    // swizzled layout, into buffer c & 1: this thread's 16-byte piece (row
    // j = tid / 8, piece tid mod 8).  Split in two so the loads can be issued
    // early and the rest interleaved with other work.
    struct WIn {
        uint4 xv;
        float wj;
    };
    auto w_load = [&](int c) {
        const uint8_t *st = sm + (c % kStages) * kStageBytes;
        const float *cs = cs_s + (c % kDtBufs) * 64, *dtv = dt_s + (c % kDtBufs) * 64;
        const int j = tid >> 3, q = tid & 7;
        WIn w;
        w.wj = ex2f(cs[kQ - 1] - cs[j]) * dtv[j];
        w.xv = *reinterpret_cast<const uint4 *>(st + kStageX + sw_chunk(j, q));
        return w;
    };
    auto w_store = [&](int c, const WIn &w) {
        uint8_t *wb = sm + kOffW + (c & 1) * 2 * kTileX;
        const int j = tid >> 3, q = tid & 7;
        const uint32_t u[4] = {w.xv.x, w.xv.y, w.xv.z, w.xv.w};
        uint32_t o[4], ol[4];
        const float2 wj2 = make_float2(w.wj, w.wj);
#pragma unroll
        for (int k = 0; k < 4; k++) {
            const float2 f = __fmul2_rn(unpack_bf16(u[k]), wj2);
            split_bf16(f.x, f.y, o[k], ol[k]);
        }
        *reinterpret_cast<uint4 *>(wb + sw_chunk(j, q)) = make_uint4(o[0], o[1], o[2], o[3]);
        *reinterpret_cast<uint4 *>(wb + kTileX + sw_chunk(j, q)) = make_uint4(ol[0], ol[1], ol[2], ol[3]);
    };

    const uint32_t idG = idesc_bf16(64, 64, 0, 0);    // C (K-major) x B (K-major)
    const uint32_t idDS = idesc_bf16(128, 128, 1, 1); // B^T (MN-major) x [W_hi | W_lo] (MN-major)
    const uint32_t idYo = idesc_bf16(64, 128, 0, 1);  // C (K-major) x [S_hi | S_lo] (MN-major)
    const uint32_t idYd = idesc_bf16(64, 64, 0, 1);   // M (K-major) x X (MN-major)

    // G = C B^T (committed on its own, so the decay matrix can start), then
    // Yo = C [S_hi | S_lo] into buffer c & 1 (no commit: dS(c), issued after
    // it, covers it)
    auto issue_G_Yo = [&](int c) {
        const uint8_t *st = sm + (c % kStages) * kStageBytes;
        const uint32_t sC = smem_u32(st + kStageC), sB = smem_u32(st + kStageB);
        const uint32_t sS = smem_u32(sm + kOffS);
#pragma unroll
        for (int kk = 0; kk < 8; kk++) {   // K = n, 8 steps of 16; two 64-wide atoms
            const uint32_t off = (kk >> 2) * kTileBC + (kk & 3) * 32;
            umma(tb + kColG, desc_sw128(sC + off, 16, 1024), desc_sw128(sB + off, 16, 1024), idG, kk > 0);
        }
        umma_commit(&bar_g);
#pragma unroll
        for (int kk = 0; kk < 8; kk++) {   // K = n; S rows n (MN-major), hi and lo blocks 16 KB apart
            const uint32_t offc = (kk >> 2) * kTileBC + (kk & 3) * 32;
            umma(tb + kColYo + (uint32_t)(c & 1) * 128, desc_sw128(sC + offc, 16, 1024),
                 desc_sw128(sS + kk * 2048, kSBytes, 1024), idYo, kk > 0);
        }
    };
    // dS = B^T [W_hi | W_lo]
    auto issue_dS = [&](int c) {
        const uint8_t *st = sm + (c % kStages) * kStageBytes;
        const uint32_t sB = smem_u32(st + kStageB);
        const uint32_t sW = smem_u32(sm + kOffW + (c & 1) * 2 * kTileX);
#pragma unroll
        for (int kk = 0; kk < 4; kk++)     // K = j (rows); B^T: two MN atoms of 64 n, 8 KB apart;
            umma(tb + kColDS, desc_sw128(sB + kk * 2048, kTileBC, 1024),      // W hi and lo 8 KB apart
                 desc_sw128(sW + kk * 2048, kTileX, 1024), idDS, kk > 0);
        umma_commit(&bar_ds);
    };
    // Yd = [M_hi, then M_lo] X
    auto issue_Yd = [&](int c) {
        const uint8_t *st = sm + (c % kStages) * kStageBytes;
        const uint32_t sM = smem_u32(sm + kOffM), sX = smem_u32(st + kStageX);
#pragma unroll
        for (int part = 0; part < 2; part++)
#pragma unroll
            for (int kk = 0; kk < 4; kk++)
                umma(tb + kColYd, desc_sw128(sM + part * kTileX + kk * 32, 16, 1024),
                     desc_sw128(sX + kk * 2048, 8192, 1024), idYd, part + kk > 0);
        umma_commit(&bar_mma2);
    };

    // S: this thread's row n (= its TMEM lane), columns [16 g, 16 g + 16), fp32
    const int row_n = wq * 32 + lane;
    float S[16];
#pragma unroll
    for (int p = 0; p < 16; p++)
        S[p] = 0.f;

    const int row_i = 16 * wq + (lane & 15);   // M = 64 accumulator row of this thread
    const int c8 = 16 * g + 8 * (lane >> 4);   // first of this thread's 8 columns

    int issued = -1;   // dt warp: the last chunk whose TMA loads were issued
    if (warp == kDtWarp) {
        // ---- the dt warp: for every chunk k, once the math threads are done
        // with chunk k - kStages (its stage and dt buffer), issue chunk k's TMA
        // loads (lane 0) and compute dt and the cumulative sum of dt A.  A
        // stage is reissued only after the math threads released it, which
        // they do only after its previous loads landed, so each stage has at
        // most one load phase in flight.
        float2 draw = load_delta2(0);
        for (int k = 0; k < nch; k++) {
            const float2 dnext = load_delta2(k + 1);
            if (k >= kStages && !wait(&bar_free[k % kStages], ((k / kStages) - 1) & 1))
                break;
            if (__any_sync(0xffffffffu, *abort))
                break;
            if (lane == 0)
                issue_tma(k);
            issued = k;
            __syncwarp();
            chunk_dt(k, draw);
            if (k != args.withhold_chunk)
                mbar_arrive(&bar_dt_full[k % kDtBufs]);
            draw = dnext;
        }
        // teardown: wait for the loads still in flight (the last phase issued
        // on each stage)
        if (lane == 0)
            for (int k = max(0, issued - kStages + 1); k <= issued; k++)
                drain_wait(&bar_tma[k % kStages], (k / kStages) & 1);
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // ---- the MMA warp: lane 0 issues each product once its operands are
        // written and its accumulator read; the warp stays converged.
        // Per chunk c: Yd(c) once M(c) is written; G, Yo and dS of chunk
        // c + 1 once W(c + 1) and S_in(c + 1) are.
        auto lane0 = [&](auto fn) {
            if (lane == 0) {
                tc_fence_after();
                fn();
            }
            __syncwarp();
        };
        bool ok = wait(&bar_sready, 0);   // W(0) written (its TMA landed); S_in(0) is zero
        if (ok)
            lane0([&] {
                issue_G_Yo(0);
                issue_dS(0);
            });
        for (int c = 0; c < nch && ok; c++) {
            ok = wait(&bar_mready, c & 1);   // M(c) written, G(c) read
            if (!ok)
                break;
            lane0([&] { issue_Yd(c); });
            if (c + 1 < nch) {
                ok = wait(&bar_sready, (c + 1) & 1);   // W(c + 1), S_in(c + 1) written, dS(c) read
                if (!ok)
                    break;
                lane0([&] {
                    issue_G_Yo(c + 1);
                    issue_dS(c + 1);
                });
            }
        }
        // teardown: one more commit tracks every MMA issued above; wait for it
        lane0([&] { umma_commit(&bar_drain); });
        if (lane == 0)
            drain_wait(&bar_drain, 0);
        __syncwarp();
    } else {
        // ---- math threads.  Prologue: W(0).  A failed wait ends this warp's
        // work (no further signals); the other roles then give up too.
        bool ok = wait(&bar_dt_full[0], 0) && wait(&bar_tma[0], 0);
        if (ok) {
            w_store(0, w_load(0));
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(&bar_sready);
        }

        for (int c = 0; c < nch && ok; c++) {
            const uint8_t *st = sm + (c % kStages) * kStageBytes;
            const float *cs = cs_s + (c % kDtBufs) * 64, *dtv = dt_s + (c % kDtBufs) * 64;
            const int t0 = c * kQ;
            const uint32_t buf = (uint32_t)(c & 1) * 64;
            // ---- 1. masked decay matrix M (bf16 hi + lo, K-major rows i) from G; hand it over
            if (!wait(&bar_g, c & 1))
                break;
            tc_fence_after();
            float e_row;   // 2^cs_i, this thread's row decay for the outputs
            {
                uint32_t gr[8];
                tmem_ld_eighth_row(tw + kColG + 16 * g, gr);
                const float csi = cs[row_i];
                float e[8];
                e_row = ex2f(csi);
#pragma unroll
                for (int k = 0; k < 8; k++) {
                    const int j = c8 + k;
                    e[k] = (j <= row_i) ? ex2f(csi - cs[j]) * dtv[j] : 0.f;
                }
                tmem_wait_ld(gr);
                uint32_t o[4], ol[4];
#pragma unroll
                for (int k = 0; k < 8; k += 2) {
                    const float2 m2 = __fmul2_rn(make_float2(__uint_as_float(gr[k]), __uint_as_float(gr[k + 1])),
                                                 make_float2(e[k], e[k + 1]));
                    split_bf16(m2.x, m2.y, o[k >> 1], ol[k >> 1]);
                }
                const int q = c8 >> 3;
                *reinterpret_cast<uint4 *>(sm + kOffM + sw_chunk(row_i, q)) = make_uint4(o[0], o[1], o[2], o[3]);
                *reinterpret_cast<uint4 *>(sm + kOffM + kTileX + sw_chunk(row_i, q)) =
                    make_uint4(ol[0], ol[1], ol[2], ol[3]);
            }
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(&bar_mready);
            // ---- 2. next chunk's W (the tensor core meanwhile finishes Yo(c), dS(c), Yd(c))
            if (c + 1 < nch) {
                if (!wait(&bar_dt_full[(c + 1) % kDtBufs], ((c + 1) / kDtBufs) & 1) ||
                    !wait(&bar_tma[(c + 1) % kStages], ((c + 1) / kStages) & 1))
                    break;
                w_store(c + 1, w_load(c + 1));
            }
            // ---- 3. state update S = exp(cs_end) S + dS; bf16 hi + lo copy S_in(c + 1); hand
            // S_in(c + 1) and W(c + 1) over
            if (!wait(&bar_ds, c & 1))   // dS(c) done, and Yo(c) before it (S_in(c) is free)
                break;
            tc_fence_after();
            {
                const float decay = dec_s[c % kDtBufs];
                uint32_t ds[16], dl[16];
                tmem_ld_row16(tw + kColDS + 16 * g, ds);
                tmem_ld_row16(tw + kColDS + 64 + 16 * g, dl);
                tmem_wait_ld(ds);
                tmem_wait_ld(dl);
                // S = decay S + (dS_hi + dS_lo), two columns per packed instruction
                const float2 dec2 = make_float2(decay, decay);
#pragma unroll
                for (int k = 0; k < 16; k += 2) {
                    const float2 d2 = __fadd2_rn(make_float2(__uint_as_float(ds[k]), __uint_as_float(ds[k + 1])),
                                                 make_float2(__uint_as_float(dl[k]), __uint_as_float(dl[k + 1])));
                    const float2 s2 = __ffma2_rn(dec2, make_float2(S[k], S[k + 1]), d2);
                    S[k] = s2.x;
                    S[k + 1] = s2.y;
                }
                if (c + 1 < nch) {
                    uint8_t *sn = sm + kOffS;
#pragma unroll
                    for (int q2 = 0; q2 < 2; q2++) {
                        uint32_t hi[4], lo[4];
#pragma unroll
                        for (int k = 0; k < 4; k++)
                            split_bf16(S[8 * q2 + 2 * k], S[8 * q2 + 2 * k + 1], hi[k], lo[k]);
                        const int q = 2 * g + q2;
                        *reinterpret_cast<uint4 *>(sn + sw_chunk(row_n, q)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                        *reinterpret_cast<uint4 *>(sn + kSBytes + sw_chunk(row_n, q)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
                    }
                }
            }
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(&bar_sready);
            // ---- 4. outputs of chunk c: y = (Yd + exp(cs_i) Yo + D x) silu(z), row i, 8 columns
            {
                const int q = c8 >> 3;
                const uint4 xv = *reinterpret_cast<const uint4 *>(st + kStageX + sw_chunk(row_i, q));
                uint4 zv = make_uint4(0, 0, 0, 0);
                if (args.has_z)
                    zv = *reinterpret_cast<const uint4 *>(st + kStageZ + sw_chunk(row_i, q));
                const float ei = e_row;
                if (!wait(&bar_mma2, c & 1))   // Yd(c) done
                    break;
                tc_fence_after();
                uint32_t yo[8], yl[8], yd[8];
                tmem_ld_eighth_row(tw + kColYo + 2 * buf + 16 * g, yo);
                tmem_ld_eighth_row(tw + kColYo + 2 * buf + 64 + 16 * g, yl);
                tmem_ld_eighth_row(tw + kColYd + 16 * g, yd);
                tmem_wait_ld(yo);
                tmem_wait_ld(yl);
                tmem_wait_ld(yd);
                const int t = t0 + row_i;
                const uint32_t xu[4] = {xv.x, xv.y, xv.z, xv.w};
                const uint32_t zu[4] = {zv.x, zv.y, zv.z, zv.w};
                uint32_t o[4];
                // two columns per packed instruction:
                // y = (Yd + e_i (Yo_hi + Yo_lo) + D x) silu(z), silu(z) = h (1 + tanh h), h = z / 2
                const float2 ei2 = make_float2(ei, ei), dh2 = make_float2(Dh, Dh);
#pragma unroll
#pragma unroll
                for (int k = 0; k < 4; k++) {
                    const float2 yo2 = __fadd2_rn(make_float2(__uint_as_float(yo[2 * k]), __uint_as_float(yo[2 * k + 1])),
                                                  make_float2(__uint_as_float(yl[2 * k]), __uint_as_float(yl[2 * k + 1])));
                    float2 y2 = __ffma2_rn(ei2, yo2, make_float2(__uint_as_float(yd[2 * k]), __uint_as_float(yd[2 * k + 1])));
                    y2 = __ffma2_rn(dh2, unpack_bf16(xu[k]), y2);
                    if (args.has_z) {
                        const float2 h2 = __fmul2_rn(unpack_bf16(zu[k]), make_float2(0.5f, 0.5f));
                        float2 t2;
                        asm("tanh.approx.f32 %0, %1;" : "=f"(t2.x) : "f"(h2.x));
                        asm("tanh.approx.f32 %0, %1;" : "=f"(t2.y) : "f"(h2.y));
                        y2 = __fmul2_rn(y2, __ffma2_rn(h2, t2, h2));
                    }
                    o[k] = pack_bf16(y2.x, y2.y);
                }
                if (t < L)
                    *reinterpret_cast<uint4 *>(args.out + (((size_t)b * L + t) * args.H + h) * kP + c8) =
                        make_uint4(o[0], o[1], o[2], o[3]);
            }
            // ---- 5. hand chunk c's stage and dt buffer back to the dt warp
            mbar_arrive(&bar_free[c % kStages]);
        }
    }

    if (args.last_state && tid < kMath) {
        float *ls = args.last_state + (size_t)bh * kP * kN;
#pragma unroll
        for (int k = 0; k < 16; k++)
            ls[(size_t)(16 * g + k) * kN + row_n] = S[k];
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tb), "r"(kTmemCols));
}

// ------------------------------------------------------------ host side

using EncodeFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                              const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                              CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn encode_fn()
{
    static EncodeFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeFn>(p);
    }
    return fn;
}

// bf16 tensor map with 128-byte swizzle; dims / strides innermost first
bool make_map(CUtensorMap *m, const void *base, int rank, const cuuint64_t *dims, const cuuint64_t *strides_bytes,
              const cuuint32_t *box)
{
    EncodeFn fn = encode_fn();
    if (!fn)
        return false;
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void *>(base), dims, strides_bytes, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

size_t ssd_workspace_bytes(int64_t, int64_t, int64_t, int64_t, int64_t, int64_t) { return 0; }

namespace {
std::atomic<int> g_stall_chunk{-1};
std::atomic<unsigned> g_stall_limit{0};
}  // namespace

void ssd_stall_set(int withhold_chunk, unsigned wait_limit)
{
    g_stall_chunk.store(withhold_chunk < 0 ? -1 : withhold_chunk);
    g_stall_limit.store(wait_limit);
}

SSDStall ssd_stall_get() { return SSDStall{g_stall_chunk.load(), g_stall_limit.load()}; }

cudaError_t launch_ssd(const SSDArgs &a, cudaStream_t stream)
{
    if (a.P != kP || a.N != kN || a.Q != kQ)
        return cudaErrorNotSupported;
    CUtensorMap mX, mZ, mB, mC;
    // x, z: (Bsz, L, H, P) -> dims (P, H, L, Bsz), box (64, 1, 64, 1)
    const cuuint64_t dx[4] = {(cuuint64_t)a.P, (cuuint64_t)a.H, (cuuint64_t)a.L, (cuuint64_t)a.Bsz};
    const cuuint64_t sx[3] = {(cuuint64_t)a.P * 2, (cuuint64_t)a.H * a.P * 2, (cuuint64_t)a.L * a.H * a.P * 2};
    const cuuint32_t bx[4] = {64, 1, 64, 1};
    // B, C: (Bsz, L, N) -> dims (N, L, Bsz), box (64, 64, 1)
    const cuuint64_t db[3] = {(cuuint64_t)a.N, (cuuint64_t)a.L, (cuuint64_t)a.Bsz};
    const cuuint64_t sb[2] = {(cuuint64_t)a.N * 2, (cuuint64_t)a.L * a.N * 2};
    const cuuint32_t bb[3] = {64, 64, 1};
    if (!make_map(&mX, a.x, 4, dx, sx, bx) || !make_map(&mB, a.B, 3, db, sb, bb) ||
        !make_map(&mC, a.C, 3, db, sb, bb))
        return cudaErrorInvalidValue;
    if (a.z) {
        if (!make_map(&mZ, a.z, 4, dx, sx, bx))
            return cudaErrorInvalidValue;
    } else {
        mZ = mX;
    }
    SSDKernelArgs k;
    k.Bsz = a.Bsz;
    k.L = a.L;
    k.H = a.H;
    k.nchunks = (a.L + kQ - 1) / kQ;
    k.softplus = a.softplus;
    k.delta = static_cast<const __nv_bfloat16 *>(a.delta);
    k.bias = a.bias;
    k.A = a.A;
    k.D = a.D;
    k.out = static_cast<__nv_bfloat16 *>(a.out);
    k.last_state = a.last_state;
    k.has_z = a.z != nullptr;
    const SSDStall stall = ssd_stall_get();
    k.wait_limit = stall.wait_limit > 0 ? (long)stall.wait_limit : kWaitLimit;
    k.withhold_chunk = stall.withhold_chunk;
    cudaError_t e = cudaFuncSetAttribute(ssd_chunk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess)
        return e;
    ssd_chunk_kernel<<<a.Bsz * a.H, kThreads, kSmemBytes, stream>>>(mX, mZ, mB, mC, k);
    return cudaGetLastError();
}

cudaError_t read_and_clear_device_error(unsigned *value, cudaStream_t stream)
{
    cudaError_t e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess)
        return e;
    e = cudaMemcpyFromSymbol(value, g_device_error, sizeof(unsigned));
    if (e != cudaSuccess)
        return e;
    const unsigned zero = 0;
    return cudaMemcpyToSymbol(g_device_error, &zero, sizeof(unsigned));
}

}  // namespace ssm
