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
// One CTA of 128 threads owns one (b, h) and walks its chunks in order.  TMA
// brings each chunk's X, Z (64 x 64 bf16 tiles) and B, C (64 x 128) into a
// two-stage shared-memory ring with 128-byte swizzle, which is directly the
// layout the tensor core reads (C and B as K-major operands of C B^T, B as
// an MN-major operand of B^T W, X as an MN-major operand of M X).  Thread 0
// issues the TMA loads and the MMAs; completion is tracked by mbarriers with
// bounded waits that set the library's error word if they give up.
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
constexpr int kThreads = 128;
constexpr float kLog2e = 1.4426950408889634f;

// shared-memory plan (byte offsets from a 1024-aligned base)
constexpr int kTileX = kQ * kP * 2;            // 8 KB  (64 rows x 128 B)
constexpr int kTileBC = kQ * 64 * 2;           // 8 KB  (one 64-wide half of B or C)
constexpr int kStageX = 0;
constexpr int kStageZ = kTileX;
constexpr int kStageB = 2 * kTileX;            // two halves (n 0..63, 64..127)
constexpr int kStageC = 2 * kTileX + 2 * kTileBC;
constexpr int kStageBytes = 2 * kTileX + 4 * kTileBC;   // 48 KB
constexpr int kOffW = 2 * kStageBytes;                  // W hi, lo: 2 x 8 KB, rows j, MN-major
constexpr int kOffM = kOffW + 2 * kTileX;               // M hi, lo: 2 x 8 KB, rows i, K-major
constexpr int kOffS = kOffM + 2 * kTileX;               // S_in [buffer][hi, lo]: 4 x 16 KB, rows n, MN-major
constexpr int kSBytes = kN * 128;
constexpr int kOffVec = kOffS + 4 * kSBytes;            // cs[64], dt[64], warp sums
constexpr int kSmemBytes = kOffVec + 3 * 64 * 4 + 1024; // + alignment slack

// TMEM columns
constexpr uint32_t kColG = 0, kColYo = 64, kColYd = 128, kColDS = 192, kTmemCols = 256;

constexpr long kWaitLimit = 1l << 26;

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

// Bounded wait on an mbarrier phase; on giving up, flag the error and return
// false (the caller carries on so that every thread still meets every barrier).
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity)
{
    const uint32_t a = smem_u32(bar);
    for (long it = 0; it < kWaitLimit; it++) {
        uint32_t ok;
        asm volatile("{.reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p;}"
                     : "=r"(ok)
                     : "r"(a), "r"(parity)
                     : "memory");
        if (ok)
            return true;
    }
    atomicExch(&g_device_error, 1u);
    return false;
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

// 32 columns of one M = 64 accumulator row: threads t < 16 of warp w get row
// 16 w + t, columns [col, col + 32); threads t >= 16 the same row, columns
// [col + 32, col + 64).
__device__ __forceinline__ void tmem_ld_half_row(uint32_t taddr, float (&v)[32])
{
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.16x32bx2.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32], 32;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int k = 0; k < 32; k++)
        v[k] = __uint_as_float(r[k]);
}

// 32 consecutive columns of this thread's lane (an M = 128 accumulator row)
__device__ __forceinline__ void tmem_ld_row32(uint32_t taddr, float *v)
{
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int k = 0; k < 32; k++)
        v[k] = __uint_as_float(r[k]);
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

// silu(z) = z sigmoid(z) = z (1 + tanh(z / 2)) / 2 (tanh.approx: rel. error 2^-11,
// far below the bf16 output rounding of this path)
__device__ __forceinline__ float silu_f(float z)
{
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * z));
    return 0.5f * z * (1.f + t);
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// v = hi + lo with hi = bf16(v) and lo = bf16(v - hi), for two values
__device__ __forceinline__ void split_bf16(float a, float b, uint32_t &hi, uint32_t &lo)
{
    hi = pack_bf16(a, b);
    const float ha = __uint_as_float(hi << 16), hb = __uint_as_float(hi & 0xffff0000u);
    lo = pack_bf16(a - ha, b - hb);
}

__device__ __forceinline__ float2 unpack_bf16(uint32_t u)
{
    return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
}

struct SSDKernelArgs {
    int Bsz, L, H, nchunks;
    int softplus;
    const __nv_bfloat16 *delta;
    const float *bias, *A, *D;
    __nv_bfloat16 *out;
    float *last_state;
    int has_z;
};

__global__ void __launch_bounds__(kThreads, 1)
    ssd_chunk_kernel(const __grid_constant__ CUtensorMap mapX, const __grid_constant__ CUtensorMap mapZ,
                     const __grid_constant__ CUtensorMap mapB, const __grid_constant__ CUtensorMap mapC,
                     const SSDKernelArgs args)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ __align__(8) uint64_t bar_tma[2];
    __shared__ __align__(8) uint64_t bar_mma1, bar_mma2;
    __shared__ uint32_t tmem_base_sh;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.x;
    const int b = bh / args.H, h = bh % args.H;
    const int L = args.L;
    float *cs_s = reinterpret_cast<float *>(sm + kOffVec);
    float *dt_s = cs_s + 64;
    float *wsum = dt_s + 64;

    const float bias = args.bias ? args.bias[h] : 0.f;
    const float Ah = args.A[h] * kLog2e;   // exponents are taken base 2
    const float Dh = args.D ? args.D[h] : 0.f;

    if (tid == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&bar_tma[0])));
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&bar_tma[1])));
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&bar_mma1)));
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&bar_mma2)));
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base_sh)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    // zero S_in buffer 0 (the state entering chunk 0)
    for (int k = tid; k < 2 * kSBytes / 16; k += kThreads)
        reinterpret_cast<uint4 *>(sm + kOffS)[k] = make_uint4(0, 0, 0, 0);
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tb = tmem_base_sh;
    const uint32_t tw = tb + ((uint32_t)(warp * 32) << 16);   // this warp's TMEM lanes

    auto issue_tma = [&](int c) {
        uint8_t *st = sm + (c & 1) * kStageBytes;
        uint64_t *bar = &bar_tma[c & 1];
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
    if (tid == 0) {
        issue_tma(0);
        if (args.nchunks > 1)
            issue_tma(1);
    }

    // delta for the first chunk (threads 0..63 hold one step each)
    auto load_delta = [&](int c) {
        const int t = c * kQ + tid;
        return (tid < kQ && t < L) ? __bfloat162float(args.delta[((size_t)b * L + t) * args.H + h]) : 0.f;
    };
    float dnext = load_delta(0);

    // S: this thread's row n = tid, 64 columns p, fp32
    float S[kP];
#pragma unroll
    for (int p = 0; p < kP; p++)
        S[p] = 0.f;

    const uint32_t idG = idesc_bf16(64, 64, 0, 0);    // C (K-major) x B (K-major)
    const uint32_t idDS = idesc_bf16(128, 64, 1, 1);  // B^T (MN-major) x W (MN-major)
    const uint32_t idYo = idesc_bf16(64, 64, 0, 1);   // C (K-major) x S_in (MN-major)
    const uint32_t idYd = idesc_bf16(64, 64, 0, 1);   // M (K-major) x X (MN-major)

    const int row_i = 16 * warp + (lane & 15);   // M = 64 accumulator row of this thread
    const int hh = lane >> 4;                    // which 32-column half

    for (int c = 0; c < args.nchunks; c++) {
        uint8_t *st = sm + (c & 1) * kStageBytes;
        const int t0 = c * kQ;
        // ---- dt and the inclusive cumulative sum of dt A inside the chunk
        float dt = 0.f;
        if (tid < kQ && t0 + tid < L) {
            dt = dnext + bias;
            if (args.softplus)
                dt = softplus_f(dt);
        }
        if (c + 1 < args.nchunks)
            dnext = load_delta(c + 1);
        float a = dt * Ah;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float v = __shfl_up_sync(0xffffffffu, a, o);
            if (lane >= o)
                a += v;
        }
        if (lane == 31 && warp < 2)
            wsum[warp] = a;
        __syncthreads();
        if (warp == 1)
            a += wsum[0];
        if (tid < kQ) {
            cs_s[tid] = a;
            dt_s[tid] = dt;
        }
        __syncthreads();
        const float cs_end = cs_s[kQ - 1];

        // ---- wait for this chunk's tiles
        const bool ok_tma = mbar_wait(&bar_tma[c & 1], (c >> 1) & 1);
        (void)ok_tma;

        // ---- W = exp(cs_end - cs_j) dt_j X[j, :], rows j, same swizzled layout as X
        {
            const int j = tid >> 1, half = tid & 1;
            const float wj = ex2f(cs_end - cs_s[j]) * dt_s[j];
#pragma unroll
            for (int q4 = 0; q4 < 4; q4++) {
                const int q = 4 * half + q4;
                const uint4 xv = *reinterpret_cast<const uint4 *>(st + kStageX + sw_chunk(j, q));
                const uint32_t u[4] = {xv.x, xv.y, xv.z, xv.w};
                uint32_t o[4], ol[4];
#pragma unroll
                for (int k = 0; k < 4; k++) {
                    const float2 f = unpack_bf16(u[k]);
                    split_bf16(f.x * wj, f.y * wj, o[k], ol[k]);
                }
                *reinterpret_cast<uint4 *>(sm + kOffW + sw_chunk(j, q)) = make_uint4(o[0], o[1], o[2], o[3]);
                *reinterpret_cast<uint4 *>(sm + kOffW + kTileX + sw_chunk(j, q)) = make_uint4(ol[0], ol[1], ol[2], ol[3]);
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();

        // ---- first MMA group: G = C B^T, Yo = C S_in, dS = B^T W
        if (tid == 0) {
            tc_fence_after();
            const uint32_t sC = smem_u32(st + kStageC), sB = smem_u32(st + kStageB);
            const uint32_t sS = smem_u32(sm + kOffS + (c & 1) * 2 * kSBytes), sW = smem_u32(sm + kOffW);
#pragma unroll
            for (int kk = 0; kk < 8; kk++) {   // K = n, 8 steps of 16; two 64-wide atoms
                const uint32_t off = (kk >> 2) * kTileBC + (kk & 3) * 32;
                umma(tb + kColG, desc_sw128(sC + off, 16, 1024), desc_sw128(sB + off, 16, 1024), idG, kk > 0);
            }
#pragma unroll
            for (int part = 0; part < 2; part++)   // S_in hi, then lo
#pragma unroll
                for (int kk = 0; kk < 8; kk++) {   // K = n; S_in rows n (MN-major, 8 rows per 1 KB)
                    const uint32_t offc = (kk >> 2) * kTileBC + (kk & 3) * 32;
                    umma(tb + kColYo, desc_sw128(sC + offc, 16, 1024),
                         desc_sw128(sS + part * kSBytes + kk * 2048, 8192, 1024), idYo, part + kk > 0);
                }
#pragma unroll
            for (int part = 0; part < 2; part++)   // W hi, then lo
#pragma unroll
                for (int kk = 0; kk < 4; kk++)     // K = j (rows); B^T: two MN atoms of 64 n, 8 KB apart
                    umma(tb + kColDS, desc_sw128(sB + kk * 2048, kTileBC, 1024),
                         desc_sw128(sW + part * kTileX + kk * 2048, 8192, 1024), idDS, part + kk > 0);
            umma_commit(&bar_mma1);
        }
        __syncwarp();
        mbar_wait(&bar_mma1, c & 1);
        tc_fence_after();

        // ---- masked decay matrix M (bf16, K-major rows i) from G
        {
            float g[32];
            tmem_ld_half_row(tw + kColG, g);
            const float csi = cs_s[row_i];
            uint32_t o[16], ol[16];
#pragma unroll
            for (int k = 0; k < 32; k += 2) {
                const int j0 = 32 * hh + k;
                const float m0 = (j0 <= row_i) ? g[k] * ex2f(csi - cs_s[j0]) * dt_s[j0] : 0.f;
                const float m1 = (j0 + 1 <= row_i) ? g[k + 1] * ex2f(csi - cs_s[j0 + 1]) * dt_s[j0 + 1] : 0.f;
                split_bf16(m0, m1, o[k >> 1], ol[k >> 1]);
            }
#pragma unroll
            for (int q4 = 0; q4 < 4; q4++) {
                *reinterpret_cast<uint4 *>(sm + kOffM + sw_chunk(row_i, 4 * hh + q4)) =
                    make_uint4(o[4 * q4], o[4 * q4 + 1], o[4 * q4 + 2], o[4 * q4 + 3]);
                *reinterpret_cast<uint4 *>(sm + kOffM + kTileX + sw_chunk(row_i, 4 * hh + q4)) =
                    make_uint4(ol[4 * q4], ol[4 * q4 + 1], ol[4 * q4 + 2], ol[4 * q4 + 3]);
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            const uint32_t sM = smem_u32(sm + kOffM), sX = smem_u32(st + kStageX);
#pragma unroll
            for (int part = 0; part < 2; part++)   // M hi, then lo
#pragma unroll
                for (int kk = 0; kk < 4; kk++)
                    umma(tb + kColYd, desc_sw128(sM + part * kTileX + kk * 32, 16, 1024),
                         desc_sw128(sX + kk * 2048, 8192, 1024), idYd, part + kk > 0);
            umma_commit(&bar_mma2);
        }
        __syncwarp();

        // ---- state update S = exp(cs_end) S + dS, row n = tid; bf16 copy for the next chunk
        {
            const float decay = ex2f(cs_end);
            float ds[32];
#pragma unroll
            for (int half = 0; half < 2; half++) {
                tmem_ld_row32(tw + kColDS + 32 * half, ds);
#pragma unroll
                for (int k = 0; k < 32; k++)
                    S[32 * half + k] = fmaf(decay, S[32 * half + k], ds[k]);
            }
            if (c + 1 < args.nchunks) {
                uint8_t *sn = sm + kOffS + ((c + 1) & 1) * 2 * kSBytes;
#pragma unroll
                for (int q = 0; q < 8; q++) {
                    uint32_t hi[4], lo[4];
#pragma unroll
                    for (int k = 0; k < 4; k++)
                        split_bf16(S[8 * q + 2 * k], S[8 * q + 2 * k + 1], hi[k], lo[k]);
                    *reinterpret_cast<uint4 *>(sn + sw_chunk(tid, q)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                    *reinterpret_cast<uint4 *>(sn + kSBytes + sw_chunk(tid, q)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
                }
            }
        }

        // ---- outputs: y = (Yd + exp(cs_i) Yo + D x) silu(z), row i, 32 columns
        {
            float yo[32], yd[32];
            tmem_ld_half_row(tw + kColYo, yo);
            mbar_wait(&bar_mma2, c & 1);
            tc_fence_after();
            tmem_ld_half_row(tw + kColYd, yd);
            const float ei = ex2f(cs_s[row_i]);
            const int t = t0 + row_i;
            uint32_t o[16];
#pragma unroll
            for (int q4 = 0; q4 < 4; q4++) {
                const int q = 4 * hh + q4;
                const uint4 xv = *reinterpret_cast<const uint4 *>(st + kStageX + sw_chunk(row_i, q));
                uint4 zv = make_uint4(0, 0, 0, 0);
                if (args.has_z)
                    zv = *reinterpret_cast<const uint4 *>(st + kStageZ + sw_chunk(row_i, q));
                const uint32_t xu[4] = {xv.x, xv.y, xv.z, xv.w};
                const uint32_t zu[4] = {zv.x, zv.y, zv.z, zv.w};
#pragma unroll
                for (int k = 0; k < 4; k++) {
                    const int col = 8 * q4 + 2 * k;   // column within this half
                    const float2 xf = unpack_bf16(xu[k]);
                    float y0 = fmaf(ei, yo[col], yd[col]) + Dh * xf.x;
                    float y1 = fmaf(ei, yo[col + 1], yd[col + 1]) + Dh * xf.y;
                    if (args.has_z) {
                        const float2 zf = unpack_bf16(zu[k]);
                        y0 *= silu_f(zf.x);
                        y1 *= silu_f(zf.y);
                    }
                    o[4 * q4 + k] = pack_bf16(y0, y1);
                }
            }
            if (t < L) {
                uint4 *dst = reinterpret_cast<uint4 *>(args.out + (((size_t)b * L + t) * args.H + h) * kP + 32 * hh);
#pragma unroll
                for (int q4 = 0; q4 < 4; q4++)
                    dst[q4] = make_uint4(o[4 * q4], o[4 * q4 + 1], o[4 * q4 + 2], o[4 * q4 + 3]);
            }
        }
        // ---- release this stage; prefetch chunk c + 2 into it
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0 && c + 2 < args.nchunks)
            issue_tma(c + 2);
    }

    if (args.last_state) {
        float *ls = args.last_state + (size_t)bh * kP * kN;
#pragma unroll
        for (int p = 0; p < kP; p++)
            ls[(size_t)p * kN + tid] = S[p];
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
