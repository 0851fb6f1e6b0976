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
// Two kernels, one thread per (b, d), a CTA holding 64 channels of one
// batch row.  s6_bwd_ckpt_kernel runs the forward recurrence once and stores
// h entering every chunk of kKc steps (padded to the template state count,
// so each channel's checkpoint is whole 16-byte vectors); its inputs arrive
// kStage steps at a time, the next stage's in flight during the current one.
// s6_bwd_kernel walks the chunks backwards: it recomputes the chunk's states
// into shared memory from the checkpoint, then sweeps the chunk backwards
// with lam in registers; the next chunk's inputs and checkpoint are copied
// (cp.async) while the current one is computed.  dB and dC are summed over a
// warp's 32 channels with a butterfly of shuffles, then added with one
// atomic per (warp, t, n).  All gradients are float32.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <string.h>

#include "internal.h"
#include "s6_math.cuh"

namespace ssm {
namespace {

constexpr int kKc = 4;         // steps per checkpointed chunk (4: the backward kernel's shared
                               // memory then allows 6 CTAs per SM, one wave for Vim-Small)
constexpr int kCta = 64;       // channels (threads) per CTA
constexpr int kStage = 16;     // steps per input stage of the checkpoint pass
constexpr int kBwdCtasPerSm = 6;   // backward kernel residency: 768 CTAs of Vim-Small in one wave
// steps of the backward sweep unrolled: all kKc of them (static shared-
// memory offsets; 1.5% faster than the rolled loop on Vim-Small)
#ifndef SSM_BWD_UNROLL
#define SSM_BWD_UNROLL 4
#endif
constexpr int kSweepUnroll = SSM_BWD_UNROLL;

template <typename T> __device__ __forceinline__ float ldv(const T *p, size_t i);
template <> __device__ __forceinline__ float ldv<float>(const float *p, size_t i) { return __ldg(p + i); }
template <> __device__ __forceinline__ float ldv<__nv_bfloat16>(const __nv_bfloat16 *p, size_t i)
{
    return __bfloat162float(__ldg(p + i));
}

__device__ __forceinline__ float dt_of(float v, int softplus) { return softplus ? softplus_f(v) : v; }
__device__ __forceinline__ float sigmoid_f(float v) { return 1.f / (1.f + ex2_mufu(-v * kLog2e)); }

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

__device__ __forceinline__ float4 lds4(const float *p) { return *reinterpret_cast<const float4 *>(p); }
__device__ __forceinline__ float2 lo2(const float4 &v) { return make_float2(v.x, v.y); }
__device__ __forceinline__ float2 hi2(const float4 &v) { return make_float2(v.z, v.w); }
__device__ __forceinline__ float2 ex2_pair(float2 v) { return make_float2(ex2_mufu(v.x), ex2_mufu(v.y)); }

// One step of the recurrence for NS states held as NS / 2 pairs (packed
// f32x2 instructions, each lane rounded as the scalar multiply / FMA):
// h = 2^(dt A log2 e) h + (dt x) B, with Brow 16-byte aligned in shared memory.
template <int NS>
__device__ __forceinline__ void recur_pairs(float2 (&h)[NS / 2], const float2 (&Al)[NS / 2], float dt, float dtx,
                                            const float *Brow)
{
    const float2 dt2 = make_float2(dt, dt), dtx2 = make_float2(dtx, dtx);
#pragma unroll
    for (int q = 0; q < NS / 4; q++) {
        const float4 B4 = lds4(Brow + 4 * q);
#pragma unroll
        for (int e = 0; e < 2; e++) {
            const int p = 2 * q + e;
            const float2 an = ex2_pair(__fmul2_rn(dt2, Al[p]));
            h[p] = __ffma2_rn(an, h[p], __fmul2_rn(dtx2, e == 0 ? lo2(B4) : hi2(B4)));
        }
    }
}

// The forward inputs of kStage steps from scan index i0: this thread's
// delta and x, and its kPer share of the steps' B rows (element e = thread +
// j kCta of the (step, state) tile).  Zero past L, N or D.
template <typename T, int NS, int kPer>
__device__ __forceinline__ void load_stage(const BwdArgs &a, int b, int dd, bool active, int i0,
                                           float (&v)[kStage], float (&xv)[kStage], float (&bq)[kPer])
{
    const T *x = static_cast<const T *>(a.x), *dl = static_cast<const T *>(a.delta);
    const T *Bm = static_cast<const T *>(a.B);
#pragma unroll
    for (int k = 0; k < kStage; k++) {
        const int i = i0 + k;
        v[k] = 0.f;
        xv[k] = 0.f;
        if (active && i < a.L) {
            const int t = a.reverse ? a.L - 1 - i : i;
            const size_t io = ((size_t)b * a.L + t) * a.D + dd;
            v[k] = ldv(dl, io);
            xv[k] = ldv(x, io);
        }
    }
#pragma unroll
    for (int j = 0; j < kPer; j++) {
        const int e = threadIdx.x + j * kCta, k = e / NS, n = e % NS, i = i0 + k;
        bq[j] = 0.f;
        if (i < a.L && n < a.N) {
            const int t = a.reverse ? a.L - 1 - i : i;
            bq[j] = ldv(Bm, ((size_t)b * a.L + t) * a.N + n);
        }
    }
}

// Forward recurrence of one (b, d) per thread, storing h entering every
// kKc-step chunk (NS floats per channel, the padding states stay zero).  The
// inputs arrive kStage steps at a time, the next stage's loads in flight
// while the current stage is computed; the stage's B rows sit in a
// double-buffered shared tile, so one barrier per stage suffices.
template <typename T, int NS>
__global__ void __launch_bounds__(kCta) s6_bwd_ckpt_kernel(const BwdArgs a)
{
    constexpr int kPer = kStage * NS / kCta;
    static_assert(kPer * kCta == kStage * NS, "stage tile must split evenly over the CTA");
    static_assert(kStage % kKc == 0, "a stage holds whole chunks");
    __shared__ __align__(16) float bs[2][kStage][NS];
    const int d = blockIdx.x * kCta + threadIdx.x;
    const int b = blockIdx.y;
    const bool active = d < a.D;
    const int dd = active ? d : 0;
    const int N = a.N, L = a.L, nch = (L + kKc - 1) / kKc, nst = (L + kStage - 1) / kStage;
    float2 Al[NS / 2], h[NS / 2];
#pragma unroll
    for (int p = 0; p < NS / 2; p++) {
        const int n = 2 * p;
        Al[p] = make_float2((active && n < N) ? a.A[(size_t)dd * N + n] * kLog2e : 0.f,
                            (active && n + 1 < N) ? a.A[(size_t)dd * N + n + 1] * kLog2e : 0.f);
        h[p] = make_float2(0.f, 0.f);
    }
    const float bias = (active && a.bias) ? a.bias[dd] : 0.f;
    float v[kStage], xv[kStage], bq[kPer];
    load_stage<T, NS, kPer>(a, b, dd, active, 0, v, xv, bq);
#pragma unroll
    for (int j = 0; j < kPer; j++) {
        const int e = threadIdx.x + j * kCta;
        bs[0][e / NS][e % NS] = bq[j];
    }
    __syncthreads();
    for (int s = 0; s < nst; s++) {
        const int i0 = s * kStage;
        const bool more = s + 1 < nst;
        float vn[kStage], xn[kStage], bn[kPer];
        if (more)
            load_stage<T, NS, kPer>(a, b, dd, active, i0 + kStage, vn, xn, bn);
        const float(*bc)[NS] = bs[s & 1];
#pragma unroll
        for (int k = 0; k < kStage; k++) {
            const int i = i0 + k;
            if (k % kKc == 0 && active && i < L) {
                float4 *ck = reinterpret_cast<float4 *>(a.ckpt + (((size_t)b * nch + i / kKc) * a.D + dd) * NS);
#pragma unroll
                for (int q = 0; q < NS / 4; q++)
                    ck[q] = make_float4(h[2 * q].x, h[2 * q].y, h[2 * q + 1].x, h[2 * q + 1].y);
            }
            const float dt = i < L ? dt_of(v[k] + bias, a.softplus) : 0.f;
            recur_pairs<NS>(h, Al, dt, dt * xv[k], bc[k]);
        }
        if (more) {
#pragma unroll
            for (int j = 0; j < kPer; j++) {
                const int e = threadIdx.x + j * kCta;
                bs[(s + 1) & 1][e / NS][e % NS] = bn[j];
            }
#pragma unroll
            for (int k = 0; k < kStage; k++) {
                v[k] = vn[k];
                xv[k] = xn[k];
            }
        }
        __syncthreads();
    }
}

// 16-byte cp.async into shared memory; src_bytes 0 writes zeros (src must
// still be a valid address, it is not read).
__device__ __forceinline__ void cp_async16z(void *smem, const void *gmem, bool valid)
{
    const unsigned sa = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    const int nbytes = valid ? 16 : 0;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(sa), "l"(gmem), "r"(nbytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

template <typename T> __device__ __forceinline__ float tof(T v);
template <> __device__ __forceinline__ float tof<float>(float v) { return v; }
template <> __device__ __forceinline__ float tof<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

// Shared memory of the backward kernel.
template <typename T, int NS>
struct BwdSmem {
    __align__(16) float hs[kKc][kCta][NS];     // the chunk's recomputed states, a row per thread
                                               // (16-byte slots swizzled by hs_slot)
    __align__(16) T raw[2][kKc][4][kCta];      // delta, x, dout, z rows of two chunks
    __align__(16) float ck[2][kCta][NS + 4];   // checkpoints of two chunks (padded rows: no bank conflicts)
    __align__(16) float bc[2][kKc][2 * NS];    // B and C rows of two chunks
    float dt[kKc][kCta];                       // this chunk's dt, a column per thread
};

// Start the copies of chunk c's delta, x, dout, z rows (16-byte pieces of
// the CTA's channel range; pieces past L or D, and a missing z, are zero
// filled) and of this thread's checkpoint into buffer `buf`; one commit group.
template <typename T, int NS>
__device__ __forceinline__ void issue_chunk(const BwdArgs &a, BwdSmem<T, NS> &sm, int buf, int b, int d0,
                                            int c, int nch)
{
    constexpr int kPieceCh = 16 / (int)sizeof(T);
    constexpr int kPiecesRow = kCta / kPieceCh;
    constexpr int kPieces = kKc * 4 * kPiecesRow;
    static_assert(kPieces % kCta == 0, "pieces split evenly over the CTA");
    const int i0 = c * kKc;
#pragma unroll
    for (int j = 0; j < kPieces / kCta; j++) {
        const int p = threadIdx.x + j * kCta, row = p / kPiecesRow, q = p % kPiecesRow;
        const int k = row >> 2, arr = row & 3, i = i0 + k, ch = d0 + q * kPieceCh;
        const void *bv = arr == 0 ? a.delta : arr == 1 ? a.x : arr == 2 ? a.dout : a.z;
        const T *base = static_cast<const T *>(bv);
        const bool valid = i < a.L && ch < a.D && base != nullptr;
        const T *g = static_cast<const T *>(a.x);
        if (valid)
            g = base + ((size_t)b * a.L + (a.reverse ? a.L - 1 - i : i)) * a.D + ch;
        cp_async16z(&sm.raw[buf][k][arr][q * kPieceCh], g, valid);
    }
    const int d = d0 + threadIdx.x;
    const bool act = d < a.D;
    const float *ck = a.ckpt + (((size_t)b * nch + c) * a.D + (act ? d : 0)) * NS;
#pragma unroll
    for (int q = 0; q < NS / 4; q++)
        cp_async16z(&sm.ck[buf][threadIdx.x][4 * q], ck + 4 * q, act);
    cp_async_commit();
}

// B and C rows of chunk c into registers (kBq per thread; element e =
// thread + j kCta of the (step, B | C, state) tile), zero past L or N.
template <typename T, int NS, int kBq>
__device__ __forceinline__ void load_bc(const BwdArgs &a, int b, int c, float (&bq)[kBq])
{
    const T *Bm = static_cast<const T *>(a.B), *Cm = static_cast<const T *>(a.C);
#pragma unroll
    for (int j = 0; j < kBq; j++) {
        const int e = threadIdx.x + j * kCta, k = e / (2 * NS), r = e % (2 * NS), n = r % NS;
        const int i = c * kKc + k;
        bq[j] = 0.f;
        if (e < kKc * 2 * NS && i < a.L && n < a.N) {
            const int t = a.reverse ? a.L - 1 - i : i;
            bq[j] = ldv(r < NS ? Bm : Cm, ((size_t)b * a.L + t) * a.N + n);
        }
    }
}

// Walks the chunks backwards.  Chunk c's inputs were fetched during chunk
// c + 1 (cp.async for the rows and the checkpoint, registers for B and C),
// so each chunk waits only for copies that had a whole chunk to land; one
// barrier per chunk.  hs and dt are per-thread columns (no barrier between
// the recompute and the sweep).
// Slot of states [4q, 4q + 4) in a thread's hs row: XOR-swizzled so that
// the 16-byte accesses of any 8 consecutive threads hit distinct banks.
template <int NS>
__device__ __forceinline__ int hs_slot(int tid, int q)
{
    constexpr int kQ = NS / 4;
    return q ^ ((tid / (8 / kQ)) % kQ);
}


// Walks the chunks backwards.  Chunk c's inputs were fetched during chunk
// c + 1 (cp.async for the rows and the checkpoint, registers for B and C),
// so each chunk waits only for copies that had a whole chunk to land; one
// barrier per chunk.  hs and dt are per-thread (no barrier between the
// recompute and the sweep).
//
// In the sweep h_{i-1} is the previous row of hs (the checkpoint for the
// chunk's first step), and
//   ddt_i = x_i sum_n lam_i[n] B_i[n] + ln 2 sum_n (lam_i[n] a_i[n] h_{i-1}[n]) A[n] log2(e)
// reuses the dx sum and the exponent's scaled A.
template <typename T, int NS>
__global__ void __launch_bounds__(kCta, kBwdCtasPerSm) s6_bwd_kernel(const BwdArgs a)
{
    constexpr int kBq = (kKc * 2 * NS + kCta - 1) / kCta;
    constexpr float kLn2 = 0.693147180559945309f;
    __shared__ BwdSmem<T, NS> sm;
    const int tid = threadIdx.x, lane = tid & 31;
    const int d0 = blockIdx.x * kCta, d = d0 + tid;
    const int b = blockIdx.y;
    const bool active = d < a.D;
    const int dd = active ? d : 0;
    const int N = a.N, L = a.L, nch = (L + kKc - 1) / kKc;
    const bool gate = a.z != nullptr;
    // state pairs (2p, 2p + 1) for the packed f32x2 instructions
    float2 Al[NS / 2], lam[NS / 2], gA[NS / 2];
#pragma unroll
    for (int p = 0; p < NS / 2; p++) {
        const int n = 2 * p;
        Al[p] = make_float2((active && n < N) ? a.A[(size_t)dd * N + n] * kLog2e : 0.f,
                            (active && n + 1 < N) ? a.A[(size_t)dd * N + n + 1] * kLog2e : 0.f);
        lam[p] = make_float2(0.f, 0.f);   // a_{i+1} lam_{i+1}, carried backwards
        gA[p] = make_float2(0.f, 0.f);    // dA: sum over steps of lam_i a_i h_{i-1} dt_i
    }
    const float bias = (active && a.bias) ? a.bias[dd] : 0.f;
    const float Dv = (active && a.Dskip) ? a.Dskip[dd] : 0.f;
    float gD = 0.f, gbias = 0.f;

    float bq[kBq];
    issue_chunk<T, NS>(a, sm, (nch - 1) & 1, b, d0, nch - 1, nch);
    load_bc<T, NS, kBq>(a, b, nch - 1, bq);
    // accumulate: the dx and ddelta already there are loaded one step ahead
    // of their use (the sweep's order: chunks and steps descending)
    const bool acc = a.accumulate && active;
    auto io_of = [&](int i) { return ((size_t)b * L + (a.reverse ? L - 1 - i : i)) * a.D + dd; };
    float nx_dx = 0.f, nx_dd = 0.f;
    if (acc) {
        nx_dx = a.dx[io_of(L - 1)];
        nx_dd = a.ddelta[io_of(L - 1)];
    }
    for (int c = nch - 1; c >= 0; c--) {
        const int buf = c & 1, i0 = c * kKc, kn = min(kKc, L - i0);
        cp_async_wait_all();
#pragma unroll
        for (int j = 0; j < kBq; j++) {
            const int e = tid + j * kCta;
            if (e < kKc * 2 * NS)
                sm.bc[buf][e / (2 * NS)][e % (2 * NS)] = bq[j];
        }
        __syncthreads();   // chunk c's copies visible; every thread is past chunk c + 1
        if (c > 0) {
            issue_chunk<T, NS>(a, sm, buf ^ 1, b, d0, c - 1, nch);
            load_bc<T, NS, kBq>(a, b, c - 1, bq);
        }
        const float(*bc)[2 * NS] = sm.bc[buf];
        const T(*raw)[4][kCta] = sm.raw[buf];
        // recompute the chunk's states from the checkpoint
        {
            float2 h[NS / 2];
#pragma unroll
            for (int q = 0; q < NS / 4; q++) {
                const float4 c4 = lds4(&sm.ck[buf][tid][4 * q]);
                h[2 * q] = lo2(c4);
                h[2 * q + 1] = hi2(c4);
            }
#pragma unroll
            for (int k = 0; k < kKc; k++) {
                const float dt = (k < kn) ? dt_of(tof(raw[k][0][tid]) + bias, a.softplus) : 0.f;
                sm.dt[k][tid] = dt;
                recur_pairs<NS>(h, Al, dt, dt * tof(raw[k][1][tid]), bc[k]);
#pragma unroll
                for (int q = 0; q < NS / 4; q++)
                    *reinterpret_cast<float4 *>(&sm.hs[k][tid][4 * hs_slot<NS>(tid, q)]) =
                        make_float4(h[2 * q].x, h[2 * q].y, h[2 * q + 1].x, h[2 * q + 1].y);
            }
        }
        // backward sweep over the chunk
#pragma unroll kSweepUnroll
        for (int k = kn - 1; k >= 0; k--) {
            const int t = a.reverse ? L - 1 - (i0 + k) : i0 + k;
            const size_t row = (size_t)b * L + t;
            const size_t io = row * a.D + dd;
            const float dt = sm.dt[k][tid], xv = tof(raw[k][1][tid]), dtx = dt * xv;
            const float gk = tof(raw[k][2][tid]);
            const float old_dx = nx_dx, old_dd = nx_dd;
            if (acc && i0 + k > 0) {
                nx_dx = a.dx[io_of(i0 + k - 1)];
                nx_dd = a.ddelta[io_of(i0 + k - 1)];
            }
            float4 hk[NS / 4], hm[NS / 4];   // h_i, h_{i-1}
            const float *prow = k > 0 ? &sm.hs[k > 0 ? k - 1 : 0][tid][0] : &sm.ck[buf][tid][0];
#pragma unroll
            for (int q = 0; q < NS / 4; q++) {
                hk[q] = lds4(&sm.hs[k][tid][4 * hs_slot<NS>(tid, q)]);
                hm[q] = lds4(prow + 4 * (k > 0 ? hs_slot<NS>(tid, q) : q));
            }
            // y_i = C . h_i + D x_i, then the gate
            float2 y2 = make_float2(0.f, 0.f);
#pragma unroll
            for (int q = 0; q < NS / 4; q++) {
                const float4 C4 = lds4(&bc[k][NS + 4 * q]);
                y2 = __ffma2_rn(lo2(C4), lo2(hk[q]), y2);
                y2 = __ffma2_rn(hi2(C4), hi2(hk[q]), y2);
            }
            const float y = fmaf(Dv, xv, y2.x + y2.y);
            float dy = gk;
            if (gate) {
                const float zk = tof(raw[k][3][tid]);
                const float s = sigmoid_f(zk);
                dy = gk * zk * s;
                if (active && a.dz)
                    a.dz[io] = gk * y * s * (1.f + zk * (1.f - s));
            }
            if (!active)
                dy = 0.f;
            const float2 dt2 = make_float2(dt, dt), dtx2 = make_float2(dtx, dtx), dy2 = make_float2(dy, dy);
            float2 dxs2 = make_float2(0.f, 0.f), dtA2 = make_float2(0.f, 0.f);
            float red[32];
#pragma unroll
            for (int q = 0; q < NS / 4; q++) {
                const float4 B4 = lds4(&bc[k][4 * q]), C4 = lds4(&bc[k][NS + 4 * q]);
#pragma unroll
                for (int e = 0; e < 2; e++) {
                    const int p = 2 * q + e, n = 2 * p;
                    const float2 Bn = e ? hi2(B4) : lo2(B4), Cn = e ? hi2(C4) : lo2(C4);
                    const float2 hcur = e ? hi2(hk[q]) : lo2(hk[q]), hprev = e ? hi2(hm[q]) : lo2(hm[q]);
                    const float2 an = ex2_pair(__fmul2_rn(dt2, Al[p]));
                    const float2 l = __ffma2_rn(dy2, Cn, lam[p]);       // lam_i
                    const float2 rb = __fmul2_rn(l, dtx2);              // dB contributions
                    const float2 rc = __fmul2_rn(dy2, hcur);            // dC contributions
                    red[n] = rb.x;
                    red[n + 1] = rb.y;
                    red[16 + n] = rc.x;
                    red[16 + n + 1] = rc.y;
                    dxs2 = __ffma2_rn(l, Bn, dxs2);
                    const float2 lah = __fmul2_rn(l, __fmul2_rn(an, hprev));   // lam_i a_i h_{i-1}
                    dtA2 = __ffma2_rn(lah, Al[p], dtA2);
                    gA[p] = __ffma2_rn(dt2, lah, gA[p]);
                    lam[p] = __fmul2_rn(an, l);                         // a_i lam_i for step i - 1
                }
            }
#pragma unroll
            for (int n = NS; n < 16; n++)
                red[n] = red[16 + n] = 0.f;
            const float dxs = dxs2.x + dxs2.y, dtA = dtA2.x + dtA2.y;
            if (active) {
                const float ddt = fmaf(xv, dxs, kLn2 * dtA);
                a.dx[io] = old_dx + fmaf(dy, Dv, dt * dxs);
                const float dv = a.softplus ? ddt * sigmoid_f(tof(raw[k][0][tid]) + bias) : ddt;
                a.ddelta[io] = old_dd + dv;
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
        for (int p = 0; p < NS / 2; p++) {
            if (2 * p < N)
                atomicAdd(a.dA + (size_t)dd * N + 2 * p, gA[p].x);
            if (2 * p + 1 < N)
                atomicAdd(a.dA + (size_t)dd * N + 2 * p + 1, gA[p].y);
        }
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
    // ask once per device for the largest shared-memory carveout (6 CTAs per SM)
    static std::atomic<uint64_t> carveout_set{0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    const uint64_t bit = 1ull << (dev & 63);
    if (!(carveout_set.load(std::memory_order_relaxed) & bit)) {
        e = cudaFuncSetAttribute(s6_bwd_kernel<T, NS>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 (int)cudaSharedmemCarveoutMaxShared);
        if (e != cudaSuccess)
            return e;
        carveout_set.fetch_or(bit, std::memory_order_relaxed);
    }
    const bool split = NS == 16 && a.N == 16 && bwd_split_enabled();
    if (!a.ckpt_given) {
        // the checkpoint pass: the split-state forward kernel when the plan
        // gives these sizes a split layout, else one thread per channel
        const int q = split ? split_threads(a.Bsz, a.L, a.D, a.N, 1) : 0;
        if (q) {
            S6Args f;
            memset(&f, 0, sizeof(f));
            f.Bsz = a.Bsz, f.L = a.L, f.D = a.D, f.N = a.N, f.S = 1, f.T = a.L;
            f.dtype = a.dtype, f.softplus = a.softplus, f.ndir = 1, f.reverse = a.reverse;
            f.x = a.x, f.delta = a.delta, f.split = q;
            if (q == 2)
                f.mix_rows2 = split_mix_rows(a.Bsz, a.D, 1);
            f.dir[0].bias = a.bias, f.dir[0].A = a.A, f.dir[0].B = a.B, f.dir[0].C = a.C;
            f.dir[0].ckpt = a.ckpt;
            if ((e = launch_s6_split_ckpt_only(f, st)) != cudaSuccess)
                return e;
        } else {
            s6_bwd_ckpt_kernel<T, NS><<<g, kCta, 0, st>>>(a);
        }
    }
    if (split) {
        if ((e = cudaGetLastError()) != cudaSuccess)
            return e;
        return launch_bwd_split(a, st);
    }
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
    const int64_t ns = N <= 4 ? 4 : N <= 8 ? 8 : 16;   // the kernels' padded state count
    return (size_t)Bsz * nch * D * ns * sizeof(float);
}

cudaError_t launch_bwd(const BwdArgs &a, cudaStream_t st)
{
    if (a.Bsz == 0 || a.L == 0 || a.D == 0)
        return cudaSuccess;
    return a.dtype == 0 ? launch_typed<float>(a, st) : launch_typed<__nv_bfloat16>(a, st);
}

}  // namespace ssm
