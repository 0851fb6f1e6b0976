// s6_scan.cu -- the S6 launch plan (segments, lane mapping) and the
// dispatch to the kernel parts (s6_part_*.cu, one element type and variant
// each, all built from s6_scan_impl.cuh).
#include "s6_scan_impl.cuh"

namespace ssm {

S6Plan plan_s6(int64_t Bsz, int64_t L, int64_t D, int64_t N, int ndir, int dtype)
{
    S6Plan p{1, (int)L, 2, 0, 0, 0, 0};
    if (L <= 0)
        return p;
    // Channels per lane: two give each thread more independent work, one
    // gives twice the threads (and fewer segments) when the problem is small.
    const int64_t lanes2 = (int64_t)ndir * Bsz * ((D + 1) / 2);
    p.cpl = SSM_S6_CPL != 0 ? SSM_S6_CPL : (lanes2 < SSM_S6_CPL1_BELOW ? 1 : 2);
    const int64_t kMinT = 16;
    int64_t S = 1;
    if (SSM_S6_WAVES > 0) {
        // Segments: as many as fill SSM_S6_WAVES waves of the main kernel's
        // resident CTAs (148 SMs x CTAs per SM for this lane mapping) -- a
        // CTA count just past a wave boundary costs a whole extra wave.
        const int64_t ch_per_cta = (ndir == 2 ? 32 : 64) * p.cpl;
        const int64_t ctas_per_seg = (D + ch_per_cta - 1) / ch_per_cta * Bsz;
        const int64_t slots = (int64_t)148 * (p.cpl == 2 ? SSM_S6_MINB : SSM_S6_MINB1) * SSM_S6_WAVES;
        if (ctas_per_seg > 0)
            S = slots / ctas_per_seg;
    } else {
        const int64_t kTargetThreads = p.cpl == 1 ? SSM_S6_TARGET1 : SSM_S6_TARGET2;
        const int64_t threads = (int64_t)ndir * Bsz * ((D + p.cpl - 1) / p.cpl);
        if (threads > 0 && threads < kTargetThreads)
            S = (kTargetThreads + threads - 1) / threads;
    }
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
    if (a.split)
        return launch_s6_split(a, st);
    const int var = (a.order || a.mask) ? 1 : (a.conv ? 2 : (a.ckpt ? 3 : 0));
    if (a.dtype == 0)
        return var == 1 ? launch_s6_f32_ord(a, st)
               : var == 2 ? launch_s6_f32_conv(a, st)
               : var == 3 ? launch_s6_f32_ckpt(a, st)
                          : launch_s6_f32(a, st);
    return var == 1 ? launch_s6_bf16_ord(a, st)
           : var == 2 ? launch_s6_bf16_conv(a, st)
           : var == 3 ? launch_s6_bf16_ckpt(a, st)
                      : launch_s6_bf16(a, st);
}

cudaError_t read_and_clear_s6_error(unsigned *value, cudaStream_t stream)
{
    cudaError_t e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess)
        return e;
    cudaError_t (*parts[])(unsigned *, bool) = {s6_error_f32,       s6_error_f32_ord,  s6_error_f32_conv,
                                                s6_error_f32_ckpt,  s6_error_bf16,     s6_error_bf16_ord,
                                                s6_error_bf16_conv, s6_error_bf16_ckpt};
    *value = 0;
    for (auto f : parts) {
        unsigned v = 0;
        if ((e = f(&v, true)) != cudaSuccess)
            return e;
        *value |= v;
    }
    return cudaSuccess;
}

}  // namespace ssm
