// ssm_capi.cu -- the extern "C" boundary of libssm.so (declared in
// include/ssm.h): argument validation, workspace sizing, dispatch.
// Every check runs before anything is launched.
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include "../../include/ssm.h"
#include "internal.h"

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool dtype_ok(int32_t dt) { return dt == SSM_F32 || dt == SSM_BF16; }

// Common S6 shape / pointer checks.  Returns SSM_OK or the first failure.
ssm_status check_s6_dims(const ssm_dims *d)
{
    if (!d)
        return SSM_ERR_INVALID_ARG;
    if (d->batch < 0 || d->seqlen < 0 || d->dim < 0 || d->dstate < 0)
        return SSM_ERR_INVALID_ARG;
    if (!dtype_ok(d->dtype))
        return SSM_ERR_UNSUPPORTED_DTYPE;
    if (d->dstate < 1 || d->dstate > 16)
        return SSM_ERR_UNSUPPORTED_SHAPE;
    // int32 indexing limits inside the kernels
    if (d->batch > INT32_MAX || d->seqlen > INT32_MAX || d->dim > INT32_MAX)
        return SSM_ERR_UNSUPPORTED_SHAPE;
    const int64_t vec = d->dtype == SSM_F32 ? 4 : 8;
    if (d->dim % vec != 0)
        return SSM_ERR_MISALIGNED;
    return SSM_OK;
}

ssm_status check_dir(const ssm_dir_params *p)
{
    if (!p || !p->A || !p->B || !p->C)
        return SSM_ERR_INVALID_ARG;
    const void *ptrs[] = {p->delta_bias, p->A, p->B, p->C, p->D, p->z, p->last_state};
    for (const void *q : ptrs)
        if (q && !aligned16(q))
            return SSM_ERR_MISALIGNED;
    return SSM_OK;
}

bool empty_s6(const ssm_dims *d) { return d->batch == 0 || d->seqlen == 0 || d->dim == 0; }

ssm_status zero_state(float *st, const ssm_dims *d, cudaStream_t s)
{
    if (!st)
        return SSM_OK;
    const size_t n = (size_t)d->batch * d->dim * d->dstate;
    if (n == 0)
        return SSM_OK;
    return cudaMemsetAsync(st, 0, n * sizeof(float), s) == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

ssm::DirArgs dir_args(const ssm_dir_params &p)
{
    return ssm::DirArgs{p.delta_bias, p.A, p.B, p.C, p.D, p.z, p.last_state};
}

ssm_status run_s6(const ssm_dims *dims, const void *x, const void *delta, int softplus, int ndir,
                  int reverse, const ssm_dir_params *dirs, void *out, void *ws, size_t ws_bytes,
                  cudaStream_t stream, const float *initial_state = nullptr, const int32_t *order = nullptr,
                  const unsigned char *mask = nullptr, const ssm_conv_params *conv = nullptr,
                  float *const *ckpt = nullptr, bool zoh = false)
{
    const int dt = dims->dtype == SSM_F32 ? 0 : 1;
    const ssm::S6Plan plan =
        ssm::plan_s6(dims->batch, dims->seqlen, dims->dim, dims->dstate, ndir, dt);
    if (plan.workspace_bytes > 0) {
        if (!ws || ws_bytes < plan.workspace_bytes)
            return SSM_ERR_WORKSPACE_TOO_SMALL;
        if (!aligned16(ws))
            return SSM_ERR_MISALIGNED;
    }
    ssm::S6Args a;
    memset(&a, 0, sizeof(a));
    a.Bsz = (int)dims->batch;
    a.L = (int)dims->seqlen;
    a.D = (int)dims->dim;
    a.N = (int)dims->dstate;
    a.S = plan.S;
    a.T = plan.T;
    a.cpl = plan.cpl;
    a.dtype = dt;
    a.softplus = softplus ? 1 : 0;
    a.ndir = ndir;
    a.reverse = reverse ? 1 : 0;
    a.x = x;
    a.delta = delta;
    for (int i = 0; i < ndir; i++)
        a.dir[i] = dir_args(dirs[i]);
    a.dir[0].init = initial_state;   // single direction only
    a.order = order;
    a.mask = mask;
    if (conv) {   // one ssm_conv_params per direction
        a.conv = 1;
        for (int i = 0; i < ndir; i++) {
            a.dir[i].conv_w = conv[i].weight;
            a.dir[i].conv_b = conv[i].bias;
            a.dir[i].conv_k = conv[i].width;
            a.dir[i].conv_silu = conv[i].silu ? 1 : 0;
        }
    }
    if (ckpt) {   // one checkpoint array per direction
        a.ckpt = 1;
        for (int i = 0; i < ndir; i++)
            a.dir[i].ckpt = ckpt[i];
    }
    a.out = out;
    // the split-state layouts also serve the checkpointing calls (their 4-step
    // groups are the checkpoint chunks); ordered and conv calls keep the
    // one-channel kernels
    int q = (order || mask || conv)
                ? 0
                : ssm::split_threads(dims->batch, dims->seqlen, dims->dim, dims->dstate, ndir);
    if (zoh) {   // the plan's split layout, else four threads per channel
        a.zoh = 1;
        q = q ? q : 4;
    }
    if (q) {
        a.split = q;   // one pass, q threads per channel
        if (q == 2 && !zoh)   // (checkpoints are the same in either layout)
            a.mix_rows2 = ssm::split_mix_rows(dims->batch, dims->dim, ndir);
        a.S = 1;
        a.T = a.L;
    }
    char *w = static_cast<char *>(ws);
    if (a.S > 1) {
        a.carry_h = reinterpret_cast<float *>(w + plan.carry_h_off);
        a.carry_s = reinterpret_cast<float *>(w + plan.carry_s_off);
    }
    if (ndir == 2)
        a.stash = dt == 0 ? static_cast<float *>(out) : reinterpret_cast<float *>(w + plan.stash_off);
    return ssm::launch_s6(a, stream) == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

}  // namespace

extern "C" {

size_t ssm_scan_workspace_size(const ssm_dims *dims)
{
    if (check_s6_dims(dims) != SSM_OK || empty_s6(dims))
        return 0;
    return ssm::plan_s6(dims->batch, dims->seqlen, dims->dim, dims->dstate, 1,
                        dims->dtype == SSM_F32 ? 0 : 1).workspace_bytes;
}

size_t bidir_scan_workspace_size(const ssm_dims *dims)
{
    if (check_s6_dims(dims) != SSM_OK || empty_s6(dims))
        return 0;
    return ssm::plan_s6(dims->batch, dims->seqlen, dims->dim, dims->dstate, 2,
                        dims->dtype == SSM_F32 ? 0 : 1).workspace_bytes;
}

ssm_status ssm_scan_plan(const ssm_dims *dims, int bidirectional, int *segments,
                         int *channels_per_lane)
{
    const ssm_status st = check_s6_dims(dims);
    if (st != SSM_OK)
        return st;
    ssm::S6Plan plan{1, 0, 2, 0, 0, 0, 0};
    const int ndir = bidirectional ? 2 : 1;
    if (!empty_s6(dims)) {
        plan = ssm::plan_s6(dims->batch, dims->seqlen, dims->dim, dims->dstate, ndir,
                            dims->dtype == SSM_F32 ? 0 : 1);
        const int q = ssm::split_threads(dims->batch, dims->seqlen, dims->dim, dims->dstate, ndir);
        if (q) {
            plan.S = 1;      // one pass
            plan.cpl = -q;   // q threads share each channel
        }
    }
    if (segments)
        *segments = plan.S;
    if (channels_per_lane)
        *channels_per_lane = plan.cpl;
    return SSM_OK;
}

}  // extern "C"

namespace {

ssm_status check_conv(const ssm_conv_params *c)
{
    if (!c || !c->weight)
        return SSM_ERR_INVALID_ARG;
    if (c->width < 1 || c->width > 4)
        return SSM_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(c->weight) || (c->bias && !aligned16(c->bias)))
        return SSM_ERR_MISALIGNED;
    return SSM_OK;
}

// Single-direction S6 with every option: the entry points below are this
// with some options off.
ssm_status scan_single(const ssm_dims *dims, const void *x, const void *delta, const float *delta_bias,
                       int delta_softplus, const float *A, const void *B, const void *C, const float *D,
                       const void *z, int reverse, const float *initial_state, const int32_t *order,
                       const unsigned char *mask, void *out, float *last_state, void *workspace,
                       size_t workspace_bytes, void *stream, const ssm_conv_params *conv = nullptr,
                       float *ckpt = nullptr, bool want_ckpt = false, bool zoh = false)
{
    ssm_status s = check_s6_dims(dims);
    if (s != SSM_OK)
        return s;
    if (conv && (s = check_conv(conv)) != SSM_OK)
        return s;
    if (want_ckpt && !empty_s6(dims)) {
        if (!ckpt)
            return SSM_ERR_INVALID_ARG;
        if (!aligned16(ckpt))
            return SSM_ERR_MISALIGNED;
    }
    if ((initial_state && !aligned16(initial_state)) || (last_state && !aligned16(last_state)))
        return SSM_ERR_MISALIGNED;
    if (order && (reinterpret_cast<uintptr_t>(order) & 3u))
        return SSM_ERR_MISALIGNED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (empty_s6(dims)) {
        // no step taken: the last state is the initial state (or zero)
        const size_t n = (size_t)dims->batch * dims->dim * dims->dstate;
        if (last_state && initial_state && dims->seqlen == 0 && n > 0) {
            if (last_state == initial_state)
                return SSM_OK;
            return cudaMemcpyAsync(last_state, initial_state, n * sizeof(float), cudaMemcpyDeviceToDevice,
                                   st) == cudaSuccess
                       ? SSM_OK
                       : SSM_ERR_CUDA;
        }
        return zero_state(last_state, dims, st);
    }
    if (!x || !delta || !out)
        return SSM_ERR_INVALID_ARG;
    ssm_dir_params p{delta_bias, A, B, C, D, z, last_state};
    if ((s = check_dir(&p)) != SSM_OK)
        return s;
    if (!aligned16(x) || !aligned16(delta) || !aligned16(out))
        return SSM_ERR_MISALIGNED;
    float *const ck[1] = {ckpt};
    return run_s6(dims, x, delta, delta_softplus, 1, reverse, &p, out, workspace, workspace_bytes, st,
                  initial_state, order, mask, conv, want_ckpt ? ck : nullptr, zoh);
}

// the zero-order-hold scans: N = 16 and a batch that fits the grid, also
// for empty problems, so that the refusal does not depend on L
ssm_status zoh_dims(const ssm_dims *dims)
{
    const ssm_status s = check_s6_dims(dims);
    if (s != SSM_OK)
        return s;
    return dims->dstate != 16 || dims->batch > 65535 ? SSM_ERR_UNSUPPORTED_SHAPE : SSM_OK;
}

ssm_status scan_bidir(const ssm_dims *dims, const void *x, const void *delta, int delta_softplus,
                      const ssm_dir_params *fwd, const ssm_dir_params *bwd, const int32_t *order,
                      const unsigned char *mask, void *out, void *workspace, size_t workspace_bytes,
                      void *stream, const ssm_conv_params *conv = nullptr, float *const *ckpt = nullptr,
                      bool zoh = false)
{
    ssm_status s = check_s6_dims(dims);
    if (s != SSM_OK)
        return s;
    if (conv && ((s = check_conv(&conv[0])) != SSM_OK || (s = check_conv(&conv[1])) != SSM_OK))
        return s;
    if (!fwd || !bwd)
        return SSM_ERR_INVALID_ARG;
    if (ckpt && !empty_s6(dims)) {
        if (!ckpt[0] || !ckpt[1])
            return SSM_ERR_INVALID_ARG;
        if (!aligned16(ckpt[0]) || !aligned16(ckpt[1]))
            return SSM_ERR_MISALIGNED;
    }
    if (order && (reinterpret_cast<uintptr_t>(order) & 3u))
        return SSM_ERR_MISALIGNED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (empty_s6(dims)) {
        if ((fwd->last_state && !aligned16(fwd->last_state)) ||
            (bwd->last_state && !aligned16(bwd->last_state)))
            return SSM_ERR_MISALIGNED;
        if ((s = zero_state(fwd->last_state, dims, st)) != SSM_OK)
            return s;
        return zero_state(bwd->last_state, dims, st);
    }
    if (!x || !delta || !out)
        return SSM_ERR_INVALID_ARG;
    if ((s = check_dir(fwd)) != SSM_OK || (s = check_dir(bwd)) != SSM_OK)
        return s;
    if ((fwd->z == nullptr) != (bwd->z == nullptr))
        return SSM_ERR_INVALID_ARG;   // both directions gated, or neither
    if (!aligned16(x) || !aligned16(delta) || !aligned16(out))
        return SSM_ERR_MISALIGNED;
    const ssm_dir_params dirs[2] = {*fwd, *bwd};
    return run_s6(dims, x, delta, delta_softplus, 2, 0, dirs, out, workspace, workspace_bytes, st, nullptr,
                  order, mask, conv, ckpt, zoh);
}

}  // namespace

extern "C" {

ssm_status ssm_scan_fwd_state(const ssm_dims *dims, const void *x, const void *delta,
                              const float *delta_bias, int delta_softplus, const float *A,
                              const void *B, const void *C, const float *D, const void *z,
                              int reverse, const float *initial_state, void *out, float *last_state,
                              void *workspace, size_t workspace_bytes, void *stream)
{
    return scan_single(dims, x, delta, delta_bias, delta_softplus, A, B, C, D, z, reverse, initial_state,
                       nullptr, nullptr, out, last_state, workspace, workspace_bytes, stream);
}

ssm_status ssm_scan_fwd_zoh(const ssm_dims *dims, const void *x, const void *delta, const float *delta_bias,
                            int delta_softplus, const float *A, const void *B, const void *C, const float *D,
                            const void *z, int reverse, const float *initial_state, void *out,
                            float *last_state, void *workspace, size_t workspace_bytes, void *stream)
{
    const ssm_status s = zoh_dims(dims);
    if (s != SSM_OK)
        return s;
    return scan_single(dims, x, delta, delta_bias, delta_softplus, A, B, C, D, z, reverse, initial_state,
                       nullptr, nullptr, out, last_state, workspace, workspace_bytes, stream, nullptr, nullptr,
                       false, true);
}

ssm_status ssm_scan_fwd_ordered(const ssm_dims *dims, const void *x, const void *delta,
                                const float *delta_bias, int delta_softplus, const float *A,
                                const void *B, const void *C, const float *D, const void *z,
                                int reverse, const int32_t *order, const unsigned char *mask, void *out,
                                float *last_state, void *workspace, size_t workspace_bytes, void *stream)
{
    return scan_single(dims, x, delta, delta_bias, delta_softplus, A, B, C, D, z, reverse, nullptr, order,
                       mask, out, last_state, workspace, workspace_bytes, stream);
}

ssm_status ssm_scan_fwd_conv(const ssm_dims *dims, const void *x_in, const ssm_conv_params *conv,
                             const void *delta, const float *delta_bias, int delta_softplus, const float *A,
                             const void *B, const void *C, const float *D, const void *z, int reverse,
                             void *out, float *last_state, void *workspace, size_t workspace_bytes,
                             void *stream)
{
    if (!conv)
        return SSM_ERR_INVALID_ARG;
    return scan_single(dims, x_in, delta, delta_bias, delta_softplus, A, B, C, D, z, reverse, nullptr,
                       nullptr, nullptr, out, last_state, workspace, workspace_bytes, stream, conv);
}

ssm_status bidir_scan_fwd_conv(const ssm_dims *dims, const void *x_in, const void *delta, int delta_softplus,
                               const ssm_dir_params *fwd, const ssm_dir_params *bwd,
                               const ssm_conv_params *conv_fwd, const ssm_conv_params *conv_bwd, void *out,
                               void *workspace, size_t workspace_bytes, void *stream)
{
    if (!conv_fwd || !conv_bwd)
        return SSM_ERR_INVALID_ARG;
    const ssm_conv_params conv[2] = {*conv_fwd, *conv_bwd};
    return scan_bidir(dims, x_in, delta, delta_softplus, fwd, bwd, nullptr, nullptr, out, workspace,
                      workspace_bytes, stream, conv);
}

ssm_status bidir_scan_fwd_ordered(const ssm_dims *dims, const void *x, const void *delta,
                                  int delta_softplus, const ssm_dir_params *fwd,
                                  const ssm_dir_params *bwd, const int32_t *order,
                                  const unsigned char *mask, void *out, void *workspace,
                                  size_t workspace_bytes, void *stream)
{
    return scan_bidir(dims, x, delta, delta_softplus, fwd, bwd, order, mask, out, workspace,
                      workspace_bytes, stream);
}

ssm_status ssm_scan_fwd(const ssm_dims *dims, const void *x, const void *delta,
                        const float *delta_bias, int delta_softplus, const float *A,
                        const void *B, const void *C, const float *D, const void *z, int reverse,
                        void *out, float *last_state, void *workspace, size_t workspace_bytes,
                        void *stream)
{
    return ssm_scan_fwd_state(dims, x, delta, delta_bias, delta_softplus, A, B, C, D, z, reverse, nullptr,
                              out, last_state, workspace, workspace_bytes, stream);
}

size_t ssm_scan_bwd_workspace_size(const ssm_dims *dims)
{
    if (check_s6_dims(dims) != SSM_OK || empty_s6(dims))
        return 0;
    return ssm::bwd_workspace_bytes(dims->batch, dims->seqlen, dims->dim, dims->dstate);
}

}  // extern "C"

namespace {

// The arguments of one direction's backward (ssm_scan_bwd, bidir_scan_bwd),
// checked before anything is launched.
ssm_status bwd_check(const ssm_dims *dims, const void *x, const void *delta, const ssm_dir_params &p,
                     const void *dout, const float *dx, const float *ddelta, const ssm_dir_grads &g,
                     const void *workspace, size_t workspace_bytes, bool ckpt_given = false)
{
    if (!x || !delta || !p.A || !p.B || !p.C || !dout || !dx || !ddelta || !g.dA || !g.dB || !g.dC)
        return SSM_ERR_INVALID_ARG;
    if ((p.D && !g.dD) || (p.z && !g.dz) || (p.delta_bias && !g.ddelta_bias))
        return SSM_ERR_INVALID_ARG;
    const void *ptrs[] = {x, delta, p.delta_bias, p.A, p.B, p.C, p.D, p.z, dout, dx, ddelta, g.dA, g.dB,
                          g.dC, g.dD, g.dz, g.ddelta_bias, workspace};
    for (const void *q : ptrs)
        if (q && !aligned16(q))
            return SSM_ERR_MISALIGNED;
    if (ckpt_given)   // the checkpoints of the checkpointing forward scan (their size is the caller's)
        return workspace ? SSM_OK : SSM_ERR_INVALID_ARG;
    const size_t need = ssm::bwd_workspace_bytes(dims->batch, dims->seqlen, dims->dim, dims->dstate);
    if (!workspace || workspace_bytes < need)
        return SSM_ERR_WORKSPACE_TOO_SMALL;
    return SSM_OK;
}

// One direction's backward launch: checks, zeroes the accumulated
// gradients, launches.  accumulate: add into dx and ddelta instead of
// writing them.
ssm_status bwd_one(const ssm_dims *dims, const void *x, const void *delta, int delta_softplus,
                   const ssm_dir_params &p, int reverse, const void *dout, float *dx, float *ddelta,
                   const ssm_dir_grads &g, void *workspace, size_t workspace_bytes, int accumulate,
                   cudaStream_t st, bool ckpt_given = false)
{
    ssm_status s = bwd_check(dims, x, delta, p, dout, dx, ddelta, g, workspace, workspace_bytes, ckpt_given);
    if (s != SSM_OK)
        return s;
    const size_t nDN = (size_t)dims->dim * dims->dstate;
    const size_t nBLN = (size_t)dims->batch * dims->seqlen * dims->dstate;
    if (cudaMemsetAsync(g.dA, 0, nDN * sizeof(float), st) != cudaSuccess ||
        cudaMemsetAsync(g.dB, 0, nBLN * sizeof(float), st) != cudaSuccess ||
        cudaMemsetAsync(g.dC, 0, nBLN * sizeof(float), st) != cudaSuccess ||
        (p.D && cudaMemsetAsync(g.dD, 0, dims->dim * sizeof(float), st) != cudaSuccess) ||
        (p.delta_bias && cudaMemsetAsync(g.ddelta_bias, 0, dims->dim * sizeof(float), st) != cudaSuccess))
        return SSM_ERR_CUDA;
    ssm::BwdArgs a;
    memset(&a, 0, sizeof(a));
    a.Bsz = (int)dims->batch;
    a.L = (int)dims->seqlen;
    a.D = (int)dims->dim;
    a.N = (int)dims->dstate;
    a.dtype = dims->dtype == SSM_F32 ? 0 : 1;
    a.softplus = delta_softplus ? 1 : 0;
    a.reverse = reverse ? 1 : 0;
    a.accumulate = accumulate;
    a.x = x;
    a.delta = delta;
    a.B = p.B;
    a.C = p.C;
    a.z = p.z;
    a.dout = dout;
    a.bias = p.delta_bias;
    a.A = p.A;
    a.Dskip = p.D;
    a.dx = dx;
    a.ddelta = ddelta;
    a.dz = p.z ? g.dz : nullptr;
    a.dA = g.dA;
    a.dB = g.dB;
    a.dC = g.dC;
    a.dD = p.D ? g.dD : nullptr;
    a.dbias = p.delta_bias ? g.ddelta_bias : nullptr;
    a.ckpt = static_cast<float *>(workspace);
    a.ckpt_given = ckpt_given ? 1 : 0;
    return ssm::launch_bwd(a, st) == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

// The gradients of an empty problem: zero over (D, N) and (D).
ssm_status bwd_empty(const ssm_dims *dims, const ssm_dir_params &p, const ssm_dir_grads &g, cudaStream_t st)
{
    const size_t nDN = (size_t)dims->dim * dims->dstate;
    if (g.dA && nDN && cudaMemsetAsync(g.dA, 0, nDN * sizeof(float), st) != cudaSuccess)
        return SSM_ERR_CUDA;
    if (p.D && g.dD && dims->dim && cudaMemsetAsync(g.dD, 0, dims->dim * sizeof(float), st) != cudaSuccess)
        return SSM_ERR_CUDA;
    if (p.delta_bias && g.ddelta_bias && dims->dim &&
        cudaMemsetAsync(g.ddelta_bias, 0, dims->dim * sizeof(float), st) != cudaSuccess)
        return SSM_ERR_CUDA;
    return SSM_OK;
}

}  // namespace

extern "C" {

ssm_status ssm_scan_bwd(const ssm_dims *dims, const void *x, const void *delta, const float *delta_bias,
                        int delta_softplus, const float *A, const void *B, const void *C, const float *D,
                        const void *z, int reverse, const void *dout, float *dx, float *ddelta, float *dA,
                        float *dB, float *dC, float *dD, float *dz, float *ddelta_bias, void *workspace,
                        size_t workspace_bytes, void *stream)
{
    ssm_status s = check_s6_dims(dims);
    if (s != SSM_OK)
        return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const ssm_dir_params p{delta_bias, A, B, C, D, z, nullptr};
    const ssm_dir_grads g{dA, dB, dC, dD, dz, ddelta_bias};
    if (empty_s6(dims))
        return bwd_empty(dims, p, g, st);
    return bwd_one(dims, x, delta, delta_softplus, p, reverse, dout, dx, ddelta, g, workspace, workspace_bytes,
                   0, st);
}

ssm_status bidir_scan_bwd(const ssm_dims *dims, const void *x, const void *delta, int delta_softplus,
                          const ssm_dir_params *fwd, const ssm_dir_params *bwd, const void *dout, float *dx,
                          float *ddelta, const ssm_dir_grads *grad_fwd, const ssm_dir_grads *grad_bwd,
                          void *workspace, size_t workspace_bytes, void *stream)
{
    ssm_status s = check_s6_dims(dims);
    if (s != SSM_OK)
        return s;
    if (!fwd || !bwd || !grad_fwd || !grad_bwd)
        return SSM_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (empty_s6(dims)) {
        if ((s = bwd_empty(dims, *fwd, *grad_fwd, st)) != SSM_OK)
            return s;
        return bwd_empty(dims, *bwd, *grad_bwd, st);
    }
    // both directions' arguments first, so that a refused call launches nothing
    if ((s = bwd_check(dims, x, delta, *fwd, dout, dx, ddelta, *grad_fwd, workspace, workspace_bytes)) != SSM_OK ||
        (s = bwd_check(dims, x, delta, *bwd, dout, dx, ddelta, *grad_bwd, workspace, workspace_bytes)) != SSM_OK)
        return s;
    // forward direction writes dx, ddelta; the reversed one adds to them (the
    // two launches share the workspace in stream order)
    if ((s = bwd_one(dims, x, delta, delta_softplus, *fwd, 0, dout, dx, ddelta, *grad_fwd, workspace,
                     workspace_bytes, 0, st)) != SSM_OK)
        return s;
    return bwd_one(dims, x, delta, delta_softplus, *bwd, 1, dout, dx, ddelta, *grad_bwd, workspace,
                   workspace_bytes, 1, st);
}

size_t ssm_scan_ckpt_size(const ssm_dims *dims)
{
    if (check_s6_dims(dims) != SSM_OK || empty_s6(dims))
        return 0;
    return ssm::bwd_workspace_bytes(dims->batch, dims->seqlen, dims->dim, dims->dstate);
}

ssm_status ssm_scan_fwd_ckpt(const ssm_dims *dims, const void *x, const void *delta, const float *delta_bias,
                             int delta_softplus, const float *A, const void *B, const void *C, const float *D,
                             const void *z, int reverse, void *out, float *last_state, float *ckpt,
                             void *workspace, size_t workspace_bytes, void *stream)
{
    return scan_single(dims, x, delta, delta_bias, delta_softplus, A, B, C, D, z, reverse, nullptr, nullptr,
                       nullptr, out, last_state, workspace, workspace_bytes, stream, nullptr, ckpt, true);
}

ssm_status bidir_scan_fwd_ckpt(const ssm_dims *dims, const void *x, const void *delta, int delta_softplus,
                               const ssm_dir_params *fwd, const ssm_dir_params *bwd, void *out, float *ckpt_fwd,
                               float *ckpt_bwd, void *workspace, size_t workspace_bytes, void *stream)
{
    float *const ck[2] = {ckpt_fwd, ckpt_bwd};
    return scan_bidir(dims, x, delta, delta_softplus, fwd, bwd, nullptr, nullptr, out, workspace,
                      workspace_bytes, stream, nullptr, ck);
}

ssm_status ssm_scan_bwd_ckpt(const ssm_dims *dims, const void *x, const void *delta, const float *delta_bias,
                             int delta_softplus, const float *A, const void *B, const void *C, const float *D,
                             const void *z, int reverse, const void *dout, float *dx, float *ddelta, float *dA,
                             float *dB, float *dC, float *dD, float *dz, float *ddelta_bias, const float *ckpt,
                             void *stream)
{
    ssm_status s = check_s6_dims(dims);
    if (s != SSM_OK)
        return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const ssm_dir_params p{delta_bias, A, B, C, D, z, nullptr};
    const ssm_dir_grads g{dA, dB, dC, dD, dz, ddelta_bias};
    if (empty_s6(dims))
        return bwd_empty(dims, p, g, st);
    return bwd_one(dims, x, delta, delta_softplus, p, reverse, dout, dx, ddelta, g, const_cast<float *>(ckpt), 0,
                   0, st, true);
}

ssm_status bidir_scan_bwd_ckpt(const ssm_dims *dims, const void *x, const void *delta, int delta_softplus,
                               const ssm_dir_params *fwd, const ssm_dir_params *bwd, const void *dout, float *dx,
                               float *ddelta, const ssm_dir_grads *grad_fwd, const ssm_dir_grads *grad_bwd,
                               const float *ckpt_fwd, const float *ckpt_bwd, void *stream)
{
    ssm_status s = check_s6_dims(dims);
    if (s != SSM_OK)
        return s;
    if (!fwd || !bwd || !grad_fwd || !grad_bwd)
        return SSM_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (empty_s6(dims)) {
        if ((s = bwd_empty(dims, *fwd, *grad_fwd, st)) != SSM_OK)
            return s;
        return bwd_empty(dims, *bwd, *grad_bwd, st);
    }
    float *cf = const_cast<float *>(ckpt_fwd), *cb = const_cast<float *>(ckpt_bwd);
    // both directions' arguments first, so that a refused call launches nothing
    if ((s = bwd_check(dims, x, delta, *fwd, dout, dx, ddelta, *grad_fwd, cf, 0, true)) != SSM_OK ||
        (s = bwd_check(dims, x, delta, *bwd, dout, dx, ddelta, *grad_bwd, cb, 0, true)) != SSM_OK)
        return s;
    if ((s = bwd_one(dims, x, delta, delta_softplus, *fwd, 0, dout, dx, ddelta, *grad_fwd, cf, 0, 0, st, true)) !=
        SSM_OK)
        return s;
    return bwd_one(dims, x, delta, delta_softplus, *bwd, 1, dout, dx, ddelta, *grad_bwd, cb, 0, 1, st, true);
}

ssm_status ssm_step(const ssm_dims *dims, const void *x, const void *delta, const float *delta_bias,
                    int delta_softplus, const float *A, const void *B, const void *C, const float *D,
                    const void *z, float *state, void *out, void *stream)
{
    ssm_status s = check_s6_dims(dims);
    if (s != SSM_OK)
        return s;
    if (dims->seqlen != 1)
        return SSM_ERR_UNSUPPORTED_SHAPE;
    if (dims->batch == 0 || dims->dim == 0)
        return SSM_OK;
    if (!x || !delta || !A || !B || !C || !state || !out)
        return SSM_ERR_INVALID_ARG;
    const void *ptrs[] = {x, delta, delta_bias, A, B, C, D, z, state, out};
    for (const void *q : ptrs)
        if (q && !aligned16(q))
            return SSM_ERR_MISALIGNED;
    ssm::StepArgs a;
    a.Bsz = (int)dims->batch;
    a.D = (int)dims->dim;
    a.N = (int)dims->dstate;
    a.dtype = dims->dtype == SSM_F32 ? 0 : 1;
    a.softplus = delta_softplus ? 1 : 0;
    a.x = x;
    a.delta = delta;
    a.B = B;
    a.C = C;
    a.z = z;
    a.bias = delta_bias;
    a.A = A;
    a.Dskip = D;
    a.state = state;
    a.out = out;
    return ssm::launch_step(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

ssm_status bidir_scan_fwd(const ssm_dims *dims, const void *x, const void *delta,
                          int delta_softplus, const ssm_dir_params *fwd,
                          const ssm_dir_params *bwd, void *out, void *workspace,
                          size_t workspace_bytes, void *stream)
{
    return scan_bidir(dims, x, delta, delta_softplus, fwd, bwd, nullptr, nullptr, out, workspace,
                      workspace_bytes, stream);
}

ssm_status bidir_scan_fwd_zoh(const ssm_dims *dims, const void *x, const void *delta, int delta_softplus,
                              const ssm_dir_params *fwd, const ssm_dir_params *bwd, void *out,
                              void *workspace, size_t workspace_bytes, void *stream)
{
    const ssm_status s = zoh_dims(dims);
    if (s != SSM_OK)
        return s;
    return scan_bidir(dims, x, delta, delta_softplus, fwd, bwd, nullptr, nullptr, out, workspace,
                      workspace_bytes, stream, nullptr, nullptr, true);
}

size_t ssd_chunk_workspace_size(const ssd_dims *d)
{
    if (!d || d->batch < 0 || d->seqlen < 0 || d->nheads < 0 || d->headdim < 0 || d->dstate < 0 ||
        d->chunk <= 0)
        return 0;
    return ssm::ssd_workspace_bytes(d->batch, d->seqlen, d->nheads, d->headdim, d->dstate, d->chunk);
}

ssm_status ssd_chunk_fwd(const ssd_dims *dims, const void *x, const void *delta,
                         const float *delta_bias, int delta_softplus, const float *A,
                         const void *B, const void *C, const float *D, const void *z, void *out,
                         float *last_state, void *workspace, size_t workspace_bytes, void *stream)
{
    if (!dims)
        return SSM_ERR_INVALID_ARG;
    if (dims->batch < 0 || dims->seqlen < 0 || dims->nheads < 0 || dims->headdim < 0 ||
        dims->dstate < 0 || dims->chunk < 0)
        return SSM_ERR_INVALID_ARG;
    if (dims->dtype != SSM_BF16)
        return SSM_ERR_UNSUPPORTED_DTYPE;
    if (dims->headdim != 64 || dims->dstate != 128 || dims->chunk != 64)
        return SSM_ERR_UNSUPPORTED_SHAPE;
    if (dims->batch > INT32_MAX || dims->seqlen > INT32_MAX || dims->nheads > INT32_MAX)
        return SSM_ERR_UNSUPPORTED_SHAPE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (dims->batch == 0 || dims->nheads == 0)
        return SSM_OK;
    if (dims->seqlen > 0 && (!x || !delta || !A || !B || !C || !out))
        return SSM_ERR_INVALID_ARG;
    const void *ptrs[] = {x, delta, delta_bias, A, B, C, D, z, out, last_state};
    for (const void *q : ptrs)
        if (q && !aligned16(q))
            return SSM_ERR_MISALIGNED;
    if (dims->seqlen == 0) {
        if (!last_state)
            return SSM_OK;
        const size_t n = (size_t)dims->batch * dims->nheads * dims->headdim * dims->dstate;
        return cudaMemsetAsync(last_state, 0, n * sizeof(float), st) == cudaSuccess ? SSM_OK
                                                                                    : SSM_ERR_CUDA;
    }
    const size_t need = ssm::ssd_workspace_bytes(dims->batch, dims->seqlen, dims->nheads,
                                                 dims->headdim, dims->dstate, dims->chunk);
    if (need > 0) {
        if (!workspace || workspace_bytes < need)
            return SSM_ERR_WORKSPACE_TOO_SMALL;
        if (!aligned16(workspace))
            return SSM_ERR_MISALIGNED;
    }
    ssm::SSDArgs a;
    memset(&a, 0, sizeof(a));
    a.Bsz = (int)dims->batch;
    a.L = (int)dims->seqlen;
    a.H = (int)dims->nheads;
    a.P = (int)dims->headdim;
    a.N = (int)dims->dstate;
    a.Q = (int)dims->chunk;
    a.softplus = delta_softplus ? 1 : 0;
    a.x = x;
    a.delta = delta;
    a.B = B;
    a.C = C;
    a.z = z;
    a.bias = delta_bias;
    a.A = A;
    a.D = D;
    a.out = out;
    a.last_state = last_state;
    a.workspace = workspace;
    const cudaError_t e = ssm::launch_ssd(a, st);
    if (e == cudaErrorNotSupported)
        return SSM_ERR_UNSUPPORTED_SHAPE;
    return e == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

ssm_status ssm_check_device(void *stream)
{
    unsigned v = 0, o = 0;
    if (ssm::read_and_clear_device_error(&v, static_cast<cudaStream_t>(stream)) != cudaSuccess ||
        ssm::read_and_clear_s6_error(&o, static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return SSM_ERR_CUDA;
    if (v)
        return SSM_ERR_DEVICE_TIMEOUT;
    return o ? SSM_ERR_INVALID_ARG : SSM_OK;
}

void ssm_debug_ssd_stall(int withhold_chunk, unsigned wait_limit) { ssm::ssd_stall_set(withhold_chunk, wait_limit); }

ssm_status ssm_debug_s6_mapping(int mode)
{
    if (mode < 0 || mode > 3)
        return SSM_ERR_INVALID_ARG;
    ssm::split_mode_set(mode);
    return SSM_OK;
}

const char *ssm_status_string(ssm_status s)
{
    switch (s) {
    case SSM_OK: return "SSM_OK";
    case SSM_ERR_INVALID_ARG: return "SSM_ERR_INVALID_ARG: NULL required pointer or negative size";
    case SSM_ERR_UNSUPPORTED_SHAPE: return "SSM_ERR_UNSUPPORTED_SHAPE: shape not supported";
    case SSM_ERR_MISALIGNED: return "SSM_ERR_MISALIGNED: pointer or dim not aligned to 16 bytes";
    case SSM_ERR_UNSUPPORTED_DTYPE: return "SSM_ERR_UNSUPPORTED_DTYPE: dtype not supported";
    case SSM_ERR_WORKSPACE_TOO_SMALL: return "SSM_ERR_WORKSPACE_TOO_SMALL: workspace too small";
    case SSM_ERR_CUDA: return "SSM_ERR_CUDA: a CUDA launch or runtime call failed";
    case SSM_ERR_DEVICE_TIMEOUT: return "SSM_ERR_DEVICE_TIMEOUT: a device-side wait gave up";
    }
    return "unknown ssm_status";
}

int ssm_version(void) { return 100; }

}  // extern "C"
