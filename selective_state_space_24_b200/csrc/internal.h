// internal.h -- launcher interface between the C-ABI shim and the kernels.
// Not part of the public ABI (include/ssm.h is).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace ssm {

// Parameters of one scan direction, device pointers.
struct DirArgs {
    const float *bias;   // (D) or nullptr
    const float *A;      // (D, N)
    const void *B;       // (Bsz, L, N)
    const void *C;       // (Bsz, L, N)
    const float *D;      // (D) or nullptr
    const void *z;       // (Bsz, L, D) or nullptr
    float *last_state;   // (Bsz, D, N) or nullptr
    const float *init;   // (Bsz, D, N) state before the first step, or nullptr (zero)
    // depthwise causal conv1d applied to x along this direction's scan order
    // (used by the kernels' conv variant only)
    const float *conv_w;   // (D, conv_k)
    const float *conv_b;   // (D) or nullptr
    int conv_k;            // 1..4
    int conv_silu;         // 1: SiLU after the conv
    // (checkpointing variant only) the state entering every 4-step chunk in
    // scan order, (Bsz, ceil(L / 4), D, NS) float32, NS = N rounded up to 4,
    // 8 or 16 -- the array the backward kernel reads
    float *ckpt;
};

// One S6 call (single direction or bidirectional).
//
// The sequence is cut into S segments of T steps (the last one may be
// shorter).  With S > 1 every segment first summarises itself (local end
// state from a zero start plus the sum of dt), a carry pass composes those
// summaries in scan order, starting from the direction's initial state, and
// the main pass then rescans each segment from its true entering state.
// carry_h / carry_s are the caller's workspace.  With S > 1 only the carry
// pass reads the initial state, so it may share a buffer with last_state.
struct S6Args {
    int Bsz, L, D, N;
    int S, T;
    int cpl;       // channels per lane: 1 or 2
    int dtype;     // 0 = float32, 1 = bf16
    int softplus;
    int ndir;      // 1 or 2
    int reverse;   // ndir == 1: 1 = the single direction runs t descending
    const void *x;
    const void *delta;
    DirArgs dir[2];  // ndir == 2: dir[0] forward, dir[1] reversed
    void *out;
    float *carry_h;  // [ndir][Bsz][S][D][N]
    float *carry_s;  // [ndir][Bsz][S][D]
    float *stash;    // ndir == 2: fp32 (Bsz, L, D) parking space for the
                     // first half of each direction's outputs (out itself
                     // when out is fp32)
    const int *order;            // (L) visiting order of the positions, or nullptr (0..L-1)
    const unsigned char *mask;   // (Bsz, L) by position, 0 = bypass the token, or nullptr
    int conv;                    // 1: x is the conv input x_in, each direction convolves it
    int ckpt;                    // 1: each direction also writes its checkpoints (DirArgs::ckpt)
    int split;                   // 2 or 4: that many threads per channel (s6_split.cu); needs
                                 // N == 16, S == 1, and none of order / mask / conv
    int zoh;                     // 1: the exact zero-order-hold input coefficient (needs split)
    int mix_rows2;               // split == 2 and 0 < mix_rows2 < Bsz: rows [mix_rows2, Bsz) take
                                 // four threads per channel in the same launch
};

struct S6Plan {
    int S, T;
    int cpl;   // channels per lane
    size_t workspace_bytes;
    size_t carry_h_off, carry_s_off, stash_off;  // byte offsets into the workspace
};

// Segment plan and lane mapping for a problem; depends on the sizes and
// dtype only.
S6Plan plan_s6(int64_t Bsz, int64_t L, int64_t D, int64_t N, int ndir, int dtype);

cudaError_t launch_s6(const S6Args &a, cudaStream_t stream);

// The kernel that splits each channel's states over two or four threads:
// how many threads per channel a plain call (no order, mask, conv or
// checkpoints) of these sizes takes (0: the one-or-two-channels-per-thread
// kernels), and its launcher.  It needs no workspace beyond the
// bidirectional bf16 stash of plan_s6.
int split_threads(int64_t Bsz, int64_t L, int64_t D, int64_t N, int ndir);
// With two threads per channel: how many leading batch rows keep it when
// the rest take four threads per channel in the same launch (0: all keep it).
int split_mix_rows(int64_t Bsz, int64_t D, int ndir);
cudaError_t launch_s6_split(const S6Args &a, cudaStream_t stream);
// The same kernel as the backward's checkpoint pass: one direction (a.dir[0],
// a.reverse), a.split threads per channel, only dir[0].ckpt written (the
// state entering every 4-step chunk; no outputs, gate or skip).
cudaError_t launch_s6_split_ckpt_only(const S6Args &a, cudaStream_t stream);
// Test setting (process-wide): 0 the cost model decides, 1 never the split
// layouts, 2 four threads per channel, 3 two, whenever supported.
void split_mode_set(int mode);

// The S6 kernel parts (s6_part_*.cu): one element type and variant each,
// and each part's error word (read, and reset if clear).
#define SSM_S6_PART_DECL(NAME)                                        \
    cudaError_t launch_s6_##NAME(const S6Args &a, cudaStream_t stream); \
    cudaError_t s6_error_##NAME(unsigned *value, bool clear);
SSM_S6_PART_DECL(f32)
SSM_S6_PART_DECL(f32_ord)
SSM_S6_PART_DECL(f32_conv)
SSM_S6_PART_DECL(bf16)
SSM_S6_PART_DECL(bf16_ord)
SSM_S6_PART_DECL(bf16_conv)
SSM_S6_PART_DECL(f32_ckpt)
SSM_S6_PART_DECL(bf16_ckpt)
#undef SSM_S6_PART_DECL

// One decode step of S6 for every (batch, channel), state updated in place.
struct StepArgs {
    int Bsz, D, N;
    int dtype;     // 0 = float32, 1 = bf16
    int softplus;
    const void *x, *delta, *B, *C, *z;   // x, delta, z (Bsz, D); B, C (Bsz, N)
    const float *bias, *A, *Dskip;       // (D), (D, N), (D)
    float *state;                        // (Bsz, D, N) in and out
    void *out;                           // (Bsz, D)
};
cudaError_t launch_step(const StepArgs &a, cudaStream_t stream);

// Gradients of one single-direction S6 call (all float32).  dB, dC, dA, dD,
// dbias are accumulated with atomics and must be zeroed by the caller;
// dx, ddelta are written, or added to when accumulate is set (the second
// direction of a bidirectional backward).
struct BwdArgs {
    int Bsz, L, D, N;
    int dtype;      // 0 = float32, 1 = bf16 (inputs and dout)
    int softplus;
    int reverse;
    int accumulate;
    const void *x, *delta, *B, *C, *z, *dout;
    const float *bias, *A, *Dskip;
    float *dx, *ddelta, *dz, *dA, *dB, *dC, *dD, *dbias;
    float *ckpt;    // workspace: (Bsz, ceil(L / 4), D, NS) states entering each 4-step chunk,
                    // NS = N rounded up to 4, 8 or 16 (16-byte aligned)
    int ckpt_given; // 1: ckpt already holds them (written by the checkpointing forward scan),
                    // so the checkpoint pass is skipped
};
size_t bwd_workspace_bytes(int64_t Bsz, int64_t L, int64_t D, int64_t N);
cudaError_t launch_bwd(const BwdArgs &a, cudaStream_t stream);
// The backward sweep with each channel's 16 states over four threads
// (s6_bwd_split.cu; N == 16), from the checkpoints in a.ckpt.
cudaError_t launch_bwd_split(const BwdArgs &a, cudaStream_t stream);
// Whether the N = 16 backward takes it: not under layout mode 1 of the
// test setting (split_mode_set).
bool bwd_split_enabled();

// One SSD call.
struct SSDArgs {
    int Bsz, L, H, P, N, Q;
    int softplus;
    const void *x, *delta, *B, *C, *z;
    const float *bias, *A, *D;
    void *out;
    float *last_state;
    void *workspace;
};

size_t ssd_workspace_bytes(int64_t Bsz, int64_t L, int64_t H, int64_t P, int64_t N, int64_t Q);

// Test setting of the SSD kernel's bounded waits (process-wide): the poll
// limit of every pipeline wait (0 = the default) and a chunk whose dt the
// producer warp never signals (-1 = none), which makes the consumers' wait
// for it run out.
struct SSDStall {
    int withhold_chunk;
    unsigned wait_limit;
};
void ssd_stall_set(int withhold_chunk, unsigned wait_limit);
SSDStall ssd_stall_get();
cudaError_t launch_ssd(const SSDArgs &a, cudaStream_t stream);

// Device-side error words: the SSD kernel's (bounded waits that gave up)
// and the S6 kernels' (an out-of-range entry of a scan order).
cudaError_t read_and_clear_device_error(unsigned *value, cudaStream_t stream);
cudaError_t read_and_clear_s6_error(unsigned *value, cudaStream_t stream);

}  // namespace ssm
