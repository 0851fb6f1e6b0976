// s6_part_bf16_ckpt.cu -- S6 kernels for bf16 data that also store the state entering
// every 4-step chunk (the checkpoints the backward pass reads).
#include "s6_scan_impl.cuh"

SSM_S6_PART(bf16_ckpt, __nv_bfloat16, 3)
