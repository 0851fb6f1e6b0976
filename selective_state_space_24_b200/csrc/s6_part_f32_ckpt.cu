// s6_part_f32_ckpt.cu -- S6 kernels for float32 data that also store the state entering
// every 4-step chunk (the checkpoints the backward pass reads).
#include "s6_scan_impl.cuh"

SSM_S6_PART(f32_ckpt, float, 3)
