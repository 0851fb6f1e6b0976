// s6_part_bf16.cu -- S6 kernels for bf16 data, plain variant.
#include "s6_scan_impl.cuh"

SSM_S6_PART(bf16, __nv_bfloat16, 0)
