// s6_part_bf16_conv.cu -- S6 kernels for bf16 data, conv input variant.
#include "s6_scan_impl.cuh"

SSM_S6_PART(bf16_conv, __nv_bfloat16, 2)
