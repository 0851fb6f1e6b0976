// s6_part_bf16_ord.cu -- S6 kernels for bf16 data, ordered / masked variant.
#include "s6_scan_impl.cuh"

SSM_S6_PART(bf16_ord, __nv_bfloat16, 1)
