// s6_part_f32_conv.cu -- S6 kernels for float32 data, conv input variant.
#include "s6_scan_impl.cuh"

SSM_S6_PART(f32_conv, float, 2)
