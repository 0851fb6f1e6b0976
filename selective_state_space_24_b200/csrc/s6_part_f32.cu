// s6_part_f32.cu -- S6 kernels for float32 data, plain variant.
#include "s6_scan_impl.cuh"

SSM_S6_PART(f32, float, 0)
