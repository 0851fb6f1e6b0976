// s6_part_f32_ord.cu -- S6 kernels for float32 data, ordered / masked variant.
#include "s6_scan_impl.cuh"

SSM_S6_PART(f32_ord, float, 1)
