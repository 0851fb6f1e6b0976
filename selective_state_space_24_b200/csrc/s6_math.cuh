// s6_math.cuh -- the scalar transcendentals of the S6 step, shared by the
// scan kernels and the one-step decode kernel so that both round alike.
#pragma once

#include <cuda_runtime.h>

namespace ssm {

constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float ex2_mufu(float v)
{
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(v));
    return r;
}

__device__ __forceinline__ float rcp_mufu(float v)
{
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(v));
    return r;
}

// softplus(v) = max(v, 0) + log1p(e), e = exp(-|v|) in (0, 1], with
// log1p(e) = e q(e) and q a degree-7 minimax polynomial for log1p(e) / e on
// [0, 1] (relative error 3.4e-7 in fp32; coefficients from fit_polys.py).
__device__ __forceinline__ float softplus_f(float v)
{
    const float e = ex2_mufu(-fabsf(v) * kLog2e);
    float q = -8.539208211e-03f;
    q = fmaf(q, e, 4.408963397e-02f);
    q = fmaf(q, e, -1.076817140e-01f);
    q = fmaf(q, e, 1.774524152e-01f);
    q = fmaf(q, e, -2.449546307e-01f);
    q = fmaf(q, e, 3.327547908e-01f);
    q = fmaf(q, e, -4.999740422e-01f);
    q = fmaf(q, e, 9.999998212e-01f);
    return fmaf(e, q, fmaxf(v, 0.f));
}

// silu(z) = z sigmoid(z).  fp32 data: z / (1 + 2^(-z log2 e)) with the MUFU
// reciprocal.  bf16 data: z (1 + tanh(z / 2)) / 2 with the single MUFU
// tanh.approx (relative error 2^-11, below the bf16 output rounding).
template <typename T>
__device__ __forceinline__ float silu_f(float z)
{
    if (sizeof(T) == 2) {
        float t;
        asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * z));
        return 0.5f * z * (1.f + t);
    }
    return z * rcp_mufu(1.f + ex2_mufu(-z * kLog2e));
}

}  // namespace ssm
