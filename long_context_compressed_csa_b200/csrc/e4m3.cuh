// E4M3 conversion shared by the key quantiser and the E4M3 indexer scan.  Reading of the
// pages' low-precision indexer ("DeepSeek-V4 Hybrid Attention: CSA and HCA from Scratch",
// section 6.4): E4M3 codes with one fp32 scale per row = max|x| / 448; code = E4M3(x /
// scale), round to nearest even, saturating at the largest finite value.
#pragma once
#include <cuda_fp8.h>

#include "common.cuh"

namespace csa {

constexpr float kE4M3Max = 448.0f;

// Row scale from the row's largest magnitude (0 for an all-zero row).
CSA_DEV float e4m3_scale(float amax) { return __fdiv_rn(amax, kE4M3Max); }

// Codes of a, b (a in the lower byte), x / scale rounded to nearest even and saturated.
CSA_DEV uint32_t e4m3x2(float a, float b, float scale)
{
    if (scale == 0.f) return 0u;
    const float2 v = make_float2(__fdiv_rn(a, scale), __fdiv_rn(b, scale));
    return (uint32_t)__nv_cvt_float2_to_fp8x2(v, __NV_SATFINITE, __NV_E4M3);
}

}  // namespace csa
