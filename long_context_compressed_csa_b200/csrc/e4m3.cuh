// E4M3 conversion shared by the key quantiser and the E4M3 indexer scan.  Reading of the
// pages' low-precision indexer ("DeepSeek-V4 Hybrid Attention: CSA and HCA from Scratch",
// section 6.4): E4M3 codes with one fp32 scale per row = max|x| / 448; code = E4M3(x *
// (448 / max|x|)), the product in fp32, rounded to nearest even, saturating at the
// largest finite value.
#pragma once
#include <cuda_fp4.h>
#include <cuda_fp8.h>

#include "common.cuh"

namespace csa {

constexpr float kE4M3Max = 448.0f;

// Dequantisation scale of a row from its largest magnitude (0 for an all-zero row).
CSA_DEV float e4m3_scale(float amax) { return __fdiv_rn(amax, kE4M3Max); }
// Quantisation factor 448 / amax (0 for an all-zero row, whose codes are then 0).
CSA_DEV float e4m3_factor(float amax) { return amax > 0.f ? __fdiv_rn(kE4M3Max, amax) : 0.f; }

// Codes of a, b (a in the lower byte): x * r rounded to nearest even and saturated.
CSA_DEV uint32_t e4m3x2(float a, float b, float r)
{
    const float2 v = make_float2(__fmul_rn(a, r), __fmul_rn(b, r));
    return (uint32_t)__nv_cvt_float2_to_fp8x2(v, __NV_SATFINITE, __NV_E4M3);
}

// E2M1 (FP4) keys: codes with one fp32 scale per row = max|x| / 6; code = E2M1(x * (6 /
// max|x|)), the product in fp32, rounded to nearest even and saturated at +-6.  Two codes
// per byte, the even column in the low nibble.
constexpr float kE2M1Max = 6.0f;

CSA_DEV float e2m1_scale(float amax) { return __fdiv_rn(amax, kE2M1Max); }
CSA_DEV float e2m1_factor(float amax) { return amax > 0.f ? __fdiv_rn(kE2M1Max, amax) : 0.f; }

// Codes of a, b (a in the low nibble): x * r rounded to nearest even and saturated.
CSA_DEV uint32_t e2m1x2(float a, float b, float r)
{
    const float2 v = make_float2(__fmul_rn(a, r), __fmul_rn(b, r));
    return (uint32_t)__nv_cvt_float2_to_fp4x2(v, __NV_E2M1, cudaRoundNearest);
}

}  // namespace csa
