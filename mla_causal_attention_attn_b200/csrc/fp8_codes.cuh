// fp8_codes.cuh -- the dynamic e4m3 activation quantisation of one 128-feature
// group (the checkpoint's FP8 format, config.json's quantization_config on page
// "Kimi K2 · Transformer blocks": e4m3, 128 x 128 weight blocks, dynamic
// activation scales): scale = amax / 448 (1 for an all-zero group), code =
// the nearest e4m3 value of x / scale.
#pragma once

#include <cstdint>

#include <cuda_fp8.h>

namespace mla {

constexpr float kE4m3Max = 448.f;  // largest finite e4m3 value

__device__ __forceinline__ float group_scale(float amax) {
  return amax > 0.f ? __fdiv_rn(amax, kE4m3Max) : 1.f;
}

// e4m3 code of x / s: fp32 quotient rounded to nearest, then the nearest
// e4m3 value (ties to even), saturating at +-448.
__device__ __forceinline__ uint32_t e4m3_code(float x, float s) {
  return uint32_t(__nv_cvt_float_to_fp8(__fdiv_rn(x, s), __NV_SATFINITE, __NV_E4M3));
}

}  // namespace mla
