// moe_mxfp8.cuh -- the MXFP8 shared-exponent rule, used by the MXFP8
// activation quantiser (moe_route.cu) and the MXFP8 GEMM1 tail
// (moe_gemm_tmx.cu).
#pragma once

#include <cstdint>

namespace moe {

// MXFP8 shared exponent of a block with maximum magnitude amax (OCP MX v1.0
// with E4M3 elements): X = floor(log2 amax) - 8, clamped to [-127, 127], and
// -127 for amax = 0 or a subnormal amax (whose floor(log2) is at most -127).
// Returns X; *scale = 2^X exactly (2^-127 is a subnormal float).
__device__ __forceinline__ int mx_e4m3_exponent(float amax, float* scale) {
  const int ef = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFFu);  // amax >= 0
  const int X = ef == 0 ? -127 : max(ef - 135, -127);
  *scale = X >= -126 ? __uint_as_float(static_cast<uint32_t>(X + 127) << 23) : __uint_as_float(0x00400000u);
  return X;
}

}  // namespace moe
