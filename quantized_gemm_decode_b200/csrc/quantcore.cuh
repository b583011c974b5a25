// Conversion steps shared by the stand-alone quantizers (quant.cu) and the
// GEMM that quantizes its own activations (gemm.cu), so both produce the same
// codes and scales bit for bit.  For a group g sharing one scale:
//   amax = max(max|x|, 1e-12f),  s = amax / qmax (448 for e4m3, 127 for
//   int8, IEEE round-to-nearest division),  q = convert(x / s) (correctly
//   rounded fp32 quotient; e4m3: round to nearest even, saturate to +-448;
//   int8: round half to even, clamp to [-127, 127]).
// Formats and scale granularities: "Building a High-Performance and Portable
// vLLM Linear Backend with Helion", section "Put algorithm selection inside
// the search space".
#pragma once

#include <cuda_fp8.h>
#include <stdint.h>

namespace qgd {
namespace {

constexpr float kE4M3Max = 448.0f;
constexpr float kInt8Max = 127.0f;
constexpr float kAmaxFloor = 1e-12f;

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ float absmax8(const uint4& v) {
  float m = fmaxf(fabsf(bf16_lo(v.x)), fabsf(bf16_hi(v.x)));
  m = fmaxf(m, fmaxf(fabsf(bf16_lo(v.y)), fabsf(bf16_hi(v.y))));
  m = fmaxf(m, fmaxf(fabsf(bf16_lo(v.z)), fabsf(bf16_hi(v.z))));
  m = fmaxf(m, fmaxf(fabsf(bf16_lo(v.w)), fabsf(bf16_hi(v.w))));
  return m;
}

__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  return static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3));
}

__device__ __forceinline__ uint32_t int8_code(float v) {
  int q = __float2int_rn(v);
  q = q > 127 ? 127 : (q < -127 ? -127 : q);
  return static_cast<uint32_t>(q) & 0xFFu;
}

// 8 bf16 values (one uint4) / s -> 8 codes packed in a uint2.
template <int kQType>
__device__ __forceinline__ uint2 encode8(const uint4& v, float s) {
  const float f[8] = {bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y),
                      bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w)};
  float d[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) d[i] = __fdiv_rn(f[i], s);
  uint2 out;
  if constexpr (kQType == 0) {
    out.x = e4m3x2(d[0], d[1]) | (e4m3x2(d[2], d[3]) << 16);
    out.y = e4m3x2(d[4], d[5]) | (e4m3x2(d[6], d[7]) << 16);
  } else {
    out.x = int8_code(d[0]) | (int8_code(d[1]) << 8) | (int8_code(d[2]) << 16) | (int8_code(d[3]) << 24);
    out.y = int8_code(d[4]) | (int8_code(d[5]) << 8) | (int8_code(d[6]) << 16) | (int8_code(d[7]) << 24);
  }
  return out;
}

// Maximum over the 32 lanes of a warp.
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

}  // namespace
}  // namespace qgd
