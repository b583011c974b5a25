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

#include <cuda_fp4.h>
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

// MXFP8 (OCP Microscaling v1.0): a 32-value block shares the scale 2^e,
// e = floor(log2(amax)) - 8 clamped to [-127, 127] (8: the exponent of
// e4m3's largest normal, 448 = 1.75 * 2^8), stored as the E8M0 byte e + 127;
// an all-zero block takes e = -127.  Codes are e4m3(v * 2^-e), round to
// nearest even, saturating: multiplying by a power of two is exact.
__device__ __forceinline__ int mx_block_exp(float amax) {
  if (amax == 0.f) return -127;
  const uint32_t bits = __float_as_uint(amax);
  const int ef = static_cast<int>((bits >> 23) & 0xFFu);
  const int fl = ef ? ef - 127 : (31 - __clz(static_cast<int>(bits & 0x7FFFFFu))) - 149;  // floor(log2(amax))
  const int e = fl - 8;
  return e < -127 ? -127 : (e > 127 ? 127 : e);
}

// 2^-e as an fp32 (exact; 2^-127 is subnormal).
__device__ __forceinline__ float mx_inv_scale(int e) {
  return e >= 127 ? __uint_as_float(0x00400000u) : __uint_as_float(static_cast<uint32_t>(127 - e) << 23);
}

// 8 bf16 values * inv -> 8 e4m3 codes.
__device__ __forceinline__ uint2 encode8_mx(const uint4& v, float inv) {
  uint2 out;
  out.x = e4m3x2(bf16_lo(v.x) * inv, bf16_hi(v.x) * inv) | (e4m3x2(bf16_lo(v.y) * inv, bf16_hi(v.y) * inv) << 16);
  out.y = e4m3x2(bf16_lo(v.z) * inv, bf16_hi(v.z) * inv) | (e4m3x2(bf16_lo(v.w) * inv, bf16_hi(v.w) * inv) << 16);
  return out;
}

// NVFP4: E2M1 values (magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6), one E4M3 scale
// per 16 values along K and an fp32 scale per row.  For a row with
// amax = max(max|x|, 1e-12f):  g = amax / 2688 (6 * 448, the largest E2M1
// value times E4M3's);  per block of 16 with maximum b:  s = e4m3(b / (6 g)),
// d = dec(s) * g,  code = e2m1(x / d) (+-0 when d is 0); every operation is
// one IEEE fp32 round-to-nearest step, E4M3 and E2M1 round to nearest even
// and saturate.  Two codes per byte, element 2i in the low nibble.
constexpr float kNvRowDiv = 2688.0f;

__device__ __forceinline__ uint32_t e2m1x2(float lo, float hi) {
  return static_cast<uint32_t>(__nv_cvt_float2_to_fp4x2(make_float2(lo, hi), __NV_E2M1, cudaRoundNearest));
}

// Value of an E4M3 code (exact in fp32).
__device__ __forceinline__ float e4m3_value(uint32_t code) {
  const __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(code), __NV_E4M3);
  return __half2float(__half(h));
}

// 16 bf16 values (two uint4) of one block -> 16 E2M1 codes in a uint2, given
// the block's fp32 divisor d (d == 0: every code +-0, keeping the sign).
__device__ __forceinline__ uint2 encode16_nv(const uint4& v0, const uint4& v1, float d) {
  const float f[16] = {bf16_lo(v0.x), bf16_hi(v0.x), bf16_lo(v0.y), bf16_hi(v0.y), bf16_lo(v0.z), bf16_hi(v0.z),
                       bf16_lo(v0.w), bf16_hi(v0.w), bf16_lo(v1.x), bf16_hi(v1.x), bf16_lo(v1.y), bf16_hi(v1.y),
                       bf16_lo(v1.z), bf16_hi(v1.z), bf16_lo(v1.w), bf16_hi(v1.w)};
  uint32_t b[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    if (d == 0.f) {
      b[i] = ((__float_as_uint(f[2 * i]) >> 31) << 3) | ((__float_as_uint(f[2 * i + 1]) >> 31) << 7);
    } else {
      b[i] = e2m1x2(__fdiv_rn(f[2 * i], d), __fdiv_rn(f[2 * i + 1], d));
    }
  }
  return make_uint2(b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24), b[4] | (b[5] << 8) | (b[6] << 16) | (b[7] << 24));
}

// Maximum over the 32 lanes of a warp.
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

}  // namespace
}  // namespace qgd
