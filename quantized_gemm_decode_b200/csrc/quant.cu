// Dynamic quantizers: bf16 -> e4m3 / int8 codes plus fp32 scales.
//
// For a group g of values sharing one scale (a row, a 1x128 group, or a
// 128x128 block):  amax = max(max|x|, 1e-12f),  s = amax / qmax  (qmax 448
// for e4m3, 127 for int8), q = convert(x / s).  Both divisions are IEEE
// round-to-nearest (__fdiv_rn); the e4m3 conversion rounds to nearest even and
// saturates to +-448 (cvt.rn.satfinite), int8 rounds half to even and clamps
// to [-127, 127].  Formats and scale granularities: "Building a
// High-Performance and Portable vLLM Linear Backend with Helion", section "Put
// algorithm selection inside the search space".
//
// Each kernel loads its group once with 16-byte vector loads, keeps it in
// registers, reduces the absolute maximum with warp shuffles, and writes the
// codes with 8-byte stores.
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <stdlib.h>

#include <utility>

#include "qgd_internal.h"
#include "quantcore.cuh"

namespace qgd {
namespace {

// Maximum over the whole CTA (blockDim.x a multiple of 32, <= 1024).
__device__ __forceinline__ float block_max(float v, float* red) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  v = warp_max(v);
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (warp == 0) {
    float t = lane < static_cast<int>(blockDim.x >> 5) ? red[lane] : 0.f;
    t = warp_max(t);
    if (lane == 0) red[32] = t;
  }
  __syncthreads();
  return red[32];
}

// ---------------------------------------------------------------------------
// One CTA per row; each thread holds kVPT vectors of 8 values.
// ---------------------------------------------------------------------------
constexpr int kRowThreads = 512;

template <int kVPT, int kQType>
__global__ void __launch_bounds__(kRowThreads) quant_rows_kernel(const uint16_t* __restrict__ x, int K, int ldx,
                                                                 uint8_t* __restrict__ q, float* __restrict__ s) {
  __shared__ float red[33];
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");  // x comes from the preceding kernel
  const size_t row = blockIdx.x;
  const uint4* xr = reinterpret_cast<const uint4*>(x + row * static_cast<size_t>(ldx));
  uint2* qr = reinterpret_cast<uint2*>(q + row * K);
  const int nvec = K / 8;
  uint4 v[kVPT];
  float amax = 0.f;
#pragma unroll
  for (int j = 0; j < kVPT; ++j) {
    const int idx = threadIdx.x + j * kRowThreads;
    if (idx < nvec) {
      v[j] = __ldg(xr + idx);
      amax = fmaxf(amax, absmax8(v[j]));
    }
  }
  amax = fmaxf(block_max(amax, red), kAmaxFloor);
  const float sc = __fdiv_rn(amax, kQType == 0 ? kE4M3Max : kInt8Max);
  if (threadIdx.x == 0) s[row] = sc;
#pragma unroll
  for (int j = 0; j < kVPT; ++j) {
    const int idx = threadIdx.x + j * kRowThreads;
    if (idx < nvec) qr[idx] = encode8<kQType>(v[j], sc);
  }
}

// ---------------------------------------------------------------------------
// 1x128 groups: a half-warp per group, 8 values per lane.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) quant_group128_kernel(const uint16_t* __restrict__ x, int M, int K, int ldx,
                                                             uint8_t* __restrict__ q, float* __restrict__ s) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");  // x comes from the preceding kernel
  const int KB = K / 128;
  const long long g = static_cast<long long>(blockIdx.x) * 16 + (threadIdx.x >> 4);
  const int sub = threadIdx.x & 15;
  const bool valid = g < static_cast<long long>(M) * KB;
  const long long gg = valid ? g : 0;
  const long long m = gg / KB, kb = gg % KB;
  const size_t off = static_cast<size_t>(m) * K + static_cast<size_t>(kb) * 128 + sub * 8;
  const size_t xoff = static_cast<size_t>(m) * ldx + static_cast<size_t>(kb) * 128 + sub * 8;
  uint4 v = make_uint4(0, 0, 0, 0);
  if (valid) v = __ldg(reinterpret_cast<const uint4*>(x + xoff));
  float amax = absmax8(v);
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  amax = fmaxf(amax, kAmaxFloor);
  const float sc = __fdiv_rn(amax, kE4M3Max);
  if (valid) {
    *reinterpret_cast<uint2*>(q + off) = encode8<0>(v, sc);
    if (sub == 0) s[static_cast<size_t>(m) * KB + kb] = sc;
  }
}

// ---------------------------------------------------------------------------
// MXFP8 blocks of 32 along a row: four lanes per block, 8 values per lane.
// x rows are ldx elements apart; q [rows][K] codes, s [rows][K/32] E8M0.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) quant_mx_kernel(const uint16_t* __restrict__ x, int rows, int K, int ldx,
                                                       uint8_t* __restrict__ q, uint8_t* __restrict__ s) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");  // x comes from the preceding kernel
  const int KB = K / 32;
  const long long b = static_cast<long long>(blockIdx.x) * 64 + (threadIdx.x >> 2);  // block index (row, kb)
  const int sub = threadIdx.x & 3;
  const bool valid = b < static_cast<long long>(rows) * KB;
  const long long bb = valid ? b : 0;
  const long long r = bb / KB, kb = bb % KB;
  uint4 v = make_uint4(0, 0, 0, 0);
  if (valid) v = __ldg(reinterpret_cast<const uint4*>(x + static_cast<size_t>(r) * ldx + kb * 32 + sub * 8));
  float amax = absmax8(v);
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
  const int e = mx_block_exp(amax);
  if (valid) {
    *reinterpret_cast<uint2*>(q + static_cast<size_t>(r) * K + kb * 32 + sub * 8) = encode8_mx(v, mx_inv_scale(e));
    if (sub == 0) s[static_cast<size_t>(r) * KB + kb] = static_cast<uint8_t>(e + 127);
  }
}

// ---------------------------------------------------------------------------
// NVFP4 rows (activations or weights): one CTA of 256 threads per row, each
// thread holding kBPT blocks of 16 values (two 16-byte vectors each) in
// registers: the row maximum over the CTA, then per block its maximum, E4M3
// scale and 16 E2M1 codes.  x rows are ldx elements apart; q [rows][K/2]
// packed codes, s [rows][K/16] E4M3 scales, g [rows] fp32 row scales.
// ---------------------------------------------------------------------------
constexpr int kNvThreads = 256;

template <int kBPT>
__global__ void __launch_bounds__(kNvThreads) quant_nv_kernel(const uint16_t* __restrict__ x, int K, int ldx,
                                                              uint8_t* __restrict__ q, uint8_t* __restrict__ s,
                                                              float* __restrict__ g) {
  __shared__ float red[33];
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");  // x comes from the preceding kernel
  const size_t row = blockIdx.x;
  const uint4* xr = reinterpret_cast<const uint4*>(x + row * static_cast<size_t>(ldx));
  const int nb = K / 16;
  uint4 v[kBPT][2];
  float bm[kBPT];
  float amax = 0.f;
#pragma unroll
  for (int j = 0; j < kBPT; ++j) {
    const int b = threadIdx.x + j * kNvThreads;
    bm[j] = 0.f;
    if (b < nb) {
      v[j][0] = __ldg(xr + 2 * b);
      v[j][1] = __ldg(xr + 2 * b + 1);
      bm[j] = fmaxf(absmax8(v[j][0]), absmax8(v[j][1]));
      amax = fmaxf(amax, bm[j]);
    }
  }
  amax = fmaxf(block_max(amax, red), kAmaxFloor);
  const float gr = __fdiv_rn(amax, kNvRowDiv);
  const float six_g = __fmul_rn(6.0f, gr);
  if (threadIdx.x == 0) g[row] = gr;
  uint2* qr = reinterpret_cast<uint2*>(q + row * static_cast<size_t>(K / 2));
  uint8_t* sr = s + row * static_cast<size_t>(nb);
#pragma unroll
  for (int j = 0; j < kBPT; ++j) {
    const int b = threadIdx.x + j * kNvThreads;
    if (b < nb) {
      const uint32_t sc = e4m3x2(__fdiv_rn(bm[j], six_g), 0.f) & 0xFFu;
      const float d = __fmul_rn(e4m3_value(sc), gr);
      qr[b] = encode16_nv(v[j][0], v[j][1], d);
      sr[b] = static_cast<uint8_t>(sc);
    }
  }
}

// ---------------------------------------------------------------------------
// 128x128 weight blocks: one CTA of 256 threads per block, 8 vectors each.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) quant_block128_kernel(const uint16_t* __restrict__ w, int K,
                                                             uint8_t* __restrict__ q, float* __restrict__ s) {
  __shared__ float red[33];
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int nb = blockIdx.y, kb = blockIdx.x, KB = gridDim.x;
  uint4 v[8];
  float amax = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int t = threadIdx.x + j * 256;  // 0..2047: row = t/16, vector = t%16
    const size_t off = static_cast<size_t>(nb * 128 + t / 16) * K + kb * 128 + (t % 16) * 8;
    v[j] = __ldg(reinterpret_cast<const uint4*>(w + off));
    amax = fmaxf(amax, absmax8(v[j]));
  }
  amax = fmaxf(block_max(amax, red), kAmaxFloor);
  const float sc = __fdiv_rn(amax, kE4M3Max);
  if (threadIdx.x == 0) s[static_cast<size_t>(nb) * KB + kb] = sc;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int t = threadIdx.x + j * 256;
    const size_t off = static_cast<size_t>(nb * 128 + t / 16) * K + kb * 128 + (t % 16) * 8;
    *reinterpret_cast<uint2*>(q + off) = encode8<0>(v[j], sc);
  }
}

// Launch with a programmatic dependency on the preceding kernel (unless
// QGD_PDL=0): the kernel may start early and waits in griddepcontrol.wait.
template <typename... Params, typename... Args>
cudaError_t launch_q(void (*kernel)(Params...), dim3 grid, dim3 block, cudaStream_t stream, Args&&... args) {
  const bool pdl = pdl_enabled();
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  return e != cudaSuccess ? e : cudaGetLastError();
}

template <int kQType>
cudaError_t launch_rows_q(const uint16_t* x, int rows, int K, int ldx, void* q, float* s, cudaStream_t st) {
  const int nvec = K / 8;
  const int vpt = (nvec + kRowThreads - 1) / kRowThreads;
  uint8_t* qb = static_cast<uint8_t*>(q);
  const dim3 grid(rows), block(kRowThreads);
  if (vpt <= 1) return launch_q(quant_rows_kernel<1, kQType>, grid, block, st, x, K, ldx, qb, s);
  if (vpt <= 2) return launch_q(quant_rows_kernel<2, kQType>, grid, block, st, x, K, ldx, qb, s);
  if (vpt <= 4) return launch_q(quant_rows_kernel<4, kQType>, grid, block, st, x, K, ldx, qb, s);
  if (vpt <= 8) return launch_q(quant_rows_kernel<8, kQType>, grid, block, st, x, K, ldx, qb, s);
  if (vpt <= 16) return launch_q(quant_rows_kernel<16, kQType>, grid, block, st, x, K, ldx, qb, s);
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_quant_rows(const uint16_t* x, int rows, int K, int ldx, int qtype, void* q, float* s,
                              cudaStream_t stream) {
  return qtype == 0 ? launch_rows_q<0>(x, rows, K, ldx, q, s, stream)
                    : launch_rows_q<1>(x, rows, K, ldx, q, s, stream);
}

cudaError_t launch_quant_group128(const uint16_t* x, int M, int K, int ldx, uint8_t* q, float* s,
                                  cudaStream_t stream) {
  const long long groups = static_cast<long long>(M) * (K / 128);
  const unsigned blocks = static_cast<unsigned>((groups + 15) / 16);
  return launch_q(quant_group128_kernel, dim3(blocks), dim3(256), stream, x, M, K, ldx, q, s);
}

cudaError_t launch_quant_mx(const uint16_t* x, int rows, int K, int ldx, uint8_t* q, uint8_t* s,
                            cudaStream_t stream) {
  const long long blocks = static_cast<long long>(rows) * (K / 32);
  const unsigned grid = static_cast<unsigned>((blocks + 63) / 64);
  return launch_q(quant_mx_kernel, dim3(grid), dim3(256), stream, x, rows, K, ldx, q, s);
}

cudaError_t launch_quant_nv(const uint16_t* x, int rows, int K, int ldx, uint8_t* q, uint8_t* s, float* g,
                            cudaStream_t stream) {
  const int per = (K / 16 + kNvThreads - 1) / kNvThreads;  // blocks of 16 per thread (K <= 65536: <= 16)
  const dim3 grid(static_cast<unsigned>(rows)), block(kNvThreads);
  if (per <= 1) return launch_q(quant_nv_kernel<1>, grid, block, stream, x, K, ldx, q, s, g);
  if (per <= 2) return launch_q(quant_nv_kernel<2>, grid, block, stream, x, K, ldx, q, s, g);
  if (per <= 4) return launch_q(quant_nv_kernel<4>, grid, block, stream, x, K, ldx, q, s, g);
  if (per <= 8) return launch_q(quant_nv_kernel<8>, grid, block, stream, x, K, ldx, q, s, g);
  return launch_q(quant_nv_kernel<16>, grid, block, stream, x, K, ldx, q, s, g);
}

cudaError_t launch_quant_block128(const uint16_t* w, int N, int K, uint8_t* q, float* s, cudaStream_t stream) {
  const dim3 grid(K / 128, N / 128);
  return launch_q(quant_block128_kernel, grid, dim3(256), stream, w, K, q, s);
}

}  // namespace qgd
