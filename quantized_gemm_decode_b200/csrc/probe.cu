// Dense tensor-core peak probe: back-to-back tcgen05.mma from operands held in
// shared memory, one CTA per SM, no global-memory traffic.  The timed FLOP
// rate of this kernel is the e4m3 / int8 denominator of the large-M
// roofline fraction, measured on the part itself rather than taken from a
// data sheet.
#include "qgd_internal.h"
#include "sm100.cuh"

namespace qgd {

__device__ unsigned int g_probe_error = 0;

namespace {

constexpr uint32_t kProbeN = 256;                  // MMA N (B operand rows)
constexpr uint32_t kProbeABytes = 128 * kTileK;    // 128 x 128 B
constexpr uint32_t kProbeBBytes = kProbeN * kTileK;  // 256 x 128 B
constexpr uint32_t kProbeCols = 256;               // one fp32/s32 accumulator of 128 x 256

__device__ __forceinline__ uint8_t* probe_align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~static_cast<uintptr_t>(1023));
}

// One thread issues `iters` groups of four K=32 MMAs (128 x 256 x 128 per
// group) into one TMEM accumulator, commits once and waits (bounded).
template <bool kInt8>
__global__ void __launch_bounds__(128, 1) mma_peak_kernel(int iters) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = probe_align1024(smem_raw);
  uint8_t* a = base;
  uint8_t* b = base + kProbeABytes;
  uint64_t* done = reinterpret_cast<uint64_t*>(b + kProbeBBytes);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  // zero operands: the product is exact and the accumulator stays finite
  for (uint32_t i = threadIdx.x; i < (kProbeABytes + kProbeBBytes) / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(base)[i] = make_uint4(0u, 0u, 0u, 0u);
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // generic writes -> tensor core reads
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    mbar_init(done, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kProbeCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (threadIdx.x == 0) {
    constexpr uint32_t idesc = idesc_mma(kInt8 ? 2 : 1, kInt8 ? 1 : 0, 128, kProbeN);
    const uint64_t ad = sdesc_kmajor_sw128(smem_u32(a));
    const uint64_t bd = sdesc_kmajor_sw128(smem_u32(b));
    for (int it = 0; it < iters; ++it) {
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_issue<kInt8>(tmem, ad + static_cast<uint64_t>((kk * 32) >> 4), bd + static_cast<uint64_t>((kk * 32) >> 4),
                         idesc, (it | kk) != 0);
    }
    mma_commit(done);
    if (!mbar_wait(done, 0)) {
      atomicCAS(&g_probe_error, 0u, static_cast<unsigned int>(kErrWaitDrain));
      // the MMAs must finish before TMEM is released: wait once more, bounded
      if (!mbar_wait(done, 0)) atomicCAS(&g_probe_error, 0u, static_cast<unsigned int>(kErrWaitDrain));
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kProbeCols);
  }
}

// Ring probe: groups of four K=32 e4m3 MMAs (128 x N x 128 per group) into
// kSlots TMEM slots in turn, each group committed to its slot's barrier.
// kWait: before reusing a slot, the issuing thread waits for that slot's
// previous group to complete (the hand-off a kernel with a ring of
// accumulators makes); otherwise it never waits.
template <uint32_t kN, uint32_t kSlots, bool kWait>
__global__ void __launch_bounds__(128, 1) mma_ring_kernel(int iters) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = probe_align1024(smem_raw);
  uint8_t* a = base;
  uint8_t* b = base + kProbeABytes;
  uint64_t* bar = reinterpret_cast<uint64_t*>(b + kN * kTileK);  // kSlots slot barriers, then `done`
  uint64_t* done = bar + kSlots;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  for (uint32_t i = threadIdx.x; i < (kProbeABytes + kN * kTileK) / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(base)[i] = make_uint4(0u, 0u, 0u, 0u);
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    for (uint32_t s = 0; s < kSlots; ++s) mbar_init(&bar[s], 1);
    mbar_init(done, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kN * kSlots);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (threadIdx.x == 0) {
    constexpr uint32_t idesc = idesc_mma(1, 0, 128, kN);
    const uint64_t ad = sdesc_kmajor_sw128(smem_u32(a));
    const uint64_t bd = sdesc_kmajor_sw128(smem_u32(b));
    for (int it = 0; it < iters; ++it) {
      const uint32_t s = static_cast<uint32_t>(it) % kSlots;
      if (kWait && it >= static_cast<int>(kSlots) &&
          !mbar_wait(&bar[s], ((static_cast<uint32_t>(it) / kSlots) - 1) & 1)) {
        atomicCAS(&g_probe_error, 0u, static_cast<unsigned int>(kErrWaitMma));
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_issue<false>(tmem + s * kN, ad + static_cast<uint64_t>((kk * 32) >> 4),
                         bd + static_cast<uint64_t>((kk * 32) >> 4), idesc, kk != 0);
      mma_commit(&bar[s]);
    }
    mma_commit(done);
    if (!mbar_wait(done, 0)) {
      atomicCAS(&g_probe_error, 0u, static_cast<unsigned int>(kErrWaitDrain));
      if (!mbar_wait(done, 0)) atomicCAS(&g_probe_error, 0u, static_cast<unsigned int>(kErrWaitDrain));
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kN * kSlots);
  }
}

template <uint32_t kN, uint32_t kSlots, bool kWait>
cudaError_t launch_ring(int iters, int ctas, cudaStream_t stream) {
  // operands, then (kSlots + 1) barriers and the TMEM address (<= 44 bytes), plus alignment slack
  static_assert((kSlots + 1) * 8 + 4 <= 64, "barrier area");
  const size_t smem = kProbeABytes + kN * kTileK + 64 + 1024;
  cudaError_t e = cudaFuncSetAttribute(mma_ring_kernel<kN, kSlots, kWait>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  mma_ring_kernel<kN, kSlots, kWait><<<ctas, 128, smem, stream>>>(iters);
  return cudaGetLastError();
}

template <bool kWait>
cudaError_t launch_ring_w(int n, int slots, int iters, int ctas, cudaStream_t stream) {
  if (n == 128 && slots == 1) return launch_ring<128, 1, kWait>(iters, ctas, stream);
  if (n == 128 && slots == 2) return launch_ring<128, 2, kWait>(iters, ctas, stream);
  if (n == 128 && slots == 4) return launch_ring<128, 4, kWait>(iters, ctas, stream);
  if (n == 256 && slots == 1) return launch_ring<256, 1, kWait>(iters, ctas, stream);
  if (n == 256 && slots == 2) return launch_ring<256, 2, kWait>(iters, ctas, stream);
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_mma_ring_probe(int n, int slots, bool wait, int iters, int ctas, cudaStream_t stream) {
  return wait ? launch_ring_w<true>(n, slots, iters, ctas, stream)
              : launch_ring_w<false>(n, slots, iters, ctas, stream);
}

size_t mma_probe_smem_bytes() { return kProbeABytes + kProbeBBytes + 64 + 1024; }

double mma_probe_flops(int iters, int ctas) {
  return 2.0 * 128.0 * kProbeN * kTileK * static_cast<double>(iters) * ctas;
}

cudaError_t launch_mma_probe(int qtype, int iters, int ctas, cudaStream_t stream) {
  const size_t smem = mma_probe_smem_bytes();
  cudaError_t e;
  if (qtype == 1) {
    e = cudaFuncSetAttribute(mma_peak_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    mma_peak_kernel<true><<<ctas, 128, smem, stream>>>(iters);
  } else {
    e = cudaFuncSetAttribute(mma_peak_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    mma_peak_kernel<false><<<ctas, 128, smem, stream>>>(iters);
  }
  return cudaGetLastError();
}

cudaError_t read_probe_error(unsigned int* code) { return cudaMemcpyFromSymbol(code, g_probe_error, sizeof(unsigned int)); }

cudaError_t clear_probe_error() {
  const unsigned int z = 0;
  return cudaMemcpyToSymbol(g_probe_error, &z, sizeof(unsigned int));
}

}  // namespace qgd
