// Quantized GEMM kernels for sm_100a: TMA-fed shared-memory ring ->
// tcgen05.mma (kind::f8f6f4 for e4m3, kind::i8 for int8) -> TMEM accumulator
// -> scale epilogue.  Two orientations:
//
//   Swap-AB   D^T[n, m] = sum_k Wq[n,k] Xq[m,k]: a CTA owns 128 weight rows
//             (the MMA's M) and all M tokens (the MMA's N, padded to 16, 32,
//             64 or 128; at most 32 for Block_FP8).  The weight stream is the
//             whole cost at decode sizes.
//   Standard  D[m, n] = sum_k Xq[m,k] Wq[n,k]: a CTA owns a 128-token x
//             tile_n-column output tile; the large-M path.
//
// Either one runs with split_k CTAs along K (Split-K).  Partials are added
// by the last CTA to arrive at a tile (in split order, deterministic), by a
// second kernel (two-pass, deterministic), atomically, or -- Swap-AB -- by
// the splits of a tile launched as one thread-block cluster, through
// distributed shared memory (in split order, deterministic).
//
// Algorithm variants and their roles follow "Building a High-Performance and
// Portable vLLM Linear Backend with Helion" (section "Como se implementa el
// kernel?" and its matmul listing); the formats follow its scope list.
//
// Warp roles (192 threads): warp 0 issues TMA loads, warp 1 owns TMEM and
// issues MMAs, warps 2-5 drain the accumulator (warp w reads TMEM lanes
// 32*(w%4) .. +31).  Every mbarrier wait is bounded; a wait that gives up
// records an error code, and the CTA unwinds, drains what it issued, frees
// TMEM and exits.
#include <cuda_bf16.h>

#include <utility>

#include "qgd_internal.h"
#include "quantcore.cuh"
#include "sm100.cuh"

namespace qgd {

// First error code recorded by any kernel of this library on this device.
__device__ unsigned int g_device_error = 0;

namespace {

__device__ __forceinline__ void record_error(unsigned int code) { atomicCAS(&g_device_error, 0u, code); }

// Developer timeline of the Swap-AB kernel: with -DQGD_TRACE each CTA stamps
// %globaltimer at up to 16 points (entry, set-up done, first loads issued,
// first stage landed, last MMA committed, last accumulator read, epilogue
// done, exit, the steps of the last segment's output, and the weight loads
// issued / the preceding kernel's completion seen before the first loads);
// qgd_debug_trace() copies the stamps out.  Compiled out otherwise.
// Launches are kept in a ring of kTraceLaunches (by the call's trace tag), so
// a chain of consecutive calls can be read back on one time line; slot 15
// holds the SM the CTA ran on.
#ifdef QGD_TRACE
constexpr int kTraceCtas = 4096;
constexpr int kTraceSlots = 16;
constexpr int kTraceLaunches = 8;
__device__ unsigned long long g_trace[kTraceLaunches * kTraceCtas * kTraceSlots];
__device__ __forceinline__ unsigned long long* trace_row(const GemmArgs& a) {
  const unsigned cta = blockIdx.x + blockIdx.y * gridDim.x;
  if (cta >= kTraceCtas) return nullptr;
  return g_trace + (static_cast<size_t>(a.trace_tag % kTraceLaunches) * kTraceCtas + cta) * kTraceSlots;
}
#define QGD_STAMP(slot)                                 \
  do {                                                  \
    unsigned long long* r_ = trace_row(a);              \
    if (r_) r_[(slot)] = globaltimer_ns();              \
    if (r_ && (slot) == 0) {                            \
      unsigned smid_;                                   \
      asm volatile("mov.u32 %0, %%smid;" : "=r"(smid_)); \
      r_[15] = smid_;                                   \
    }                                                   \
  } while (0)
#else
#define QGD_STAMP(slot) \
  do {                  \
  } while (0)
#endif

constexpr uint32_t kBarBytes = 1024;  // mbarriers, flags and staged token scales, after the rings

struct SmemCtl {
  uint64_t full[kMaxStages];
  uint64_t xfull[kMaxStages];  // fused Swap-AB: the stage's activation codes are written (one arrival per warp)
  uint64_t empty[kMaxStages];
  uint64_t tfull[4];
  uint64_t tempty[4];
  uint64_t accfull;
  uint64_t drain;
  uint64_t recv_bar;  // Swap-AB cluster Split-K: peers' partial rows have landed here
  uint32_t tmem_base;
  int abort_flag;
  int last_flag;
  int epi_ok;
  float sx_s[128];  // Swap-AB, per-token formats: the M token scales, staged once
};
static_assert(sizeof(SmemCtl) <= kBarBytes, "control block too large");

// Fused Swap-AB: shared memory after the control block (and the cluster
// receive buffer) for the per-row maxima of the per-token pre-pass (128 rows
// x 4 warps) and a ring of Block_FP8 group scales, kScaleRing K slices deep
// (the quantizer runs at most (stages + 1) x 2 slices ahead of the promotion).
constexpr int kScaleRing = 36;
constexpr uint32_t kFusedBytes = 128 * 4 * 4 + kScaleRing * 32 * 4;

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  const uint32_t a = smem_u32(p);
  return p + (((a + 1023u) & ~1023u) - a);
}

// Wait on an mbarrier with the whole warp and agree on the outcome.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity) {
  const bool ok = mbar_wait(bar, parity);
  return __all_sync(0xffffffffu, ok);
}

// Hand a TMEM accumulator back: one arrival per warp (the barrier counts
// warps), after every lane's reads have completed and been fenced.  One
// shared-memory atomic per warp instead of per thread: with 128-512 epilogue
// threads arriving on one barrier per K block, the arrivals themselves had
// become the Block_FP8 promotion's bottleneck.
__device__ __forceinline__ void warp_release(uint64_t* bar) {
  tc_fence_before();
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

template <int kCols>
__device__ __forceinline__ void tmem_load_cols(uint32_t taddr, uint32_t (&r)[kCols]) {
  static_assert(kCols % 16 == 0, "columns come in groups of 16");
#pragma unroll
  for (int c = 0; c < kCols / 16; ++c) {
    uint32_t t[16];
    tmem_ld16(taddr + c * 16, t);
#pragma unroll
    for (int j = 0; j < 16; ++j) r[c * 16 + j] = t[j];
  }
}

__device__ __forceinline__ uint16_t bf16_bits(float v) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(v));
}

// Accumulator word (fp32 bits, or int32 for INT8) -> final fp32 value.
template <int kFmt>
__device__ __forceinline__ float scale_out(uint32_t accbits, int m, int n, const GemmArgs& a) {
  if constexpr (kFmt == kFmtBlock || kFmt == kFmtMX) {
    return __uint_as_float(accbits);  // scales were applied per K block (MXFP8: by the tensor core)
  } else if constexpr (kFmt == kFmtINT8) {
    return (static_cast<float>(static_cast<int32_t>(accbits)) * __ldg(a.sx + m)) * __ldg(a.sw + n);
  } else {
    return (__uint_as_float(accbits) * __ldg(a.sx + m)) * __ldg(a.sw + n);
  }
}

template <int kFmt>
__device__ __forceinline__ uint32_t add_acc(uint32_t x, uint32_t y) {
  if constexpr (kFmt == kFmtINT8)
    return static_cast<uint32_t>(static_cast<int32_t>(x) + static_cast<int32_t>(y));
  else
    return __float_as_uint(__uint_as_float(x) + __uint_as_float(y));
}

template <int kFmt>
__device__ __forceinline__ void atomic_acc(void* base, size_t idx, uint32_t v) {
  if constexpr (kFmt == kFmtINT8)
    atomicAdd(static_cast<int*>(base) + idx, static_cast<int>(v));
  else
    atomicAdd(static_cast<float*>(base) + idx, __uint_as_float(v));
}

// Store one finished element (y in bf16, or the raw accumulator).
template <int kFmt>
__device__ __forceinline__ void store_final(uint32_t accbits, int m, int n, const GemmArgs& a) {
  const size_t idx = static_cast<size_t>(m) * a.N + n;
  if (a.raw) {
    static_cast<uint32_t*>(a.raw)[idx] = accbits;
  } else {
    a.y[idx] = bf16_bits(scale_out<kFmt>(accbits, m, n, a));
  }
}

// Swap-AB output of one element from on-chip operands only: token scale from
// shared memory, channel scale prefetched into a register.  Same arithmetic
// as scale_out: ((acc * sx[m]) * sw[n]) for the per-token formats.
template <int kFmt>
__device__ __forceinline__ void store_swap_final(uint32_t accbits, int m, int n, float swv, const float* sx_s,
                                                 const GemmArgs& a) {
  const size_t idx = static_cast<size_t>(m) * a.N + n;
  if (a.raw) {
    static_cast<uint32_t*>(a.raw)[idx] = accbits;
    return;
  }
  uint16_t v;
  if constexpr (kFmt == kFmtBlock || kFmt == kFmtMX) {
    v = bf16_bits(__uint_as_float(accbits));
  } else if constexpr (kFmt == kFmtINT8) {
    v = bf16_bits((static_cast<float>(static_cast<int32_t>(accbits)) * sx_s[m]) * swv);
  } else {
    v = bf16_bits((__uint_as_float(accbits) * sx_s[m]) * swv);
  }
  if (a.tp_ranks == 0) {
    a.y[idx] = v;
  } else {
    // column-parallel: this element of the full output, on every rank
    const size_t full = static_cast<size_t>(m) * a.tp_ldy + a.tp_col0 + n;
    for (int r = 0; r < a.tp_ranks; ++r) a.tp_y[r][full] = v;
  }
}

// Column-parallel completion: after every CTA's output is out, the last CTA
// to finish advances this rank's call counter (word `ranks` of its own flag
// array; 0 is skipped when it wraps) and publishes the new value in entry
// `rank` of every rank's flag array (system scope: the readers are other
// GPUs).  The counter lives on the device, so a captured graph advances it on
// every replay.  Called by all threads of a CTA at its end.
__device__ __forceinline__ void tp_signal_done(const GemmArgs& a) {
  if (a.tp_ranks == 0) return;
  __syncthreads();  // every thread's output stores, to every rank, precede thread 0's fence
  if (threadIdx.x == 0) {
    const unsigned total = gridDim.x * gridDim.y * gridDim.z;
    unsigned prev;
    // the arrival releases this CTA's stores (the barrier above ordered every
    // thread's before it); the last arrival acquires every other CTA's, and its
    // system-scope releases below pass them all on to the other ranks
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(prev) : "l"(a.tp_done) : "memory");
    if (prev == total - 1) {
      unsigned* own = a.tp_flag[a.tp_rank];
      unsigned epoch = *reinterpret_cast<volatile unsigned*>(own + a.tp_ranks) + 1u;
      if (epoch == 0u) epoch = 1u;
      own[a.tp_ranks] = epoch;  // read by this rank's wait, after this kernel in stream order
      // one system-scope fence releases the output to every rank's flag (a
      // fence followed by strong stores); a release per store costs a fence each
      asm volatile("fence.acq_rel.sys;" ::: "memory");
      for (int r = 0; r < a.tp_ranks; ++r)
        asm volatile("st.relaxed.sys.global.u32 [%0], %1;" ::"l"(a.tp_flag[r] + a.tp_rank), "r"(epoch)
                     : "memory");
      *a.tp_done = 0u;  // ready for the next call
    }
  }
}

__device__ __forceinline__ uint32_t ldcg_u32(const void* p) {
  return __ldcg(static_cast<const unsigned int*>(p));
}

// Teardown shared by both kernels: drain on abort, then free TMEM.
__device__ __forceinline__ void teardown(SmemCtl* ctl, int warp, int lane, int issued, int stages,
                                         uint32_t tmem, uint32_t ncols) {
  tc_fence_before();
  __syncthreads();
  if (ctl->abort_flag) {
    if (warp == 0 && lane == 0) {
      // the last load issued into each stage must land before the CTA exits
      for (int i = issued > stages ? issued - stages : 0; i < issued; ++i) {
        if (!mbar_wait(&ctl->full[i % stages], (i / stages) & 1)) {
          record_error(kErrWaitDrain);
          break;
        }
      }
    }
    if (warp == 1 && lane == 0) {
      mma_commit(&ctl->drain);  // arrives once every MMA issued so far is done
      if (!mbar_wait(&ctl->drain, 0)) record_error(kErrWaitDrain);
    }
    __syncthreads();
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, ncols);
  }
}

// Epilogue-only barrier: the epilogue warps are warps 2.. of the CTA
// (128 threads, or 256 for the Block_FP8 Standard kernel).
__device__ __forceinline__ void epi_sync(uint32_t nthreads = 128) { named_bar_sync(1, nthreads); }

// After the epilogue's waits: agree (uniformly) on whether to write output.
__device__ __forceinline__ bool epi_agree_ok(SmemCtl* ctl, uint32_t nthreads = 128) {
  epi_sync(nthreads);
  if (threadIdx.x == 64) ctl->epi_ok = (ctl->abort_flag == 0);
  epi_sync(nthreads);
  return ctl->epi_ok != 0;
}

// Split-K arrival: returns true in every epilogue thread of the last CTA to
// arrive at tile `tile`.  Called after this CTA's partials are written: the
// barrier orders every epilogue thread's stores before one thread's
// acquire-release atomic at GPU scope, and the barrier after it orders that
// acquire before the last CTA's reads of the other partials.
__device__ __forceinline__ bool epi_arrive_last(SmemCtl* ctl, const GemmArgs& a, int tile, int expected,
                                                uint32_t nthreads = 128) {
  epi_sync(nthreads);
  if (threadIdx.x == 64) {
    unsigned int old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(old) : "l"(a.tickets + tile) : "memory");
    ctl->last_flag = (old == static_cast<unsigned int>(expected - 1));
  }
  epi_sync(nthreads);
  return ctl->last_flag != 0;
}

// ===========================================================================
// Swap-AB kernel (decode token counts; up to 128 tokens for the per-token formats).
//
// Work is the linear sequence of units u = tile * nku + kp (tile = 128 weight
// rows, kp = the kp-th group of a.kps consecutive 128-wide K slices, one
// pipeline stage; nku = ceil(nkt / kps) units per tile).  Every CTA takes a
// contiguous range of units; the range breaks into segments, one per tile it
// touches.
//   grid schedule       grid (n_tiles, split_k): CTA (t, s) owns the s-th of
//                       split_k near-equal K ranges of tile t (Split-K).
//   persistent schedule grid (G): CTA c owns units [c*U/G, (c+1)*U/G) of all
//                       U units, so every SM streams the same number of
//                       weight bytes (the Split-K partition chosen per CTA).
// A tile whose units all belong to one CTA is written straight to Y; a tile
// shared by several CTAs is finished by the last of them to arrive, which
// adds the partials in contributor order (deterministic), or the partials
// are added atomically, or by a second kernel.
// ===========================================================================
__device__ __forceinline__ int sk_owner(long long u, long long G, long long U) {
  return static_cast<int>(((u + 1) * G - 1) / U);
}

// Contributors to tile t and this CTA's index among them.
__device__ __forceinline__ void tile_contributors(const GemmArgs& a, int t, int nku, long long U, int cta,
                                                  int& ncontrib, int& j) {
  if (a.persistent) {
    const int first = sk_owner(static_cast<long long>(t) * nku, a.ctas, U);
    const int last = sk_owner(static_cast<long long>(t) * nku + nku - 1, a.ctas, U);
    ncontrib = last - first + 1;
    j = cta - first;
  } else {
    ncontrib = a.splits;
    j = cta;
  }
}

template <int kMpad>
__device__ __forceinline__ uint32_t* swap_slot(const GemmArgs& a, int t, int j, int row) {
  return static_cast<uint32_t*>(a.partial) +
         ((static_cast<size_t>(t) * a.maxc + j) * kSwapTileN + row) * static_cast<size_t>(a.mstride);
}

// Sum of the contributors' partial rows of tile t (this thread's weight row),
// in contributor order.  Loads are issued kBatch contributors at a time so
// that one memory round trip serves many partials; kVec 16-byte vectors per
// partial row (only the first nvec are live).  Contributor `own` (or -1) is
// taken from `own_acc` instead of memory.
template <int kFmt, int kMpad, int kVec, int kBatch>
__device__ __forceinline__ void fixup_sum_t(const GemmArgs& a, int t, int row, int ncontrib, int nvec, int own,
                                            const uint32_t (&own_acc)[kMpad], uint32_t (&sum)[kMpad]) {
  static_assert(kVec * 4 <= kMpad, "vector count exceeds the accumulator");
  for (int j0 = 0; j0 < ncontrib; j0 += kBatch) {
    uint4 buf[kBatch][kVec];
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      const int j = j0 + b;
      if (j < ncontrib && j != own) {
        const uint4* src = reinterpret_cast<const uint4*>(swap_slot<kMpad>(a, t, j, row));
#pragma unroll
        for (int v = 0; v < kVec; ++v)
          if (v < nvec) buf[b][v] = __ldcg(src + v);
      }
    }
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      const int j = j0 + b;
      if (j < ncontrib) {
#pragma unroll
        for (int v = 0; v < kVec; ++v) {
          if (v < nvec) {
            uint4 w4 = buf[b][v];
            if (j == own) w4 = make_uint4(own_acc[4 * v], own_acc[4 * v + 1], own_acc[4 * v + 2], own_acc[4 * v + 3]);
            if (j == 0) {
              sum[4 * v] = w4.x; sum[4 * v + 1] = w4.y; sum[4 * v + 2] = w4.z; sum[4 * v + 3] = w4.w;
            } else {
              sum[4 * v] = add_acc<kFmt>(sum[4 * v], w4.x);
              sum[4 * v + 1] = add_acc<kFmt>(sum[4 * v + 1], w4.y);
              sum[4 * v + 2] = add_acc<kFmt>(sum[4 * v + 2], w4.z);
              sum[4 * v + 3] = add_acc<kFmt>(sum[4 * v + 3], w4.w);
            }
          }
        }
      }
    }
  }
}

// The same sum through shared memory: the contributors' partial rows are
// requested with cp.async (no register cost while in flight), `chunk`
// contributors per round trip, then added from shared memory in contributor
// order.  Vector v of contributor j for weight row `row` sits at 16-byte index
// (j * nvec + v) * 128 + row, so a warp's 32 threads touch 32 consecutive
// 16-byte words (no bank conflicts).  `stage` holds 128 * chunk * nvec * 16
// bytes.
template <int kFmt, int kMpad>
__device__ __forceinline__ void fixup_sum_smem(const GemmArgs& a, int t, int row, int ncontrib, int nvec, int chunk,
                                               uint8_t* stage, uint32_t (&sum)[kMpad]) {
  uint4* area = reinterpret_cast<uint4*>(stage);
  for (int j0 = 0; j0 < ncontrib; j0 += chunk) {
    const int nj = (ncontrib - j0) < chunk ? (ncontrib - j0) : chunk;
    for (int jj = 0; jj < nj; ++jj) {
      const uint4* src = reinterpret_cast<const uint4*>(swap_slot<kMpad>(a, t, j0 + jj, row));
      for (int v = 0; v < nvec; ++v) cp_async16(area + (jj * nvec + v) * kSwapTileN + row, src + v);
    }
    cp_async_wait_all();
    for (int jj = 0; jj < nj; ++jj) {
#pragma unroll
      for (int v = 0; v < kMpad / 4; ++v) {
        if (v < nvec) {
          const uint4 w4 = area[(jj * nvec + v) * kSwapTileN + row];
          if (j0 + jj == 0) {
            sum[4 * v] = w4.x; sum[4 * v + 1] = w4.y; sum[4 * v + 2] = w4.z; sum[4 * v + 3] = w4.w;
          } else {
            sum[4 * v] = add_acc<kFmt>(sum[4 * v], w4.x);
            sum[4 * v + 1] = add_acc<kFmt>(sum[4 * v + 1], w4.y);
            sum[4 * v + 2] = add_acc<kFmt>(sum[4 * v + 2], w4.z);
            sum[4 * v + 3] = add_acc<kFmt>(sum[4 * v + 3], w4.w);
          }
        }
      }
    }
  }
}

// Contributors' vectors [v0, v0 + nv) of weight row `row` of tile t, added in
// contributor order (more than 32 tokens: one 32-token chunk of the row).
// With chunk > 0 the drained ring stages them, `chunk` contributors per round
// trip (same layout as fixup_sum_smem); otherwise one contributor per round
// trip through registers.
template <int kFmt, int kAcc, int kMpad>
__device__ __forceinline__ void fixup_sum_range(const GemmArgs& a, int t, int row, int ncontrib, int v0, int nv,
                                                int chunk, uint8_t* stage, uint32_t (&sum)[kAcc]) {
  for (int j0 = 0; j0 < ncontrib; j0 += (chunk > 0 ? chunk : 1)) {
    const int nj = chunk > 0 ? ((ncontrib - j0) < chunk ? (ncontrib - j0) : chunk) : 1;
    uint4 buf[kAcc / 4];
    uint4* area = reinterpret_cast<uint4*>(stage);
    if (chunk > 0) {
      for (int jj = 0; jj < nj; ++jj) {
        const uint4* src = reinterpret_cast<const uint4*>(swap_slot<kMpad>(a, t, j0 + jj, row)) + v0;
        for (int v = 0; v < nv; ++v) cp_async16(area + (jj * nv + v) * kSwapTileN + row, src + v);
      }
      cp_async_wait_all();
    }
    for (int jj = 0; jj < nj; ++jj) {
      const int j = j0 + jj;
      if (chunk > 0) {
#pragma unroll
        for (int v = 0; v < kAcc / 4; ++v)
          if (v < nv) buf[v] = area[(jj * nv + v) * kSwapTileN + row];
      } else {
        const uint4* src = reinterpret_cast<const uint4*>(swap_slot<kMpad>(a, t, j, row)) + v0;
#pragma unroll
        for (int v = 0; v < kAcc / 4; ++v)
          if (v < nv) buf[v] = __ldcg(src + v);
      }
#pragma unroll
      for (int v = 0; v < kAcc / 4; ++v) {
        if (v < nv) {
          const uint4 w4 = buf[v];
          if (j == 0) {
            sum[4 * v] = w4.x; sum[4 * v + 1] = w4.y; sum[4 * v + 2] = w4.z; sum[4 * v + 3] = w4.w;
          } else {
            sum[4 * v] = add_acc<kFmt>(sum[4 * v], w4.x);
            sum[4 * v + 1] = add_acc<kFmt>(sum[4 * v + 1], w4.y);
            sum[4 * v + 2] = add_acc<kFmt>(sum[4 * v + 2], w4.z);
            sum[4 * v + 3] = add_acc<kFmt>(sum[4 * v + 3], w4.w);
          }
        }
      }
    }
  }
}

template <int kFmt, int kMpad>
__device__ __forceinline__ void fixup_sum(const GemmArgs& a, int t, int row, int ncontrib, int nvec, int own,
                                       const uint32_t (&own_acc)[kMpad], uint32_t (&sum)[kMpad]) {
  // a fixed budget of kMpad/4 16-byte loads per round trip, spent on more
  // contributors when each partial row is short
  // contributors when each partial row is short (M > 16 always has 5+ vectors)
  constexpr int kV = kMpad / 4;
  if constexpr (kMpad == 16) {
    if (nvec == 1) fixup_sum_t<kFmt, kMpad, 1, kV>(a, t, row, ncontrib, nvec, own, own_acc, sum);
    else if (nvec == 2) fixup_sum_t<kFmt, kMpad, 2, kV / 2>(a, t, row, ncontrib, nvec, own, own_acc, sum);
    else fixup_sum_t<kFmt, kMpad, kV, 1>(a, t, row, ncontrib, nvec, own, own_acc, sum);
  } else {
    fixup_sum_t<kFmt, kMpad, kV, 1>(a, t, row, ncontrib, nvec, own, own_acc, sum);
  }
}

// Two CTAs per SM must always fit (the persistent grid size assumes it), so
// the register budget is capped at 65536 / (2 * 192) per thread.
//
// kFused: the activation quantizer runs inside the kernel.  The epilogue
// warps, idle while the weights stream, read the bf16 activations, quantize
// them with the stand-alone quantizers' arithmetic (per token: every CTA
// first takes each row's maximum over all of K; Block_FP8: one scale per
// 1x128 group, inside the K slice) and write the codes into each stage's
// activation tile in the layout the TMA would have written (128-byte rows,
// 16-byte chunk c of row m at chunk c ^ (m % 8)), staying far enough ahead of
// the MMA that neither waits on the other in a cycle (see quant_until).
template <int kFmt, int kMpad, bool kFused>
__global__ void __launch_bounds__(kGemmThreads, 2)
    swapab_kernel(const __grid_constant__ CUtensorMap tw, const __grid_constant__ CUtensorMap tx,
                  const GemmArgs a) {
  constexpr bool kInt = (kFmt == kFmtINT8);
  constexpr bool kBlock = (kFmt == kFmtBlock);
  // MXFP8 / NVFP4: the tensor core applies the block scales (E8M0 per 32 /
  // E4M3 per 16 values), which the epilogue warps write into tensor memory
  // stage by stage; NVFP4's operands are E2M1 codes, two per byte, and its K
  // here counts bytes (K / 2 values), so a 128-byte slice holds 256 values
  constexpr bool kMX = (kFmt == kFmtMX);
  constexpr bool kNV = (kFmt == kFmtNV);
  constexpr bool kBS = kMX || kNV;
  // Block_FP8: a ring of per-K-block accumulators; otherwise one accumulator
  // per segment, double-buffered so the next segment's MMAs overlap the drain.
  constexpr int kSlots = kBlock ? 4 : 2;
  constexpr uint32_t kCols = kSlots * kMpad <= 32 ? 32 : (kSlots * kMpad <= 64 ? 64 : (kSlots * kMpad <= 128 ? 128 : 256));
  static_assert(!kBlock || kMpad <= 32, "Block_FP8 Swap-AB covers at most 32 tokens");
  static_assert(!(kBS && kFused), "the block-scaled formats take quantized activations");
  // MXFP8 scale-factor columns per ring slot: a 4-column group for the
  // weights (lane quadrant q reads column q), then one for the tokens (token m
  // in lane m % 32 of every quadrant, column m / 32; kSFB columns used)
  constexpr uint32_t kSFB = kMpad > 32 ? kMpad / 32 : 1;
  constexpr uint32_t kSFSlot = kNV ? kNvSlotCols : kMxSlotCols;
  static_assert(kSFB <= 4, "token scales fit one 4-column group");
  // the epilogue walks the accumulator row in chunks of at most 32 token columns
  constexpr int kAcc = kMpad > 32 ? 32 : kMpad;
  constexpr int kChunks = kMpad / kAcc;
  constexpr uint32_t kWBytes = kSwapTileN * kTileK;
  constexpr uint32_t kXBytes = kMpad * kTileK;
  constexpr uint32_t kIdesc = idesc_mma(kInt ? 2 : 1, kInt ? 1 : 0, kSwapTileN, kMpad);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = align1024(smem_raw);
  const int stages = a.stages;
  const int kps = a.kps;                     // K slices per stage
  const uint32_t stage_w = kps * kWBytes;    // weight bytes per stage
  const uint32_t stage_x = kps * kXBytes;    // activation bytes per stage
  uint8_t* w_ring = base;
  uint8_t* x_ring = base + stages * stage_w;
  SmemCtl* ctl = reinterpret_cast<SmemCtl*>(x_ring + stages * stage_x);
  // cluster Split-K: S x ceil(128 / S) <= 128 + 7 rows of kMpad words
  uint8_t* recv_buf = reinterpret_cast<uint8_t*>(ctl) + kBarBytes;
  // fused: per-row maxima [128][4] and the Block_FP8 group-scale ring [kScaleRing][kMpad]
  float* row_red = reinterpret_cast<float*>(recv_buf + (a.reduce == kCluster ? (kSwapTileN + 8) * kMpad * 4 : 0));
  float* scale_ring = row_red + 128 * 4;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nkt = (a.K + kTileK - 1) / kTileK;
  const int nku = (nkt + kps - 1) / kps;
  const int n_tiles = (a.N + kSwapTileN - 1) / kSwapTileN;
  const long long U = static_cast<long long>(n_tiles) * nku;
  long long ub, ue;
  int cta;  // index among the contributors' numbering (persistent: CTA id; grid: split id)
  if (a.persistent) {
    cta = blockIdx.x;
    ub = static_cast<long long>(blockIdx.x) * U / gridDim.x;
    ue = static_cast<long long>(blockIdx.x + 1) * U / gridDim.x;
  } else {
    cta = blockIdx.y;
    const long long t0 = static_cast<long long>(blockIdx.x) * nku;
    ub = t0 + static_cast<long long>(blockIdx.y) * nku / a.splits;
    ue = t0 + static_cast<long long>(blockIdx.y + 1) * nku / a.splits;
  }
  const int nk = static_cast<int>(ue - ub);
  const uint32_t ncols = kBS ? mx_tmem_cols(kMpad, stages, kps, kFmt) : kCols;
  if (threadIdx.x == 0) QGD_STAMP(0);

  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tw);
    if (!kFused) tma_prefetch_desc(&tx);
    for (int i = 0; i < stages; ++i) {
      mbar_init(&ctl->full[i], 1);
      mbar_init(&ctl->xfull[i], 4);  // fused: one arrival per quantizing (epilogue) warp
      mbar_init(&ctl->empty[i], 1);
    }
    for (int i = 0; i < kSlots; ++i) {
      mbar_init(&ctl->tfull[i], 1);
      mbar_init(&ctl->tempty[i], 4);  // one arrival per epilogue warp
    }
    mbar_init(&ctl->accfull, 1);
    mbar_init(&ctl->drain, 1);
    {
      // cluster Split-K: one arrival per (owned weight row, contributor)
      const int S = a.splits > 0 ? a.splits : 1;
      const int j = blockIdx.y;
      const int lo = (j * kSwapTileN + S - 1) / S, hi = ((j + 1) * kSwapTileN + S - 1) / S;
      const int cnt = (a.reduce == kCluster && !a.persistent && S > 1) ? (hi - lo) * S : kSwapTileN;
      mbar_init(&ctl->recv_bar, cnt > 0 ? cnt : 1);
    }
    ctl->abort_flag = 0;
    ctl->last_flag = 0;
    ctl->epi_ok = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&ctl->tmem_base, ncols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // cluster Split-K: every CTA's receive barrier is initialised before any
  // peer can arrive on it
  if (a.reduce == kCluster) cluster_sync_all();
  griddep_launch_dependents();
  const uint32_t tmem = ctl->tmem_base;
  int issued = 0;
  if (threadIdx.x == 0) QGD_STAMP(1);

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_x = policy_evict_last();
      // Weights do not depend on the preceding kernel: start streaming them
      // before waiting for it, then fetch the activations.
      // (fused: the stage's activation half is written by the epilogue warps)
      const uint32_t x_tx = kFused ? 0u : kXBytes;
      const int pre = nk < stages ? nk : stages;
      for (int i = 0; i < pre; ++i) {
        const long long u = ub + i;
        const int k0 = static_cast<int>(u % nku) * kps;   // first K slice of the unit
        const int ns = (nkt - k0) < kps ? (nkt - k0) : kps;
        mbar_arrive_expect_tx(&ctl->full[i], ns * (kWBytes + x_tx));
        for (int j = 0; j < ns; ++j)
          tma_load_2d(w_ring + i * stage_w + j * kWBytes, &tw, &ctl->full[i], (k0 + j) * kTileK,
                      static_cast<int>(u / nku) * kSwapTileN, pol_w);
      }
      QGD_STAMP(13);
      if (!kFused) {
        griddep_wait();
        QGD_STAMP(14);
        for (int i = 0; i < pre; ++i) {
          const int k0 = static_cast<int>((ub + i) % nku) * kps;
          const int ns = (nkt - k0) < kps ? (nkt - k0) : kps;
          for (int j = 0; j < ns; ++j)
            tma_load_2d(x_ring + i * stage_x + j * kXBytes, &tx, &ctl->full[i], (k0 + j) * kTileK, 0, pol_x);
        }
      }
      issued = pre;
      QGD_STAMP(2);
      for (int i = pre; i < nk; ++i) {
        const int s = i % stages;
        const uint32_t round = i / stages;
        if (!mbar_wait(&ctl->empty[s], (round & 1) ^ 1)) {
          record_error(kErrWaitProducer);
          ctl->abort_flag = 1;
          break;
        }
        if (*reinterpret_cast<volatile int*>(&ctl->abort_flag)) break;
        const long long u = ub + i;
        const int k0 = static_cast<int>(u % nku) * kps;
        const int ns = (nkt - k0) < kps ? (nkt - k0) : kps;
        mbar_arrive_expect_tx(&ctl->full[s], ns * (kWBytes + x_tx));
        for (int j = 0; j < ns; ++j) {
          tma_load_2d(w_ring + s * stage_w + j * kWBytes, &tw, &ctl->full[s], (k0 + j) * kTileK,
                      static_cast<int>(u / nku) * kSwapTileN, pol_w);
          if (!kFused)
            tma_load_2d(x_ring + s * stage_x + j * kXBytes, &tx, &ctl->full[s], (k0 + j) * kTileK, 0, pol_x);
        }
        issued = i + 1;
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t w_base = smem_u32(w_ring), x_base = smem_u32(x_ring);
      int seg = 0;
      int sl = 0;  // Block_FP8: K slices consumed so far (one TMEM slot each)
      bool stop = false;
      for (int i = 0; i < nk && !stop; ++i) {
        const int s = i % stages;
        const uint32_t round = i / stages;
        if (!mbar_wait(&ctl->full[s], round & 1) ||
            ((kFused || kBS) && !mbar_wait(&ctl->xfull[s], round & 1))) {
          record_error(kErrWaitMma);
          ctl->abort_flag = 1;
          break;
        }
        if (i == 0) QGD_STAMP(3);
        const int kp = static_cast<int>((ub + i) % nku);
        const int ns = (nkt - kp * kps) < kps ? (nkt - kp * kps) : kps;
        const bool seg_start = (i == 0) || (kp == 0);
        const bool seg_end = (i == nk - 1) || (kp == nku - 1);
        if (!kBlock && seg_start) {
          if (!mbar_wait(&ctl->tempty[seg & 1], ((seg >> 1) & 1) ^ 1)) {
            record_error(kErrWaitMma);
            ctl->abort_flag = 1;
            break;
          }
        }
        for (int j = 0; j < ns; ++j) {
          const int slot = kBlock ? sl % kSlots : (seg & 1);
          if (kBlock && !mbar_wait(&ctl->tempty[slot], ((sl / kSlots) & 1) ^ 1)) {
            record_error(kErrWaitMma);
            ctl->abort_flag = 1;
            stop = true;
            break;
          }
          if (*reinterpret_cast<volatile int*>(&ctl->abort_flag)) {
            stop = true;
            break;
          }
          tc_fence_after();
          const uint32_t d = tmem + slot * kMpad;
          // MXFP8 / NVFP4: this slot's scale-factor columns.  Every group
          // starts on a multiple of 4 columns (by construction; checked, so
          // that a mistake aborts the CTA instead of faulting)
          const uint32_t sfa = tmem + 2 * kMpad + static_cast<uint32_t>(s * kps + j) * kSFSlot;
          if (kBS && (sfa & 3u) != 0u) {
            record_error(kErrBadOperand);
            ctl->abort_flag = 1;
            stop = true;
            break;
          }
#pragma unroll
          for (int kk = 0; kk < kTileK / 32; ++kk) {
            const uint64_t ad = sdesc_kmajor_sw128(w_base + s * stage_w + j * kWBytes + kk * 32);
            const uint64_t bd = sdesc_kmajor_sw128(x_base + s * stage_x + j * kXBytes + kk * 32);
            const uint32_t accumulate = kBlock ? (kk > 0) : !(seg_start && j == 0 && kk == 0);
            if constexpr (kMX) {
              const uint32_t sel = static_cast<uint32_t>(kk) << 30;  // the 32-wide K block's byte
              mma_issue_mx(d, ad, bd, idesc_mx(kSwapTileN, kMpad, kk, kk), sfa | sel, (sfa + 4) | sel,
                           accumulate);
            } else if constexpr (kNV) {
              // 64 values per MMA: weight-scale group kk, token-scale group 4 + kk
              mma_issue_nv(d, ad, bd, idesc_nv(kSwapTileN, kMpad), sfa + 4 * kk, sfa + 16 + 4 * kk, accumulate);
            } else {
              mma_issue<kInt>(d, ad, bd, kIdesc, accumulate);
            }
          }
          if (kBlock) {
            if (!a.withhold_acc) mma_commit(&ctl->tfull[slot]);
            ++sl;
          }
        }
        if (stop) break;
        mma_commit(&ctl->empty[s]);
        // (withhold_acc: the failure-detection test leaves the epilogue's
        // accumulator barrier unsignalled, so its bounded wait runs out)
        if (!kBlock && seg_end && !a.withhold_acc) mma_commit(&ctl->tfull[seg & 1]);
        if (seg_end) ++seg;
      }
      QGD_STAMP(4);
    }
    __syncwarp();
  } else {
    // ---------------- epilogue (warps 2..5) ----------------
    griddep_wait();  // scales and outputs: only after the preceding kernel is done
    const int q = warp & 3;
    const int row = q * 32 + lane;  // TMEM lane = weight row inside the tile
    const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16);
    const int M = a.M, N = a.N;
    const int KB = a.K / kTileK;
    const int nvec = (M + 3) / 4;  // float4 groups of the M accumulators
    const bool scaled = (kFmt != kFmtBlock) && !kMX && !a.raw;  // NVFP4: the fp32 row scales
    const int et = static_cast<int>(threadIdx.x) - 64;  // 0..127 among the epilogue threads
    if constexpr (kFused && !kBlock) {
      // per-token scales: every CTA takes each row's maximum over all of K
      // (four rows at a time, the loads of a row group in flight together)
      const int nv8 = a.K / 8;
      for (int m0 = 0; m0 < M; m0 += 4) {
        float am[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 2
        for (int v = et; v < nv8; v += 128) {
          uint4 r[4];
#pragma unroll
          for (int k = 0; k < 4; ++k)
            if (m0 + k < M) r[k] = __ldg(reinterpret_cast<const uint4*>(a.xbf + static_cast<size_t>(m0 + k) * a.ldxb) + v);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            if (m0 + k < M) am[k] = fmaxf(am[k], absmax8(r[k]));
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float w = warp_max(am[k]);
          if (lane == 0 && m0 + k < M) row_red[(m0 + k) * 4 + q] = w;
        }
      }
      epi_sync();
      for (int m = et; m < M; m += 128) {
        const float* rr = row_red + m * 4;
        const float amax = fmaxf(fmaxf(fmaxf(rr[0], rr[1]), fmaxf(rr[2], rr[3])), kAmaxFloor);
        const float sc = __fdiv_rn(amax, kInt ? kInt8Max : kE4M3Max);
        ctl->sx_s[m] = sc;
        if (a.sx_out && ub == 0) a.sx_out[m] = sc;  // the CTA owning unit 0
      }
    } else if (scaled) {
      for (int m = et; m < M; m += kSwapTileN) ctl->sx_s[m] = __ldg(a.sx + m);
    }
    epi_sync();
    // Fused: write the activation codes of stages [qnext, limit) into the
    // ring.  Quantizing stage q needs the MMA to have released the ring slot,
    // i.e. consumed stage q - stages; callers keep q - stages inside segments
    // whose accumulator slot is already free (non-Block: the segment after
    // the one being drained; Block_FP8: K slices at most 4 past the one being
    // promoted), so the quantizer and the MMA never wait on each other in a
    // cycle.  Each warp arrives on the stage's xfull barrier after its share;
    // a warp whose wait gives up records the error and stops quantizing.
    int qnext = 0, qslice = 0;
    bool qdead = false;
    auto quant_until = [&](int limit) {
      if constexpr (kNV) {
        // NVFP4: each stage's E4M3 block scales into its tensor-memory slot
        // once the MMA has released the stage: per K slice (256 values) four
        // MMAs, each reading one 4-column group of weight scales (lane
        // quadrant q in column q; a word = the 4 blocks of 16 of its 64
        // values) and one of token scales (token m in lane m % 32 of every
        // quadrant, column m / 32)
        if (limit > nk) limit = nk;
        const int KB16 = a.K / 8;  // block scales per row: (2 K) / 16
        for (; qnext < limit && !qdead; ++qnext) {
          const int s = qnext % stages;
          const uint32_t round = qnext / stages;
          if (*reinterpret_cast<volatile int*>(&ctl->abort_flag) || !warp_wait(&ctl->empty[s], (round & 1) ^ 1)) {
            if (lane == 0) {
              record_error(kErrWaitEpilogue);
              ctl->abort_flag = 1;
            }
            qdead = true;
            break;
          }
          const long long u = ub + qnext;
          const int t = static_cast<int>(u / nku);
          const int k0 = static_cast<int>(u % nku) * kps;
          const int ns = (nkt - k0) < kps ? (nkt - k0) : kps;
          tc_fence_after();
          const uint32_t lanes = static_cast<uint32_t>(q * 32) << 16;
          const int n = t * kSwapTileN + q * 32 + lane;
          for (int j = 0; j < ns; ++j) {
            const uint32_t col = 2 * kMpad + static_cast<uint32_t>(s * kps + j) * kSFSlot;
            const int b0 = (k0 + j) * 16;  // first block of 16 of the slice
            const uint4 wsf = n < N ? __ldg(reinterpret_cast<const uint4*>(a.sw8 + static_cast<size_t>(n) * KB16 + b0))
                                    : make_uint4(0, 0, 0, 0);
            tmem_st32(tmem + lanes + col + 0 + q, wsf.x);
            tmem_st32(tmem + lanes + col + 4 + q, wsf.y);
            tmem_st32(tmem + lanes + col + 8 + q, wsf.z);
            tmem_st32(tmem + lanes + col + 12 + q, wsf.w);
#pragma unroll
            for (uint32_t w = 0; w < kSFB; ++w) {
              const int m = static_cast<int>(w) * 32 + lane;
              const uint4 xsf = m < M ? __ldg(reinterpret_cast<const uint4*>(a.sx8 + static_cast<size_t>(m) * KB16 + b0))
                                      : make_uint4(0, 0, 0, 0);
              tmem_st32(tmem + lanes + col + 16 + w, xsf.x);
              tmem_st32(tmem + lanes + col + 20 + w, xsf.y);
              tmem_st32(tmem + lanes + col + 24 + w, xsf.z);
              tmem_st32(tmem + lanes + col + 28 + w, xsf.w);
            }
          }
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&ctl->xfull[s]);
        }
      } else if constexpr (kMX) {
        // MXFP8: write each stage's block scales into its tensor-memory slot
        // once the MMA has released the stage (its empty barrier)
        if (limit > nk) limit = nk;
        const int KB32 = a.K / 32;
        for (; qnext < limit && !qdead; ++qnext) {
          const int s = qnext % stages;
          const uint32_t round = qnext / stages;
          if (*reinterpret_cast<volatile int*>(&ctl->abort_flag) || !warp_wait(&ctl->empty[s], (round & 1) ^ 1)) {
            if (lane == 0) {
              record_error(kErrWaitEpilogue);
              ctl->abort_flag = 1;
            }
            qdead = true;
            break;
          }
          const long long u = ub + qnext;
          const int t = static_cast<int>(u / nku);
          const int k0 = static_cast<int>(u % nku) * kps;
          const int ns = (nkt - k0) < kps ? (nkt - k0) : kps;
          tc_fence_after();
          for (int j = 0; j < ns; ++j) {
            const uint32_t col = 2 * kMpad + static_cast<uint32_t>(s * kps + j) * kSFSlot;
            const uint32_t lanes = static_cast<uint32_t>(q * 32) << 16;
            // weight rows of this lane quadrant: 4 E8M0 bytes (the 128-wide K slice) per row
            const int n = t * kSwapTileN + q * 32 + lane;
            const uint32_t wsf = n < N ? __ldg(reinterpret_cast<const unsigned*>(a.sw8 + static_cast<size_t>(n) * KB32) + (k0 + j))
                                       : 0u;
            tmem_st32(tmem + lanes + col + q, wsf);
#pragma unroll
            for (uint32_t w = 0; w < kSFB; ++w) {
              const int m = static_cast<int>(w) * 32 + lane;
              const uint32_t xsf =
                  m < M ? __ldg(reinterpret_cast<const unsigned*>(a.sx8 + static_cast<size_t>(m) * KB32) + (k0 + j)) : 0u;
              tmem_st32(tmem + lanes + col + 4 + w, xsf);
            }
          }
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&ctl->xfull[s]);
        }
      } else if constexpr (kFused) {
        if (limit > nk) limit = nk;
        for (; qnext < limit && !qdead; ++qnext) {
          const int s = qnext % stages;
          const uint32_t round = qnext / stages;
          if (*reinterpret_cast<volatile int*>(&ctl->abort_flag) || !warp_wait(&ctl->empty[s], (round & 1) ^ 1)) {
            if (lane == 0) {
              record_error(kErrWaitEpilogue);
              ctl->abort_flag = 1;
            }
            qdead = true;
            break;
          }
          const long long u = ub + qnext;
          const int t = static_cast<int>(u / nku);
          const int k0 = static_cast<int>(u % nku) * kps;
          const int ns = (nkt - k0) < kps ? (nkt - k0) : kps;
          const int rows_w = round == 0 ? kMpad : M;  // the padding rows are zeroed once
          for (int j = 0; j < ns; ++j, ++qslice) {
            uint8_t* xs = x_ring + s * stage_x + j * kXBytes;
            const int kk0 = (k0 + j) * kTileK;
            for (int base = 0; base < rows_w * 8; base += 128) {
              const int item = base + et;  // (row, 16-byte chunk); a row's 8 chunks are 8 adjacent lanes
              const bool valid = item < rows_w * 8;
              const int m = item >> 3, c = item & 7;
              // past K (the last slice of a K that is not a multiple of 128;
              // K % 16 == 0, so a chunk is all in or all out): zero codes, as
              // the TMA's out-of-range fill gives the weights there
              const bool live = valid && m < M && kk0 + c * 16 < a.K;
              uint4 v0 = make_uint4(0, 0, 0, 0), v1 = v0;
              if (live) {
                const uint4* src = reinterpret_cast<const uint4*>(a.xbf + static_cast<size_t>(m) * a.ldxb + kk0 + c * 16);
                v0 = __ldg(src);
                v1 = __ldg(src + 1);
              }
              float sc;
              if constexpr (kBlock) {
                float am = fmaxf(absmax8(v0), absmax8(v1));
                am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));
                am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 2));
                am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 4));
                sc = __fdiv_rn(fmaxf(am, kAmaxFloor), kE4M3Max);
                if (live && c == 0) {
                  scale_ring[(qslice % kScaleRing) * kMpad + m] = sc;
                  if (a.sx_out && t == 0) a.sx_out[static_cast<size_t>(m) * KB + k0 + j] = sc;
                }
              } else {
                sc = live ? ctl->sx_s[m] : 1.f;
              }
              uint4 code = make_uint4(0, 0, 0, 0);
              if (live) {
                const uint2 lo = encode8<kInt ? 1 : 0>(v0, sc), hi = encode8<kInt ? 1 : 0>(v1, sc);
                code = make_uint4(lo.x, lo.y, hi.x, hi.y);
              }
              if (valid) st_shared_v4(xs + m * 128 + ((c ^ (m & 7)) << 4), code);
              if (live && a.xq_out && t == 0)
                *reinterpret_cast<uint4*>(a.xq_out + static_cast<size_t>(m) * a.K + kk0 + c * 16) = code;
            }
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&ctl->xfull[s]);
        }
      }
    };
    int i = 0, seg = 0;
    int sl = 0;  // Block_FP8: K slices consumed so far (same sequence as the MMA issuer's)
    while (i < nk) {
      const long long u = ub + i;
      const int t = static_cast<int>(u / nku);
      const int kp_first = static_cast<int>(u % nku);
      const int len = (nku - kp_first) < (nk - i) ? (nku - kp_first) : (nk - i);
      const int n = t * kSwapTileN + row;
      // the channel scale is known before the accumulator is: fetch it now
      const float swv = (scaled && n < N) ? __ldg(a.sw + n) : 0.f;
      uint32_t acc[kAcc];
      const int slot_nb = seg & 1;  // non-Block: this segment's accumulator slot
      if constexpr (kBlock) {
        float facc[kMpad];
#pragma unroll
        for (int m = 0; m < kMpad; ++m) facc[m] = 0.f;
        const int kb_first = kp_first * kps;
        const int kb_end = (kp_first + len) * kps < nkt ? (kp_first + len) * kps : nkt;
        for (int kb = kb_first; kb < kb_end; ++kb, ++sl) {
          const int slot = sl % kSlots;
          const int kstage = i + kb / kps - kp_first;  // the stage holding this K slice
          quant_until(kstage + stages);
          if (!warp_wait(&ctl->tfull[slot], (sl / kSlots) & 1)) {
            if (lane == 0) {
              record_error(kErrWaitEpilogue);
              ctl->abort_flag = 1;
            }
            break;
          }
          tc_fence_after();
          uint32_t r[kMpad];
          tmem_load_cols<kMpad>(taddr + slot * kMpad, r);
          tmem_wait_ld();
          warp_release(&ctl->tempty[slot]);
          const float swv = __ldg(a.sw + static_cast<size_t>(t) * KB + kb);  // one weight block per tile
          if constexpr (kFused) {
            // the slice's group scales, written by all four warps before their
            // arrivals on the stage's xfull barrier (whose phase is still this
            // one: the quantizer stays less than `stages` stages ahead)
            if (!warp_wait(&ctl->xfull[kstage % stages], (kstage / stages) & 1)) {
              if (lane == 0) {
                record_error(kErrWaitEpilogue);
                ctl->abort_flag = 1;
              }
              break;
            }
            const float* sxs = scale_ring + (sl % kScaleRing) * kMpad;
#pragma unroll
            for (int m = 0; m < kMpad; ++m)
              if (m < M) facc[m] = fmaf(__uint_as_float(r[m]), sxs[m] * swv, facc[m]);
          } else {
#pragma unroll
            for (int m = 0; m < kMpad; ++m) {
              if (m < M)
                facc[m] = fmaf(__uint_as_float(r[m]), __ldg(a.sx + static_cast<size_t>(m) * KB + kb) * swv, facc[m]);
            }
          }
        }
#pragma unroll
        for (int m = 0; m < kMpad; ++m) acc[m] = __float_as_uint(facc[m]);
      } else {
        quant_until(i + len + nku);  // this segment and the next one
        if (!warp_wait(&ctl->tfull[slot_nb], (seg >> 1) & 1)) {
          if (lane == 0) {
            record_error(kErrWaitEpilogue);
            ctl->abort_flag = 1;
          }
        } else if constexpr (kChunks == 1) {
          tc_fence_after();
          tmem_load_cols<kMpad>(taddr + slot_nb * kMpad, acc);
          tmem_wait_ld();
          warp_release(&ctl->tempty[slot_nb]);
        }
      }
      // More than 32 tokens: chunk cc of the accumulator row is read on demand
      // (the slot is handed back after the last chunk).
      auto load_chunk = [&](int cc) {
        if constexpr (kChunks > 1) {
          tc_fence_after();
          tmem_load_cols<kAcc>(taddr + slot_nb * kMpad + cc * kAcc, acc);
          tmem_wait_ld();
          if (cc == kChunks - 1) warp_release(&ctl->tempty[slot_nb]);
        }
      };
      if (!epi_agree_ok(ctl)) break;
      if (threadIdx.x == 64 && i + len >= nk) QGD_STAMP(5);

      const bool in_n = n < N;
      const bool last_seg = i + len >= nk;
      int ncontrib, jslot;
      tile_contributors(a, t, nku, U, cta, ncontrib, jslot);
      if (ncontrib == 1) {
        for (int cc = 0; cc < kChunks; ++cc) {
          load_chunk(cc);
          if (in_n) {
#pragma unroll
            for (int mm = 0; mm < kAcc; ++mm)
              if (cc * kAcc + mm < M) store_swap_final<kFmt>(acc[mm], cc * kAcc + mm, n, swv, ctl->sx_s, a);
          }
        }
        if (threadIdx.x == 64 && last_seg) QGD_STAMP(8);
      } else if (a.reduce == kCluster) {
        // Split-K inside a thread-block cluster (the grid schedule's S splits
        // of one tile, 2 <= S <= 8, any S): CTA j owns weight rows
        // [ceil(128 j / S), ceil(128 (j + 1) / S)) of the tile, i.e. row r
        // belongs to CTA floor(r S / 128).  Every CTA writes each of its
        // partial rows into the owner's shared memory (at most ceil(128 / S)
        // rows per contributor) and arrives on the owner's barrier; each owner
        // then adds the S contributions of its rows in CTA order.
        const int S = ncontrib;
        const int Rm = (kSwapTileN + S - 1) / S;  // most rows any owner holds
        const int owner = (row * S) / kSwapTileN;
        const int lr = row - (owner * kSwapTileN + S - 1) / S;
        const uint32_t dst = mapa_shared(smem_u32(recv_buf), static_cast<uint32_t>(owner));
        // owner's layout: [contributor][vector][row], 16 bytes each
        for (int cc = 0; cc < kChunks; ++cc) {
          load_chunk(cc);
#pragma unroll
          for (int v = 0; v < kAcc / 4; ++v) {
            const int vg = cc * (kAcc / 4) + v;
            if (vg < nvec)
              st_cluster_v4(dst + static_cast<uint32_t>(((jslot * nvec + vg) * Rm + lr) * 16), acc[4 * v],
                            acc[4 * v + 1], acc[4 * v + 2], acc[4 * v + 3]);
          }
        }
        mbar_arrive_remote(mapa_shared(smem_u32(&ctl->recv_bar), static_cast<uint32_t>(owner)));
        if (!mbar_wait_cluster(&ctl->recv_bar, 0)) {
          record_error(kErrWaitEpilogue);
          ctl->abort_flag = 1;
        } else {
          const uint4* rb = reinterpret_cast<const uint4*>(recv_buf);
          const int my_lo = (jslot * kSwapTileN + S - 1) / S;
          const int R = ((jslot + 1) * kSwapTileN + S - 1) / S - my_lo;
          for (int idx = row; idx < R * nvec; idx += kSwapTileN) {
            const int v = idx / R, r = idx % R;
            uint4 s4 = rb[v * Rm + r];
            for (int j = 1; j < S; ++j) {
              const uint4 w4 = rb[(j * nvec + v) * Rm + r];
              s4.x = add_acc<kFmt>(s4.x, w4.x);
              s4.y = add_acc<kFmt>(s4.y, w4.y);
              s4.z = add_acc<kFmt>(s4.z, w4.z);
              s4.w = add_acc<kFmt>(s4.w, w4.w);
            }
            const int nn = t * kSwapTileN + my_lo + r;
            if (nn < N) {
              const float swn = scaled ? __ldg(a.sw + nn) : 0.f;
              const uint32_t vals[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
              for (int q = 0; q < 4; ++q)
                if (4 * v + q < M) store_swap_final<kFmt>(vals[q], 4 * v + q, nn, swn, ctl->sx_s, a);
            }
          }
        }
      } else {
        for (int cc = 0; cc < kChunks; ++cc) {
          load_chunk(cc);
          if (in_n) {
            if (a.reduce == kAtomic) {
#pragma unroll
              for (int mm = 0; mm < kAcc; ++mm)
                if (cc * kAcc + mm < M)
                  atomic_acc<kFmt>(a.accum, static_cast<size_t>(cc * kAcc + mm) * N + n, acc[mm]);
            } else {
              uint4* dst = reinterpret_cast<uint4*>(swap_slot<kMpad>(a, t, jslot, row)) + cc * (kAcc / 4);
#pragma unroll
              for (int v = 0; v < kAcc / 4; ++v)
                if (cc * (kAcc / 4) + v < nvec)
                  dst[v] = make_uint4(acc[4 * v], acc[4 * v + 1], acc[4 * v + 2], acc[4 * v + 3]);
            }
          }
        }
        if (threadIdx.x == 64 && last_seg) QGD_STAMP(9);
        if (a.reduce != kTwoPass && epi_arrive_last(ctl, a, t, ncontrib)) {
          if (threadIdx.x == 64 && last_seg) QGD_STAMP(10);
          if (in_n) {
            if (a.reduce == kAtomic) {
#pragma unroll 4
              for (int m = 0; m < kMpad; ++m)
                if (m < M)
                  store_swap_final<kFmt>(ldcg_u32(static_cast<uint32_t*>(a.accum) + static_cast<size_t>(m) * N + n),
                                         m, n, swv, ctl->sx_s, a);
            } else if constexpr (kChunks == 1) {
              uint32_t sum[kMpad];
              // in the CTA's last segment every ring stage has been consumed,
              // so the ring's shared memory can stage the partials
              const size_t ring_bytes = static_cast<size_t>(stages) * (stage_w + stage_x);
              const int chunk = static_cast<int>(ring_bytes / (static_cast<size_t>(kSwapTileN) * nvec * 16));
              if (last_seg && chunk >= 1)
                fixup_sum_smem<kFmt, kMpad>(a, t, row, ncontrib, nvec, chunk, w_ring, sum);
              else
                fixup_sum<kFmt, kMpad>(a, t, row, ncontrib, nvec, -1, acc, sum);  // own partial re-read from L2
              if (threadIdx.x == 64 && last_seg) QGD_STAMP(11);
#pragma unroll
              for (int m = 0; m < kMpad; ++m)
                if (m < M) store_swap_final<kFmt>(sum[m], m, n, swv, ctl->sx_s, a);
            } else {
              // more than 32 tokens: the contributors' rows, 32 tokens at a time
              const size_t ring_bytes = static_cast<size_t>(stages) * (stage_w + stage_x);
              for (int cc = 0; cc < kChunks; ++cc) {
                const int v0 = cc * (kAcc / 4);
                const int nv = (nvec - v0) < kAcc / 4 ? (nvec - v0) : kAcc / 4;
                if (nv <= 0) break;
                uint32_t sum[kAcc];
                const int chunk = static_cast<int>(ring_bytes / (static_cast<size_t>(kSwapTileN) * nv * 16));
                fixup_sum_range<kFmt, kAcc, kMpad>(a, t, row, ncontrib, v0, nv, last_seg ? chunk : 0, w_ring, sum);
#pragma unroll
                for (int mm = 0; mm < kAcc; ++mm)
                  if (cc * kAcc + mm < M) store_swap_final<kFmt>(sum[mm], cc * kAcc + mm, n, swv, ctl->sx_s, a);
              }
            }
          }
          if (threadIdx.x == 64) a.tickets[t] = 0u;
          if (threadIdx.x == 64 && last_seg) QGD_STAMP(12);
        }
      }
      i += len;
      ++seg;
    }
    if (threadIdx.x == 64) QGD_STAMP(6);
  }

  teardown(ctl, warp, lane, issued, stages, tmem, ncols);
  if (threadIdx.x == 32) QGD_STAMP(7);
  tp_signal_done(a);
}

// Two-pass reduction for the Swap-AB layout: one CTA per tile, one thread per
// weight row; contributors' partials added in contributor order.
template <int kFmt, int kMpad>
__global__ void __launch_bounds__(kSwapTileN) swapab_reduce_kernel(const GemmArgs a) {
  griddep_wait();
  const int t = blockIdx.x, row = threadIdx.x;
  const int nkt = (a.K + kTileK - 1) / kTileK;
  const int nku = (nkt + a.kps - 1) / a.kps;
  const long long U = static_cast<long long>((a.N + kSwapTileN - 1) / kSwapTileN) * nku;
  int ncontrib = a.splits, j0;
  if (a.persistent) tile_contributors(a, t, nku, U, 0, ncontrib, j0);
  const int n = t * kSwapTileN + row;
  if (ncontrib == 1 || n >= a.N) return;  // written directly by its only contributor
  const int M = a.M, nvec = (M + 3) / 4;
  uint32_t sum[kMpad], none[kMpad];
#pragma unroll
  for (int m = 0; m < kMpad; ++m) none[m] = 0u;
  fixup_sum<kFmt, kMpad>(a, t, row, ncontrib, nvec, -1, none, sum);
#pragma unroll
  for (int m = 0; m < kMpad; ++m)
    if (m < M) store_final<kFmt>(sum[m], m, n, a);
}

// Split-K fixup by the last-arriving CTA: this thread's row m, columns
// [n0, n0 + kCols), 32 at a time, partials added in split order s = 0, 1, ...
// (or the atomic accumulator read).  Every load of a chunk -- its partials and
// its channel scales -- is issued before any of its stores, and the stores
// are vectorised, so a chunk costs one L2 round trip per split rather than
// one per 16 columns plus one per element's scales.
template <int kFmt, int kCols>
__device__ __forceinline__ void std_reduce_tile(const GemmArgs& a, int m, int n0, bool in_m) {
  if (!in_m) return;
  constexpr bool kScaled = !(kFmt == kFmtBlock || kFmt == kFmtMX);
  const int M = a.M, N = a.N;
  const float sxm = (kScaled && !a.raw) ? __ldg(a.sx + m) : 1.f;
  for (int nc0 = n0; nc0 < n0 + kCols && nc0 < N; nc0 += 32) {
    const int nq = (N - nc0 < 32 ? N - nc0 : 32) / 4;  // 16-byte groups in this chunk: 4 or 8 (N % 16 == 0)
    const size_t idx = static_cast<size_t>(m) * N + nc0;
    const uint4* src = reinterpret_cast<const uint4*>(
        static_cast<const uint32_t*>(a.reduce == kAtomic ? a.accum : a.partial) + idx);
    uint4 v[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) v[q] = q < nq ? __ldcg(src + q) : make_uint4(0u, 0u, 0u, 0u);
    float sw32[32];
    if (kScaled && !a.raw) {
      const float4* swv = reinterpret_cast<const float4*>(a.sw + nc0);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float4 t4 = q < nq ? __ldg(swv + q) : make_float4(0.f, 0.f, 0.f, 0.f);
        sw32[4 * q] = t4.x;
        sw32[4 * q + 1] = t4.y;
        sw32[4 * q + 2] = t4.z;
        sw32[4 * q + 3] = t4.w;
      }
    }
    if (a.reduce != kAtomic) {
      for (int sp = 1; sp < a.splits; ++sp) {
        const uint4* ps = reinterpret_cast<const uint4*>(static_cast<const uint32_t*>(a.partial) +
                                                         static_cast<size_t>(sp) * M * N + idx);
        uint4 t[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) t[q] = q < nq ? __ldcg(ps + q) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          v[q].x = add_acc<kFmt>(v[q].x, t[q].x);
          v[q].y = add_acc<kFmt>(v[q].y, t[q].y);
          v[q].z = add_acc<kFmt>(v[q].z, t[q].z);
          v[q].w = add_acc<kFmt>(v[q].w, t[q].w);
        }
      }
    }
    if (a.raw) {
      uint4* dst = reinterpret_cast<uint4*>(static_cast<uint32_t*>(a.raw) + idx);
#pragma unroll
      for (int q = 0; q < 8; ++q)
        if (q < nq) dst[q] = v[q];
      continue;
    }
    uint32_t w[32];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      w[4 * q] = v[q].x;
      w[4 * q + 1] = v[q].y;
      w[4 * q + 2] = v[q].z;
      w[4 * q + 3] = v[q].w;
    }
    uint32_t pk[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      float f0, f1;
      if constexpr (kFmt == kFmtINT8) {
        f0 = (static_cast<float>(static_cast<int32_t>(w[2 * j])) * sxm) * sw32[2 * j];
        f1 = (static_cast<float>(static_cast<int32_t>(w[2 * j + 1])) * sxm) * sw32[2 * j + 1];
      } else if constexpr (kScaled) {
        f0 = (__uint_as_float(w[2 * j]) * sxm) * sw32[2 * j];
        f1 = (__uint_as_float(w[2 * j + 1]) * sxm) * sw32[2 * j + 1];
      } else {
        f0 = __uint_as_float(w[2 * j]);
        f1 = __uint_as_float(w[2 * j + 1]);
      }
      pk[j] = static_cast<uint32_t>(bf16_bits(f0)) | (static_cast<uint32_t>(bf16_bits(f1)) << 16);
    }
    uint4* dst = reinterpret_cast<uint4*>(a.y + idx);
#pragma unroll
    for (int q = 0; q < 4; ++q)
      if (2 * q < nq) dst[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
  }
}

// Split-K of the Standard kernel inside a thread-block cluster (grid schedule:
// the S = a.splits CTAs of a tile are one cluster, CTA rank = split).  Row r of
// the tile (TMEM lane r) belongs to CTA floor(r S / 128); after every CTA's
// MMAs are done (first cluster barrier: each epilogue has waited for its
// accumulator, so every ring is idle), each CTA writes its partial rows that
// others own into the owner's ring through distributed shared memory, and
// after the second barrier each owner adds the S partials of its rows in
// split order -- its own straight from tensor memory -- and stores them.
// Called by every thread of the CTA (the barriers need all of them).  The
// host checks that (S - 1) ceil(128 / S) kTileN * 4 bytes fit in the ring.
template <int kFmt, int kTileN>
__device__ __forceinline__ void std_cluster_reduce(const GemmArgs& a, SmemCtl* ctl, uint8_t* ring, uint32_t tmem,
                                                   int warp, int lane) {
  const int S = a.splits;
  const int self = static_cast<int>(cluster_ctarank());
  const int tile = static_cast<int>(blockIdx.x) / S;
  const int m_tiles = (a.M + kStdTileM - 1) / kStdTileM;
  const int m_tile = tile % m_tiles, n_tile = tile / m_tiles;
  const int Rm = (kStdTileM + S - 1) / S;  // most rows any owner holds
  tc_fence_before();
  __syncwarp();  // the role branches leave warps diverged; the cluster barrier is warp-aligned
  cluster_sync_all();
  // an aborted CTA may still have copies landing in its ring: no exchange then
  bool abort = false;
  for (int j = 0; j < S; ++j)
    abort |= ld_cluster_u32(mapa_shared(smem_u32(&ctl->abort_flag), static_cast<uint32_t>(j))) != 0u;
  const int q = warp & 3, r = q * 32 + lane;  // this thread's tile row (TMEM lane), epilogue warps only
  const int owner = (r * S) / kStdTileM;     // (an owner's band may start inside a warp: the TMEM
  const int lr = r - (owner * kStdTileM + S - 1) / S;  // loads stay warp-wide, the rest per lane)
  const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16);  // accumulator buffer 0
  if (warp >= 2 && !abort) {
    tc_fence_after();
    const int jslot = self < owner ? self : self - 1;  // this CTA's slot in the owner's buffer
    const uint32_t dst = mapa_shared(smem_u32(ring), static_cast<uint32_t>(owner)) +
                         static_cast<uint32_t>((jslot * Rm + lr) * kTileN * 4);
#pragma unroll 1
    for (int c4 = 0; c4 < kTileN / 64; ++c4) {
      uint32_t vv[4][16];
      __syncwarp();
#pragma unroll
      for (int h = 0; h < 4; ++h) tmem_ld16(taddr + c4 * 64 + h * 16, vv[h]);
      tmem_wait_ld();
      if (owner != self) {
#pragma unroll
        for (int h = 0; h < 4; ++h)
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const int ch = (16 * c4 + 4 * h + g) ^ (lr & 7);  // 16-byte chunk, swizzled against bank conflicts
            st_cluster_v4(dst + static_cast<uint32_t>(ch * 16), vv[h][4 * g], vv[h][4 * g + 1], vv[h][4 * g + 2],
                          vv[h][4 * g + 3]);
          }
      }
    }
  }
  tc_fence_before();
  __syncwarp();
  cluster_sync_all();
  if (warp < 2) return;
  if (abort) {
    if (lane == 0) record_error(kErrWaitEpilogue);
    return;
  }
  tc_fence_after();
  const int M = a.M, N = a.N;
  const int m = m_tile * kStdTileM + r;
  const int n0 = n_tile * kTileN;
  const bool mine = owner == self && m < M;
  const float sxm = (mine && !a.raw) ? __ldg(a.sx + m) : 0.f;
#pragma unroll 1
  for (int c4 = 0; c4 < kTileN / 64; ++c4) {
    uint32_t own4[4][16];
    __syncwarp();
#pragma unroll
    for (int h = 0; h < 4; ++h) tmem_ld16(taddr + c4 * 64 + h * 16, own4[h]);
    tmem_wait_ld();
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const int c = 4 * c4 + h;
      const int nc = n0 + c * 16;
      const uint32_t (&own)[16] = own4[h];
      if (!mine || nc >= N) continue;
      uint32_t v[16];
      for (int j = 0; j < S; ++j) {
        uint32_t p[16];
        if (j == self) {
#pragma unroll
          for (int e = 0; e < 16; ++e) p[e] = own[e];
        } else {
          const int js = j < self ? j : j - 1;
          const uint8_t* src = ring + static_cast<size_t>((js * Rm + lr) * kTileN * 4);
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const uint4 t = *reinterpret_cast<const uint4*>(src + (((4 * c + g) ^ (lr & 7)) * 16));
            p[4 * g] = t.x;
            p[4 * g + 1] = t.y;
            p[4 * g + 2] = t.z;
            p[4 * g + 3] = t.w;
          }
        }
#pragma unroll
        for (int e = 0; e < 16; ++e) v[e] = j == 0 ? p[e] : add_acc<kFmt>(v[e], p[e]);  // split order
      }
      const size_t idx = static_cast<size_t>(m) * N + nc;
      if (a.raw) {
        uint4* dst = reinterpret_cast<uint4*>(static_cast<uint32_t*>(a.raw) + idx);
#pragma unroll
        for (int g = 0; g < 4; ++g) dst[g] = make_uint4(v[4 * g], v[4 * g + 1], v[4 * g + 2], v[4 * g + 3]);
        continue;
      }
      const float4* swv = reinterpret_cast<const float4*>(a.sw + nc);
      float sw16[16];
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const float4 t = __ldg(swv + g);
        sw16[4 * g] = t.x;
        sw16[4 * g + 1] = t.y;
        sw16[4 * g + 2] = t.z;
        sw16[4 * g + 3] = t.w;
      }
      uint32_t pk[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float f0, f1;
        if constexpr (kFmt == kFmtINT8) {
          f0 = (static_cast<float>(static_cast<int32_t>(v[2 * j])) * sxm) * sw16[2 * j];
          f1 = (static_cast<float>(static_cast<int32_t>(v[2 * j + 1])) * sxm) * sw16[2 * j + 1];
        } else {
          f0 = (__uint_as_float(v[2 * j]) * sxm) * sw16[2 * j];
          f1 = (__uint_as_float(v[2 * j + 1]) * sxm) * sw16[2 * j + 1];
        }
        pk[j] = static_cast<uint32_t>(bf16_bits(f0)) | (static_cast<uint32_t>(bf16_bits(f1)) << 16);
      }
      uint4* dst = reinterpret_cast<uint4*>(a.y + idx);
      dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
    }
  }
}

// ===========================================================================
// Standard kernel (larger M): D[m, n] over 128 x kTileN output tiles.
//
// Work items are (tile, split) pairs, tiles ordered token-tile fastest so
// CTAs running side by side share a weight tile in L2.  CTA c takes items c,
// c + G, c + 2G, ... of the grid's G CTAs: with G = #items every CTA does
// one item (the grid schedule, needed for Split-K), with G = #SMs the CTAs
// persist and the TMEM accumulator is double-buffered, so the epilogue of
// one tile overlaps the mainloop of the next.
// ===========================================================================
// Threads of the Standard kernel: producer warp, MMA warp, then 4 epilogue
// warps -- 8 for Block_FP8, whose per-K-block promotion (TMEM read, scale,
// add) is the busiest part: two warps per TMEM lane quadrant, each taking half
// the columns (16 warps measured slower on B200).
constexpr int kBlockEpiGroups = 2;
template <int kFmt>
__host__ __device__ constexpr int std_threads() {
  return kFmt == kFmtBlock ? 64 + 128 * kBlockEpiGroups : kGemmThreads;
}

template <int kFmt, int kTileN, int kKps>
__global__ void __launch_bounds__(std_threads<kFmt>(), 1)
    standard_kernel(const __grid_constant__ CUtensorMap tx, const __grid_constant__ CUtensorMap tw,
                    const GemmArgs a) {
  constexpr bool kInt = (kFmt == kFmtINT8);
  constexpr bool kBlock = (kFmt == kFmtBlock);
  constexpr uint32_t kEpi = std_threads<kFmt>() - 64;  // epilogue threads
  constexpr int kHalf = kBlock ? kTileN / kBlockEpiGroups : kTileN;  // columns per epilogue thread
  // Block_FP8: a ring of per-K-block accumulators (4 x 128 columns, or 2 x
  // 256 for tiles two weight blocks wide, whose epilogue warp pairs then each
  // own one weight block); else: a per-tile double buffer.
  static_assert(!kBlock || kTileN == 128 || kTileN == 256, "Block_FP8 tiles are one or two weight blocks wide");
  constexpr int kSlots = kBlock ? (kTileN == 128 ? 4 : 2) : 2;
  constexpr uint32_t kCols = kSlots * kTileN;  // 512 (4 x 128 or 2 x 256) or 256
  constexpr uint32_t kXBytes = kStdTileM * kTileK;
  constexpr uint32_t kWBytes = kTileN * kTileK;
  constexpr uint32_t kIdesc = idesc_mma(kInt ? 2 : 1, kInt ? 1 : 0, kStdTileM, kTileN);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = align1024(smem_raw);
  const int stages = a.stages;
  // K blocks per pipeline stage (1 or 2, a compile-time constant so that the
  // stage loops are straight-line code): one full/empty hand-off and one MMA
  // commit per stage, so two blocks per stage halve those per FLOP
  static_assert(kKps == 1 || kKps == 2, "one or two K blocks per stage");
  constexpr int kps = kKps;
  const uint32_t stage_x = kps * kXBytes, stage_w = kps * kWBytes;
  uint8_t* x_ring = base;
  uint8_t* w_ring = base + stages * stage_x;
  SmemCtl* ctl = reinterpret_cast<SmemCtl*>(w_ring + stages * stage_w);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nkt = (a.K + kTileK - 1) / kTileK;
  const int m_tiles = (a.M + kStdTileM - 1) / kStdTileM;
  const int n_tiles = (a.N + kTileN - 1) / kTileN;
  const int S = a.splits;
  const long long items = static_cast<long long>(m_tiles) * n_tiles * S;

  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tx);
    tma_prefetch_desc(&tw);
    for (int i = 0; i < stages; ++i) {
      mbar_init(&ctl->full[i], 1);
      mbar_init(&ctl->empty[i], 1);
    }
    for (int i = 0; i < kSlots; ++i) {
      mbar_init(&ctl->tfull[i], 1);
      mbar_init(&ctl->tempty[i], kEpi / 32);  // one arrival per epilogue warp
    }
    mbar_init(&ctl->accfull, 1);
    mbar_init(&ctl->drain, 1);
    ctl->abort_flag = 0;
    ctl->last_flag = 0;
    ctl->epi_ok = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&ctl->tmem_base, kCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  griddep_launch_dependents();
  const uint32_t tmem = ctl->tmem_base;
  int issued = 0;

  if (warp == 0) {
    // ---------------- TMA producer: items x K slices, one ring ----------------
    if (lane == 0) {
      const uint64_t pol_x = policy_evict_last();
      const uint64_t pol_w = policy_evict_last();
      griddep_wait();  // activations come from the preceding kernel
      int i = 0;
      bool stop = false;
      for (long long w = blockIdx.x; w < items && !stop; w += gridDim.x) {
        const int tile = static_cast<int>(w / S), split = static_cast<int>(w % S);
        const int m_tile = tile % m_tiles, n_tile = tile / m_tiles;
        const int kt0 = static_cast<int>(static_cast<long long>(split) * nkt / S);
        const int kt1 = static_cast<int>(static_cast<long long>(split + 1) * nkt / S);
        for (int kt = kt0; kt < kt1; kt += kps, ++i) {
          const int s = i % stages;
          const uint32_t round = i / stages;
          if (!mbar_wait(&ctl->empty[s], (round & 1) ^ 1)) {
            record_error(kErrWaitProducer);
            ctl->abort_flag = 1;
            stop = true;
            break;
          }
          if (*reinterpret_cast<volatile int*>(&ctl->abort_flag)) {
            stop = true;
            break;
          }
          const int ns = (kt1 - kt) < kps ? (kt1 - kt) : kps;  // K blocks in this stage
          mbar_arrive_expect_tx(&ctl->full[s], ns * (kXBytes + kWBytes));
#pragma unroll
          for (int h = 0; h < kps; ++h) {
            if (h >= ns) break;
            tma_load_2d(x_ring + s * stage_x + h * kXBytes, &tx, &ctl->full[s], (kt + h) * kTileK,
                        m_tile * kStdTileM, pol_x);
            tma_load_2d(w_ring + s * stage_w + h * kWBytes, &tw, &ctl->full[s], (kt + h) * kTileK,
                        n_tile * kTileN, pol_w);
          }
          issued = i + 1;
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t x_base = smem_u32(x_ring), w_base = smem_u32(w_ring);
      int i = 0, li = 0, ib = 0;  // stages, items and (Block_FP8) K blocks consumed
      bool stop = false;
      for (long long w = blockIdx.x; w < items && !stop; w += gridDim.x, ++li) {
        const int split = static_cast<int>(w % S);
        const int kt0 = static_cast<int>(static_cast<long long>(split) * nkt / S);
        const int kt1 = static_cast<int>(static_cast<long long>(split + 1) * nkt / S);
        const int buf = li & 1;
        if constexpr (!kBlock) {
          if (!mbar_wait(&ctl->tempty[buf], ((li >> 1) & 1) ^ 1)) {
            record_error(kErrWaitMma);
            ctl->abort_flag = 1;
            break;
          }
        }
        for (int kt = kt0; kt < kt1 && !stop; kt += kps, ++i) {
          const int s = i % stages;
          const uint32_t round = i / stages;
          if (!mbar_wait(&ctl->full[s], round & 1)) {
            record_error(kErrWaitMma);
            ctl->abort_flag = 1;
            stop = true;
            break;
          }
          const int ns = (kt1 - kt) < kps ? (kt1 - kt) : kps;
#pragma unroll
          for (int h = 0; h < kps; ++h) {
            if (h >= ns) break;
            uint32_t d = tmem + buf * kTileN;
            if constexpr (kBlock) {
              // every K block accumulates into its own TMEM slot
              const int slot = ib % kSlots;
              if (!mbar_wait(&ctl->tempty[slot], ((ib / kSlots) & 1) ^ 1)) {
                record_error(kErrWaitMma);
                ctl->abort_flag = 1;
                stop = true;
                break;
              }
              d = tmem + slot * kTileN;
            }
            if (*reinterpret_cast<volatile int*>(&ctl->abort_flag)) {
              stop = true;
              break;
            }
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < kTileK / 32; ++kk) {
              const uint64_t ad = sdesc_kmajor_sw128(x_base + s * stage_x + h * kXBytes + kk * 32);
              const uint64_t bd = sdesc_kmajor_sw128(w_base + s * stage_w + h * kWBytes + kk * 32);
              const uint32_t accumulate = kBlock ? (kk > 0) : (kt + h > kt0 || kk > 0);
              mma_issue<kInt>(d, ad, bd, kIdesc, accumulate);
            }
            if constexpr (kBlock) mma_commit(&ctl->tfull[ib % kSlots]);
            ++ib;
          }
          if (stop) break;
          mma_commit(&ctl->empty[s]);
        }
        if (stop) break;
        if constexpr (!kBlock) mma_commit(&ctl->tfull[buf]);
      }
    }
    __syncwarp();
  } else {
    // ---------------- epilogue (warps 2..) ----------------
    griddep_wait();  // scales and outputs: only after the preceding kernel is done
    const int q = warp & 3;
    const int half = kBlock ? (warp - 2) / 4 : 0;  // Block_FP8: which column group (of kBlockEpiGroups)
    const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16);
    const int M = a.M, N = a.N;
    int i = 0, li = 0;
    for (long long w = blockIdx.x; w < items; w += gridDim.x, ++li) {
      const int tile = static_cast<int>(w / S), split = static_cast<int>(w % S);
      const int m_tile = tile % m_tiles, n_tile = tile / m_tiles;
      const int kt0 = static_cast<int>(static_cast<long long>(split) * nkt / S);
      const int kt1 = static_cast<int>(static_cast<long long>(split + 1) * nkt / S);
      const int m = m_tile * kStdTileM + q * 32 + lane;  // TMEM lane = token row
      const int n0 = n_tile * kTileN + half * kHalf;     // this thread's first column
      const bool in_m = m < M;

      if constexpr (kBlock) {
        const int KB = a.K / kTileK;
        float facc[kHalf];
#pragma unroll
        for (int j = 0; j < kHalf; ++j) facc[j] = 0.f;
        // this thread's columns lie in one 128-row weight block (n0 / 128); in
        // a 256-wide tile past N (N an odd number of blocks) the second half
        // has no block and no scale
        const bool live = in_m && n0 < N;
        const float* sxrow = a.sx + static_cast<size_t>(in_m ? m : 0) * KB;
        const float* swrow = a.sw + static_cast<size_t>(n0 < N ? n0 / 128 : 0) * KB;
        // scales one K block ahead, so their load latency hides behind a block
        float sc_next = (live && kt0 < kt1) ? __ldg(sxrow + kt0) * __ldg(swrow + kt0) : 0.f;
        for (int kt = kt0; kt < kt1; ++kt, ++i) {
          const int slot = i % kSlots;
          const float sc = sc_next;
          if (kt + 1 < kt1) sc_next = live ? __ldg(sxrow + kt + 1) * __ldg(swrow + kt + 1) : 0.f;
          if (!warp_wait(&ctl->tfull[slot], (i / kSlots) & 1)) {
            if (lane == 0) {
              record_error(kErrWaitEpilogue);
              ctl->abort_flag = 1;
            }
            break;
          }
          tc_fence_after();
          // this thread's columns: 64 in one TMEM wait, or a 128-column half in
          // rounds of 32 (its running sums already hold 128 registers; 32-column
          // rounds measured 4 % faster than 64)
          constexpr int kRound = kHalf <= 64 ? kHalf : 32;
#pragma unroll
          for (int c0 = 0; c0 < kHalf; c0 += kRound) {
            uint32_t r[kRound / 16][16];
#pragma unroll
            for (int c = 0; c < kRound / 16; ++c)
              tmem_ld16(taddr + slot * kTileN + half * kHalf + c0 + c * 16, r[c]);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < kRound / 16; ++c)
#pragma unroll
              for (int j = 0; j < 16; ++j)
                facc[c0 + c * 16 + j] = fmaf(__uint_as_float(r[c][j]), sc, facc[c0 + c * 16 + j]);
          }
          warp_release(&ctl->tempty[slot]);
        }
        if (!epi_agree_ok(ctl, kEpi)) break;
        if (S == 1) {
          if (in_m) {
#pragma unroll
            for (int c = 0; c < kHalf / 16; ++c) {
              const int nc = n0 + c * 16;
              if (nc >= N) break;
              if (a.raw) {
                uint4* dst = reinterpret_cast<uint4*>(static_cast<float*>(a.raw) + static_cast<size_t>(m) * N + nc);
#pragma unroll
                for (int v = 0; v < 4; ++v)
                  dst[v] = make_uint4(__float_as_uint(facc[c * 16 + 4 * v]), __float_as_uint(facc[c * 16 + 4 * v + 1]),
                                      __float_as_uint(facc[c * 16 + 4 * v + 2]), __float_as_uint(facc[c * 16 + 4 * v + 3]));
              } else {
                uint32_t pk[8];
#pragma unroll
                for (int j = 0; j < 8; ++j)
                  pk[j] = static_cast<uint32_t>(bf16_bits(facc[c * 16 + 2 * j])) |
                          (static_cast<uint32_t>(bf16_bits(facc[c * 16 + 2 * j + 1])) << 16);
                uint4* dst = reinterpret_cast<uint4*>(a.y + static_cast<size_t>(m) * N + nc);
                dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
              }
            }
          }
        } else {
          if (in_m) {
#pragma unroll
            for (int c = 0; c < kHalf / 16; ++c) {
              const int nc = n0 + c * 16;
              if (nc >= N) break;
              const size_t idx = static_cast<size_t>(m) * N + nc;
              if (a.reduce == kAtomic) {
#pragma unroll
                for (int j = 0; j < 16; ++j) atomic_acc<kFmt>(a.accum, idx + j, __float_as_uint(facc[c * 16 + j]));
              } else {
                uint4* dst = reinterpret_cast<uint4*>(static_cast<float*>(a.partial) + static_cast<size_t>(split) * M * N + idx);
#pragma unroll
                for (int v = 0; v < 4; ++v)
                  dst[v] = make_uint4(__float_as_uint(facc[c * 16 + 4 * v]), __float_as_uint(facc[c * 16 + 4 * v + 1]),
                                      __float_as_uint(facc[c * 16 + 4 * v + 2]), __float_as_uint(facc[c * 16 + 4 * v + 3]));
              }
            }
          }
          if (a.reduce != kTwoPass && epi_arrive_last(ctl, a, tile, S, kEpi)) {
            std_reduce_tile<kFmt, kHalf>(a, m, n0, in_m);
            if (threadIdx.x == 64) a.tickets[tile] = 0u;
          }
        }
      } else {
        const int buf = li & 1;
        const bool ok = warp_wait(&ctl->tfull[buf], (li >> 1) & 1);
        if (!ok && lane == 0) {
          record_error(kErrWaitEpilogue);
          ctl->abort_flag = 1;
        }
        if (ok) tc_fence_after();
        if (!epi_agree_ok(ctl)) break;
        if (a.reduce == kCluster) continue;  // the cluster reduction below reads the accumulator
        const float sxm = (in_m && !a.raw) ? __ldg(a.sx + m) : 0.f;
        const uint32_t tbuf = taddr + buf * kTileN;
        // 64 columns per TMEM wait: four loads in flight instead of one
#pragma unroll 1
        for (int c4 = 0; c4 < kTileN / 64; ++c4) {
          uint32_t rr[4][16];
          __syncwarp();
#pragma unroll
          for (int g = 0; g < 4; ++g) tmem_ld16(tbuf + c4 * 64 + g * 16, rr[g]);
          tmem_wait_ld();
          if (c4 == kTileN / 64 - 1) {
            // the whole accumulator is in registers: hand the buffer back
            warp_release(&ctl->tempty[buf]);
          }
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const uint32_t (&r)[16] = rr[g];
            const int nc = n0 + (c4 * 4 + g) * 16;
            if (!in_m || nc >= N) continue;
            const size_t idx = static_cast<size_t>(m) * N + nc;
            if (S > 1) {
              if (a.reduce == kAtomic) {
#pragma unroll
                for (int j = 0; j < 16; ++j) atomic_acc<kFmt>(a.accum, idx + j, r[j]);
              } else {
                uint4* dst = reinterpret_cast<uint4*>(static_cast<uint32_t*>(a.partial) + static_cast<size_t>(split) * M * N + idx);
#pragma unroll
                for (int v = 0; v < 4; ++v) dst[v] = make_uint4(r[4 * v], r[4 * v + 1], r[4 * v + 2], r[4 * v + 3]);
              }
            } else if (a.raw) {
              uint4* dst = reinterpret_cast<uint4*>(static_cast<uint32_t*>(a.raw) + idx);
#pragma unroll
              for (int v = 0; v < 4; ++v) dst[v] = make_uint4(r[4 * v], r[4 * v + 1], r[4 * v + 2], r[4 * v + 3]);
            } else {
              const float4* swv = reinterpret_cast<const float4*>(a.sw + nc);
              float sw16[16];
#pragma unroll
              for (int v = 0; v < 4; ++v) {
                const float4 t = __ldg(swv + v);
                sw16[4 * v] = t.x;
                sw16[4 * v + 1] = t.y;
                sw16[4 * v + 2] = t.z;
                sw16[4 * v + 3] = t.w;
              }
              uint32_t pk[8];
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                float v0, v1;
                if constexpr (kInt) {
                  v0 = (static_cast<float>(static_cast<int32_t>(r[2 * j])) * sxm) * sw16[2 * j];
                  v1 = (static_cast<float>(static_cast<int32_t>(r[2 * j + 1])) * sxm) * sw16[2 * j + 1];
                } else {
                  v0 = (__uint_as_float(r[2 * j]) * sxm) * sw16[2 * j];
                  v1 = (__uint_as_float(r[2 * j + 1]) * sxm) * sw16[2 * j + 1];
                }
                pk[j] = static_cast<uint32_t>(bf16_bits(v0)) | (static_cast<uint32_t>(bf16_bits(v1)) << 16);
              }
              uint4* dst = reinterpret_cast<uint4*>(a.y + idx);
              dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
              dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
            }
          }
        }
        if (S > 1 && a.reduce != kTwoPass && epi_arrive_last(ctl, a, tile, S)) {
          std_reduce_tile<kFmt, kTileN>(a, m, n0, in_m);
          if (threadIdx.x == 64) a.tickets[tile] = 0u;
        }
      }
    }
  }

  if constexpr (!kBlock) {
    if (a.reduce == kCluster) std_cluster_reduce<kFmt, kTileN>(a, ctl, x_ring, tmem, warp, lane);
  }
  teardown(ctl, warp, lane, issued, stages, tmem, kCols);
}

// ===========================================================================
// Standard tiles of 256 tokens x 256 weight rows computed by a CTA pair (a
// 2-CTA cluster, tcgen05 .cta_group::2), FP8_Dynamic and W8A8_INT8.
//
// CTA r of the pair loads X rows [256 mt + 128 r, +128) and W rows
// [256 nt + 128 r, +128) into its own shared memory; the leader (r = 0)
// issues one M = 256, N = 256 MMA per 32-wide K step that reads both CTAs'
// tiles, and each CTA's tensor memory receives its 128 token rows x 256
// weight columns.  Per CTA and K block that is 32 KB of operands for the
// same 8.4 MFLOP a one-CTA 128 x 256 tile does with 48 KB: the L2-to-SM
// traffic per FLOP, which bounds the one-CTA kernel at large M, drops by a
// third.  The accumulator is double-buffered in all 512 TMEM columns, so the
// epilogue of one tile overlaps the next tile's mainloop.  (A 256 x 512 tile,
// two N = 256 halves sharing each X tile, cuts the traffic further but leaves
// no second accumulator: measured slower on B200 at every larger-M shape,
// the drain of each tile no longer hidden.)  Both CTAs' copies complete on
// the leader's `full` barrier (its expect-tx counts both); the leader's
// commits arrive on `empty` / `tfull` in both CTAs; both CTAs' epilogue warps
// hand the accumulator back on the leader's `tempty`.  Work items are pair
// tiles, token-tile fastest, dealt to the pairs round-robin.  A failed
// (bounded) wait in either CTA sets both CTAs' abort flags.
// ===========================================================================
constexpr int kPairTileM = 256;  // tokens per pair tile (MMA M)
constexpr int kPairTileN = 256;  // weight rows per pair tile (MMA N)

// Output staging for the tensor stores of Y: per epilogue warp two buffers of
// 32 rows x 64 bf16 columns (4 KB each), 128-byte swizzled like the tensor
// map's box, so that a warp's 32 rows are written without bank conflicts and
// leave as whole 128-byte lines.
constexpr uint32_t kPairStageBytes = 4 * 2 * 32 * 128;

template <int kFmt, bool kSplitK>
__global__ void __launch_bounds__(kGemmThreads, 1)
    standard_pair_kernel(const __grid_constant__ CUtensorMap tx, const __grid_constant__ CUtensorMap tw,
                         const __grid_constant__ CUtensorMap ty, const GemmArgs a) {
  constexpr bool kInt = (kFmt == kFmtINT8);
  static_assert(kFmt == kFmtFP8 || kFmt == kFmtINT8, "per-token / per-channel formats only");
  constexpr uint32_t kXBytes = (kPairTileM / 2) * kTileK;  // this CTA's 128 token rows of a K block
  constexpr uint32_t kWBytes = (kPairTileN / 2) * kTileK;  // this CTA's 128 weight rows of a K block
  constexpr uint32_t kCols = 2 * kPairTileN;               // double-buffered 128 x 256 accumulator
  constexpr uint32_t kIdesc = idesc_mma(kInt ? 2 : 1, kInt ? 1 : 0, kPairTileM, kPairTileN);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = align1024(smem_raw);
  const int stages = a.stages;
  const int kps = a.kps > 1 ? 2 : 1;
  const uint32_t stage_x = kps * kXBytes, stage_w = kps * kWBytes;
  uint8_t* x_ring = base;
  uint8_t* w_ring = base + stages * stage_x;
  uint8_t* y_stage = w_ring + stages * stage_w;  // 1024-aligned: the rings are whole 16 KB blocks
  SmemCtl* ctl = reinterpret_cast<SmemCtl*>(y_stage + kPairStageBytes);

  const uint32_t rank = cluster_ctarank();  // 0: the leader, which issues the MMAs
  const int pair = static_cast<int>(blockIdx.x >> 1), npairs = static_cast<int>(gridDim.x >> 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nkt = (a.K + kTileK - 1) / kTileK;
  const int m_tiles = (a.M + kPairTileM - 1) / kPairTileM;
  const int n_tiles = (a.N + kPairTileN - 1) / kPairTileN;
  // work items: (pair tile, K split), the splits of a tile adjacent; with
  // Split-K (a separate instantiation, so that the one-split kernel keeps its
  // own code) each split writes its partial for a second kernel to add
  const int S = kSplitK ? a.splits : 1;
  const long long items = static_cast<long long>(m_tiles) * n_tiles * S;

  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tx);
    tma_prefetch_desc(&tw);
    if (!a.raw || S > 1) tma_prefetch_desc(&ty);
    for (int i = 0; i < stages; ++i) {
      mbar_init(&ctl->full[i], 1);
      mbar_init(&ctl->empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ctl->tfull[i], 1);
      mbar_init(&ctl->tempty[i], 8);  // the 4 epilogue warps of each CTA of the pair
    }
    mbar_init(&ctl->drain, 1);
    ctl->abort_flag = 0;
    ctl->last_flag = 0;
    ctl->epi_ok = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(&ctl->tmem_base, kCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers and tensor memory exist before any traffic between them
  tc_fence_after();
  griddep_launch_dependents();
  const uint32_t tmem = ctl->tmem_base;
  const uint32_t partner_abort = mapa_shared(smem_u32(&ctl->abort_flag), rank ^ 1u);
  auto fail = [&](unsigned int code) {
    record_error(code);
    ctl->abort_flag = 1;
    st_cluster_u32(partner_abort, 1u);
  };
  auto aborted = [&]() { return *reinterpret_cast<volatile int*>(&ctl->abort_flag) != 0; };
  int issued = 0;

  if (warp == 0) {
    // ---------------- TMA producer (both CTAs): this CTA's halves ----------------
    if (lane == 0) {
      const uint64_t pol_x = policy_evict_last();
      const uint64_t pol_w = policy_evict_last();
      const uint32_t full0 = mapa_shared(smem_u32(&ctl->full[0]), 0);  // the leader's barriers
      griddep_wait();  // activations come from the preceding kernel
      int i = 0;
      bool stop = false;
      for (long long w = pair; w < items && !stop; w += npairs) {
        const long long tile = w / S;
        const int split = static_cast<int>(w % S);
        const int mt = static_cast<int>(tile % m_tiles), nt = static_cast<int>(tile / m_tiles);
        const int kt0 = static_cast<int>(static_cast<long long>(split) * nkt / S);
        const int kt1 = static_cast<int>(static_cast<long long>(split + 1) * nkt / S);
        const int xrow = mt * kPairTileM + static_cast<int>(rank) * (kPairTileM / 2);
        const int wrow = nt * kPairTileN + static_cast<int>(rank) * (kPairTileN / 2);
        for (int kt = kt0; kt < kt1; kt += kps, ++i) {
          const int s = i % stages;
          const uint32_t round = i / stages;
          if (!mbar_wait(&ctl->empty[s], (round & 1) ^ 1)) {
            fail(kErrWaitProducer);
            stop = true;
            break;
          }
          if (aborted()) {
            stop = true;
            break;
          }
          const int ns = (kt1 - kt) < kps ? (kt1 - kt) : kps;
          // the leader's barrier expects both CTAs' bytes (a copy may land first)
          if (rank == 0) mbar_arrive_expect_tx(&ctl->full[s], 2u * ns * (kXBytes + kWBytes));
          const uint32_t fb = full0 + static_cast<uint32_t>(s) * 8u;
          for (int h = 0; h < ns; ++h) {
            tma_load_2d_pair(x_ring + s * stage_x + h * kXBytes, &tx, fb, (kt + h) * kTileK, xrow, pol_x);
            tma_load_2d_pair(w_ring + s * stage_w + h * kWBytes, &tw, fb, (kt + h) * kTileK, wrow, pol_w);
          }
          issued = i + 1;
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer: the leader only ----------------
    if (rank == 0 && lane == 0) {
      const uint32_t x_base = smem_u32(x_ring), w_base = smem_u32(w_ring);
      int i = 0, li = 0;
      bool stop = false;
      for (long long w = pair; w < items && !stop; w += npairs, ++li) {
        const int split = static_cast<int>(w % S);
        const int kt0 = static_cast<int>(static_cast<long long>(split) * nkt / S);
        const int kt1 = static_cast<int>(static_cast<long long>(split + 1) * nkt / S);
        const int buf = li & 1;
        if (!mbar_wait(&ctl->tempty[buf], ((li >> 1) & 1) ^ 1)) {
          fail(kErrWaitMma);
          break;
        }
        const uint32_t d = tmem + buf * kPairTileN;
        for (int kt = kt0; kt < kt1 && !stop; kt += kps, ++i) {
          const int s = i % stages;
          const uint32_t round = i / stages;
          if (!mbar_wait(&ctl->full[s], round & 1)) {
            fail(kErrWaitMma);
            stop = true;
            break;
          }
          if (aborted()) {
            stop = true;
            break;
          }
          tc_fence_after();
          const int ns = (kt1 - kt) < kps ? (kt1 - kt) : kps;
          for (int h = 0; h < ns; ++h) {
#pragma unroll
            for (int kk = 0; kk < kTileK / 32; ++kk) {
              const uint64_t ad = sdesc_kmajor_sw128(x_base + s * stage_x + h * kXBytes + kk * 32);
              const uint64_t bd = sdesc_kmajor_sw128(w_base + s * stage_w + h * kWBytes + kk * 32);
              mma_issue_pair<kInt>(d, ad, bd, kIdesc, (kt + h > kt0 || kk > 0) ? 1u : 0u);
            }
          }
          mma_commit_pair(&ctl->empty[s], 0x3);
        }
        if (stop) break;
        mma_commit_pair(&ctl->tfull[buf], 0x3);
      }
    }
    __syncwarp();
  } else {
    // ---------------- epilogue (warps 2..5 of both CTAs) ----------------
    griddep_wait();  // scales and outputs: only after the preceding kernel is done
    const int q = warp & 3;
    const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16);
    const uint32_t tempty0 = mapa_shared(smem_u32(&ctl->tempty[0]), 0);  // the leader's
    const int M = a.M, N = a.N;
    uint8_t* ybuf = y_stage + q * (2 * 32 * 128);  // this warp's two 4 KB staging buffers
    int nstore = 0;                                // tensor stores this warp has issued
    int li = 0;
    for (long long w = pair; w < items; w += npairs, ++li) {
      const long long tile = w / S;
      const int split = static_cast<int>(w % S);
      const int mt = static_cast<int>(tile % m_tiles), nt = static_cast<int>(tile / m_tiles);
      const int row0 = mt * kPairTileM + static_cast<int>(rank) * (kPairTileM / 2) + q * 32;  // this warp's rows
      const int m = row0 + lane;
      const bool in_m = m < M;
      const float sxm = (in_m && !a.raw) ? __ldg(a.sx + m) : 0.f;
      {
        const int buf = li & 1;
        const bool ok = warp_wait(&ctl->tfull[buf], (li >> 1) & 1);
        if (!ok && lane == 0) fail(kErrWaitEpilogue);
        if (ok) tc_fence_after();
        if (!epi_agree_ok(ctl)) break;
        const uint32_t tbuf = taddr + buf * kPairTileN;
        const int ncol0 = nt * kPairTileN;  // first weight column of the tile
        // 64 columns at a time: four TMEM loads, one wait
#pragma unroll 1
        for (int grp = 0; grp < kPairTileN / 64; ++grp) {
          const int nc0 = ncol0 + grp * 64;
          uint32_t r[4][16];
          __syncwarp();
#pragma unroll
          for (int g = 0; g < 4; ++g) tmem_ld16(tbuf + grp * 64 + g * 16, r[g]);
          tmem_wait_ld();
          if (grp == kPairTileN / 64 - 1) {
            // the whole accumulator row is in registers: hand the buffer back to the leader
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(tempty0 + static_cast<uint32_t>(buf) * 8u);
          }
          if constexpr (kSplitK) {
            // Split-K partial (raw accumulator bits) of row m, columns nc0 ..
            // nc0 + 63: both 4 KB buffers, 32 columns each (the same 128-byte
            // swizzle), then two tensor stores into split plane `split`
            if (lane == 0 && nstore >= 1) bulk_wait_group_read<0>();  // the last group has read them
            __syncwarp();
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              uint8_t* row = ybuf + (g >> 1) * (32 * 128) + lane * 128;
#pragma unroll
              for (int v = 0; v < 4; ++v)
                st_shared_v4(row + ((((g & 1) * 4 + v) ^ (lane & 7)) << 4),
                             make_uint4(r[g][4 * v], r[g][4 * v + 1], r[g][4 * v + 2], r[g][4 * v + 3]));
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              if (row0 < M && nc0 < N) {
                tma_store_3d(&ty, ybuf, nc0, row0, split);
                if (nc0 + 32 < N) tma_store_3d(&ty, ybuf + 32 * 128, nc0 + 32, row0, split);
              }
              bulk_commit_group();
            }
            ++nstore;
            continue;
          }
          if (a.raw) {  // int32 accumulators (test hook): plain stores
            if (in_m) {
              uint32_t* out = static_cast<uint32_t*>(a.raw);
#pragma unroll
              for (int g = 0; g < 4; ++g) {
                const int nc = nc0 + g * 16;
                if (nc >= N) break;
                uint4* dst = reinterpret_cast<uint4*>(out + static_cast<size_t>(m) * N + nc);
#pragma unroll
                for (int v = 0; v < 4; ++v)
                  dst[v] = make_uint4(r[g][4 * v], r[g][4 * v + 1], r[g][4 * v + 2], r[g][4 * v + 3]);
              }
            }
            continue;
          }
          // row m, columns nc0 .. nc0 + 63 -> bf16 in a staging buffer (the
          // 16-byte chunk j of a row sits at j ^ (row % 8)), then one tensor store
          uint8_t* sb = ybuf + (nstore & 1) * (32 * 128);
          if (lane == 0 && nstore >= 2) bulk_wait_group_read<1>();  // this buffer's last store has read it
          __syncwarp();
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const int nc = nc0 + g * 16;
            float sw16[16];
            if (nc < N) {
              const float4* swv = reinterpret_cast<const float4*>(a.sw + nc);
#pragma unroll
              for (int v = 0; v < 4; ++v) {
                const float4 t4 = __ldg(swv + v);
                sw16[4 * v] = t4.x;
                sw16[4 * v + 1] = t4.y;
                sw16[4 * v + 2] = t4.z;
                sw16[4 * v + 3] = t4.w;
              }
            } else {
#pragma unroll
              for (int j = 0; j < 16; ++j) sw16[j] = 0.f;
            }
            uint32_t pk[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              float v0, v1;
              if constexpr (kInt) {
                v0 = (static_cast<float>(static_cast<int32_t>(r[g][2 * j])) * sxm) * sw16[2 * j];
                v1 = (static_cast<float>(static_cast<int32_t>(r[g][2 * j + 1])) * sxm) * sw16[2 * j + 1];
              } else {
                v0 = (__uint_as_float(r[g][2 * j]) * sxm) * sw16[2 * j];
                v1 = (__uint_as_float(r[g][2 * j + 1]) * sxm) * sw16[2 * j + 1];
              }
              pk[j] = static_cast<uint32_t>(bf16_bits(v0)) | (static_cast<uint32_t>(bf16_bits(v1)) << 16);
            }
            st_shared_v4(sb + lane * 128 + (((2 * g) ^ (lane & 7)) << 4), make_uint4(pk[0], pk[1], pk[2], pk[3]));
            st_shared_v4(sb + lane * 128 + (((2 * g + 1) ^ (lane & 7)) << 4), make_uint4(pk[4], pk[5], pk[6], pk[7]));
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            // a group per buffer use, empty when the box lies wholly past M or N,
            // so that "one group still reading" always means the other buffer
            if (row0 < M && nc0 < N) tma_store_2d(&ty, sb, nc0, row0);
            bulk_commit_group();
          }
          ++nstore;
        }
      }
    }
    if (lane == 0) bulk_wait_group_all();  // the stores are done before the CTA ends
  }

  // ---------------- teardown ----------------
  tc_fence_before();
  // one answer for every thread (the partner may set the flag at any time)
  if (__syncthreads_or(ctl->abort_flag != 0)) {
    if (rank == 0 && warp == 0 && lane == 0) {
      // the last copies issued into each stage (both CTAs') must land before either CTA exits
      for (int i = issued > stages ? issued - stages : 0; i < issued; ++i) {
        if (!mbar_wait(&ctl->full[i % stages], (i / stages) & 1)) {
          record_error(kErrWaitDrain);
          break;
        }
      }
    }
    if (rank == 0 && warp == 1 && lane == 0) {
      mma_commit_pair(&ctl->drain, 0x1);  // arrives once every MMA issued so far is done
      if (!mbar_wait(&ctl->drain, 0)) record_error(kErrWaitDrain);
    }
    __syncthreads();
  }
  cluster_sync_all();  // neither CTA leaves while its partner may still signal its barriers
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kCols);
  }
}

// ===========================================================================
// Tensor-parallel wait: one thread takes the epoch of this rank's last call
// from word `ranks` of its own flag array, then reads each rank's entry
// (acquire, system scope) until it holds that epoch (or a later one: a rank
// may already have finished its next call), giving up after about
// kWaitLimitNs per rank (error kErrWaitPeers).  Launched in stream order after
// this rank's GEMM, so it never waits on a kernel of its own GPU; the kernels
// after it read the full output.
// ===========================================================================
__global__ void __launch_bounds__(32) tp_wait_kernel(const unsigned* flags, int ranks) {
  griddep_launch_dependents();  // the next kernel may set up and stream its weights meanwhile
  griddep_wait();               // this rank's GEMM (which advanced the count) is complete
  if (threadIdx.x != 0) return;
  const unsigned epoch = *reinterpret_cast<const volatile unsigned*>(flags + ranks);
  for (int r = 0; r < ranks; ++r) {
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t i = 0;; ++i) {
      unsigned v;
      asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(flags + r) : "memory");
      if (static_cast<int>(v - epoch) >= 0) break;  // this call's epoch or a later one (wraps)
      if ((i & 63u) == 63u && globaltimer_ns() - t0 > kWaitLimitNs) {
        record_error(kErrWaitPeers);
        return;
      }
    }
  }
}

// ===========================================================================
// Two-pass Split-K reduction: one thread per output element, partials added
// in split order s = 0, 1, ..., splits-1.
// ===========================================================================
template <int kFmt>
__global__ void __launch_bounds__(256) splitk_reduce_kernel(const GemmArgs a) {
  // four adjacent outputs per thread (N % 16 == 0 keeps them in one row);
  // up to eight splits' partials in flight before they are added in order
  griddep_wait();
  const size_t total = static_cast<size_t>(a.M) * a.N;
  const size_t quad = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (quad * 4 >= total) return;
  const uint4* p = reinterpret_cast<const uint4*>(a.partial);
  const size_t stride = total / 4;
  uint32_t acc[4];
  for (int s0 = 0; s0 < a.splits; s0 += 8) {
    uint4 v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (s0 + j < a.splits) v[j] = p[static_cast<size_t>(s0 + j) * stride + quad];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (s0 + j < a.splits) {
        if (s0 + j == 0) {
          acc[0] = v[j].x; acc[1] = v[j].y; acc[2] = v[j].z; acc[3] = v[j].w;
        } else {
          acc[0] = add_acc<kFmt>(acc[0], v[j].x);
          acc[1] = add_acc<kFmt>(acc[1], v[j].y);
          acc[2] = add_acc<kFmt>(acc[2], v[j].z);
          acc[3] = add_acc<kFmt>(acc[3], v[j].w);
        }
      }
    }
  }
  const size_t idx = quad * 4;
  const int m = static_cast<int>(idx / a.N), n = static_cast<int>(idx % a.N);
#pragma unroll
  for (int j = 0; j < 4; ++j) store_final<kFmt>(acc[j], m, n + j, a);
}

// Launch with dynamic shared memory and, when `pdl` is set, a programmatic
// dependency on the preceding kernel in the stream; clusters of
// cluster_x x cluster_y CTAs when either is above 1.
template <typename... Params, typename... Args>
cudaError_t launch_ex_cluster_xy(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                                 bool pdl, int cluster_x, int cluster_y, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  int n = 0;
  if (pdl) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  if (cluster_x > 1 || cluster_y > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = static_cast<unsigned>(cluster_x);
    attr[n].val.clusterDim.y = static_cast<unsigned>(cluster_y);
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <typename... Params, typename... Args>
cudaError_t launch_ex_cluster(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              bool pdl, int cluster_y, Args&&... args) {
  return launch_ex_cluster_xy(kernel, grid, block, smem, stream, pdl, 1, cluster_y, std::forward<Args>(args)...);
}

template <typename... Params, typename... Args>
cudaError_t launch_ex(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                      bool pdl, Args&&... args) {
  return launch_ex_cluster(kernel, grid, block, smem, stream, pdl, 1, std::forward<Args>(args)...);
}

template <typename Kern>
cudaError_t set_smem_attr(Kern kernel, bool& done) {
  if (done) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem_budget()));
  if (e == cudaSuccess) done = true;
  return e;
}

}  // namespace

size_t swapab_smem_bytes(int mpad, int stages, int kps, bool cluster, bool fused) {
  return 1024 + static_cast<size_t>(stages) * kps * (kSwapTileN * kTileK + mpad * kTileK) + kBarBytes +
         (cluster ? static_cast<size_t>(kSwapTileN + 8) * mpad * 4 : 0) + (fused ? kFusedBytes : 0);
}

size_t standard_smem_bytes(int tile_n, int stages, int kps) {
  return 1024 + static_cast<size_t>(stages) * kps * (kStdTileM * kTileK + tile_n * kTileK) + kBarBytes;
}

int swapab_max_stages(int mpad, int kps, bool cluster, bool fused) {
  const size_t fixed = 1024 + kBarBytes + (cluster ? static_cast<size_t>(kSwapTileN + 8) * mpad * 4 : 0) +
                       (fused ? kFusedBytes : 0);
  int s = static_cast<int>((smem_budget() - fixed) / (kps * (kSwapTileN * kTileK + mpad * kTileK)));
  return s > kMaxStages ? kMaxStages : s;
}

// At least half an SM's shared memory, so that no two CTAs of this kernel share
// an SM: each allocates all 512 tensor-memory columns together with its
// partner, and a CTA whose allocation waited on another pair's CTA on its SM
// could wait for good.
size_t pair_smem_bytes(int stages, int kps) {
  const size_t need = 1024 +
                      static_cast<size_t>(stages) * kps * ((kPairTileM / 2) * kTileK + (kPairTileN / 2) * kTileK) +
                      kPairStageBytes + kBarBytes;
  return need > kSmemPerSM / 2 ? need : kSmemPerSM / 2;
}

int pair_max_stages(int kps) {
  int s = static_cast<int>((smem_budget() - 1024 - kPairStageBytes - kBarBytes) /
                           (kps * ((kPairTileM / 2) * kTileK + (kPairTileN / 2) * kTileK)));
  return s > kMaxStages ? kMaxStages : s;
}

int standard_max_stages(int tile_n, int kps) {
  int s = static_cast<int>((smem_budget() - 1024 - kBarBytes) / (kps * (kStdTileM * kTileK + tile_n * kTileK)));
  return s > kMaxStages ? kMaxStages : s;
}

template <int kFmt, int kMpad, bool kFused>
static cudaError_t launch_swapab_t(const CUtensorMap& tw, const CUtensorMap& tx, const GemmArgs& a,
                                   cudaStream_t stream) {
  static bool attr_done = false;
  cudaError_t e = set_smem_attr(swapab_kernel<kFmt, kMpad, kFused>, attr_done);
  if (e != cudaSuccess) return e;
  const dim3 grid = a.persistent ? dim3(a.ctas, 1, 1)
                                 : dim3((a.N + kSwapTileN - 1) / kSwapTileN, a.splits, 1);
  const bool cluster = a.reduce == kCluster;
  return launch_ex_cluster(swapab_kernel<kFmt, kMpad, kFused>, grid, dim3(kGemmThreads),
                           swapab_smem_bytes(kMpad, a.stages, a.kps, cluster, kFused), stream, a.pdl != 0,
                           cluster ? a.splits : 1, tw, tx, a);
}

template <bool kFused>
static cudaError_t launch_swapab_f(int fmt, int mpad, const CUtensorMap& tw, const CUtensorMap& tx,
                                   const GemmArgs& a, cudaStream_t stream) {
  if (fmt == kFmtFP8) {
    switch (mpad) {
      case 16: return launch_swapab_t<kFmtFP8, 16, kFused>(tw, tx, a, stream);
      case 32: return launch_swapab_t<kFmtFP8, 32, kFused>(tw, tx, a, stream);
      case 64: return launch_swapab_t<kFmtFP8, 64, kFused>(tw, tx, a, stream);
      case 128: return launch_swapab_t<kFmtFP8, 128, kFused>(tw, tx, a, stream);
    }
  } else if (fmt == kFmtINT8) {
    switch (mpad) {
      case 16: return launch_swapab_t<kFmtINT8, 16, kFused>(tw, tx, a, stream);
      case 32: return launch_swapab_t<kFmtINT8, 32, kFused>(tw, tx, a, stream);
      case 64: return launch_swapab_t<kFmtINT8, 64, kFused>(tw, tx, a, stream);
      case 128: return launch_swapab_t<kFmtINT8, 128, kFused>(tw, tx, a, stream);
    }
  } else if (fmt == kFmtBlock) {
    switch (mpad) {
      case 16: return launch_swapab_t<kFmtBlock, 16, kFused>(tw, tx, a, stream);
      case 32: return launch_swapab_t<kFmtBlock, 32, kFused>(tw, tx, a, stream);
    }
  } else if (fmt == kFmtMX) {
    if constexpr (!kFused) {
      switch (mpad) {
        case 16: return launch_swapab_t<kFmtMX, 16, false>(tw, tx, a, stream);
        case 32: return launch_swapab_t<kFmtMX, 32, false>(tw, tx, a, stream);
        case 64: return launch_swapab_t<kFmtMX, 64, false>(tw, tx, a, stream);
        case 128: return launch_swapab_t<kFmtMX, 128, false>(tw, tx, a, stream);
      }
    }
  } else if (fmt == kFmtNV) {
    if constexpr (!kFused) {
      switch (mpad) {
        case 16: return launch_swapab_t<kFmtNV, 16, false>(tw, tx, a, stream);
        case 32: return launch_swapab_t<kFmtNV, 32, false>(tw, tx, a, stream);
        case 64: return launch_swapab_t<kFmtNV, 64, false>(tw, tx, a, stream);
        case 128: return launch_swapab_t<kFmtNV, 128, false>(tw, tx, a, stream);
      }
    }
  }
  return cudaErrorInvalidValue;
}

template <int kFmt, int kTileN, int kKps>
static cudaError_t launch_standard_k(const CUtensorMap& tx, const CUtensorMap& tw, const GemmArgs& a,
                                     cudaStream_t stream) {
  static bool attr_done = false;
  cudaError_t e = set_smem_attr(standard_kernel<kFmt, kTileN, kKps>, attr_done);
  if (e != cudaSuccess) return e;
  const long long items = static_cast<long long>((a.N + kTileN - 1) / kTileN) *
                          ((a.M + kStdTileM - 1) / kStdTileM) * a.splits;
  const dim3 grid(static_cast<unsigned>(a.persistent && a.ctas < items ? a.ctas : items));
  // cluster Split-K (grid schedule): the a.splits CTAs of a tile, consecutive along x, are one cluster
  return launch_ex_cluster_xy(standard_kernel<kFmt, kTileN, kKps>, grid, dim3(std_threads<kFmt>()),
                              standard_smem_bytes(kTileN, a.stages, kKps), stream, a.pdl != 0,
                              a.reduce == kCluster ? a.splits : 1, 1, tx, tw, a);
}

template <int kFmt, int kTileN>
static cudaError_t launch_standard_t(const CUtensorMap& tx, const CUtensorMap& tw, const GemmArgs& a,
                                     cudaStream_t stream) {
  return a.kps > 1 ? launch_standard_k<kFmt, kTileN, 2>(tx, tw, a, stream)
                   : launch_standard_k<kFmt, kTileN, 1>(tx, tw, a, stream);
}

template <int kFmt, bool kSplitK>
static cudaError_t launch_standard_pair_split_t(const CUtensorMap& tx, const CUtensorMap& tw, const CUtensorMap& ty,
                                                const GemmArgs& a, cudaStream_t stream) {
  static bool attr_done = false;
  cudaError_t e = set_smem_attr(standard_pair_kernel<kFmt, kSplitK>, attr_done);
  if (e != cudaSuccess) return e;
  const long long items = static_cast<long long>((a.N + kPairTileN - 1) / kPairTileN) *
                          ((a.M + kPairTileM - 1) / kPairTileM) * (kSplitK ? a.splits : 1);
  const long long pairs = a.persistent && a.ctas / 2 < items ? a.ctas / 2 : items;
  return launch_ex_cluster_xy(standard_pair_kernel<kFmt, kSplitK>, dim3(static_cast<unsigned>(2 * pairs)),
                              dim3(kGemmThreads), pair_smem_bytes(a.stages, a.kps > 1 ? 2 : 1), stream, a.pdl != 0, 2,
                              1, tx, tw, ty, a);
}

template <int kFmt>
static cudaError_t launch_standard_pair_t(const CUtensorMap& tx, const CUtensorMap& tw, const CUtensorMap& ty,
                                          const GemmArgs& a, cudaStream_t stream) {
  if (a.splits > 1) return launch_standard_pair_split_t<kFmt, true>(tx, tw, ty, a, stream);
  return launch_standard_pair_split_t<kFmt, false>(tx, tw, ty, a, stream);
}

cudaError_t launch_standard_pair(int fmt, const CUtensorMap& tx, const CUtensorMap& tw, const CUtensorMap& ty,
                                 const GemmArgs& a, cudaStream_t stream) {
  if (fmt == kFmtFP8) return launch_standard_pair_t<kFmtFP8>(tx, tw, ty, a, stream);
  if (fmt == kFmtINT8) return launch_standard_pair_t<kFmtINT8>(tx, tw, ty, a, stream);
  return cudaErrorInvalidValue;
}

template <int kFmt>
static int pair_clusters_t(cudaLaunchConfig_t& cfg) {
  static bool done = false;
  if (set_smem_attr(standard_pair_kernel<kFmt, false>, done) != cudaSuccess) return 0;
  int n = 0;  // (the Split-K instantiation has the same shared memory and block)
  if (cudaOccupancyMaxActiveClusters(&n, standard_pair_kernel<kFmt, false>, &cfg) != cudaSuccess) {
    (void)cudaGetLastError();
    return 0;
  }
  return n;
}

// Pair clusters that fit on the GPU at once with this shared memory (0 if the
// query fails): the persistent pair schedule launches no more than that.
int pair_max_active_clusters(int fmt, int stages, int kps) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * 74);
  cfg.blockDim = dim3(kGemmThreads);
  cfg.dynamicSmemBytes = pair_smem_bytes(stages, kps);
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = 2;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  return fmt == kFmtINT8 ? pair_clusters_t<kFmtINT8>(cfg) : pair_clusters_t<kFmtFP8>(cfg);
}

cudaError_t launch_swapab(int fmt, int mpad, bool fused, const CUtensorMap& tw, const CUtensorMap& tx,
                          const GemmArgs& a, cudaStream_t stream) {
  return fused ? launch_swapab_f<true>(fmt, mpad, tw, tx, a, stream)
               : launch_swapab_f<false>(fmt, mpad, tw, tx, a, stream);
}

cudaError_t launch_standard(int fmt, int tile_n, const CUtensorMap& tx, const CUtensorMap& tw,
                            const GemmArgs& a, cudaStream_t stream) {
  if (fmt == kFmtFP8) return tile_n == 256 ? launch_standard_t<kFmtFP8, 256>(tx, tw, a, stream)
                                           : launch_standard_t<kFmtFP8, 128>(tx, tw, a, stream);
  if (fmt == kFmtINT8) return tile_n == 256 ? launch_standard_t<kFmtINT8, 256>(tx, tw, a, stream)
                                            : launch_standard_t<kFmtINT8, 128>(tx, tw, a, stream);
  if (fmt == kFmtBlock) return tile_n == 256 ? launch_standard_t<kFmtBlock, 256>(tx, tw, a, stream)
                                             : launch_standard_t<kFmtBlock, 128>(tx, tw, a, stream);
  return cudaErrorInvalidValue;
}

#ifdef QGD_TRACE
extern "C" __attribute__((visibility("default"))) int qgd_debug_trace(unsigned long long* host, size_t count) {
  const size_t cap = static_cast<size_t>(kTraceLaunches) * kTraceCtas * kTraceSlots;
  const size_t n = count < cap ? count : cap;
  return static_cast<int>(cudaMemcpyFromSymbol(host, g_trace, n * sizeof(unsigned long long)));
}
#endif

cudaError_t launch_tp_wait(const unsigned* flags, int ranks, bool pdl, cudaStream_t stream) {
  // with a programmatic dependency it starts early and reads the count only
  // after its griddepcontrol.wait, once this rank's GEMM is complete
  return launch_ex(tp_wait_kernel, dim3(1), dim3(32), 0, stream, pdl, flags, ranks);
}

cudaError_t read_device_error(unsigned int* code) {
  return cudaMemcpyFromSymbol(code, g_device_error, sizeof(unsigned int));
}

cudaError_t clear_device_error() {
  const unsigned int zero = 0;
  return cudaMemcpyToSymbol(g_device_error, &zero, sizeof(unsigned int));
}

cudaError_t launch_splitk_reduce(int fmt, const GemmArgs& a, cudaStream_t stream) {
  const size_t total = static_cast<size_t>(a.M) * a.N;
  const unsigned blocks = static_cast<unsigned>((total / 4 + 255) / 256);
  const bool pdl = a.pdl != 0;
  if (fmt == kFmtFP8) return launch_ex(splitk_reduce_kernel<kFmtFP8>, dim3(blocks), dim3(256), 0, stream, pdl, a);
  if (fmt == kFmtINT8) return launch_ex(splitk_reduce_kernel<kFmtINT8>, dim3(blocks), dim3(256), 0, stream, pdl, a);
  return launch_ex(splitk_reduce_kernel<kFmtBlock>, dim3(blocks), dim3(256), 0, stream, pdl, a);
}

cudaError_t launch_swapab_reduce(int fmt, int mpad, const GemmArgs& a, cudaStream_t stream) {
  const dim3 grid((a.N + kSwapTileN - 1) / kSwapTileN);
  const dim3 block(kSwapTileN);
  const bool pdl = a.pdl != 0;
  if (mpad != 16 && mpad != 32) return cudaErrorInvalidValue;  // two-pass covers at most 32 tokens
  switch (fmt * 2 + (mpad == 32 ? 1 : 0)) {
    case 0: return launch_ex(swapab_reduce_kernel<kFmtFP8, 16>, grid, block, 0, stream, pdl, a);
    case 1: return launch_ex(swapab_reduce_kernel<kFmtFP8, 32>, grid, block, 0, stream, pdl, a);
    case 2: return launch_ex(swapab_reduce_kernel<kFmtINT8, 16>, grid, block, 0, stream, pdl, a);
    case 3: return launch_ex(swapab_reduce_kernel<kFmtINT8, 32>, grid, block, 0, stream, pdl, a);
    case 4: return launch_ex(swapab_reduce_kernel<kFmtBlock, 16>, grid, block, 0, stream, pdl, a);
    case 5: return launch_ex(swapab_reduce_kernel<kFmtBlock, 32>, grid, block, 0, stream, pdl, a);
  }
  return cudaErrorInvalidValue;
}

}  // namespace qgd
