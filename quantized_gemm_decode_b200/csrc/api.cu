// C ABI of the library (declared in include/qgd.h): argument checking, plan
// selection from the dispatch table, workspace layout, TMA descriptor
// encoding, and kernel launch on the caller's stream.
#include <cudaTypedefs.h>
#include <stdarg.h>
#include <stdio.h>

#include <atomic>
#include <cstdlib>
#include <cstring>
#include <fstream>
#include <map>
#include <mutex>
#include <sstream>
#include <string>
#include <tuple>

#include "../../include/qgd.h"
#include "qgd_internal.h"

using namespace qgd;

namespace {

thread_local std::string g_err;

qgd_status fail(qgd_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_err = buf;
  if (getenv("QGD_LOG")) fprintf(stderr, "[qgd] %s\n", buf);
  return st;
}

qgd_status cuda_fail(cudaError_t e, const char* what) {
  return fail(QGD_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ---------------------------------------------------------------------------
// Device checks (per device, cached)
// ---------------------------------------------------------------------------
constexpr int kMaxDevices = 64;
int g_dev_ok[kMaxDevices];  // 0 unknown, 1 ok, -1 not sm_100
int g_num_sms = 148;         // used by the default plan; refreshed from the device

qgd_status check_device() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(QGD_ERR_DEVICE, "device index %d out of range", dev);
  if (g_dev_ok[dev] == 0) {
    int major = 0, minor = 0, sms = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (sms > 0) g_num_sms = sms;
    g_dev_ok[dev] = (major == 10 && minor == 0) ? 1 : -1;
  }
  if (g_dev_ok[dev] < 0) return fail(QGD_ERR_DEVICE, "device %d is not an sm_100 GPU; this library is built for sm_100a only", dev);
  return QGD_OK;
}

// ---------------------------------------------------------------------------
// TMA descriptors.  cuTensorMapEncodeTiled is a host-only driver function;
// it is looked up once through the runtime.
// ---------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

qgd_status get_encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &qr) == cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  if (!g_encode) return fail(QGD_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  return QGD_OK;
}

// 2-D byte matrix [rows, cols] (cols contiguous), box = box_rows x 128 bytes,
// 128-byte swizzle; out-of-range rows/columns read as zero.
// bf16 output [rows, cols] (cols contiguous) for tensor stores: boxes of
// 32 rows x 64 columns (128 bytes), 128-byte swizzle; parts of a box past the
// extent are not written.
qgd_status encode_out_bf16(CUtensorMap* map, void* base, int rows, int cols) {
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
  cuuint32_t box[2] = {64, 32};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(QGD_ERR_CUDA, "cuTensorMapEncodeTiled (output) failed (%d) rows=%d cols=%d", (int)r, rows, cols);
  return QGD_OK;
}

// Split-K partials as a 3-D tensor [splits][rows][cols] of 32-bit words
// (fp32 or int32 accumulator bits), boxes of 32 rows x 32 words, 128-byte
// swizzle: a box clips at `rows` within its own split.
qgd_status encode_partial_u32(CUtensorMap* map, void* base, int splits, int rows, int cols) {
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(splits)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(cols) * 4, static_cast<cuuint64_t>(rows) * cols * 4};
  cuuint32_t box[3] = {32, 32, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, base, dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(QGD_ERR_CUDA, "cuTensorMapEncodeTiled (partials) failed (%d) splits=%d rows=%d cols=%d", (int)r, splits,
                rows, cols);
  return QGD_OK;
}

qgd_status encode_kmajor(CUtensorMap* map, const void* base, int rows, int cols, int box_rows) {
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(kTileK), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(QGD_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d) rows=%d cols=%d box_rows=%d", (int)r, rows, cols, box_rows);
  return QGD_OK;
}

// ---------------------------------------------------------------------------
// Dispatch: table (format, N, K, M-bucket) -> plan; override per format.
// ---------------------------------------------------------------------------
// Workspace layout: a fixed header of per-tile arrival counters that every
// call leaves zero, then the Split-K data (partials, or the atomic
// accumulator, which is zeroed by a memset node at the start of the call).
// No call ever writes data into the header, so calls with different shapes
// and plans can share one workspace.
constexpr size_t kTicketBytes = 64 * 1024;
constexpr size_t kMaxTickets = kTicketBytes / 4;
const int kBuckets[] = {1, 2, 4, 8, 16, 24, 32, 64, 128, 512, 2048, 8192};
constexpr int kNumBuckets = sizeof(kBuckets) / sizeof(kBuckets[0]);
constexpr int kDecodeMaxM = 32;   // decode token counts: Swap-AB by default
constexpr int kSwapMaxM = 128;    // largest token count the Swap-AB kernel covers (FP8_Dynamic, W8A8_INT8)
// MXFP8 / NVFP4: at most 128 tokens.  Up to 64 tokens a CTA takes at most 256
// tensor-memory columns, so that two CTAs always fit in an SM's 512 (a CTA
// whose allocation had to wait for a cluster peer on the same SM would never
// be released); at 128 tokens it takes all 512 (two 128-column accumulators
// and the scale slots), and its ring holds at least four K slices, so that
// its shared memory keeps it alone on its SM.
constexpr int kMxMaxM = 128;
constexpr unsigned kMxMaxCols = 256;
constexpr int kMxWideSlices = 4;  // K slices in the ring of a 128-token CTA, at least

// Token columns of the Swap-AB MMA (its N): the next of 16, 32, 64, 128.
int swap_mpad(int M) { return M <= 16 ? 16 : (M <= 32 ? 32 : (M <= 64 ? 64 : 128)); }

struct Entry {
  int variant, split_k, reduce, stages, tile_n, schedule, occupancy, k_slices, fused;
};
using Key = std::tuple<int, int, int, int>;
std::mutex g_mu;
std::map<Key, Entry> g_table;
struct Override {
  int variant = -1, split_k = -1, reduce = -1, stages = 0, tile_n = 0, schedule = -1, occupancy = 0, k_slices = 0;
  int fused = -1;  // layer calls: -1 = table/default, 0/1 forced
} g_override[kNumFmts];

int bucket_of(int M) {
  for (int i = 0; i < kNumBuckets; ++i)
    if (M <= kBuckets[i]) return kBuckets[i];
  return kBuckets[kNumBuckets - 1];
}

int floor_pow2(int v) {
  int p = 1;
  while (p * 2 <= v) p *= 2;
  return p;
}

int fmt_from_name(const std::string& s) {
  if (s == "fp8_dynamic" || s == "fp8") return kFmtFP8;
  if (s == "w8a8_int8" || s == "int8") return kFmtINT8;
  if (s == "block_fp8" || s == "block") return kFmtBlock;
  if (s == "mxfp8" || s == "mx") return kFmtMX;
  if (s == "nvfp4" || s == "nv") return kFmtNV;
  return -1;
}

int variant_from_name(const std::string& s) {
  if (s == "standard") return kStandard;
  if (s == "swap_ab" || s == "swapab") return kSwapAB;
  if (s == "standard_pair") return kStandardPair;
  return -1;
}

int schedule_from_name(const std::string& s) {
  if (s == "grid") return kGrid;
  if (s == "persistent") return kPersistent;
  return -1;
}

int reduce_from_name(const std::string& s) {
  if (s == "last_cta") return kLastCta;
  if (s == "two_pass") return kTwoPass;
  if (s == "atomic") return kAtomic;
  if (s == "cluster") return kCluster;
  return -1;
}

// layer: the plan of a layer call from bf16 activations (the qlinear_*_bf16
// entry points), the only calls that can fuse the activation quantizer.
// K as the kernels count it: NVFP4 packs two values per byte
int kernel_k(int fmt, int K) { return fmt == kFmtNV ? K / 2 : K; }

// tp: a column-parallel call (qlinear_tp_bf16), whose output epilogue exists
// in the Swap-AB kernel only and must be the last kernel of the call.
qgd_plan make_plan(int fmt, int M, int N, int K, bool layer = false, bool tp = false) {
  const int nkt = (kernel_k(fmt, K) + kTileK - 1) / kTileK;
  qgd_plan p;
  p.source = 0;
  p.fused = 0;
  p.reduce = kLastCta;
  p.stages = 0;
  p.schedule = kGrid;
  p.occupancy = 0;
  p.k_slices = 0;
  if (M <= kDecodeMaxM) {
    // Decode: Swap-AB (the hand-written rule the method replaces with
    // measurement), persistent over all (tile, K-slice) units so that every
    // SM streams the same share of the weights.
    p.variant = kSwapAB;
    p.tile_n = kSwapTileN;
    p.schedule = kPersistent;
    const int tiles = (N + kSwapTileN - 1) / kSwapTileN;
    int s = 1;
    while (tiles * s < g_num_sms && s * 2 <= nkt && s < 256) s *= 2;
    p.split_k = s;  // used by the grid schedule
  } else {
    // Larger M: Standard tiles, one persistent CTA per SM (Block_FP8: two
    // weight blocks per tile, which keeps the tensor pipe twice as busy)
    p.variant = kStandard;
    p.tile_n = 256;
    p.split_k = 1;
    p.schedule = kPersistent;
  }
  {
    std::lock_guard<std::mutex> lk(g_mu);
    auto it = g_table.find(Key(fmt, N, K, bucket_of(M)));
    if (it != g_table.end()) {
      const Entry& e = it->second;
      p.variant = e.variant;
      p.split_k = e.split_k;
      p.reduce = e.reduce;
      p.stages = e.stages;
      p.tile_n = e.tile_n;
      p.schedule = e.schedule;
      p.occupancy = e.occupancy;
      p.k_slices = e.k_slices;
      p.fused = e.fused;
      p.source = 1;
    }
    const Override& o = g_override[fmt];
    if (o.variant >= 0 || o.split_k >= 0 || o.reduce >= 0 || o.stages > 0 || o.tile_n > 0 || o.schedule >= 0 ||
        o.occupancy > 0 || o.k_slices > 0) {
      if (o.variant >= 0) p.variant = o.variant;
      if (o.split_k >= 0) p.split_k = o.split_k;
      if (o.reduce >= 0) p.reduce = o.reduce;
      if (o.stages > 0) p.stages = o.stages;
      if (o.tile_n > 0) p.tile_n = o.tile_n;
      if (o.schedule >= 0) p.schedule = o.schedule;
      if (o.occupancy > 0) p.occupancy = o.occupancy;
      if (o.k_slices > 0) p.k_slices = o.k_slices;
      p.source = 2;
    }
    if (o.fused >= 0) {
      p.fused = o.fused;
      p.source = 2;
    }

  }
  // Make the plan legal for this shape.  (MXFP8 runs in the Swap-AB kernel
  // only, up to 128 tokens, and has no two-pass reduction kernel.)
  if (fmt == kFmtMX || fmt == kFmtNV || tp) {
    p.variant = kSwapAB;
    if (p.reduce == kTwoPass) p.reduce = kLastCta;
  }
  if (p.variant == kSwapAB && M > (fmt == kFmtBlock ? kDecodeMaxM : kSwapMaxM)) p.variant = kStandard;
  // CTA-pair tiles: the per-token / per-channel formats; Split-K with the
  // two-pass reduction only
  if (p.variant == kStandardPair && fmt != kFmtFP8 && fmt != kFmtINT8) p.variant = kStandard;
  if (p.variant < kStandard || p.variant > kStandardPair) p.variant = kStandard;
  if (p.variant == kSwapAB) p.tile_n = kSwapTileN;
  else if (p.variant == kStandardPair) p.tile_n = 256;
  else if (p.tile_n != 128 && p.tile_n != 256) p.tile_n = (fmt == kFmtBlock) ? 128 : 256;
  if (p.schedule != kPersistent) p.schedule = kGrid;
  // 128-wide K slices (K blocks) per pipeline stage: 1 or 2, at most the K extent
  if (p.k_slices < 1 || nkt < 2) p.k_slices = 1;
  if (p.k_slices > 2) p.k_slices = 2;
  const int nku = (nkt + p.k_slices - 1) / p.k_slices;  // K units per tile
  int smax = nku < 256 ? nku : 256;
  if (smax < 1) smax = 1;
  if (p.split_k < 1) p.split_k = 1;
  if (p.split_k > smax) p.split_k = smax;
  // a power of two, except in a cluster, whose reduction takes any 2..8, and
  // in pair tiles, whose two-pass reduction takes any count
  const bool any_split = p.reduce == kCluster || p.variant == kStandardPair;
  if (!any_split) p.split_k = floor_pow2(p.split_k);
  if (p.reduce < kLastCta || p.reduce > kCluster) p.reduce = kLastCta;
  // the two-pass reduction kernel covers at most 32 tokens
  if (p.variant == kSwapAB && M > kDecodeMaxM && p.reduce == kTwoPass) p.reduce = kLastCta;
  // cluster Split-K: the S splits of a tile form one thread-block cluster
  // (Swap-AB, or the one-CTA Standard kernel for FP8_Dynamic / W8A8_INT8;
  // grid schedule, 2 <= S <= 8)
  const bool std_cluster_ok = p.variant == kStandard && (fmt == kFmtFP8 || fmt == kFmtINT8);
  if (p.reduce == kCluster && ((p.variant != kSwapAB && !std_cluster_ok) || p.schedule != kGrid || p.split_k < 2 ||
                               p.split_k > kMaxClusterSplit))
    p.reduce = kLastCta;
  if (p.reduce != kCluster && p.variant != kStandardPair) p.split_k = floor_pow2(p.split_k);
  if (p.variant == kStandardPair) p.reduce = p.split_k > 1 ? kTwoPass : kLastCta;
  if (p.reduce != kTwoPass && p.variant != kStandardPair) {  // (pair tiles take no arrival counters)
    const size_t tiles = p.variant == kSwapAB
                             ? static_cast<size_t>((N + kSwapTileN - 1) / kSwapTileN)
                             : static_cast<size_t>((N + p.tile_n - 1) / p.tile_n) * ((M + kStdTileM - 1) / kStdTileM);
    if (tiles > kMaxTickets) p.reduce = kTwoPass;  // more tiles than arrival counters
  }
  // the fused quantizer exists in the Swap-AB kernel only; its two-pass
  // reduction would need the activation scales in memory, so it takes the
  // last-arriving CTA instead
  if (!layer || p.variant != kSwapAB || fmt == kFmtMX || fmt == kFmtNV) p.fused = 0;
  p.fused = p.fused ? 1 : 0;
  if (p.fused && p.reduce == kTwoPass) p.reduce = kLastCta;
  const int mpad = swap_mpad(M);
  const int max_st = p.variant == kSwapAB ? swapab_max_stages(mpad, p.k_slices, p.reduce == kCluster, p.fused != 0)
                     : p.variant == kStandardPair ? pair_max_stages(p.k_slices)
                                                  : standard_max_stages(p.tile_n, p.k_slices);
  if (p.stages <= 0 || p.stages > max_st) p.stages = max_st;
  if (p.stages < 2) p.stages = 2;
  // the Standard cluster reduction receives the other splits' rows in the
  // ring: (S - 1) ceil(128 / S) rows of tile_n fp32 values must fit there
  if (p.variant == kStandard && p.reduce == kCluster) {
    const size_t recv = static_cast<size_t>(p.split_k - 1) * ((kStdTileM + p.split_k - 1) / p.split_k) * p.tile_n * 4;
    const size_t ring = static_cast<size_t>(p.stages) * p.k_slices * (kStdTileM + p.tile_n) * kTileK;
    if (recv > ring) {
      p.reduce = kLastCta;
      p.split_k = floor_pow2(p.split_k);
    }
  }
  if (fmt == kFmtMX || fmt == kFmtNV) {
    if (mpad < 128) {
      while (p.stages > 2 && mx_tmem_cols(mpad, p.stages, p.k_slices, fmt) > kMxMaxCols) --p.stages;
    } else {
      // 128 tokens: all 512 columns, and a ring deep enough to fill more than
      // half of the SM's shared memory (one CTA per SM)
      while (p.stages * p.k_slices < kMxWideSlices && p.stages < max_st) ++p.stages;
      while (p.stages > 2 && mx_tmem_cols(mpad, p.stages, p.k_slices, fmt) > 512u) --p.stages;
    }
  }
  // CTAs per SM for the persistent grid: at most what shared memory (and, for
  // the Standard kernel, TMEM) allows, at most 2; 0 asks for that maximum.
  int fit = 1;
  if (p.schedule == kPersistent) {
    const size_t bytes = (p.variant == kSwapAB ? swapab_smem_bytes(mpad, p.stages, p.k_slices, false, p.fused != 0)
                                               : standard_smem_bytes(p.tile_n, p.stages, p.k_slices)) + 1024;
    fit = static_cast<int>(kSmemPerSM / bytes);
    fit = fit < 1 ? 1 : (fit > 2 ? 2 : fit);
    if (p.variant == kStandard && (p.tile_n == 256 || fmt == kFmtBlock)) fit = 1;  // all 512 TMEM columns
    if (p.variant == kStandardPair) fit = 1;

  }
  if (p.occupancy <= 0 || p.occupancy > fit) p.occupancy = fit;
  if (p.schedule != kPersistent) p.occupancy = 1;
  return p;
}

size_t align256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

// How many CTA-pair clusters fit on the current device at once, per
// (format, stages, K blocks per stage); queried once each (0 if unknown).
int pair_clusters_that_fit(int fmt, int stages, int kps) {
  static std::mutex mu;
  static std::map<std::tuple<int, int, int, int>, int> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  const auto key = std::make_tuple(dev, fmt, stages, kps);
  std::lock_guard<std::mutex> lk(mu);
  auto it = cache.find(key);
  if (it != cache.end()) return it->second;
  const int n = pair_max_active_clusters(fmt, stages, kps);
  cache[key] = n;
  return n;
}

long long sk_owner(long long u, long long G, long long U) { return ((u + 1) * G - 1) / U; }

// Everything a launch derives from the plan and the shape: the persistent
// schedule's CTA count, the partial-slot geometry and the workspace layout.
struct Exec {
  bool persistent = false;
  int ctas = 0;     // persistent schedule: CTAs launched
  int maxc = 1;     // most CTAs sharing one output tile
  int mpad = 16;    // Swap-AB: token columns per MMA (16, 32, 64 or 128)
  int mstride = 4;  // Swap-AB: partial row stride in words
  size_t tiles = 0;  // output tiles (arrival counters)
  size_t data_off = 0, data_bytes = 0, total = 0;
};

Exec make_exec(int fmt, const qgd_plan& p, int M, int N, int K) {
  Exec e;
  const int nkt = (kernel_k(fmt, K) + kTileK - 1) / kTileK;
  e.mpad = swap_mpad(M);
  e.mstride = (M + 3) / 4 * 4;
  if (M <= 0) return e;
  if (p.variant == kSwapAB) {
    const int n_tiles = (N + kSwapTileN - 1) / kSwapTileN;
    const int nku = (nkt + p.k_slices - 1) / p.k_slices;  // K units (stages) per tile
    e.tiles = n_tiles;
    if (p.schedule == kPersistent) {
      const long long U = static_cast<long long>(n_tiles) * nku;
      const long long cap = static_cast<long long>(g_num_sms) * p.occupancy;
      const long long G = U < cap ? U : cap;
      e.persistent = true;
      e.ctas = static_cast<int>(G);
      int maxc = 1;
      for (int t = 0; t < n_tiles; ++t) {
        const long long c = sk_owner(static_cast<long long>(t) * nku + nku - 1, G, U) -
                            sk_owner(static_cast<long long>(t) * nku, G, U) + 1;
        if (c > maxc) maxc = static_cast<int>(c);
      }
      e.maxc = maxc;
    } else {
      e.maxc = p.split_k;
    }
    if (e.maxc > 1 && p.reduce != kCluster)  // the cluster reduction needs no workspace
      e.data_bytes = p.reduce == kAtomic
                         ? align256(static_cast<size_t>(M) * N * 4)
                         : align256(static_cast<size_t>(n_tiles) * e.maxc * kSwapTileN * e.mstride * 4);
  } else if (p.variant == kStandardPair) {
    // 256 x 256 pair tiles dealt to CTA pairs (two CTAs each, one per SM);
    // the launch lowers the pair count to what fits on the GPU at once
    // ((tile, split) items with Split-K, whose fp32 partials a second kernel adds)
    e.maxc = p.split_k;
    e.tiles = static_cast<size_t>((N + 255) / 256) * ((M + 255) / 256);
    if (p.schedule == kPersistent) {
      const long long items = static_cast<long long>(e.tiles) * p.split_k;
      const long long pairs = g_num_sms / 2;
      e.persistent = true;
      e.ctas = static_cast<int>(2 * (items < pairs ? items : pairs));
    }
    if (p.split_k > 1) e.data_bytes = align256(static_cast<size_t>(M) * N * 4 * p.split_k);
  } else {
    e.maxc = p.split_k;
    e.tiles = static_cast<size_t>((N + p.tile_n - 1) / p.tile_n) * ((M + kStdTileM - 1) / kStdTileM);
    if (p.schedule == kPersistent) {
      // (tile, split) items dealt round-robin over the SMs; a CTA whose
      // accumulators take all 512 TMEM columns (2 x 256, or Block_FP8's
      // 4 x 128) leaves room for no second CTA on its SM
      const long long items = static_cast<long long>(e.tiles) * p.split_k;
      const long long cap = static_cast<long long>(g_num_sms) * p.occupancy;
      e.persistent = true;
      e.ctas = static_cast<int>(items < cap ? items : cap);
    }
    if (p.split_k > 1 && p.reduce != kCluster)  // the cluster reduction needs no workspace
      e.data_bytes = align256(static_cast<size_t>(M) * N * 4 * (p.reduce == kAtomic ? 1 : p.split_k));
  }
  if (e.data_bytes) {
    e.data_off = kTicketBytes;
    e.total = e.data_off + e.data_bytes;
  }
  return e;
}

// Programmatic dependent launch: on unless QGD_PDL=0 (read once, at the first
// launch) or qgd_set_pdl(0).  -1: not yet decided.
std::atomic<int> g_pdl{-1};

}  // namespace

bool qgd::pdl_enabled() {
  int v = g_pdl.load(std::memory_order_relaxed);
  if (v < 0) {
    const char* e = getenv("QGD_PDL");
    v = (e && e[0] == '0') ? 0 : 1;
    g_pdl.store(v, std::memory_order_relaxed);
  }
  return v != 0;
}

namespace {

std::atomic<int> g_call_seq{0};  // numbers GEMM calls for the developer timeline
std::atomic<int> g_withhold_acc{0};  // qgd_test_withhold_accumulator

qgd_status check_shape(int fmt, int M, int N, int K) {
  if (M < 0 || N <= 0 || K <= 0) return fail(QGD_ERR_INVALID, "sizes must be positive (M=%d N=%d K=%d)", M, N, K);
  if (N % 16 != 0) return fail(QGD_ERR_UNSUPPORTED, "N=%d must be a multiple of 16", N);
  if (K % 16 != 0) return fail(QGD_ERR_UNSUPPORTED, "K=%d must be a multiple of 16", K);
  if (fmt == kFmtBlock && (K % 128 != 0 || N % 128 != 0))
    return fail(QGD_ERR_UNSUPPORTED, "Block_FP8 needs N and K multiples of 128 (N=%d K=%d)", N, K);
  if (fmt == kFmtMX && K % 128 != 0) return fail(QGD_ERR_UNSUPPORTED, "MXFP8 needs K a multiple of 128 (K=%d)", K);
  if (fmt == kFmtMX && M > kMxMaxM)
    return fail(QGD_ERR_UNSUPPORTED, "MXFP8 covers at most %d tokens (M=%d)", kMxMaxM, M);
  if (fmt == kFmtNV && K % 256 != 0) return fail(QGD_ERR_UNSUPPORTED, "NVFP4 needs K a multiple of 256 (K=%d)", K);
  if (fmt == kFmtNV && M > kMxMaxM)
    return fail(QGD_ERR_UNSUPPORTED, "NVFP4 covers at most %d tokens (M=%d)", kMxMaxM, M);
  if (static_cast<long long>(M) * N > (1LL << 31)) return fail(QGD_ERR_UNSUPPORTED, "M*N too large");
  return QGD_OK;
}

std::atomic<void*> g_capture_xq{nullptr};    // qgd_test_capture_fused
std::atomic<float*> g_capture_sx{nullptr};

// One GEMM launch (plus its memset / second reduction kernel) for a plan.
// xbf != null: the fused layer call -- the kernel quantizes the bf16
// activations (rows ldxb elements apart) itself and xq/sx are unused.
// follows_memset: the caller has just enqueued a memset on `stream`, so the
// GEMM is launched without a programmatic dependency (that relaxation is
// defined between two kernels only).
// NVFP4: sx / sw are the fp32 row scales, sx8 / sw8 the E4M3 block scales.
// tp != null: a column-parallel call; the output goes to every rank's full Y
// (tp->y) and tp_done is this rank's completion counter (zero between calls).
qgd_status run_gemm_plan(int fmt, const qgd_plan& p, const void* xq, const float* sx, const uint16_t* xbf, int ldxb,
                         const void* wq, const float* sw, void* y, void* raw, int M, int N, int K, void* ws,
                         size_t ws_bytes, void* stream, bool follows_memset, const uint8_t* sx8 = nullptr,
                         const uint8_t* sw8 = nullptr, const qgd_tp* tp = nullptr, unsigned* tp_done = nullptr) {
  qgd_status st;
  if ((st = check_device()) != QGD_OK) return st;
  if ((st = get_encoder()) != QGD_OK) return st;
  const bool fused = xbf != nullptr;
  if (fused && (!p.fused || p.variant != kSwapAB)) return fail(QGD_ERR_INVALID, "internal: fused launch without a fused plan");
  if (tp && (p.variant != kSwapAB || p.reduce == kTwoPass || raw || !tp_done))
    return fail(QGD_ERR_INVALID, "internal: column-parallel launch without a one-kernel Swap-AB plan");
  const Exec ex = make_exec(fmt, p, M, N, K);
  if (ex.total > 0 && (!ws || ws_bytes < ex.total))
    return fail(QGD_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", ex.total, ws ? ws_bytes : 0);
  if (ex.total > 0 && !aligned16(ws)) return fail(QGD_ERR_INVALID, "workspace must be 16-byte aligned");

  GemmArgs a{};
  a.sx = sx;
  a.sw = sw;
  a.y = static_cast<uint16_t*>(y);
  a.raw = raw;
  a.partial = nullptr;
  a.accum = nullptr;
  a.tickets = nullptr;
  if (ex.total > 0) {
    uint8_t* wsb = static_cast<uint8_t*>(ws);
    a.tickets = reinterpret_cast<unsigned int*>(wsb);
    if (p.reduce == kAtomic) a.accum = wsb + ex.data_off;
    else a.partial = wsb + ex.data_off;
  }
  a.M = M;
  a.N = N;
  a.K = kernel_k(fmt, K);  // NVFP4: bytes of packed codes
  a.splits = p.split_k;
  a.reduce = p.reduce;
  a.stages = p.stages;
  a.persistent = ex.persistent ? 1 : 0;
  a.ctas = ex.ctas;
  a.maxc = ex.maxc;
  a.mstride = ex.mstride;
  a.kps = p.k_slices;
  a.pdl = (pdl_enabled() && !follows_memset) ? 1 : 0;
  a.trace_tag = g_call_seq.fetch_add(1, std::memory_order_relaxed) & 0x7fffffff;
  a.withhold_acc = g_withhold_acc.load(std::memory_order_relaxed);
  a.xbf = xbf;
  a.ldxb = ldxb;
  a.xq_out = fused ? static_cast<uint8_t*>(g_capture_xq.load()) : nullptr;
  a.sx_out = fused ? g_capture_sx.load() : nullptr;
  a.sx8 = fmt == kFmtMX ? reinterpret_cast<const uint8_t*>(sx) : fmt == kFmtNV ? sx8 : nullptr;
  a.sw8 = fmt == kFmtMX ? reinterpret_cast<const uint8_t*>(sw) : fmt == kFmtNV ? sw8 : nullptr;
  a.tp_ranks = 0;  // a plain call unless column-parallel
  a.tp_rank = 0;
  a.tp_col0 = 0;
  a.tp_ldy = 0;
  a.tp_done = nullptr;
  for (int r = 0; r < kMaxTpRanks; ++r) {
    a.tp_y[r] = nullptr;
    a.tp_flag[r] = nullptr;
  }
  if (tp) {
    a.tp_ranks = tp->ranks;
    a.tp_rank = tp->rank;
    a.tp_col0 = tp->col0;
    a.tp_ldy = tp->ldy;
    a.tp_done = tp_done;
    for (int r = 0; r < tp->ranks; ++r) {
      a.tp_y[r] = static_cast<uint16_t*>(tp->y[r]);
      a.tp_flag[r] = tp->flags[r];
    }
  }

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  CUtensorMap tw, tx;
  memset(&tx, 0, sizeof tx);
  cudaError_t e;
  if (a.accum) {
    e = cudaMemsetAsync(a.accum, 0, static_cast<size_t>(M) * N * 4, s);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync (atomic Split-K accumulator)");
    a.pdl = 0;  // the GEMM follows a memset, not a kernel
  }
  if (p.variant == kSwapAB) {
    if ((st = encode_kmajor(&tw, wq, N, a.K, kSwapTileN)) != QGD_OK) return st;
    if (!fused && (st = encode_kmajor(&tx, xq, M, a.K, ex.mpad)) != QGD_OK) return st;
    e = launch_swapab(fmt, ex.mpad, fused, tw, tx, a, s);
  } else if (p.variant == kStandardPair) {
    // each CTA of a pair loads 128 token rows and 128 weight rows per K block
    if ((st = encode_kmajor(&tx, xq, M, K, kStdTileM)) != QGD_OK) return st;
    if ((st = encode_kmajor(&tw, wq, N, K, 128)) != QGD_OK) return st;
    CUtensorMap ty;
    memset(&ty, 0, sizeof ty);
    if (a.splits > 1) {  // fp32 / int32 partials, one plane per split, for the two-pass reduction
      if ((st = encode_partial_u32(&ty, a.partial, a.splits, M, N)) != QGD_OK) return st;
    } else if (!raw && (st = encode_out_bf16(&ty, y, M, N)) != QGD_OK) {
      return st;
    }
    if (a.persistent) {
      const int fit = pair_clusters_that_fit(fmt, p.stages, p.k_slices);
      if (fit > 0 && a.ctas > 2 * fit) a.ctas = 2 * fit;
    }
    e = launch_standard_pair(fmt, tx, tw, ty, a, s);
  } else {
    if ((st = encode_kmajor(&tx, xq, M, K, kStdTileM)) != QGD_OK) return st;
    if ((st = encode_kmajor(&tw, wq, N, K, p.tile_n)) != QGD_OK) return st;
    e = launch_standard(fmt, p.tile_n, tx, tw, a, s);
  }
  if (e != cudaSuccess) return cuda_fail(e, "GEMM launch");
  if (ex.maxc > 1 && p.reduce == kTwoPass) {
    a.pdl = pdl_enabled() ? 1 : 0;
    e = p.variant == kSwapAB ? launch_swapab_reduce(fmt, ex.mpad, a, s) : launch_splitk_reduce(fmt, a, s);
    if (e != cudaSuccess) return cuda_fail(e, "Split-K reduce launch");
  }
  return QGD_OK;
}

qgd_status run_gemm(int fmt, const void* xq, const float* sx, const void* wq, const float* sw, void* y, void* raw,
                    int M, int N, int K, void* ws, size_t ws_bytes, void* stream, bool follows_memset = false,
                    const uint8_t* sx8 = nullptr, const uint8_t* sw8 = nullptr) {
  qgd_status st = check_shape(fmt, M, N, K);
  if (st != QGD_OK) return st;
  if (M == 0) return QGD_OK;
  if (!xq || !wq || (!y && !raw)) return fail(QGD_ERR_INVALID, "null operand pointer");
  if (!raw && (!sx || !sw)) return fail(QGD_ERR_INVALID, "null scale pointer");
  if (fmt == kFmtNV && (!sx8 || !sw8)) return fail(QGD_ERR_INVALID, "null block-scale pointer");
  if (!aligned16(xq) || !aligned16(wq) || !aligned16(y) || !aligned16(raw) || !aligned16(sx) || !aligned16(sw) ||
      !aligned16(sx8) || !aligned16(sw8))
    return fail(QGD_ERR_INVALID, "operand pointers must be 16-byte aligned");
  return run_gemm_plan(fmt, make_plan(fmt, M, N, K), xq, sx, nullptr, 0, wq, sw, y, raw, M, N, K, ws, ws_bytes,
                       stream, follows_memset, sx8, sw8);
}

// Workspace of a layer call from bf16 activations: the GEMM's own part first
// (its counter header must lead), then -- unless the plan fuses the
// quantizer -- the activation codes and their scales.  The codes never go
// into the counter header, even when this call's GEMM needs no workspace:
// a workspace serves calls of every shape and plan, and the header must stay
// zero between them.
struct LayerWs {
  qgd_plan plan;
  Exec ex;
  size_t xq_off = 0, sx_off = 0, sb_off = 0, total = 0;
};

// tp: a column-parallel call, whose completion counter lives in the last
// word of the counter header, so its workspace always holds the header.
LayerWs layer_ws(int fmt, int M, int N, int K, bool tp = false) {
  LayerWs l;
  l.plan = make_plan(fmt, M, N, K, true, tp);
  l.ex = make_exec(fmt, l.plan, M, N, K);
  l.total = l.ex.total;
  if (tp && l.total < kTicketBytes) l.total = kTicketBytes;
  if (!l.plan.fused && M > 0) {
    l.xq_off = align256(l.total > kTicketBytes ? l.total : kTicketBytes);
    l.sx_off = align256(l.xq_off + static_cast<size_t>(M) * kernel_k(fmt, K));
    // scales: fp32 per row or per 1x128 group; MXFP8: one byte per 32 values;
    // NVFP4: fp32 per row, then (sb_off) one byte per 16 values
    const size_t nsx = fmt == kFmtBlock ? static_cast<size_t>(M) * (K / kTileK)
                       : fmt == kFmtMX  ? (static_cast<size_t>(M) * (K / 32) + 3) / 4
                                        : static_cast<size_t>(M);
    l.total = align256(l.sx_off + nsx * 4);
    if (fmt == kFmtNV) {
      l.sb_off = l.total;
      l.total = align256(l.sb_off + static_cast<size_t>(M) * (K / 16));
    }
  }
  return l;
}

// tp != null: a column-parallel call (checked by the caller); y is unused.
qgd_status run_layer(int fmt, const void* x_bf16, int ldx, const void* wq, const float* sw, void* y, int M, int N,
                     int K, void* ws, size_t ws_bytes, void* stream, const uint8_t* sw8 = nullptr,
                     const qgd_tp* tp = nullptr) {
  qgd_status st = check_shape(fmt, M, N, K);
  if (st != QGD_OK) return st;
  if (ldx < K || ldx % 8 != 0)
    return fail(QGD_ERR_INVALID, "row stride ldx=%d must be >= K=%d and a multiple of 8", ldx, K);
  if (K > 65536) return fail(QGD_ERR_UNSUPPORTED, "K=%d must be <= 65536", K);
  if (M == 0) return QGD_OK;
  if (!x_bf16 || !wq || !sw || (!y && !tp) || (fmt == kFmtNV && !sw8))
    return fail(QGD_ERR_INVALID, "null operand pointer");
  if (!aligned16(x_bf16) || !aligned16(wq) || !aligned16(y) || !aligned16(sw) || !aligned16(sw8))
    return fail(QGD_ERR_INVALID, "operand pointers must be 16-byte aligned");
  const LayerWs l = layer_ws(fmt, M, N, K, tp != nullptr);
  if (l.total > 0 && (!ws || ws_bytes < l.total))
    return fail(QGD_ERR_WORKSPACE, "layer workspace of %zu bytes needed, %zu given", l.total, ws ? ws_bytes : 0);
  if (l.total > 0 && !aligned16(ws)) return fail(QGD_ERR_INVALID, "workspace must be 16-byte aligned");
  // column-parallel: the completion counter is the last word of the header
  unsigned* tp_done = tp ? static_cast<unsigned*>(ws) + (kMaxTickets - 1) : nullptr;
  const uint16_t* xb = static_cast<const uint16_t*>(x_bf16);
  if (l.plan.fused)
    return run_gemm_plan(fmt, l.plan, nullptr, nullptr, xb, ldx, wq, sw, y, nullptr, M, N, K, ws, ws_bytes, stream,
                         false, nullptr, nullptr, tp, tp_done);
  if ((st = check_device()) != QGD_OK) return st;
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  void* xq = wsb + l.xq_off;
  float* sx = reinterpret_cast<float*>(wsb + l.sx_off);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* sb = wsb + l.sb_off;  // NVFP4 block scales
  cudaError_t e = fmt == kFmtBlock ? launch_quant_group128(xb, M, K, ldx, static_cast<uint8_t*>(xq), sx, s)
                 : fmt == kFmtMX  ? launch_quant_mx(xb, M, K, ldx, static_cast<uint8_t*>(xq),
                                                    reinterpret_cast<uint8_t*>(sx), s)
                 : fmt == kFmtNV  ? launch_quant_nv(xb, M, K, ldx, static_cast<uint8_t*>(xq), sb, sx, s)
                                  : launch_quant_rows(xb, M, K, ldx, fmt == kFmtINT8 ? 1 : 0, xq, sx, s);
  if (e != cudaSuccess) return cuda_fail(e, "activation quantizer launch");
  return run_gemm_plan(fmt, l.plan, xq, sx, nullptr, 0, wq, sw, y, nullptr, M, N, K, ws, l.ex.total, stream, false,
                       fmt == kFmtNV ? sb : nullptr, sw8, tp, tp_done);
}

// ---------------------------------------------------------------------------
// Built-in scratch for qlinear_fp8_dynamic_noalloc.  Some callers must not
// allocate device memory once they are running: an engine that carves all
// device memory into fixed pools at start-up has none left to give, and a
// cudaMalloc in a latency-critical loop can block until the device is idle.
// They get the Split-K workspace from this fixed array instead.  Every GPU
// that loads the library holds it until the process exits.  Its first 64 KiB
// are the arrival-counter header (zero at load, left zero by every call, and
// cleared again at the start of each call that splits K); the rest holds
// Split-K partials.
// ---------------------------------------------------------------------------
constexpr size_t kNoAllocScratchBytes = 8u << 20;  // 8 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_addr[kMaxDevices];

// Device address of the scratch array on the current device.  In host code
// `g_noalloc_scratch` names a host-side stand-in, never the device memory, so
// the address is looked up once per device (with that device current).
qgd_status noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(QGD_ERR_DEVICE, "device index %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress (built-in Split-K scratch)");
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return QGD_OK;
}

}  // namespace

extern "C" {

qgd_status quant_act_per_token_strided(const void* x_bf16, int M, int K, int ldx, int qtype, void* xq, float* sx,
                                       void* stream) {
  if (M < 0 || K <= 0) return fail(QGD_ERR_INVALID, "sizes must be positive (M=%d K=%d)", M, K);
  if (qtype != QGD_QTYPE_E4M3 && qtype != QGD_QTYPE_INT8) return fail(QGD_ERR_INVALID, "bad qtype %d", qtype);
  if (K % 8 != 0 || K > 65536) return fail(QGD_ERR_UNSUPPORTED, "K=%d must be a multiple of 8 and <= 65536", K);
  if (ldx < K || ldx % 8 != 0) return fail(QGD_ERR_INVALID, "row stride ldx=%d must be >= K=%d and a multiple of 8", ldx, K);
  if (M == 0) return QGD_OK;
  if (!x_bf16 || !xq || !sx) return fail(QGD_ERR_INVALID, "null pointer");
  if (!aligned16(x_bf16) || !aligned16(xq) || (reinterpret_cast<uintptr_t>(sx) & 3u))
    return fail(QGD_ERR_INVALID, "x and xq must be 16-byte aligned, sx 4-byte aligned");
  qgd_status st = check_device();
  if (st != QGD_OK) return st;
  cudaError_t e = launch_quant_rows(static_cast<const uint16_t*>(x_bf16), M, K, ldx, qtype, xq, sx,
                                    static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? QGD_OK : cuda_fail(e, "quant_act_per_token launch");
}

qgd_status quant_act_per_token(const void* x_bf16, int M, int K, int qtype, void* xq, float* sx, void* stream) {
  return quant_act_per_token_strided(x_bf16, M, K, K, qtype, xq, sx, stream);
}

qgd_status quant_act_group128_strided(const void* x_bf16, int M, int K, int ldx, void* xq, float* sx,
                                      void* stream) {
  if (M < 0 || K <= 0) return fail(QGD_ERR_INVALID, "sizes must be positive (M=%d K=%d)", M, K);
  if (K % 128 != 0) return fail(QGD_ERR_UNSUPPORTED, "K=%d must be a multiple of 128", K);
  if (ldx < K || ldx % 8 != 0) return fail(QGD_ERR_INVALID, "row stride ldx=%d must be >= K=%d and a multiple of 8", ldx, K);
  if (M == 0) return QGD_OK;
  if (!x_bf16 || !xq || !sx) return fail(QGD_ERR_INVALID, "null pointer");
  if (!aligned16(x_bf16) || !aligned16(xq) || (reinterpret_cast<uintptr_t>(sx) & 3u))
    return fail(QGD_ERR_INVALID, "x and xq must be 16-byte aligned, sx 4-byte aligned");
  qgd_status st = check_device();
  if (st != QGD_OK) return st;
  cudaError_t e = launch_quant_group128(static_cast<const uint16_t*>(x_bf16), M, K, ldx, static_cast<uint8_t*>(xq),
                                        sx, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? QGD_OK : cuda_fail(e, "quant_act_group128 launch");
}

qgd_status quant_act_group128(const void* x_bf16, int M, int K, void* xq, float* sx, void* stream) {
  return quant_act_group128_strided(x_bf16, M, K, K, xq, sx, stream);
}

qgd_status quant_act_mx(const void* x_bf16, int M, int K, int ldx, void* xq, void* s_e8m0, void* stream) {
  if (M < 0 || K <= 0) return fail(QGD_ERR_INVALID, "sizes must be positive (M=%d K=%d)", M, K);
  if (K % 32 != 0) return fail(QGD_ERR_UNSUPPORTED, "K=%d must be a multiple of 32", K);
  if (ldx < K || ldx % 8 != 0)
    return fail(QGD_ERR_INVALID, "row stride ldx=%d must be >= K=%d and a multiple of 8", ldx, K);
  if (M == 0) return QGD_OK;
  if (!x_bf16 || !xq || !s_e8m0) return fail(QGD_ERR_INVALID, "null pointer");
  if (!aligned16(x_bf16) || !aligned16(xq)) return fail(QGD_ERR_INVALID, "x and xq must be 16-byte aligned");
  qgd_status st = check_device();
  if (st != QGD_OK) return st;
  cudaError_t e = launch_quant_mx(static_cast<const uint16_t*>(x_bf16), M, K, ldx, static_cast<uint8_t*>(xq),
                                  static_cast<uint8_t*>(s_e8m0), static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? QGD_OK : cuda_fail(e, "quant_act_mx launch");
}

qgd_status quant_nvfp4(const void* x_bf16, int rows, int K, int ldx, void* q, void* s_e4m3, float* g, void* stream) {
  if (rows < 0 || K <= 0) return fail(QGD_ERR_INVALID, "sizes must be positive (rows=%d K=%d)", rows, K);
  if (K % 16 != 0 || K > 65536) return fail(QGD_ERR_UNSUPPORTED, "K=%d must be a multiple of 16, at most 65536", K);
  if (ldx < K || ldx % 8 != 0)
    return fail(QGD_ERR_INVALID, "row stride ldx=%d must be >= K=%d and a multiple of 8", ldx, K);
  if (rows == 0) return QGD_OK;
  if (!x_bf16 || !q || !s_e4m3 || !g) return fail(QGD_ERR_INVALID, "null pointer");
  if (!aligned16(x_bf16) || (reinterpret_cast<uintptr_t>(q) & 7u) || (reinterpret_cast<uintptr_t>(g) & 3u))
    return fail(QGD_ERR_INVALID, "x must be 16-byte aligned, q 8-byte and g 4-byte aligned");
  qgd_status st = check_device();
  if (st != QGD_OK) return st;
  cudaError_t e = launch_quant_nv(static_cast<const uint16_t*>(x_bf16), rows, K, ldx, static_cast<uint8_t*>(q),
                                  static_cast<uint8_t*>(s_e4m3), g, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? QGD_OK : cuda_fail(e, "quant_nvfp4 launch");
}

qgd_status quant_weight_block128(const void* w_bf16, int N, int K, void* wq, float* sw, void* stream) {
  if (N <= 0 || K <= 0) return fail(QGD_ERR_INVALID, "sizes must be positive (N=%d K=%d)", N, K);
  if (N % 128 != 0 || K % 128 != 0) return fail(QGD_ERR_UNSUPPORTED, "N=%d and K=%d must be multiples of 128", N, K);
  if (!w_bf16 || !wq || !sw) return fail(QGD_ERR_INVALID, "null pointer");
  if (!aligned16(w_bf16) || !aligned16(wq) || (reinterpret_cast<uintptr_t>(sw) & 3u))
    return fail(QGD_ERR_INVALID, "w and wq must be 16-byte aligned, sw 4-byte aligned");
  qgd_status st = check_device();
  if (st != QGD_OK) return st;
  cudaError_t e = launch_quant_block128(static_cast<const uint16_t*>(w_bf16), N, K, static_cast<uint8_t*>(wq), sw,
                                        static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? QGD_OK : cuda_fail(e, "quant_weight_block128 launch");
}

qgd_status qlinear_fp8_dynamic(const void* xq, const float* sx, const void* wq, const float* sw, void* y_bf16,
                               int M, int N, int K, void* ws, size_t ws_bytes, void* stream) {
  return run_gemm(kFmtFP8, xq, sx, wq, sw, y_bf16, nullptr, M, N, K, ws, ws_bytes, stream);
}

qgd_status qlinear_w8a8_int8(const void* xq, const float* sx, const void* wq, const float* sw, void* y_bf16,
                             int M, int N, int K, void* ws, size_t ws_bytes, void* stream) {
  return run_gemm(kFmtINT8, xq, sx, wq, sw, y_bf16, nullptr, M, N, K, ws, ws_bytes, stream);
}

qgd_status qlinear_block_fp8(const void* xq, const float* sx, const void* wq, const float* sw, void* y_bf16,
                             int M, int N, int K, void* ws, size_t ws_bytes, void* stream) {
  return run_gemm(kFmtBlock, xq, sx, wq, sw, y_bf16, nullptr, M, N, K, ws, ws_bytes, stream);
}

qgd_status qlinear_mxfp8(const void* xq, const void* sx_e8m0, const void* wq, const void* sw_e8m0, void* y_bf16,
                         int M, int N, int K, void* ws, size_t ws_bytes, void* stream) {
  // the E8M0 scale rows are read as 32-bit words (4 blocks = one 128-wide K slice)
  if ((reinterpret_cast<uintptr_t>(sx_e8m0) & 3u) || (reinterpret_cast<uintptr_t>(sw_e8m0) & 3u))
    return fail(QGD_ERR_INVALID, "MXFP8 scale arrays must be 4-byte aligned");
  return run_gemm(kFmtMX, xq, static_cast<const float*>(sx_e8m0), wq, static_cast<const float*>(sw_e8m0), y_bf16,
                  nullptr, M, N, K, ws, ws_bytes, stream);
}

qgd_status qlinear_nvfp4(const void* xq, const void* sx_e4m3, const float* gx, const void* wq, const void* sw_e4m3,
                         const float* gw, void* y_bf16, int M, int N, int K, void* ws, size_t ws_bytes, void* stream) {
  return run_gemm(kFmtNV, xq, gx, wq, gw, y_bf16, nullptr, M, N, K, ws, ws_bytes, stream, false,
                  static_cast<const uint8_t*>(sx_e4m3), static_cast<const uint8_t*>(sw_e4m3));
}

qgd_status qlinear_nvfp4_bf16(const void* x_bf16, int ldx, const void* wq, const void* sw_e4m3, const float* gw,
                              void* y_bf16, int M, int N, int K, void* ws, size_t ws_bytes, void* stream) {
  return run_layer(kFmtNV, x_bf16, ldx, wq, gw, y_bf16, M, N, K, ws, ws_bytes, stream,
                   static_cast<const uint8_t*>(sw_e4m3));
}

qgd_status qlinear_fp8_dynamic_bf16(const void* x_bf16, int ldx, const void* wq, const float* sw, void* y_bf16,
                                    int M, int N, int K, void* ws, size_t ws_bytes, void* stream) {
  return run_layer(kFmtFP8, x_bf16, ldx, wq, sw, y_bf16, M, N, K, ws, ws_bytes, stream);
}

qgd_status qlinear_w8a8_int8_bf16(const void* x_bf16, int ldx, const void* wq, const float* sw, void* y_bf16,
                                  int M, int N, int K, void* ws, size_t ws_bytes, void* stream) {
  return run_layer(kFmtINT8, x_bf16, ldx, wq, sw, y_bf16, M, N, K, ws, ws_bytes, stream);
}

qgd_status qlinear_block_fp8_bf16(const void* x_bf16, int ldx, const void* wq, const float* sw, void* y_bf16,
                                  int M, int N, int K, void* ws, size_t ws_bytes, void* stream) {
  return run_layer(kFmtBlock, x_bf16, ldx, wq, sw, y_bf16, M, N, K, ws, ws_bytes, stream);
}

qgd_status qlinear_mxfp8_bf16(const void* x_bf16, int ldx, const void* wq, const void* sw_e8m0, void* y_bf16,
                              int M, int N, int K, void* ws, size_t ws_bytes, void* stream) {
  return run_layer(kFmtMX, x_bf16, ldx, wq, static_cast<const float*>(sw_e8m0), y_bf16, M, N, K, ws, ws_bytes,
                   stream);
}

// ---------------------------------------------------------------------------
// Column-parallel (tensor-parallel) layer call: this rank's N-shard of the
// weights, its output tile written straight into every rank's full Y.
size_t qgd_tp_workspace_size(int fmt, int M, int N, int K) {
  if (fmt < 0 || fmt >= kNumFmts || M <= 0 || N <= 0 || K <= 0) return 0;
  return layer_ws(fmt, M, N, K, true).total;
}

qgd_status qlinear_tp_bf16(int fmt, const void* x_bf16, int ldx, const void* wq, const void* sw,
                           const void* sw_block, int M, int N, int K, const qgd_tp* tp, void* ws, size_t ws_bytes,
                           void* stream) {
  if (fmt < 0 || fmt >= kNumFmts) return fail(QGD_ERR_INVALID, "bad format %d", fmt);
  if (!tp) return fail(QGD_ERR_INVALID, "null tensor-parallel descriptor");
  if (tp->ranks < 1 || tp->ranks > kMaxTpRanks || tp->rank < 0 || tp->rank >= tp->ranks)
    return fail(QGD_ERR_INVALID, "rank %d of %d ranks (1..%d ranks)", tp->rank, tp->ranks, kMaxTpRanks);
  if (N <= 0 || tp->col0 < 0 || tp->ldy % 8 != 0 || static_cast<long long>(tp->col0) + N > tp->ldy)
    return fail(QGD_ERR_INVALID, "shard columns [%d, %d) outside a full output %d wide (a multiple of 8)", tp->col0,
                tp->col0 + N, tp->ldy);
  for (int r = 0; r < tp->ranks; ++r) {
    if (!tp->y[r] || !tp->flags[r]) return fail(QGD_ERR_INVALID, "null output or flag pointer of rank %d", r);
    if (!aligned16(tp->y[r]) || reinterpret_cast<uintptr_t>(tp->flags[r]) % 4 != 0)
      return fail(QGD_ERR_INVALID, "rank %d: output must be 16-byte aligned, flags 4-byte aligned", r);
  }
  const int max_m = fmt == kFmtBlock ? kDecodeMaxM : (fmt == kFmtMX || fmt == kFmtNV) ? kMxMaxM : kSwapMaxM;
  if (M > max_m)
    return fail(QGD_ERR_UNSUPPORTED, "column-parallel calls cover at most %d tokens in this format (M=%d)", max_m, M);
  if (static_cast<long long>(M) * tp->ldy > (1LL << 31)) return fail(QGD_ERR_UNSUPPORTED, "M*ldy too large");
  if (static_cast<size_t>((N + kSwapTileN - 1) / kSwapTileN) >= kMaxTickets)
    return fail(QGD_ERR_UNSUPPORTED, "N=%d has more output tiles than the counter header holds", N);
  if (!ws) return fail(QGD_ERR_WORKSPACE, "column-parallel calls need a workspace");
  return run_layer(fmt, x_bf16, ldx, wq, static_cast<const float*>(sw), nullptr, M, N, K, ws, ws_bytes, stream,
                   static_cast<const uint8_t*>(sw_block), tp);
}

qgd_status qgd_tp_wait(const unsigned int* flags, int ranks, void* stream) {
  if (!flags || reinterpret_cast<uintptr_t>(flags) % 4 != 0) return fail(QGD_ERR_INVALID, "null or misaligned flags");
  if (ranks < 1 || ranks > kMaxTpRanks) return fail(QGD_ERR_INVALID, "%d ranks (1..%d)", ranks, kMaxTpRanks);
  qgd_status st;
  if ((st = check_device()) != QGD_OK) return st;
  const cudaError_t e = launch_tp_wait(flags, ranks, pdl_enabled(), static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "tensor-parallel wait launch");
  return QGD_OK;
}

static_assert(sizeof(cudaIpcMemHandle_t) == QGD_IPC_HANDLE_BYTES, "IPC handle size");
static_assert(QGD_MAX_TP_RANKS == kMaxTpRanks, "tensor-parallel rank limit");

qgd_status qgd_ipc_malloc(size_t bytes, void** dptr, void* handle) {
  if (!dptr || !handle || bytes == 0) return fail(QGD_ERR_INVALID, "null pointer or zero size");
  *dptr = nullptr;
  qgd_status st;
  if ((st = check_device()) != QGD_OK) return st;
  void* p = nullptr;
  cudaError_t e = cudaMalloc(&p, bytes);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMalloc (shared buffer)");
  e = cudaMemset(p, 0, bytes);
  cudaIpcMemHandle_t h;
  if (e == cudaSuccess) e = cudaIpcGetMemHandle(&h, p);
  if (e != cudaSuccess) {
    cudaFree(p);
    return cuda_fail(e, "zeroing or exporting a shared buffer");
  }
  memcpy(handle, &h, sizeof h);
  *dptr = p;
  return QGD_OK;
}

qgd_status qgd_ipc_open(const void* handle, void** dptr) {
  if (!handle || !dptr) return fail(QGD_ERR_INVALID, "null pointer");
  *dptr = nullptr;
  qgd_status st;
  if ((st = check_device()) != QGD_OK) return st;
  cudaIpcMemHandle_t h;
  memcpy(&h, handle, sizeof h);
  const cudaError_t e = cudaIpcOpenMemHandle(dptr, h, cudaIpcMemLazyEnablePeerAccess);
  if (e != cudaSuccess) return cuda_fail(e, "cudaIpcOpenMemHandle");
  return QGD_OK;
}

qgd_status qgd_ipc_close(void* dptr) {
  if (!dptr) return fail(QGD_ERR_INVALID, "null pointer");
  const cudaError_t e = cudaIpcCloseMemHandle(dptr);
  if (e != cudaSuccess) return cuda_fail(e, "cudaIpcCloseMemHandle");
  return QGD_OK;
}

qgd_status qgd_ipc_free(void* dptr) {
  if (!dptr) return fail(QGD_ERR_INVALID, "null pointer");
  const cudaError_t e = cudaFree(dptr);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFree (shared buffer)");
  return QGD_OK;
}

size_t qgd_layer_workspace_size(int fmt, int M, int N, int K) {
  if (fmt < 0 || fmt >= kNumFmts || M <= 0 || N <= 0 || K <= 0) return 0;
  return layer_ws(fmt, M, N, K).total;
}

qgd_status qgd_get_layer_plan(int fmt, int M, int N, int K, qgd_plan* plan) {
  if (!plan) return fail(QGD_ERR_INVALID, "null plan");
  if (fmt < 0 || fmt >= kNumFmts) return fail(QGD_ERR_INVALID, "bad format %d", fmt);
  if (M < 0 || N <= 0 || K <= 0) return fail(QGD_ERR_INVALID, "bad sizes");
  *plan = make_plan(fmt, M < 1 ? 1 : M, N, K, true);
  return QGD_OK;
}

qgd_status qgd_set_fused_override(int fmt, int fused) {
  if (fmt < 0 || fmt >= kNumFmts) return fail(QGD_ERR_INVALID, "bad format %d", fmt);
  if (fused < -1 || fused > 1) return fail(QGD_ERR_INVALID, "fused must be -1, 0 or 1");
  std::lock_guard<std::mutex> lk(g_mu);
  g_override[fmt].fused = fused;
  return QGD_OK;
}

qgd_status qgd_test_capture_fused(void* xq, float* sx) {
  g_capture_xq.store(xq);
  g_capture_sx.store(sx);
  return QGD_OK;
}

qgd_status qgd_w8a8_int8_acc32(const void* xq, const void* wq, int32_t* acc, int M, int N, int K, void* ws,
                               size_t ws_bytes, void* stream) {
  if (M > 0 && !acc) return fail(QGD_ERR_INVALID, "null accumulator pointer");
  return run_gemm(kFmtINT8, xq, nullptr, wq, nullptr, nullptr, acc, M, N, K, ws, ws_bytes, stream);
}

qgd_status qlinear_fp8_dynamic_noalloc(const void* xq, const float* sx, const void* wq, const float* sw,
                                       void* y_bf16, int M, int N, int K, void* stream) {
  qgd_status st = check_shape(kFmtFP8, M, N, K);
  if (st != QGD_OK) return st;
  if (M == 0) return QGD_OK;
  const qgd_plan p = make_plan(kFmtFP8, M, N, K);
  const Exec ex = make_exec(kFmtFP8, p, M, N, K);
  if (ex.total > kNoAllocScratchBytes)
    return fail(QGD_ERR_WORKSPACE,
                "qlinear_fp8_dynamic_noalloc: this plan (split_k=%d, M=%d, N=%d) needs %zu bytes of Split-K "
                "scratch but the built-in scratch holds %zu; use qlinear_fp8_dynamic with a workspace or a "
                "smaller split_k",
                p.split_k, M, N, ex.total, kNoAllocScratchBytes);
  if ((st = check_device()) != QGD_OK) return st;
  void* scratch = nullptr;
  if ((st = noalloc_scratch(&scratch)) != QGD_OK) return st;
  if (ex.total > 0) {
    // the counters this call uses must start at zero whatever an earlier
    // (possibly interrupted) call left behind
    cudaError_t e = cudaMemsetAsync(scratch, 0, ex.tiles * 4, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync (built-in scratch counters)");
  }
  return run_gemm(kFmtFP8, xq, sx, wq, sw, y_bf16, nullptr, M, N, K, scratch, kNoAllocScratchBytes, stream,
                  ex.total > 0);
}

size_t qgd_workspace_size(int fmt, int M, int N, int K) {
  if (fmt < 0 || fmt >= kNumFmts || M <= 0 || N <= 0 || K <= 0) return 0;
  return make_exec(fmt, make_plan(fmt, M, N, K), M, N, K).total;
}

qgd_status qgd_load_dispatch_table(const char* path) {
  if (!path) return fail(QGD_ERR_INVALID, "null path");
  std::ifstream in(path);
  if (!in) return fail(QGD_ERR_TABLE, "cannot open dispatch table %s", path);
  std::map<Key, Entry> t;
  std::string line;
  int lineno = 0;
  while (std::getline(in, line)) {
    ++lineno;
    const size_t hash = line.find('#');
    if (hash != std::string::npos) line.resize(hash);
    std::istringstream ls(line);
    std::string fmt_s, var_s, red_s, sch_s;
    int N, K, Mb, split, stages, tile_n, occ, kslices = 0;
    if (!(ls >> fmt_s)) continue;  // blank line
    if (!(ls >> N >> K >> Mb >> var_s >> split >> red_s >> stages >> tile_n >> sch_s >> occ))
      return fail(QGD_ERR_TABLE,
                  "%s:%d: expected 11 to 13 fields: fmt N K M_bucket variant split_k reduce stages tile_n schedule "
                  "occupancy [k_slices [fused]]",
                  path, lineno);
    std::string extra;
    int fused = 0;
    if (ls >> extra) {
      char* end = nullptr;
      const long v = strtol(extra.c_str(), &end, 10);
      if (*end != '\0' || v < 0 || v > 2) return fail(QGD_ERR_TABLE, "%s:%d: bad k_slices '%s'", path, lineno, extra.c_str());
      kslices = static_cast<int>(v);
      if (ls >> extra) {
        const long f = strtol(extra.c_str(), &end, 10);
        if (*end != '\0' || f < 0 || f > 1) return fail(QGD_ERR_TABLE, "%s:%d: bad fused '%s'", path, lineno, extra.c_str());
        fused = static_cast<int>(f);
        if (ls >> extra) return fail(QGD_ERR_TABLE, "%s:%d: trailing field '%s'", path, lineno, extra.c_str());
      }
    }
    const int fmt = fmt_from_name(fmt_s), var = variant_from_name(var_s), red = reduce_from_name(red_s);
    const int sch = schedule_from_name(sch_s);
    if (fmt < 0 || var < 0 || red < 0 || sch < 0)
      return fail(QGD_ERR_TABLE, "%s:%d: unknown format/variant/reduce/schedule name", path, lineno);
    if (N <= 0 || K <= 0 || bucket_of(Mb) != Mb)
      return fail(QGD_ERR_TABLE, "%s:%d: bad N/K or M bucket %d", path, lineno, Mb);
    if (split < 1 || split > 256 ||
        ((split & (split - 1)) != 0 && !(red == kCluster && split <= kMaxClusterSplit) && var != kStandardPair))
      return fail(QGD_ERR_TABLE,
                  "%s:%d: split_k %d is not a power of two in 1..256 (or 2..8 with cluster, any with pair tiles)",
                  path, lineno, split);
    if (stages < 0 || stages > kMaxStages || (tile_n != 0 && tile_n != 128 && tile_n != 256) || occ < 0 ||
        occ > 2)
      return fail(QGD_ERR_TABLE, "%s:%d: bad stages/tile_n/occupancy", path, lineno);
    t[Key(fmt, N, K, Mb)] = Entry{var, split, red, stages, tile_n, sch, occ, kslices, fused};
  }
  std::lock_guard<std::mutex> lk(g_mu);
  g_table.swap(t);
  return QGD_OK;
}

qgd_status qgd_clear_dispatch_table(void) {
  std::lock_guard<std::mutex> lk(g_mu);
  g_table.clear();
  return QGD_OK;
}

qgd_status qgd_set_override(int fmt, int variant, int split_k, int reduce, int stages, int tile_n, int schedule,
                            int occupancy, int k_slices) {
  if (fmt < 0 || fmt >= kNumFmts) return fail(QGD_ERR_INVALID, "bad format %d", fmt);
  if (variant > 2 || reduce > 3 || split_k > 256 || stages > kMaxStages || stages < 0 || schedule > 1 ||
      occupancy < 0 || occupancy > 2 || k_slices < 0 || k_slices > 2 ||
      (tile_n != 0 && tile_n != 128 && tile_n != 256))
    return fail(QGD_ERR_INVALID, "bad override");
  if (split_k > 0 && (split_k & (split_k - 1)) != 0 && !(reduce == kCluster && split_k <= kMaxClusterSplit) &&
      variant != kStandardPair)
    return fail(QGD_ERR_INVALID,
                "split_k must be a power of two (any 2..8 with the cluster reduction, any with pair tiles)");
  std::lock_guard<std::mutex> lk(g_mu);
  Override& o = g_override[fmt];
  o.variant = variant < 0 ? -1 : variant;
  o.split_k = split_k <= 0 ? -1 : split_k;
  o.reduce = reduce < 0 ? -1 : reduce;
  o.stages = stages;
  o.tile_n = tile_n;
  o.schedule = schedule < 0 ? -1 : schedule;
  o.occupancy = occupancy;
  o.k_slices = k_slices;
  return QGD_OK;
}

qgd_status qgd_get_plan(int fmt, int M, int N, int K, qgd_plan* plan) {
  if (!plan) return fail(QGD_ERR_INVALID, "null plan");
  if (fmt < 0 || fmt >= kNumFmts) return fail(QGD_ERR_INVALID, "bad format %d", fmt);
  if (M < 0 || N <= 0 || K <= 0) return fail(QGD_ERR_INVALID, "bad sizes");
  *plan = make_plan(fmt, M < 1 ? 1 : M, N, K);
  return QGD_OK;
}

int qgd_m_bucket(int M) { return bucket_of(M < 1 ? 1 : M); }

const char* qgd_status_string(int status) {
  switch (status) {
    case QGD_OK: return "ok";
    case QGD_ERR_INVALID: return "invalid argument";
    case QGD_ERR_UNSUPPORTED: return "unsupported shape";
    case QGD_ERR_WORKSPACE: return "workspace too small";
    case QGD_ERR_CUDA: return "CUDA error";
    case QGD_ERR_TABLE: return "dispatch table error";
    case QGD_ERR_DEVICE: return "unsupported device";
  }
  return "unknown status";
}

const char* qgd_last_error_message(void) { return g_err.c_str(); }

qgd_status qgd_device_error(unsigned int* code) {
  if (!code) return fail(QGD_ERR_INVALID, "null code");
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
  e = read_device_error(code);
  if (e == cudaSuccess && *code == 0) e = read_probe_error(code);
  return e == cudaSuccess ? QGD_OK : cuda_fail(e, "read device error flag");
}

qgd_status qgd_clear_device_error(void) {
  cudaError_t e = clear_device_error();
  if (e == cudaSuccess) e = clear_probe_error();
  return e == cudaSuccess ? QGD_OK : cuda_fail(e, "clear device error flag");
}

qgd_status qgd_mma_peak_probe(int qtype, int iters, double* flops, void* stream) {
  if (qtype != QGD_QTYPE_E4M3 && qtype != QGD_QTYPE_INT8) return fail(QGD_ERR_INVALID, "bad qtype %d", qtype);
  if (iters < 1 || iters > 200000) return fail(QGD_ERR_INVALID, "iters=%d must be in [1, 200000]", iters);
  qgd_status st = check_device();
  if (st != QGD_OK) return st;
  if (flops) *flops = mma_probe_flops(iters, g_num_sms);
  cudaError_t e = launch_mma_probe(qtype, iters, g_num_sms, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? QGD_OK : cuda_fail(e, "qgd_mma_peak_probe launch");
}

qgd_status qgd_mma_ring_probe(int n, int slots, int wait, int iters, double* flops, void* stream) {
  if ((n != 128 && n != 256) || (slots != 1 && slots != 2 && slots != 4) || n * slots > 512 || (wait != 0 && wait != 1))
    return fail(QGD_ERR_INVALID, "n=%d slots=%d wait=%d: n in {128, 256}, slots in {1, 2, 4}, n*slots <= 512",
                n, slots, wait);
  if (iters < 1 || iters > 200000) return fail(QGD_ERR_INVALID, "iters=%d must be in [1, 200000]", iters);
  qgd_status st = check_device();
  if (st != QGD_OK) return st;
  if (flops) *flops = 2.0 * 128.0 * n * kTileK * static_cast<double>(iters) * g_num_sms;
  cudaError_t e = launch_mma_ring_probe(n, slots, wait != 0, iters, g_num_sms, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? QGD_OK : cuda_fail(e, "qgd_mma_ring_probe launch");
}

qgd_status qgd_set_pdl(int on) {
  if (on < -1 || on > 1) return fail(QGD_ERR_INVALID, "on=%d must be -1, 0 or 1", on);
  g_pdl.store(on, std::memory_order_relaxed);  // -1: QGD_PDL decides again at the next launch
  return QGD_OK;
}

qgd_status qgd_test_withhold_accumulator(int on) {
  g_withhold_acc.store(on ? 1 : 0, std::memory_order_relaxed);
  return QGD_OK;
}

const char* qgd_version(void) { return "0.1.0"; }

}  // extern "C"
