// Shared declarations between the C-ABI layer (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace qgd {

enum Fmt : int { kFmtFP8 = 0, kFmtINT8 = 1, kFmtBlock = 2, kFmtMX = 3, kFmtNV = 4 };
constexpr int kNumFmts = 5;
// kStandardPair: Standard tiles of 256 x 256 computed by a CTA pair (FP8_Dynamic, W8A8_INT8)
enum Variant : int { kStandard = 0, kSwapAB = 1, kStandardPair = 2 };
enum Reduce : int { kLastCta = 0, kTwoPass = 1, kAtomic = 2, kCluster = 3 };
constexpr int kMaxClusterSplit = 8;  // portable thread-block cluster size
constexpr int kMaxTpRanks = 8;       // tensor-parallel ranks of one NVLink domain
enum Schedule : int { kGrid = 0, kPersistent = 1 };

constexpr int kTileK = 128;           // K elements (= bytes) per pipeline stage
constexpr int kSwapTileN = 128;       // weight rows per Swap-AB CTA (MMA M)
constexpr int kStdTileM = 128;        // token rows per Standard CTA (MMA M)
constexpr int kMaxStages = 16;
constexpr int kGemmThreads = 192;     // producer warp, MMA warp, 4 epilogue warps
// Opt-in dynamic shared memory per CTA on sm_100 (227 KB).
constexpr size_t kSmemBudget = 232448;
// Shared memory per SM on sm_100 (228 KB), shared by the CTAs resident on it.
constexpr size_t kSmemPerSM = 233472;
inline size_t smem_budget() { return kSmemBudget; }

// Runtime arguments common to both GEMM orientations.
struct GemmArgs {
  const float* sx;      // FP8/INT8: [M]; Block: [M][K/128]; NVFP4: the fp32 row scales [M]
  const float* sw;      // FP8/INT8: [N]; Block: [N/128][K/128]; NVFP4: [N]
  uint16_t* y;          // bf16 [M][N]
  void* raw;            // when non-null: fp32/int32 accumulator [M][N] instead of y
  void* partial;        // Split-K partials, 4-byte [splits][M][N]
  void* accum;          // atomic Split-K accumulator, 4-byte [M][N], zero on entry
  unsigned int* tickets;  // per output tile arrival counters (workspace header), zero on entry and exit
  int M, N, K;
  int splits;      // grid schedule: CTAs along K per tile
  int reduce;
  int stages;
  int persistent;  // Swap-AB: 1 = persistent schedule over all (tile, K-slice) units
  int ctas;        // persistent schedule: number of CTAs
  int maxc;        // Swap-AB partial slots per tile (largest contributor count)
  int mstride;     // Swap-AB partial row stride in words (M rounded up to 4)
  int kps;         // Swap-AB: 128-wide K slices per pipeline stage (1 or 2)
  int pdl;         // launch with a programmatic dependency on the preceding kernel
  int trace_tag;   // sequence number of the call (developer timeline builds file stamps by it)
  int withhold_acc;  // failure-detection test: Swap-AB never signals a finished accumulator
  // Swap-AB with the activation quantizer fused in: the kernel reads bf16
  // activations and writes their codes into its shared-memory stages itself.
  const uint16_t* xbf;  // bf16 activations [M] rows, ldxb elements apart
  int ldxb;
  uint8_t* xq_out;      // test capture (may be null): the codes [M][K] the kernel made
  float* sx_out;        // test capture (may be null): their scales, [M] or [M][K/128]
  // MXFP8: E8M0 block-scale bytes, one per 32 values along K ([M][K/32],
  // [N][K/32]); NVFP4: E4M3 block-scale bytes, one per 16 ([M][K/16],
  // [N][K/16]; the kernel's K then counts the packed bytes, K/2)
  const uint8_t* sx8;
  const uint8_t* sw8;
  // Column-parallel tensor parallelism (Swap-AB): this rank's output columns
  // (its weight shard's N) go to columns [tp_col0, tp_col0 + N) of every
  // rank's full bf16 output, tp_ldy columns wide, through the ranks' pointers
  // (peer memory); the last CTA to finish then advances this rank's call
  // counter (word tp_ranks of its own flag array) and writes the new value to
  // entry tp_rank of every rank's flag array.  tp_ranks == 0: a plain call.
  int tp_ranks;
  int tp_rank;
  int tp_col0;
  int tp_ldy;
  unsigned* tp_done;  // CTAs finished this call (zero on entry and exit)
  uint16_t* tp_y[kMaxTpRanks];
  unsigned* tp_flag[kMaxTpRanks];
};

// Tensor-memory columns of the block-scaled Swap-AB kernels: two accumulators
// of mpad columns, then per ring slot (stage, K slice) the slice's scale
// factors, in 4-column, 128-bit groups that each start on a multiple of 4:
// MXFP8 one group of weight scales and one of token scales (the slice's four
// MMAs each pick one byte of a word); NVFP4 a group of each per MMA (an MMA
// of 64 values reads all four bytes, one per 16).  Rounded up to a power of two.
constexpr unsigned kMxSlotCols = 8;
constexpr unsigned kNvSlotCols = 32;
__host__ __device__ inline unsigned slot_cols(int fmt) { return fmt == kFmtNV ? kNvSlotCols : kMxSlotCols; }
__host__ __device__ inline unsigned mx_tmem_cols(int mpad, int stages, int kps, int fmt = kFmtMX) {
  const unsigned need = 2u * mpad + static_cast<unsigned>(stages * kps) * slot_cols(fmt);
  unsigned c = 32;
  while (c < need) c *= 2;
  return c;
}

// Launchers (gemm.cu).  Each returns the cudaError_t of the launch.
// fused: the kernel quantizes a.xbf itself (tx unused)
cudaError_t launch_swapab(int fmt, int mpad, bool fused, const CUtensorMap& tw, const CUtensorMap& tx,
                          const GemmArgs& a, cudaStream_t stream);
cudaError_t launch_standard(int fmt, int tile_n, const CUtensorMap& tx, const CUtensorMap& tw,
                            const GemmArgs& a, cudaStream_t stream);
// ty: the bf16 output as a tensor map (boxes of 32 rows x 64 columns, 128-byte swizzle)
cudaError_t launch_standard_pair(int fmt, const CUtensorMap& tx, const CUtensorMap& tw, const CUtensorMap& ty,
                                 const GemmArgs& a, cudaStream_t stream);
int pair_max_active_clusters(int fmt, int stages, int kps);
cudaError_t launch_splitk_reduce(int fmt, const GemmArgs& a, cudaStream_t stream);
// Tensor parallelism: wait (bounded) until flags[0..ranks) all reach the
// epoch in flags[ranks] (this rank's call counter)
cudaError_t launch_tp_wait(const unsigned* flags, int ranks, bool pdl, cudaStream_t stream);
// Programmatic dependent launch for every kernel of the library: on unless
// QGD_PDL=0 (read once) or qgd_set_pdl(0)
bool pdl_enabled();
cudaError_t launch_swapab_reduce(int fmt, int mpad, const GemmArgs& a, cudaStream_t stream);
cudaError_t read_device_error(unsigned int* code);
cudaError_t clear_device_error();
size_t swapab_smem_bytes(int mpad, int stages, int kps, bool cluster, bool fused);
size_t standard_smem_bytes(int tile_n, int stages, int kps);
int swapab_max_stages(int mpad, int kps, bool cluster, bool fused);
int standard_max_stages(int tile_n, int kps);
size_t pair_smem_bytes(int stages, int kps);
int pair_max_stages(int kps);

// Tensor-core peak probe (probe.cu).
cudaError_t launch_mma_probe(int qtype, int iters, int ctas, cudaStream_t stream);
double mma_probe_flops(int iters, int ctas);
cudaError_t launch_mma_ring_probe(int n, int slots, bool wait, int iters, int ctas, cudaStream_t stream);
cudaError_t read_probe_error(unsigned int* code);
cudaError_t clear_probe_error();

// Quantizer launchers (quant.cu).
// x rows are ldx elements apart (ldx >= K); q and s are dense.
cudaError_t launch_quant_rows(const uint16_t* x, int rows, int K, int ldx, int qtype, void* q, float* s,
                              cudaStream_t stream);
cudaError_t launch_quant_group128(const uint16_t* x, int M, int K, int ldx, uint8_t* q, float* s,
                                  cudaStream_t stream);
cudaError_t launch_quant_block128(const uint16_t* w, int N, int K, uint8_t* q, float* s, cudaStream_t stream);
// MXFP8: rows of 32-value blocks -> e4m3 codes q [rows][K], E8M0 bytes s [rows][K/32]
// NVFP4 rows: q [rows][K/2] packed E2M1 codes, s [rows][K/16] E4M3 block
// scales, g [rows] fp32 row scales
cudaError_t launch_quant_nv(const uint16_t* x, int rows, int K, int ldx, uint8_t* q, uint8_t* s, float* g,
                            cudaStream_t stream);
cudaError_t launch_quant_mx(const uint16_t* x, int rows, int K, int ldx, uint8_t* q, uint8_t* s,
                            cudaStream_t stream);

}  // namespace qgd
