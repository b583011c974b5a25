/*
 * qgd.h - C ABI of a B200 (sm_100a) library for the quantized linear layer
 *
 *     Y[M,N] = dequant(Xq)[M,K] . dequant(Wq)[N,K]^T      (Y in bf16)
 *
 * at decode-sized token counts M (1..32) and beyond, in the three formats of
 * "Building a High-Performance and Portable vLLM Linear Backend with Helion"
 * (section "Put algorithm selection inside the search space", and the scope
 * list "Alcance" of its Spanish translation):
 *
 *   FP8_Dynamic  e4m3 activations with one scale per token (row of X) and
 *                e4m3 weights with one scale per output channel (row of W);
 *   W8A8_INT8    the same granularity with symmetric int8 codes;
 *   Block_FP8    e4m3 with one activation scale per 1x128 group of a row and
 *                one weight scale per 128x128 block.
 *
 * The GEMM comes in the article's algorithm variants (section "Como se
 * implementa el kernel?" and its matmul listing): Standard (each CTA owns an
 * output tile and reduces all of K), Split-K (K is cut into split_k parts,
 * split_k a power of two from 1 to 256 -- any count from 2 to 8 when the
 * splits reduce inside a thread-block cluster, and any count in CTA-pair
 * tiles -- whose partial sums are then added)
 * and Swap-AB (the product is computed as (W . X^T)^T so the wide N dimension
 * fills the MMA's M slot).  Which one runs for a shape is chosen from a
 * measured dispatch table (section "Hybrid dispatch" / "Despacho hibrido":
 * the token counts 1, 2, 4, 8, 16, 24 and 32 are tuned separately).
 *
 * Conventions for every call below
 *   - All matrices are row-major with K contiguous ("K-major"): X/Xq [M,K],
 *     W/Wq [N,K], Y [M,N].  bf16 is passed as its 16-bit storage.
 *   - Data pointers are DEVICE pointers owned by the caller and must be
 *     16-byte aligned.  The library never allocates device memory (except
 *     qgd_ipc_malloc, on request), never frees caller memory and never
 *     synchronizes the stream.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Work is
 *     enqueued asynchronously.  The quantizers and the qlinear_* calls that
 *     take a workspace can be captured into a CUDA graph (nothing inside them
 *     allocates or synchronizes).
 *   - Errors are returned as a qgd_status and nothing is launched when the
 *     arguments are rejected.  qgd_last_error_message() describes the last
 *     failure on the calling thread.  A device-side wait that gives up (about
 *     one second without progress) is reported through qgd_device_error().
 *   - M == 0 is a valid empty call: it returns QGD_OK and launches nothing.
 */
#ifndef QGD_H
#define QGD_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define QGD_API __attribute__((visibility("default")))
#else
#define QGD_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  QGD_OK = 0,
  QGD_ERR_INVALID = -1,     /* null or misaligned pointer, negative size, bad enum */
  QGD_ERR_UNSUPPORTED = -2, /* shape outside the supported set (see each call) */
  QGD_ERR_WORKSPACE = -3,   /* workspace missing or smaller than qgd_workspace_size() */
  QGD_ERR_CUDA = -4,        /* a CUDA runtime/driver call failed */
  QGD_ERR_TABLE = -5,       /* dispatch table file unreadable or malformed */
  QGD_ERR_DEVICE = -6       /* current device is not an sm_100 part */
} qgd_status;

typedef enum {
  QGD_FMT_FP8_DYNAMIC = 0,
  QGD_FMT_W8A8_INT8 = 1,
  QGD_FMT_BLOCK_FP8 = 2,
  QGD_FMT_MXFP8 = 3,
  QGD_FMT_NVFP4 = 4
} qgd_format;
typedef enum { QGD_QTYPE_E4M3 = 0, QGD_QTYPE_INT8 = 1 } qgd_qtype;
/* Standard: X is the MMA's A operand (128-token tiles).  Swap-AB: Y^T = W X^T, the weight rows fill
 * the MMA's 128-row slot and the tokens its N (16/32/64/128); up to 32 tokens for Block_FP8 and up
 * to 128 for FP8_Dynamic / W8A8_INT8 (a plan asking for more gets Standard).  Standard pair: the
 * Standard orientation with 256-token x 256-weight-row tiles, each computed by two CTAs on two SMs
 * (one 2-CTA cluster, tcgen05 cta_group::2): each CTA loads half of the tile's token rows and half
 * of its weight rows, so operand traffic per FLOP is two thirds of a one-CTA 128 x 256 tile's.
 * FP8_Dynamic and W8A8_INT8 only (other formats get Standard); Split-K only with the two-pass
 * reduction (any split_k above 1 takes it, not only powers of two), table name "standard_pair". */
typedef enum {
  QGD_VARIANT_AUTO = -1,
  QGD_VARIANT_STANDARD = 0,
  QGD_VARIANT_SWAP_AB = 1,
  QGD_VARIANT_STANDARD_PAIR = 2
} qgd_variant;
typedef enum {
  QGD_REDUCE_AUTO = -1,
  QGD_REDUCE_LAST_CTA = 0, /* split partials to workspace; the last CTA of each tile adds them in split order */
  QGD_REDUCE_TWO_PASS = 1, /* split partials to workspace; a second kernel adds them in split order
                              (Swap-AB: at most 32 tokens, else the last CTA adds them) */
  QGD_REDUCE_ATOMIC = 2,   /* split partials added atomically into a zeroed workspace (fp32 order varies) */
  QGD_REDUCE_CLUSTER = 3   /* grid schedule, 2 <= split_k <= 8 (not only powers of two): the splits of
                              a tile form one thread-block cluster and add their partials in split
                              order through distributed shared memory (no workspace).  Swap-AB, and
                              the one-CTA Standard kernel for FP8_Dynamic / W8A8_INT8 when the other
                              splits' rows fit the ring (else the last CTA adds them) */
} qgd_reduce;

typedef enum {
  QGD_SCHEDULE_AUTO = -1,
  QGD_SCHEDULE_GRID = 0,      /* one CTA per (output tile, K split): split_k CTAs along K */
  QGD_SCHEDULE_PERSISTENT = 1 /* about one CTA per SM.  Swap-AB: all (tile, K unit) units are
                                 dealt out in equal contiguous ranges, shared tiles finished by the last
                                 CTA.  Standard: (tile, split) items dealt round-robin, the TMEM
                                 accumulator double-buffered across a CTA's tiles */
} qgd_schedule;

/* The execution plan for one (format, M, N, K). */
typedef struct {
  int variant;  /* qgd_variant (never AUTO here) */
  int split_k;  /* grid schedule: CTAs along K, 1..256, at most ceil(K/128); a power of two
                   except with QGD_REDUCE_CLUSTER, which takes any 2..8, and in Standard pair
                   tiles, which take any count */
  int reduce;   /* qgd_reduce, used when several CTAs share an output tile */
  int stages;   /* depth of the shared-memory operand ring */
  int tile_n;   /* Standard: output columns per CTA (128 or 256); Swap-AB: 128 */
  int schedule;  /* qgd_schedule (never AUTO here) */
  int occupancy; /* persistent schedule: CTAs per SM the grid is sized for (1 or 2).  With 1 and a
                    ring under half the SM's shared memory, the next GEMM's CTA can be resident
                    beside this one and do its set-up and first weight loads before this one ends */
  int source;    /* 0 = built-in default, 1 = dispatch table, 2 = override */
  int k_slices;  /* 128-wide K slices (K blocks) per pipeline stage, 1 or 2, in both kernels.  Each
                    stage costs a fixed hand-off between the copy engine and the MMA (and one MMA
                    commit), so one Swap-AB CTA per SM keeps up with HBM only with two slices
                    (32 KB of weights) per stage, and the Standard kernel's tensor pipe idles
                    between one-block stages */
  int fused;     /* layer calls (qlinear_*_bf16) only: 1 = the activation quantizer runs inside the
                    Swap-AB GEMM kernel, 0 = a separate quantizer kernel first.  Always 0 in the plan
                    of the qlinear_* calls, which take quantized activations */
} qgd_plan;

/* ---------------------------------------------------------------------
 * Dynamic quantizers ("Fused Quantization Ops"; per-token / per-group
 * scaling of the three formats).  For each row (or 1x128 group, or 128x128
 * block) g:
 *     amax = max(max |x| over g, 1e-12f)
 *     s    = amax / qmax            (qmax = 448 for e4m3, 127 for int8;
 *                                    correctly rounded fp32 division)
 *     q    = convert(x / s)         (correctly rounded fp32 quotient, then
 *                                    round-to-nearest-even; e4m3 saturates to
 *                                    +-448 and keeps the sign of zero; int8 is
 *                                    clamped to [-127, 127])
 * ------------------------------------------------------------------- */

/* Per-row scales.  x_bf16 [M,K] -> xq [M,K] (e4m3 bytes or int8), sx [M]
 * fp32.  Also the weight quantizer for FP8_Dynamic / W8A8_INT8 (rows = N).
 * Requires K % 8 == 0 and K <= 65536. */
QGD_API qgd_status quant_act_per_token(const void* x_bf16, int M, int K, int qtype, void* xq, float* sx, void* stream);

/* 1x128 activation groups (Block_FP8).  x_bf16 [M,K] -> xq e4m3 [M,K],
 * sx [M][K/128] fp32 row-major.  Requires K % 128 == 0. */
QGD_API qgd_status quant_act_group128(const void* x_bf16, int M, int K, void* xq, float* sx, void* stream);

/* The same two quantizers reading x rows `ldx` elements apart (ldx >= K,
 * ldx % 8 == 0; the row starts stay 16-byte aligned), e.g. the first K
 * columns of a wider activation such as a fused projection's output.  xq
 * and sx are dense as above.  ldx < K or not a multiple of 8 ->
 * QGD_ERR_INVALID. */
QGD_API qgd_status quant_act_per_token_strided(const void* x_bf16, int M, int K, int ldx, int qtype, void* xq,
                                               float* sx, void* stream);
QGD_API qgd_status quant_act_group128_strided(const void* x_bf16, int M, int K, int ldx, void* xq, float* sx,
                                              void* stream);

/* 128x128 weight blocks (Block_FP8).  w_bf16 [N,K] -> wq e4m3 [N,K],
 * sw [N/128][K/128] fp32 row-major.  Requires N % 128 == 0, K % 128 == 0. */
QGD_API qgd_status quant_weight_block128(const void* w_bf16, int N, int K, void* wq, float* sw, void* stream);

/* ---------------------------------------------------------------------
 * Quantized GEMMs.  y_bf16 [M,N] = round_bf16( sum_k xq*wq * scales ):
 *   FP8_Dynamic / W8A8_INT8: acc[m,n] = sum_k Xq[m,k] Wq[n,k] (fp32 / exact
 *     int32 accumulation); Y = (acc * sx[m]) * sw[n].
 *   Block_FP8: for each 128-wide K block kb, P_kb = sum over the block;
 *     Y = sum_kb P_kb * (sx[m][kb] * sw[n/128][kb]).
 * Shapes: M >= 0; N % 16 == 0; K % 16 == 0 (FP8_Dynamic, W8A8_INT8) or
 * K % 128 == 0 and N % 128 == 0 (Block_FP8).
 * Workspace: `ws` (device, >= qgd_workspace_size() bytes for the same
 * arguments) holds, when the plan splits K, a 64 KiB header of per-tile
 * arrival counters followed by the Split-K partials (or the atomic
 * accumulator, which the call zeroes itself with a memset node).  The header
 * must be zero-filled once after allocation; every call leaves it zero again
 * and never writes anything else there, so one workspace can serve calls of
 * different shapes and plans.  Calls that share a workspace must not run
 * concurrently.  ws may be NULL when qgd_workspace_size() returns 0.
 * ------------------------------------------------------------------- */
QGD_API qgd_status qlinear_fp8_dynamic(const void* xq, const float* sx, const void* wq, const float* sw, void* y_bf16,
                               int M, int N, int K, void* ws, size_t ws_bytes, void* stream);
QGD_API qgd_status qlinear_w8a8_int8(const void* xq, const float* sx, const void* wq, const float* sw, void* y_bf16,
                             int M, int N, int K, void* ws, size_t ws_bytes, void* stream);
QGD_API qgd_status qlinear_block_fp8(const void* xq, const float* sx, const void* wq, const float* sw, void* y_bf16,
                             int M, int N, int K, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------
 * Layer calls from bf16 activations: dynamic activation quantization and
 * the GEMM in one call ("Fused Quantization Ops" of the explore.n1n.ai
 * page's architecture diagram; the formats as above).
 *     y_bf16 [M,N] = qlinear_*(quantize(x_bf16 [M,K]), wq, sw)
 * with exactly the codes and scales quant_act_per_token /
 * quant_act_group128 would produce.  x rows are `ldx` elements apart (ldx
 * >= K, ldx % 8 == 0; 16-byte aligned base), so x may be the first K
 * columns of a wider activation.  The layer plan (qgd_get_layer_plan)
 * decides how:
 *   fused = 1  one Swap-AB kernel: its epilogue warps read x, quantize it
 *              into the shared-memory stages the MMA consumes (per-token
 *              scales: every CTA first takes each row's maximum over all of
 *              K; Block_FP8: per 1x128 group inside the K slice).  No
 *              activation codes reach global memory.
 *   fused = 0  the quantizer kernel writes codes and scales into the
 *              workspace, then the GEMM runs as qlinear_* would.
 * Workspace: >= qgd_layer_workspace_size() bytes (same rules as for
 * qlinear_*: zero-filled once after allocation; calls sharing it must not
 * overlap), ws may be NULL when that size is 0.  Shapes as qlinear_*, and
 * K <= 65536.  Errors as qlinear_*; ldx < K or not a multiple of 8 ->
 * QGD_ERR_INVALID.
 * ------------------------------------------------------------------- */
QGD_API qgd_status qlinear_fp8_dynamic_bf16(const void* x_bf16, int ldx, const void* wq, const float* sw,
                                            void* y_bf16, int M, int N, int K, void* ws, size_t ws_bytes,
                                            void* stream);
QGD_API qgd_status qlinear_w8a8_int8_bf16(const void* x_bf16, int ldx, const void* wq, const float* sw,
                                          void* y_bf16, int M, int N, int K, void* ws, size_t ws_bytes,
                                          void* stream);
QGD_API qgd_status qlinear_block_fp8_bf16(const void* x_bf16, int ldx, const void* wq, const float* sw,
                                          void* y_bf16, int M, int N, int K, void* ws, size_t ws_bytes,
                                          void* stream);

/* MXFP8 layer call: quant_act_mx into the workspace, then qlinear_mxfp8
 * (there is no fused MXFP8 kernel).  sw_e8m0 [N][K/32] bytes, 16-byte
 * aligned; otherwise as the calls above. */
QGD_API qgd_status qlinear_mxfp8_bf16(const void* x_bf16, int ldx, const void* wq, const void* sw_e8m0,
                                      void* y_bf16, int M, int N, int K, void* ws, size_t ws_bytes, void* stream);

/* Bytes of workspace a layer call for (fmt, M, N, K) needs under the layer
 * plan in force (0 when none). */
QGD_API size_t qgd_layer_workspace_size(int fmt, int M, int N, int K);

/* ---------------------------------------------------------------------
 * MXFP8, a fourth format beside Block_FP8 for Blackwell's block-scaled
 * tensor cores (the pages list further vLLM formats and name Blackwell as
 * the next target; the format is the OCP Microscaling (MX) v1.0 definition):
 * every 32 consecutive values of a row along K share one power-of-two scale
 * 2^e, stored as an E8M0 byte e + 127; the values are e4m3.
 *     e = clamp(floor(log2(max |x| over the block)) - 8, -127, 127)
 *         (8: the exponent of e4m3's largest normal; an all-zero block
 *          takes e = -127),   q = e4m3_rne_satfinite(x * 2^-e).
 * The GEMM multiplies in hardware (tcgen05.mma kind::mxf8f6f4 with E8M0
 * block scales read from tensor memory): Y = sum over 32-wide K blocks of
 * (Xq . Wq^T)_block * 2^(ex + ew), fp32 accumulation, bf16 out.
 * ------------------------------------------------------------------- */

/* MX quantizer: x_bf16 [M,K] (rows ldx elements apart, ldx >= K, ldx % 8 ==
 * 0) -> xq e4m3 [M,K], s_e8m0 [M][K/32] bytes.  Also the weight quantizer
 * (rows = N).  Requires K % 32 == 0; x and xq 16-byte aligned. */
QGD_API qgd_status quant_act_mx(const void* x_bf16, int M, int K, int ldx, void* xq, void* s_e8m0, void* stream);

/* MXFP8 GEMM: y_bf16 [M,N] from xq [M,K], sx_e8m0 [M][K/32], wq [N,K],
 * sw_e8m0 [N][K/32].  Swap-AB kernel only: 0 <= M <= 128 (more ->
 * QGD_ERR_UNSUPPORTED); K % 128 == 0, N % 16 == 0; all pointers 16-byte
 * aligned.  The block scales sit in tensor memory beside the accumulators
 * (at most 256 columns per CTA up to 64 tokens, which caps the ring depth;
 * at 65..128 tokens all 512, with a ring of at least four K slices so that
 * the CTA has its SM to itself).  Workspace as qlinear_fp8_dynamic (same
 * plans; no two-pass reduction, whose requests take the last-arriving CTA). */
QGD_API qgd_status qlinear_mxfp8(const void* xq, const void* sx_e8m0, const void* wq, const void* sw_e8m0,
                                 void* y_bf16, int M, int N, int K, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------
 * NVFP4, the 4-bit format the pages list among vLLM's ("NVFP4"): E2M1
 * values (magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6), one E4M3 scale per 16
 * consecutive values of a row along K, and one fp32 scale per row -- per
 * token for the activations (computed at run time, as FP8_Dynamic's) and
 * per output channel for the weights.  For a row with
 * amax = max(max |x|, 1e-12f):
 *     g = amax / 2688                     (6 * 448: the largest E2M1 value
 *                                          times the largest E4M3)
 *     per block of 16 with maximum b:
 *     s = e4m3(b / (6 g)),  d = dec(s) * g,  q = e2m1(x / d)   (q = +-0
 *                                          where d is 0)
 * each operation one IEEE fp32 round-to-nearest step; E4M3 and E2M1 round to
 * nearest even and saturate.  Codes are packed two per byte, value 2i in the
 * low nibble of byte i.  The GEMM multiplies in hardware (tcgen05.mma
 * kind::mxf4nvf4 with E4M3 scale factors read from tensor memory, K = 64 per
 * instruction) and the epilogue applies the row scales:
 *     Y[m,n] = bf16( gx[m] gw[n] sum_b dec(sx[m,b]) dec(sw[n,b]) sum_{k in b} q_x q_w )
 * ------------------------------------------------------------------- */

/* NVFP4 quantizer: x_bf16 [rows,K] (rows ldx elements apart, ldx >= K, ldx %
 * 8 == 0) -> q [rows][K/2] packed codes, s_e4m3 [rows][K/16] block scales,
 * g [rows] fp32 row scales.  For activations (rows = M) and weights (rows =
 * N).  Requires K % 16 == 0, K <= 65536; x 16-byte, q 8-byte and g 4-byte
 * aligned. */
QGD_API qgd_status quant_nvfp4(const void* x_bf16, int rows, int K, int ldx, void* q, void* s_e4m3, float* g,
                               void* stream);

/* NVFP4 GEMM: y_bf16 [M,N] from xq [M][K/2], sx_e4m3 [M][K/16], gx [M], wq
 * [N][K/2], sw_e4m3 [N][K/16], gw [N].  Swap-AB kernel only: 0 <= M <= 128
 * (more -> QGD_ERR_UNSUPPORTED); K % 256 == 0, N % 16 == 0; all pointers
 * 16-byte aligned.  The block scales sit in tensor memory beside the
 * accumulators, 32 columns per ring slot (at most 256 columns per CTA up to
 * 64 tokens, which caps the ring depth; at 65..128 tokens all 512, as for
 * MXFP8).  Workspace as qlinear_fp8_dynamic (same plans; no two-pass
 * reduction, whose requests take the last-arriving CTA). */
QGD_API qgd_status qlinear_nvfp4(const void* xq, const void* sx_e4m3, const float* gx, const void* wq,
                                 const void* sw_e4m3, const float* gw, void* y_bf16, int M, int N, int K, void* ws,
                                 size_t ws_bytes, void* stream);

/* NVFP4 layer call: quant_nvfp4 of x_bf16 into the workspace, then
 * qlinear_nvfp4.  Workspace: qgd_layer_workspace_size(QGD_FMT_NVFP4, ...);
 * otherwise as the calls above. */
QGD_API qgd_status qlinear_nvfp4_bf16(const void* x_bf16, int ldx, const void* wq, const void* sw_e4m3,
                                      const float* gw, void* y_bf16, int M, int N, int K, void* ws, size_t ws_bytes,
                                      void* stream);

/* ---------------------------------------------------------------------
 * Column-parallel (tensor-parallel) layer call with the all-gather fused
 * into the GEMM's output stores.  The pages run one GPU only (tensor
 * parallelism of one: "Building a High-Performance and Portable vLLM Linear
 * Backend with Helion", section "Preserve the conditions when moving from
 * kernels to serving"); this is the library's own extension of the same
 * operation to G GPUs.  The full layer Y[M, ldy] = dequant(Xq) . dequant(W)^T
 * has its weight rows (output columns) split over G ranks: rank r holds the
 * rows [col0_r, col0_r + N_r) of W, quantized as for the layer calls above,
 * and the replicated activations x_bf16 [M,K].  Each rank's call quantizes x
 * as the layer call would and computes its Y columns with the Swap-AB kernel,
 * whose epilogue stores every finished element to ALL ranks' full outputs
 * (peer memory over NVLink), so that after qgd_tp_wait every rank holds the
 * whole Y.  The numbers are exactly those of a single-GPU layer call on the
 * shard with the same plan.
 *
 *   ranks      G, 1..QGD_MAX_TP_RANKS
 *   rank       this rank, 0..G-1 (the index of its own entries below)
 *   col0, ldy  this shard's first column in the full output, and the full
 *              output's width (its row stride in elements; ldy % 8 == 0,
 *              col0 + N <= ldy)
 *   y[r]       rank r's full bf16 output [M, ldy] as addressed from this
 *              process (this GPU's own buffer at y[rank]; the others opened
 *              with qgd_ipc_open, or plain pointers when every "rank" runs on
 *              one GPU), 16-byte aligned
 *   flags[r]   rank r's flag array as addressed from this process: G + 1
 *              uint32 words, zero-filled before the first call.  Entry j
 *              holds the number of calls rank j has completed; word G is
 *              rank r's own call counter
 *
 * After the last of this call's CTAs has stored its output, the kernel adds
 * one to this rank's counter (word G of flags[rank]; 0 is skipped when it
 * wraps) and writes the new count to entry `rank` of every rank's flag array
 * (a system-scope release).  The count lives on the device, so the call can
 * be captured in a CUDA graph and replayed.  Every rank must make the same
 * sequence of calls on the same flag arrays.  A rank reads the full Y only
 * after qgd_tp_wait on its own flags in stream order after its own call.
 * Because another rank may already run its next call and write into this
 * rank's Y while this rank still reads the previous result, alternate
 * between two output buffers (the flags need no second copy).  A kernel that
 * gave up on one of its bounded waits still advances and raises its count
 * (every rank stays in step), so its share of Y is then incomplete: every
 * rank should check qgd_device_error() before trusting a result.
 *
 * Plan: the layer plan for (fmt, M, N, K) forced to Swap-AB (the Standard
 * kernels have no such epilogue) and to a reduction inside the GEMM kernel
 * (a two-pass request takes the last-arriving CTA).  M <= 128 (FP8_Dynamic,
 * W8A8_INT8, MXFP8, NVFP4), <= 32 (Block_FP8); more ->
 * QGD_ERR_UNSUPPORTED.  M == 0 launches nothing and sets no flag: skip the
 * wait for such a call.  sw: the weight scales of the format (fp32 per
 * channel or per block; MXFP8 E8M0 bytes; NVFP4 the fp32 row scales), and
 * sw_block the NVFP4 E4M3 block scales (NULL otherwise).  Workspace:
 * qgd_tp_workspace_size() bytes, never NULL (the 64 KiB counter header is
 * always present; its last word counts this call's finished CTAs), the usual
 * rules otherwise.  Errors as the layer calls; a bad descriptor ->
 * QGD_ERR_INVALID.
 * ------------------------------------------------------------------- */
#define QGD_MAX_TP_RANKS 8
typedef struct {
  int ranks;
  int rank;
  int col0;
  int ldy;
  void* y[QGD_MAX_TP_RANKS];
  unsigned int* flags[QGD_MAX_TP_RANKS];
} qgd_tp;

QGD_API size_t qgd_tp_workspace_size(int fmt, int M, int N, int K);
QGD_API qgd_status qlinear_tp_bf16(int fmt, const void* x_bf16, int ldx, const void* wq, const void* sw,
                                   const void* sw_block, int M, int N, int K, const qgd_tp* tp, void* ws,
                                   size_t ws_bytes, void* stream);

/* Enqueue, on `stream`, a one-thread kernel that reads this rank's call
 * count e from word `ranks` of its own flag array `flags` and waits until
 * every one of flags[0..ranks-1] holds e or a later count (compared modulo
 * 2^32), with acquire semantics at system scope, so that kernels after it on
 * the stream see every rank's output.  A flag still behind after about one
 * second makes the kernel record device error 6 (qgd_device_error) and
 * return; the output is then incomplete.  Launch it only after this rank's
 * own qlinear_tp_bf16 in the same stream: it must never wait for a kernel of
 * its own GPU. */
QGD_API qgd_status qgd_tp_wait(const unsigned int* flags, int ranks, void* stream);

/* Buffers shared between processes (CUDA IPC).  qgd_ipc_malloc allocates
 * `bytes` of device memory on the current device, zero-fills it
 * (synchronously) and writes its QGD_IPC_HANDLE_BYTES-byte handle to
 * `handle`; free it with qgd_ipc_free after every importer has closed it.
 * qgd_ipc_open maps another process's buffer from its handle (peer access
 * enabled on demand) and qgd_ipc_close unmaps it.  A process cannot open its
 * own handles. */
#define QGD_IPC_HANDLE_BYTES 64
QGD_API qgd_status qgd_ipc_malloc(size_t bytes, void** dptr, void* handle);
QGD_API qgd_status qgd_ipc_open(const void* handle, void** dptr);
QGD_API qgd_status qgd_ipc_close(void* dptr);
QGD_API qgd_status qgd_ipc_free(void* dptr);

/* Test hook: the W8A8_INT8 mainloop and Split-K reduction of the plan in
 * force, writing the exact int32 accumulator acc[M][N] instead of Y. */
QGD_API qgd_status qgd_w8a8_int8_acc32(const void* xq, const void* wq, int32_t* acc, int M, int N, int K, void* ws,
                               size_t ws_bytes, void* stream);

/* FP8_Dynamic GEMM for callers that cannot allocate device memory while they
 * run -- for example an inference engine that splits all device memory into
 * fixed pools at start-up and has none left for a per-call workspace, or a
 * latency-critical loop where a cudaMalloc may block until the device is
 * idle.  It is qlinear_fp8_dynamic without the workspace arguments: the
 * caller still passes inputs and output, and the Split-K scratch comes from a
 * fixed 8 MiB array inside the library (held by every GPU that loads it until
 * exit).  The pages have no counterpart; this is an addition of this library.
 *   - The plan is the same as qlinear_fp8_dynamic's; a plan whose Split-K
 *     scratch exceeds 8 MiB (64 KiB of counters + partials) is rejected with
 *     QGD_ERR_WORKSPACE before anything is launched.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.
 *   - All calls share the one array, which keeps what the last call left in
 *     it: calls that overlap on the GPU (other streams, other threads) race
 *     and give undefined results.  A call that splits K first clears the
 *     counters it uses with a memset, then runs the GEMM (launched without a
 *     programmatic dependency, since it follows a memset).
 *   - Nothing is allocated or freed: no cudaMalloc/cudaFree, no allocating
 *     library routine. */
QGD_API qgd_status qlinear_fp8_dynamic_noalloc(const void* xq, const float* sx, const void* wq, const float* sw,
                                               void* y_bf16, int M, int N, int K, void* stream);

/* Bytes of workspace the plan for (fmt, M, N, K) needs (0 when it needs
 * none).  Re-query after changing the override or the dispatch table. */
QGD_API size_t qgd_workspace_size(int fmt, int M, int N, int K);

/* ---------------------------------------------------------------------
 * Dispatch (host only; no GPU needed).
 * ------------------------------------------------------------------- */

/* Load a dispatch table: a text file with one line per (format, N, K,
 * M-bucket) and '#' comments,
 *     fmt N K M_bucket variant split_k reduce stages tile_n schedule occupancy [k_slices]
 * fmt in {fp8_dynamic, w8a8_int8, block_fp8, mxfp8, nvfp4}; variant in {standard, swap_ab, standard_pair};
 * reduce in {last_cta, two_pass, atomic, cluster}; schedule in {grid, persistent};
 * stages/tile_n/occupancy/k_slices 0 (or k_slices absent) = default.
 * Replaces the table in force.  On
 * QGD_ERR_TABLE the table in force is unchanged.  Not thread-safe against
 * concurrent qlinear_* calls. */
QGD_API qgd_status qgd_load_dispatch_table(const char* path);

/* (An optional 13th field, fused = 0 or 1, sets the layer plan's `fused`.) */

/* Drop the table in force; the built-in defaults apply again. */
QGD_API qgd_status qgd_clear_dispatch_table(void);

/* Force a plan for one format (tests and the tuner).  Any argument < 0 keeps
 * the table/default choice for that field; stages/tile_n/occupancy/k_slices
 * 0 = default.  qgd_set_override(fmt, -1, -1, -1, 0, 0, -1, 0, 0) removes it. */
QGD_API qgd_status qgd_set_override(int fmt, int variant, int split_k, int reduce, int stages, int tile_n,
                                    int schedule, int occupancy, int k_slices);

/* The plan a qlinear_* call with these arguments would run. */
QGD_API qgd_status qgd_get_plan(int fmt, int M, int N, int K, qgd_plan* plan);

/* The plan a layer call (qlinear_*_bf16) with these arguments would run: the
 * same table entry, with its `fused` field in effect. */
QGD_API qgd_status qgd_get_layer_plan(int fmt, int M, int N, int K, qgd_plan* plan);

/* Force the `fused` field of layer plans for one format (tests and the
 * tuner): -1 = table / default (not fused), 0 = quantizer kernel first,
 * 1 = fused (Swap-AB plans only; others stay unfused).  Independent of
 * qgd_set_override.  Other values -> QGD_ERR_INVALID. */
QGD_API qgd_status qgd_set_fused_override(int fmt, int fused);

/* M-bucket of a token count: the smallest tuned count >= M among
 * 1, 2, 4, 8, 16, 24, 32, 64, 128, 512, 2048, 8192 (the last one beyond). */
QGD_API int qgd_m_bucket(int M);

/* ---------------------------------------------------------------------
 * Status
 * ------------------------------------------------------------------- */
QGD_API const char* qgd_status_string(int status);
QGD_API const char* qgd_last_error_message(void);

/* Device error flag of the current device (0 = none).  Nonzero means a
 * kernel gave up a bounded wait and returned without finishing; its outputs
 * are undefined and the workspace must be zero-filled again.  Synchronizes
 * the device.  qgd_clear_device_error() resets the flag. */
QGD_API qgd_status qgd_device_error(unsigned int* code);
QGD_API qgd_status qgd_clear_device_error(void);

/* ---------------------------------------------------------------------
 * Measurement aid (no counterpart on the pages, whose roofline takes the
 * dense tensor peak from the data sheet).  Launches one CTA per SM, each
 * issuing `iters` groups of four back-to-back tcgen05.mma (M=128, N=256,
 * K=32 each; kind::f8f6f4 for QGD_QTYPE_E4M3, kind::i8 for QGD_QTYPE_INT8)
 * from zeroed operands in shared memory into one TMEM accumulator; nothing
 * is read from or written to global memory.  The caller times the launch on
 * `stream`; *flops (host pointer, may be NULL) receives the launch's
 * 2*M*N*K operation count.  1 <= iters <= 200000 (about 50 ms at most), else
 * QGD_ERR_INVALID.  A wait that gives up is reported by qgd_device_error().
 * --------------------------------------------------------------------- */
QGD_API qgd_status qgd_mma_peak_probe(int qtype, int iters, double* flops, void* stream);

/* Measurement aid: the tensor pipe with a ring of accumulators.  One CTA per
 * SM issues `iters` groups of four e4m3 tcgen05.mma (128 x n x 32 each) into
 * `slots` TMEM slots of n columns in turn, committing each group to its
 * slot's mbarrier; with wait = 1 the issuing thread first waits for the
 * slot's previous group to complete (the hand-off of a kernel whose
 * accumulators form a ring), with wait = 0 it never waits.  n in {128, 256},
 * slots in {1, 2, 4}, n * slots <= 512, 1 <= iters <= 200000, else
 * QGD_ERR_INVALID.  *flops and timing as qgd_mma_peak_probe. */
QGD_API qgd_status qgd_mma_ring_probe(int n, int slots, int wait, int iters, double* flops, void* stream);

/* Programmatic dependent launch (each kernel starts while the one before it
 * on the stream finishes, and waits only where it reads that kernel's
 * output): on = 1 (the default), 0 = plain stream order, -1 = as the
 * environment variable QGD_PDL says (QGD_PDL=0 turns it off), read at the
 * next launch.  The setting is read once and then cached, not looked up per
 * launch.  Other values -> QGD_ERR_INVALID. */
QGD_API qgd_status qgd_set_pdl(int on);

/* Test hook for the failure-detection path (the pages have no counterpart).
 * While on (on != 0), GEMMs launched from then on in the Swap-AB orientation
 * never signal the epilogue that an accumulator is complete -- a flag that
 * nothing sets -- so the epilogue's bounded wait runs out after about one
 * second.  The kernel then records error 3 (epilogue wait) for
 * qgd_device_error(), waits for the copies and MMAs it issued, frees its
 * tensor memory and returns without writing Y; the context stays usable.
 * No other kernel is affected.  Host-global, for tests only; not
 * thread-safe against concurrent qlinear_* calls.  Always QGD_OK. */
QGD_API qgd_status qgd_test_withhold_accumulator(int on);

/* Test hook for the fused layer calls (the pages have no counterpart):
 * while xq (device, [M][K] bytes) and sx (device, [M] or [M][K/128] fp32)
 * are non-null, every fused launch also writes the activation codes and
 * scales it made there, so they can be compared with the oracle's; both
 * NULL turns it off.  Host-global, for tests only.  Always QGD_OK. */
QGD_API qgd_status qgd_test_capture_fused(void* xq, float* sx);

/* Library version, "major.minor.patch". */
QGD_API const char* qgd_version(void);

#ifdef __cplusplus
}
#endif

#endif /* QGD_H */
