/*
 * moefp8.h -- C ABI of libmoefp8.so: the forward pass of one DeepSeekMoE layer
 * with FP8 (E4M3) block-scaled expert GEMMs, as hand-written sm_100a kernels.
 *
 * Sources (web pages on DeepSeek-V3/V4):
 *   [ANN]   "DeepSeek_V3_Report：Annotation" -- eqs. (12)-(16), "Node-Limited
 *           Routing", "Auxiliary-Loss-Free Load Balancing", "Fine-Grained
 *           Quantization", "Online Quantization", "Low-Precision Communication",
 *           SwiGLU operator notes.
 *   [INFRA] "DeepSeek V3 / V4 Infra：把 all-to-all 藏进计算" -- 6hd FLOPs per
 *           token-expert pair (gate, up, down projections).
 *
 * Conventions shared by every call:
 *   - All pointers are DEVICE pointers unless stated.  The caller owns every
 *     buffer; the library allocates nothing and keeps no state between calls
 *     (scratch comes from the caller through `ws`, sized by the matching
 *     *_workspace_size query).
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream) and returns a moe_status.  Argument, shape and
 *     alignment errors are detected on the host before anything is launched
 *     and returned synchronously; a failed launch returns MOE_ERR_CUDA.
 *   - Faults that only the device can see (inconsistent segment tables, a
 *     bounded wait that ran out) are recorded in the caller's `dev_err`
 *     (one int32 in device memory, 0 = none; first error wins) and read by
 *     the caller after synchronising.  `dev_err` may be NULL, which drops them.
 *   - bf16 tensors are passed as uint16_t bit patterns.  FP8 tensors are
 *     E4M3 bytes (bias 7, max 448, no infinities).
 *   - Device pointers must be 16-byte aligned; leading dimensions are in
 *     elements and must keep every row 16-byte aligned.  Widths that are
 *     tiled by 128 (d, I, N, K) must be multiples of 128.
 *   - Scales are fp32 dequantisation multipliers: x ~= e4m3_value * scale,
 *     scale = max(amax, 1e-4) / 448 computed in fp32, and the stored byte is
 *     E4M3(x / scale) with the division in fp32 (IEEE, round to nearest even)
 *     and round-to-nearest-even, saturating conversion.
 *   - No call throws; no exception crosses the ABI.
 */
#ifndef MOEFP8_H
#define MOEFP8_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1, /* NULL where a buffer is required, negative size */
  MOE_ERR_SHAPE = 2,       /* a width not a multiple of 128, K % M != 0, ... */
  MOE_ERR_ALIGN = 3,       /* pointer or leading dimension not 16-byte aligned */
  MOE_ERR_UNSUPPORTED = 4, /* shape outside the kernels' limits (e.g. E > 1024) */
  MOE_ERR_CUDA = 5,        /* a CUDA call or kernel launch failed */
  MOE_ERR_WORKSPACE = 6    /* workspace smaller than the size query returned */
} moe_status;

typedef enum {
  MOE_EP_F32 = 0,         /* D is fp32 [rows][N] */
  MOE_EP_SWIGLU_QUANT = 1 /* D is E4M3 [rows][N/2] with d_scale fp32 [rows][N/256] */
} moe_epilogue;

/* Codes the kernels write into dev_err. */
#define MOE_DEVERR_TIMEOUT 1   /* a bounded wait gave up; results are invalid */
#define MOE_DEVERR_BAD_TABLE 2 /* segment offsets / tile table inconsistent */
#define MOE_DEVERR_BAD_INDEX 3 /* an expert index outside [0, E) */
#define MOE_DEVERR_BAD_SCALE 4 /* a scale that is not a positive power of two reached the
                                  power-of-two GEMM */

typedef void* moe_stream_t; /* cudaStream_t */

/* Human-readable text for a status (static storage, never NULL). */
const char* moe_status_string(moe_status s);

/* ABI version of this header (bumped on any incompatible change); this
 * header is version 4. */
int moe_abi_version(void);

/* ---------------------------------------------------------------------------
 * fp8_quant_1x128 -- online 1x128 activation quantisation.
 * [ANN] "Fine-Grained Quantization" (activations grouped and scaled per token
 * per 128 channels) and "Online Quantization" (scale from the tile's own
 * max |x|, s = Q_max / max(A_max, eps), Q_max = 448 for E4M3).
 *   x     bf16 [rows][ldx], first `cols` columns used; ldx >= cols, ldx % 8 == 0
 *   q     E4M3 [rows][cols] (dense, row stride cols)
 *   scale fp32 [rows][cols/128]
 * cols % 128 == 0; rows >= 0 (rows == 0 launches nothing).
 */
moe_status fp8_quant_1x128(const uint16_t* x, int64_t ldx, int rows, int cols, uint8_t* q,
                           float* scale, moe_stream_t stream);

/* ---------------------------------------------------------------------------
 * fp8_quant_128x128 -- online 128x128 weight-block quantisation.
 * [ANN] "Fine-Grained Quantization" (weights grouped per 128 input x 128
 * output channels) and "Online Quantization".
 *   w     bf16 [rows][ldw] in nn.Linear layout (output channels x input
 *         channels, input channels contiguous); stacks of experts are passed
 *         as rows = experts * N when N % 128 == 0
 *   q     E4M3 [rows][cols];  scale fp32 [ceil(rows/128)][cols/128]
 * cols % 128 == 0; a ragged last row-block takes its amax over its real rows.
 */
moe_status fp8_quant_128x128(const uint16_t* w, int64_t ldw, int rows, int cols, uint8_t* q,
                             float* scale, moe_stream_t stream);

/* ---------------------------------------------------------------------------
 * fp8_quant_1x128_pow2 / fp8_quant_128x128_pow2 -- the same quantisers with
 * power-of-two scales.  [ANN] "Low-Precision Storage and Communication": the
 * activations quantised before the dispatch carry scaling factors that are
 * integral powers of 2.  Each tile's or block's scale max(amax, 1e-4)/448 is
 * rounded UP to the next power of two (so nothing saturates and the tile
 * maximum lands in [224, 448]); x / scale is then exact and q is its E4M3
 * rounding.  Arguments, layouts, limits and errors as above; the scales are
 * still written as fp32 values (each an exact power of two, i.e. a UE8M0
 * exponent), ready for grouped_gemm_fp8_pow2.
 */
moe_status fp8_quant_1x128_pow2(const uint16_t* x, int64_t ldx, int rows, int cols, uint8_t* q,
                                float* scale, moe_stream_t stream);
moe_status fp8_quant_128x128_pow2(const uint16_t* w, int64_t ldw, int rows, int cols,
                                  uint8_t* q, float* scale, moe_stream_t stream);

/* ---------------------------------------------------------------------------
 * moe_balance_loss -- state and outputs of the complementary sequence-wise
 * balance loss ([ANN] "Complementary Sequence-Wise Auxiliary Loss", eqs.
 * (17)-(20)) when moe_route computes it in its selection pass.  For each
 * sequence q of seq_len consecutive tokens:
 *   L_q = alpha * sum_i f_i P_i,  f_i = E/(K S) * #{t : i in TopK_K(s_t)},
 *   P_i = (1/S) sum_t s'_{i,t},   s'_{i,t} = s_{i,t} / sum_j s_{j,t},
 * the TopK over the raw affinities of all E experts (no bias, no group
 * limit, ties to the lower index, K the routing K).  Each block of 8 tokens
 * adds its sums with integer atomics -- s' in fixed point with 32 fraction
 * bits, so the sum does not depend on the order of the additions and the
 * result is deterministic -- and the last block of a sequence forms f, P and
 * the loss (a fixed-order tree over the experts) and zeroes the sequence's
 * state again.  The caller owns every buffer:
 *   acc   int64 [T/seq_len][E], cnt int32 [T/seq_len][E], done int32
 *         [T/seq_len]: all zero before the first call (cudaMemset); every
 *         call leaves them zero.  One state serves one call at a time.
 *   loss  fp32 [T/seq_len];  f, P fp32 [T/seq_len][E] or NULL.
 * Limits: seq_len % 8 == 0, T % seq_len == 0, seq_len <= 2^30.
 */
typedef struct moe_balance_loss {
  int seq_len;
  float alpha;
  int64_t* acc;
  int32_t* cnt;
  int32_t* done;
  float* loss;
  float* f;
  float* P;
} moe_balance_loss;

/* ---------------------------------------------------------------------------
 * moe_route -- sigmoid router with bias-based, group-limited top-K selection.
 * [ANN] eqs. (13)-(16): s_{i,t} = Sigmoid(u_t . e_i); the top-K is taken over
 * s_{i,t} + b_i, the gate g_{i,t} = s_{i,t} / sum of the chosen s; "Node-
 * Limited Routing": at most M of G groups, groups ranked by the sum of their
 * top K/M biased scores.  Ties go to the lower index (groups and experts);
 * the K outputs of a token are ordered by biased score, descending.
 * The logits are a bf16 x bf16 -> fp32 tensor-core GEMM; everything after
 * them runs in fp32.
 *   u          bf16 [T][ldu];  centroids bf16 [E][d];  bias fp32 [E]
 *   topk_idx   int32 [T][K];   topk_gate fp32 [T][K]
 *   logits_out fp32 [T][E] or NULL (the logits the selection used)
 *   aux        NULL, or the balance loss to compute from the same affinities
 *              in the same pass (see moe_balance_loss)
 *   ws         scratch of moe_route_workspace_size() bytes (may be NULL if 0)
 * Limits: d % 128 == 0, E % 16 == 0, 16 <= E <= 1024, E % G == 0,
 * 1 <= M <= G <= 32, K <= E, K % M == 0 when M < G, K <= 32.
 */
moe_status moe_route_workspace_size(int T, int d, int E, size_t* bytes);
moe_status moe_route(const uint16_t* u, int64_t ldu, const uint16_t* centroids,
                     const float* bias, int T, int d, int E, int G, int M, int K,
                     int32_t* topk_idx, float* topk_gate, float* logits_out,
                     const moe_balance_loss* aux, void* ws, size_t ws_bytes,
                     int32_t* dev_err, moe_stream_t stream);

/* ---------------------------------------------------------------------------
 * moe_permute -- local permutation of (token, expert) pairs by expert, the
 * single-GPU stand-in for the dispatch step.  [ANN] "Low-Precision
 * Communication" (activations are quantised to FP8 before dispatch, so the
 * permutation moves FP8 rows and their scales) and "No Token-Dropping" (no
 * capacity limit: every pair gets a row).
 * Pair (t, k) goes to row dst_of[t][k]; rows of expert e are
 * [offsets[e], offsets[e+1]) in ascending token order.  With with_shared != 0
 * the shared expert is group E whose T rows [T*K, T*K+T) the caller fills
 * with the unpermuted quantised tokens (offsets has E+2 entries then).
 *   topk_idx int32 [T][K] (each token's experts distinct, in [0, E))
 *   xq E4M3 [T][d], xscale fp32 [T][d/128]   (the quantised tokens)
 *   counts int32 [E] (routed pairs per expert), offsets int32 [E+1 (+1)]
 *   src_row int32 [T*K], dst_of int32 [T][K]
 *   xq_perm E4M3 [T*K][d], xscale_perm fp32 [T*K][d/128]  (rows 0..T*K-1)
 *   tile_group int32 [moe_max_m_tiles()], tile_start int32 [groups+1],
 *   n_tiles int32 [1]: the 128-row tiles of every segment, for the grouped
 *   GEMM (tile j covers rows of group tile_group[j]).
 * An out-of-range expert index records MOE_DEVERR_BAD_INDEX.
 */
int moe_max_m_tiles(int T, int K, int E, int with_shared);
moe_status moe_permute_workspace_size(int T, int K, int E, size_t* bytes);
moe_status moe_permute(const int32_t* topk_idx, int T, int K, int E, int with_shared,
                       const uint8_t* xq, const float* xscale, int d, int32_t* counts,
                       int32_t* offsets, int32_t* src_row, int32_t* dst_of, uint8_t* xq_perm,
                       float* xscale_perm, int32_t* tile_group, int32_t* tile_start,
                       int32_t* n_tiles, void* ws, size_t ws_bytes, int32_t* dev_err,
                       moe_stream_t stream);

/* ---------------------------------------------------------------------------
 * moe_permute_index -- moe_permute without moving any row: counts, offsets,
 * src_row, dst_of and the tile table only (same arguments, layouts, limits
 * and errors, minus xq/xscale/d/xq_perm/xscale_perm).  The rows are then
 * written by fp8_quant_1x128_scatter, which quantises each token once and
 * stores its FP8 bytes straight at every destination row ([ANN]
 * "Low-Precision Communication": the tokens are quantised to FP8 and the FP8
 * rows are what the dispatch moves).
 */
moe_status moe_permute_index(const int32_t* topk_idx, int T, int K, int E, int with_shared,
                             int32_t* counts, int32_t* offsets, int32_t* src_row,
                             int32_t* dst_of, int32_t* tile_group, int32_t* tile_start,
                             int32_t* n_tiles, void* ws, size_t ws_bytes, int32_t* dev_err,
                             moe_stream_t stream);

/* ---------------------------------------------------------------------------
 * fp8_quant_1x128_scatter -- fp8_quant_1x128 (or its power-of-two form,
 * pow2 != 0) with the permutation's gather fused in: every 1x128 tile of row
 * t is quantised once ([ANN] "Fine-Grained Quantization", "Online
 * Quantization") and written to the token-order copy q_tok / s_tok (row t;
 * both may be NULL) and to row dst_of[t][k] of q_perm / s_perm for every k
 * with dst_of[t][k] >= 0 (moe_permute_index's output; a -1 entry, left by a
 * flagged bad expert index, writes nothing).  The bytes and scales equal
 * fp8_quant_1x128 followed by moe_permute's gather.
 *   x bf16 [rows][ldx]; dst_of int32 [rows][K]; q_tok E4M3 [rows][cols],
 *   s_tok fp32 [rows][cols/128]; q_perm E4M3 [rows*K][cols], s_perm fp32
 *   [rows*K][cols/128].
 * Limits: cols % 128 == 0, 1 <= K <= 16.
 */
moe_status fp8_quant_1x128_scatter(const uint16_t* x, int64_t ldx, int rows, int cols,
                                   const int32_t* dst_of, int K, int pow2, uint8_t* q_tok,
                                   float* s_tok, uint8_t* q_perm, float* s_perm,
                                   moe_stream_t stream);

/* ---------------------------------------------------------------------------
 * moe_permute_noalloc -- moe_permute without a caller workspace.  The pages
 * have no counterpart: it is a deployment convenience.  It serves callers
 * that cannot allocate device memory at call time -- plugins of inference
 * runtimes whose host framework owns and plans all device memory and gives
 * the plugin no workspace, and latency-critical paths that must not incur
 * cudaMalloc's implicit device-wide synchronisation.
 * Arguments, outputs and errors are those of moe_permute minus ws/ws_bytes.
 * Its scratch is a fixed 1 MiB file-scope device array (262144 int32), held
 * by every device that loads the library until the library is unloaded; a
 * batch whose moe_permute_workspace_size exceeds 1 MiB (ceil(T/128) * E int32
 * entries) returns MOE_ERR_UNSUPPORTED before anything is launched.  The
 * first call on a device looks up the array's device address
 * (cudaGetSymbolAddress); make that first call before any stream capture.
 * All calls share the array and it keeps the last call's contents (nothing in
 * it needs clearing); calls that overlap on the GPU race on it, so the caller
 * must serialise them.  It allocates nothing.
 */
moe_status moe_permute_noalloc(const int32_t* topk_idx, int T, int K, int E, int with_shared,
                               const uint8_t* xq, const float* xscale, int d, int32_t* counts,
                               int32_t* offsets, int32_t* src_row, int32_t* dst_of,
                               uint8_t* xq_perm, float* xscale_perm, int32_t* tile_group,
                               int32_t* tile_start, int32_t* n_tiles, int32_t* dev_err,
                               moe_stream_t stream);

/* ---------------------------------------------------------------------------
 * moe_tile_table -- the 128-row tile table of arbitrary segment offsets (for
 * grouped GEMM calls whose segments do not come from moe_permute).
 *   offsets int32 [groups+1], non-decreasing, device
 *   tile_group int32 [max_tiles], tile_start int32 [groups+1], n_tiles int32 [1]
 * Inconsistent offsets or too small a max_tiles record MOE_DEVERR_BAD_TABLE.
 */
moe_status moe_tile_table(const int32_t* offsets, int groups, int max_tiles,
                          int32_t* tile_group, int32_t* tile_start, int32_t* n_tiles,
                          int32_t* dev_err, moe_stream_t stream);

/* ---------------------------------------------------------------------------
 * moe_segment_ids -- expert parallelism: the group of every row of a receive
 * buffer that holds, for each source rank s in order, its rows of this rank's
 * E local experts sorted by expert ([ANN] "Low-Precision Communication": FP8
 * rows dispatched to the experts' ranks).  counts int32 [n_segments] (=
 * [sources][E], row-major).  With lead_rows == 0: ids int32 [n_rows], row r of
 * segment s gets s % E.  With lead_rows > 0 the buffer starts with lead_rows
 * rows of group 0 (the rank's own tokens, which the shared expert takes) and
 * the received rows after them get 1 + s % E.  The ids feed moe_permute
 * (K = 1) to regroup the rows by group.  Counts that do not sum to n_rows -
 * lead_rows, or negative counts, record MOE_DEVERR_BAD_TABLE.
 * Limits: n_segments % E == 0, n_segments <= 1024, 0 <= lead_rows <= n_rows. */
moe_status moe_segment_ids(const int32_t* counts, int n_segments, int E, int64_t lead_rows,
                           int64_t n_rows, int32_t* ids, int32_t* dev_err, moe_stream_t stream);

/* ---------------------------------------------------------------------------
 * grouped_gemm_fp8_blockscaled -- D_g = A_g . B_g^T for every segment g, with
 * FP8 operands, per-128-K block scales and fp32 accumulation.
 * [ANN] "Fine-Grained Quantization" (per-group scales along the inner
 * dimension K) and "Increasing Accumulation Precision" (partial results
 * promoted to fp32 and scaled every 128 elements of K).  Here each 128-wide
 * K block is one tensor-core (tcgen05) accumulation in TMEM, which is then
 * scaled by sa * sb and added to an fp32 register accumulator.
 *   A  E4M3 [a_rows][K], sa fp32 [a_rows][K/128]  (1x128 tiles)
 *   B  E4M3 [groups][N][K], sb fp32 [groups][N/128][K/128] (128x128 blocks)
 *   offsets int32 [groups+1] (segment g = rows [offsets[g], offsets[g+1]))
 *   tile_group / tile_start / n_tiles: as written by moe_permute or
 *   moe_tile_table; max_tiles = capacity of tile_group.  The kernel walks
 *   (group, n-tile, m-tile) work items from tile_start (the per-group tile
 *   prefix) and offsets; max_tiles bounds its grid.
 *   ep == MOE_EP_F32:  D fp32 [a_rows][N] (rows outside every segment are
 *                      left untouched); d_scale unused.  d_rows (optional,
 *                      int32 [a_rows], NULL = identity) sends A row j's
 *                      output to D row d_rows[j]: expert parallelism writes
 *                      the outputs of rows regrouped by expert straight back
 *                      in receive order ([ANN] "Low-Precision
 *                      Communication": the combine's rows return to their
 *                      senders).  A map entry outside [0, a_rows) records
 *                      MOE_DEVERR_BAD_TABLE and its row is not written.
 *   ep == MOE_EP_SWIGLU_QUANT: B rows are gate/up block-interleaved (rows
 *      [256j, 256j+128) gate channels 128j.., the next 128 the matching up
 *      channels); D is E4M3 h [a_rows][N/2] with h = SiLU(gate) * up
 *      ([ANN] SwiGLU operator notes, Swish with beta = 1) quantised 1x128 as
 *      in fp8_quant_1x128, d_scale fp32 [a_rows][N/256]; d_rows must be NULL.
 *   sched: one int32 of device scratch, or NULL.  With it the kernel hands
 *      out its (group, n-tile, m-tile) work items dynamically (an atomic
 *      counter, zeroed by the call on `stream`; calls that overlap on the GPU
 *      must not share it); NULL keeps a static round-robin order.  The results
 *      are the same either way.  The pow2 variant ignores it.
 *   An m-tile of at most 32 rows (an expert's tail past its whole 128-row
 *   tiles, or an expert with few rows) is computed transposed -- the weight
 *   tile's halves as the tensor core's M side, the rows as N = 32 -- with the
 *   same per-128-K scaled fp32 accumulation (K <= 8192).
 * Limits: K % 128 == 0, N % 256 == 0.
 */
moe_status grouped_gemm_fp8_blockscaled(const uint8_t* A, const float* sa, int64_t a_rows,
                                        const uint8_t* B, const float* sb,
                                        const int32_t* offsets, const int32_t* tile_group,
                                        const int32_t* tile_start, const int32_t* n_tiles,
                                        int max_tiles, int groups, int N, int K,
                                        moe_epilogue ep, void* D, float* d_scale,
                                        const int32_t* d_rows, int32_t* sched,
                                        int32_t* dev_err, moe_stream_t stream);

/* ---------------------------------------------------------------------------
 * grouped_gemm_fp8_pow2 -- grouped_gemm_fp8_blockscaled for operands whose
 * every scale is a power of two (from the _pow2 quantisers).  [ANN] "Low-
 * Precision Storage and Communication" (power-of-two scaling factors) and
 * "Suggestions on Hardware Design" / "Support for Tile- and Block-Wise
 * Quantization" (tensor cores that apply the group scales themselves, with
 * no copy of partial results to the CUDA cores): each scale's exponent is handed to the tensor core as a
 * UE8M0 scale factor (tcgen05 kind::mxf8f6f4 block scaling, one exponent
 * per row per 32-element K slice, the 1x128 / 128x128 scale repeated over
 * its four slices), and the whole K extent accumulates in the tensor core's
 * fp32 TMEM accumulator with no promotion step.
 * Arguments, layouts and limits as in grouped_gemm_fp8_blockscaled; with
 * MOE_EP_SWIGLU_QUANT the scales of h are rounded up to powers of two as in
 * fp8_quant_1x128_pow2.  A scale that is not a positive normal power of two
 * records MOE_DEVERR_BAD_SCALE (its exponent is used as if the mantissa were
 * zero).
 */
moe_status grouped_gemm_fp8_pow2(const uint8_t* A, const float* sa, int64_t a_rows,
                                 const uint8_t* B, const float* sb, const int32_t* offsets,
                                 const int32_t* tile_group, const int32_t* tile_start,
                                 const int32_t* n_tiles, int max_tiles, int groups, int N, int K,
                                 moe_epilogue ep, void* D, float* d_scale,
                                 const int32_t* d_rows, int32_t* sched, int32_t* dev_err,
                                 moe_stream_t stream);

/* ===========================================================================
 * Backward of the expert FFNs.  [ANN] "Mixed Precision Framework": Fprop,
 * Dgrad (activation gradient) and Wgrad (weight gradient) GEMMs all take FP8
 * inputs; weight gradients stay fp32.  "Low-Precision Activation": the
 * SwiGLU input is cached in FP8 and the SwiGLU output recomputed.  "Low-
 * Precision Communication": the gradient before the down projection is
 * quantised to FP8 with power-of-two scales.  "Support for Transposed GEMM
 * Operations": an operand reduced over tokens is re-quantised in 128x1 tiles.
 * Every gradient quantisation here is 1x128 along channels (or 128x1 along
 * tokens for Wgrad) with power-of-two scales.  The Dgrad GEMMs are
 * grouped_gemm_fp8_blockscaled / grouped_gemm_fp8_pow2 with A = the
 * quantised gradient and B = the transposed weights (fp8_transpose_128x128).
 * =========================================================================== */

/* fp8_quant_1x128_f32 -- 1x128 quantisation of fp32 rows (the SwiGLU input
 * cache); pow2 != 0 rounds each scale up to a power of two.
 *   x fp32 [rows][ldx];  q E4M3 [rows][cols];  scale fp32 [rows][cols/128]
 * Limits: cols % 128 == 0, ldx % 4 == 0. */
moe_status fp8_quant_1x128_f32(const float* x, int64_t ldx, int rows, int cols, int pow2,
                               uint8_t* q, float* scale, moe_stream_t stream);

/* moe_combine_backward -- the gradient at every expert output row of the
 * permuted layout (the backward of eq. (12)): dy[dst_of[t][k]] = fl32(gate
 * [t][k] * dout[t]), dy[T*K + t] = dout[t], quantised 1x128 with power-of-two
 * scales.  Rows with dst_of < 0 are skipped.
 *   dout fp32 [T][d];  dyq E4M3 [T*K+T][d];  dys fp32 [T*K+T][d/128]
 *   dy fp32 [T*K+T][d] or NULL (the unquantised values, for the Wgrad operand)
 * Limits: d % 128 == 0, K <= 32. */
moe_status moe_combine_backward(const float* dout, const int32_t* dst_of, const float* topk_gate,
                                int T, int K, int d, uint8_t* dyq, float* dys, float* dy,
                                moe_stream_t stream);

/* swiglu_backward -- from dh [rows][I] (Dgrad of the down projection) and the
 * cached SwiGLU input gu (E4M3 [rows][2I], 1x128 scales [rows][2I/128], gate/
 * up blocks interleaved as in the forward): sigma = 1/(1+e^-g), dg = dh * u *
 * sigma (1 + g (1 - sigma)), du = dh * g sigma, in fp32; dgu (same
 * interleaving) quantised 1x128 with power-of-two scales.
 *   dguq E4M3 [rows][2I], dgus fp32 [rows][2I/128]
 *   dgu fp32 [rows][2I] or NULL;  h fp32 [rows][I] or NULL (the recomputed
 *   SwiGLU output g sigma u, for the Wgrad of the down projection)
 * Limits: I % 128 == 0. */
moe_status swiglu_backward(const float* dh, const uint8_t* guq, const float* gus, int rows, int I,
                           uint8_t* dguq, float* dgus, float* dgu, float* h, moe_stream_t stream);

/* fp8_quant_128x1_pow2 / fp8_requant_128x1_pow2 -- token-major (transposed)
 * re-quantisation for Wgrad.  For every 128-token tile i of the segment table
 * (tile_group, tile_start, n_tiles as written by moe_permute or
 * moe_tile_table), rows offsets[g] + 128 (i - tile_start[g]) .. (zero past
 * the segment's end): qt[c][128 i + r] = E4M3(src[row r][c] / st[c][i]), st
 * = the power-of-two scale of the 128 tokens of channel c.  The _requant form
 * reads an FP8 source with 1x128 scales (the cached x) and dequantises it
 * first.
 *   src fp32 [rows][ld_src]  (or q E4M3 [rows][ld_src], scale [rows][ld_src/128])
 *   qt E4M3 [C][ldt], st fp32 [C][ldt/128], ldt >= 128 * max_tiles
 *   sf_atoms NULL or [C/128][ldt/512][512] bytes (ldt % 512 == 0): the
 *   exponents (UE8M0) of st arranged for grouped_gemm_fp8_wgrad (byte
 *   16 r + 4 j + b of atom (cb, a) = channel 128 cb + 32 j + r, tile 4a + b)
 * Limits: C % 128 == 0. */
moe_status fp8_quant_128x1_pow2(const float* src, int64_t ld_src, const int32_t* offsets,
                                const int32_t* tile_group, const int32_t* tile_start,
                                const int32_t* n_tiles, int max_tiles, int C, uint8_t* qt,
                                int64_t ldt, float* st, uint8_t* sf_atoms, moe_stream_t stream);
moe_status fp8_requant_128x1_pow2(const uint8_t* q, const float* scale, int64_t ld_src,
                                  const int32_t* offsets, const int32_t* tile_group,
                                  const int32_t* tile_start, const int32_t* n_tiles,
                                  int max_tiles, int C, uint8_t* qt, int64_t ldt, float* st,
                                  uint8_t* sf_atoms, moe_stream_t stream);

/* fp8_transpose_128x128 -- FP8 weight stack [groups][N][K] with 128x128
 * scales [groups][N/128][K/128] -> [groups][K][N] and [groups][K/128][N/128]
 * (exact: every block keeps its scale); the B operand of a Dgrad GEMM.
 * Limits: N % 128 == 0, K % 128 == 0. */
moe_status fp8_transpose_128x128(const uint8_t* q, const float* scale, int groups, int N, int K,
                                 uint8_t* qt, float* scale_t, moe_stream_t stream);

/* moe_unpermute_add -- du[t] = dout[t] + dx[T*K + t] + sum_k dx[dst_of[t][k]]
 * (fp32, added in that order): the gradient of the layer input through the
 * residual and the experts (the router's share is not included).
 *   dx fp32 [T*K+T][d] (Dgrad of the up projection by permuted row) */
moe_status moe_unpermute_add(const float* dx, const int32_t* dst_of, const float* dout, int T,
                             int K, int d, float* du, moe_stream_t stream);

/* grouped_gemm_fp8_wgrad -- dW[g] = At[:, tiles of g] . Bt[:, tiles of g]^T,
 * fp32 [groups][Ma][Nb], for every group g with tiles tile_start[g] ..
 * tile_start[g+1] (128 tokens each) of both token-major operands; a group
 * without tiles gets a zero gradient.  The exponents of both operands (one
 * per row per 128 tokens, from fp8_quant_128x1_pow2's sf_atoms) are applied
 * by the tensor core (block-scaled tcgen05 MMA), fp32 accumulation in TMEM.
 *   At E4M3 [Ma][ldt], Bt E4M3 [Nb][ldt]; sfa_atoms / sfb_atoms as above
 * Limits: Ma % 128 == 0, Nb % 256 == 0, ldt % 512 == 0. */
moe_status grouped_gemm_fp8_wgrad(const uint8_t* At, const uint8_t* sfa_atoms, const uint8_t* Bt,
                                  const uint8_t* sfb_atoms, int64_t ldt, int Ma, int Nb,
                                  const int32_t* tile_start, int groups, float* dW,
                                  int32_t* dev_err, moe_stream_t stream);

/* ---------------------------------------------------------------------------
 * swiglu_quant -- standalone SwiGLU + 1x128 quantisation of fp32 GEMM output
 * in the block-interleaved layout above; bit-identical to the fused epilogue
 * on identical input.  [ANN] SwiGLU operator notes: h = Swish(gate) * up with
 * Swish(x) = x * Sigmoid(x); "Fine-Grained Quantization": the input of the
 * down projection is FP8 like every GEMM input, quantised per token per 128
 * channels ("Online Quantization": scale from the tile's own max |h|).
 * swiglu_quant_pow2 rounds each scale up to a power of two ([ANN]
 * "Low-Precision Storage and Communication").
 *   gu fp32 [rows][2I];  h E4M3 [rows][I];  h_scale fp32 [rows][I/128]
 */
moe_status swiglu_quant(const float* gu, int rows, int I, uint8_t* h, float* h_scale,
                        moe_stream_t stream);
/* swiglu_quant_pow2 -- the same with the scales of h rounded up to powers of
 * two (bit-identical to grouped_gemm_fp8_pow2's fused epilogue on identical
 * input). */
moe_status swiglu_quant_pow2(const float* gu, int rows, int I, uint8_t* h, float* h_scale,
                             moe_stream_t stream);

/* ---------------------------------------------------------------------------
 * moe_combine -- [ANN] eq. (12): out_t = u_t + FFN_shared(u_t)
 *                                        + sum_k gate[t][k] * Y[dst_of[t][k]],
 * summed in fp32 in that order (k ascending), deterministic.
 *   Y fp32 [>= T*K][d] (routed expert outputs by permuted row)
 *   Y_shared fp32 [T][d] or NULL;  u bf16 [T][d];  out fp32 [T][d]
 */
moe_status moe_combine(const float* Y, const int32_t* dst_of, const float* topk_gate,
                       const float* Y_shared, const uint16_t* u, int T, int K, int d,
                       float* out, moe_stream_t stream);

/* ---------------------------------------------------------------------------
 * moe_bias_update -- [ANN] "Auxiliary-Loss-Free Load Balancing": after the
 * step, b_i -= gamma for an expert loaded above the batch mean T*K/E, b_i +=
 * gamma below it, unchanged at it (fp32).  counts are routed pairs per
 * expert over the whole batch of T tokens (sum over data-parallel ranks).
 *   counts int32 [E], bias fp32 [E] (updated in place)
 */
moe_status moe_bias_update(const int32_t* counts, int E, int64_t T, int K, float gamma,
                           float* bias, moe_stream_t stream);

/* ---------------------------------------------------------------------------
 * moe_seq_balance_loss -- the complementary sequence-wise balance loss,
 * [ANN] "Complementary Sequence-Wise Auxiliary Loss", eqs. (17)-(20), for
 * every sequence of seq_len consecutive tokens:
 *   L = alpha * sum_i f_i P_i,  f_i = E / (K * seq_len) * #{t : i in TopK(s_t)},
 *   P_i = (1/seq_len) * sum_t s_{i,t} / sum_j s_{j,t},  s = Sigmoid(logits);
 * the TopK over the raw affinities of all E routed experts (no bias, no group
 * limit), ties to the lower index.  DeepSeek-V3 uses alpha = 1e-4.
 * Deterministic (fixed reduction orders, no atomics); fp32 arithmetic.
 *   logits fp32 [T][E] (moe_route's logits_out);  T % seq_len == 0
 *   loss fp32 [T/seq_len]; f, P fp32 [T/seq_len][E] (each may be NULL)
 *   ws: moe_seq_balance_loss_workspace_size bytes (T*E floats plus the
 *       per-32-token partials)
 * Limits: K <= min(E, 32), E <= 1024.
 */
moe_status moe_seq_balance_loss_workspace_size(int T, int E, int seq_len, size_t* bytes);
moe_status moe_seq_balance_loss(const float* logits, int T, int E, int K, int seq_len,
                                float alpha, float* loss, float* f, float* P, void* ws,
                                size_t ws_bytes, moe_stream_t stream);

/* ---------------------------------------------------------------------------
 * moe_fp8_mma_peak -- measurement helper: the dense FP8 tensor-core rate of
 * this GPU, the denominator of the expert GEMMs' roofline ([ANN]
 * "Fine-Grained Quantization": both GEMM operands are E4M3; "Suggestions on
 * Hardware Design" asks for tensor cores that take the group scales, which
 * block_scaled = 1 exercises).  One CTA per SM (ctas of them) runs `iters` K
 * blocks of four 128x256x32 E4M3 tcgen05 MMAs from shared memory into TMEM
 * and touches no global memory except sink.  block_scaled = 0:
 * kind::f8f6f4 (what grouped_gemm_fp8_blockscaled issues); 1:
 * kind::mxf8f6f4.block_scale with unit UE8M0 scales (what
 * grouped_gemm_fp8_pow2 issues).  The caller times the launch:
 *   FLOPs = ctas * iters * 4 * (2 * 128 * 256 * 32).
 *   sink fp32 [ctas] (one accumulator value per CTA, ignore it)
 * Limits: 1 <= iters <= 2^21 (the kernel's bounded wait is 2 s); a wait that
 * gives up records MOE_DEVERR_TIMEOUT.
 */
moe_status moe_fp8_mma_peak(int block_scaled, int iters, int ctas, float* sink,
                            int32_t* dev_err, moe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOEFP8_H */
