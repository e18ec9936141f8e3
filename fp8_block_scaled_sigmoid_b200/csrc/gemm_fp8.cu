// Block-scaled FP8 grouped GEMM for sm_100a (tcgen05 + TMEM + TMA).
//
// "DeepSeek_V3_Report：Annotation", "Fine-Grained Quantization" and
// "Increasing Accumulation Precision": activations carry one fp32 scale per
// 1x128 tile, weights one per 128x128 block, so the scales change along the
// inner dimension K every 128 elements; the pages promote the tensor core's
// partial sums to fp32 registers every N_C = 128 elements and apply the
// scales there.  On Blackwell the same contract maps onto:
//
//   * one 128x256x128 block product per K block = 4 tcgen05.mma (K=32 each)
//     from a TMA-fed, swizzled shared-memory ring into a fresh TMEM
//     accumulator (two 256-column buffers, ping-pong);
//   * two epilogue warpgroups drain each finished buffer with tcgen05.ld and
//     fold it into fp32 register accumulators: acc += (sa[row,kb] *
//     sb[nblk,kb]) * partial (packed fp32x2 FMA), while the tensor core fills
//     the other buffer;
//   * a persistent grid walks the (expert, n-tile, m-tile) work list derived
//     on the device from the segment offsets and the tile table's per-expert
//     tile prefix, so the ragged expert segments need no host
//     synchronisation; the m-tiles of one expert that share a weight tile run
//     next to each other for L2 reuse.  With a caller work counter the items
//     are handed out dynamically; an m-tile of at most 32 rows is computed
//     transposed (the weight tile's halves as M, its rows as N), and a
//     partial m-tile loads only the 32-row groups of A that hold its rows.
//
// The shared-memory ring is staged in K slices of SK bytes (128, or 64 with
// the 64-byte swizzle): a stage is released as soon as the MMAs of its slice
// complete.  Measured on V3-prefill shapes, 128-byte slices are faster (the
// 64-byte ones halve the contiguous bytes each weight row contributes to a
// TMA box), so 128 is the default.
//
// One CTA computes a 128 x 256 tile (tcgen05 cta_group::1).  A CTA-pair form
// (cta_group::2, 256 x 256 tiles, each CTA staging half of A and of the
// weight tile) was measured slower on every workload here: its cross-CTA
// handshakes cost more than the halved shared-memory ingress saves.
//
// Warp roles (384 threads): warp 0 = TMA producer, warp 1 = MMA issuer and
// TMEM owner, warp 2 stages the tile prefix then idles with warp 3 (the first
// warpgroup gives registers to the other two), warps 4..11 = epilogue (warp w
// reads TMEM lanes 32*(w%4)..).  Epilogues: fp32 rows, or SwiGLU + 1x128 E4M3
// requantisation of h (the W1 rows are gate/up block-interleaved so one
// 256-wide tile holds 128 gate and the matching 128 up channels).  Every
// wait is bounded (MOE_DEVERR_TIMEOUT).
#include <algorithm>

#include "epi_math.cuh"
#include "moe_common.cuh"

// Stage width (build-time choice).
#ifndef MOE_GEMM_SK
#define MOE_GEMM_SK 128
#endif

namespace moe {
namespace {

constexpr int kBM = 128, kBN = 256, kBK = 128;
constexpr int kThreads = 384;       // 3 warpgroups
constexpr int kEpiThreads = 256;    // warpgroups 1 and 2
// Register split (setmaxnreg), checked against the launch budget of
// 384 threads x 168 registers = 64512: 128 x 56 + 256 x 224 = 64512.
constexpr int kRegsCtl = 56;
constexpr int kRegsEpi = 224;
constexpr uint32_t kTmemCols = 512;
constexpr int kRingBytes = 192 * 1024;
constexpr int kMaxGroups = 1024;
constexpr size_t kSmemBytes = 1024 + kRingBytes + 512 + (kMaxGroups + 1) * 4 + 2048 + 64;
// Tail m-tiles of at most kTailRows rows (an expert's last rows past a whole
// 128-row tile, or an expert with few rows) take the swapped path below.
// Its promotion factors sa * sb for every (K block, weight half, row) are
// staged in shared memory: 2 x kTailRows x kTailMaxKB floats.
constexpr int kTailRows = 32;
constexpr int kTailMaxKB = 64;
constexpr int kTailFactorBytes = 2 * kTailRows * kTailMaxKB * 4;
// work queue (4 slots) and the tail path's barriers and amax exchange
constexpr int kWQ = 4;
constexpr int kQueueBytes = 1024;     // barriers, slots and amax; the factors start at +640
constexpr int kTailFactorOffset = 640;
constexpr size_t kSmemPromoteBytes = kSmemBytes + kQueueBytes + kTailFactorBytes;
static_assert(kSmemPromoteBytes <= 232448, "shared memory per CTA");

struct GemmArgs {
  const float* sa;
  int64_t a_rows;
  const float* sb;
  const int32_t* offsets;
  const int32_t* tile_group;
  const int32_t* tile_start;
  const int32_t* n_tiles;
  int max_tiles, groups, N, K;
  void* D;
  float* d_scale;
  int32_t* dev_err;
  const int32_t* d_rows;  // fp32 epilogue: output row of A row j (NULL: row j)
  int32_t* sched;         // work counter (zeroed before the launch), NULL: static schedule
};

// Tensor maps of A with boxes of 32, 64, 96 and 128 rows: an m-tile loads
// only the 32-row groups that hold its rows (the MMA still reads 128 rows;
// the rest of the stage holds older bytes, whose results land in rows that
// are never written out).
struct ATmaps {
  CUtensorMap box[4];
};

// index of the smallest A box holding `rows` rows
__device__ __forceinline__ int a_box(int rows) { return min(3, max(0, (rows - 1) >> 5)); }

struct Work {
  int e, n_idx, row0, rows;  // expert, n-tile, first row and valid rows of the m-tile
  bool ok;
  bool swp;  // a tail tile for the swapped path (rows <= kTailRows)
};

template <int SK>
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t addr) {
  static_assert(SK == 128 || SK == 64, "stage K width");
  return SK == 128 ? smem_desc_sw128(addr) : smem_desc_sw64(addr);
}

// rstart[g] = number of 128-row tiles of the groups before g: the tile
// table's tile_start (written by moe_permute / moe_tile_table), staged in
// shared memory by one warp.
__device__ __forceinline__ void load_tile_prefix(const GemmArgs& a, int* rstart, int lane) {
  for (int g = lane; g <= a.groups; g += 32) rstart[g] = __ldg(a.tile_start + g);
}

// Work item w -> (expert, n-tile, RT-row tile); the items of expert e occupy
// [nN*rstart[e], nN*rstart[e+1]) and the row tile varies fastest inside.
template <int RT>
__device__ __forceinline__ Work decode_work(int w, int nN, const int* rstart, const GemmArgs& a) {
  Work t{0, 0, 0, 0, false, false};
  const int j = w / nN;
  int lo = 0, hi = a.groups - 1;
  while (lo < hi) {  // last group whose first tile index is <= j
    const int mid = (lo + hi + 1) >> 1;
    if (rstart[mid] <= j) lo = mid;
    else hi = mid - 1;
  }
  const int e = lo;
  const int tc = rstart[e + 1] - rstart[e];
  if (tc <= 0 || j < rstart[e] || j >= rstart[e] + tc) return t;
  const int local = w - nN * rstart[e];
  t.n_idx = local / tc;
  const int mt = local - t.n_idx * tc;
  const int seg0 = __ldg(a.offsets + e), seg1 = __ldg(a.offsets + e + 1);
  const int tile0 = seg0 + RT * mt;
  if (tile0 >= seg1 || seg1 > a.a_rows || t.n_idx >= nN) return t;
  t.row0 = tile0;
  t.rows = min(RT, seg1 - tile0);
  t.e = e;
  t.ok = true;
  t.swp = t.rows <= kTailRows && a.K / kBK <= kTailMaxKB;
  return t;
}

// ------------------------------------------------------------------ epilogue
// Writes one finished tile from this thread's fp32 accumulators: row r_in of
// the tile, columns c_lo..c_lo+63 and c_hi..c_hi+63 as 64 packed pairs.  POW2
// rounds the requantisation scale of h up to a power of two.  Returns false
// if a bounded wait gave up.
template <int EP, bool POW2>
__device__ __forceinline__ bool write_tile(const GemmArgs& args, const Work& t, float2 (&acc)[64],
                                           int warp, int lane, int N, int& xtile, uint64_t* xbar,
                                           float* amax_x, volatile int* abort_v) {
  const int g = (warp - 4) >> 2;
  const int r_in = (warp & 3) * 32 + lane;
  const int64_t arow = static_cast<int64_t>(t.row0) + r_in;
  const bool row_ok = r_in < t.rows;
  if (EP == MOE_EP_F32) {
    // Each lane holds one row (128 columns).  Per 32-column chunk, the 8
    // lanes of each group (rows rb..rb+7) transpose their 8 x 8 block of
    // float4 with three xor-butterfly exchange rounds: afterwards lane rb+i
    // holds columns 4i..4i+3 of every row of the group, so one store
    // instruction writes 4 rows x 128 contiguous bytes (whole lines).
    const int li = lane & 7;
    const int rb = r_in - li;  // first row of this lane's group inside the tile
    // output row of each of the group's 8 rows: the tile's own rows, or the
    // caller's row map (lane rb + j reads row rb + j's entry and the group's
    // lanes exchange them); a bad map entry skips its row
    int my_drow = -1;
    if (args.d_rows != nullptr && row_ok) {
      my_drow = __ldg(args.d_rows + arow);
      if (static_cast<uint32_t>(my_drow) >= static_cast<uint32_t>(args.a_rows)) {
        set_dev_err(args.dev_err, MOE_DEVERR_BAD_TABLE);
        my_drow = -1;
      }
    }
    int drow[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
      drow[j] = args.d_rows != nullptr ? __shfl_sync(0xffffffffu, my_drow, (lane & ~7) | j)
                                       : t.row0 + rb + j;
    float* const D0 = static_cast<float*>(args.D) + t.n_idx * kBN + 128 * g + 4 * li;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      float4 e[8];  // e[j] = columns 32b + 4j .. 32b + 4j + 3 of this lane's row
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float2 x0 = acc[16 * b + 2 * j], x1 = acc[16 * b + 2 * j + 1];
        e[j] = make_float4(x0.x, x0.y, x1.x, x1.y);
      }
      // round s: for each pair (j0, j0 | s), a lane with bit s set sends e[j0]
      // and receives its partner's e[j0 | s] into e[j0]; the other sends
      // e[j0 | s] and receives into it
#pragma unroll
      for (int sft = 1; sft < 8; sft <<= 1) {
        const bool hi = (lane & sft) != 0;
#pragma unroll
        for (int j0 = 0; j0 < 8; ++j0) {
          if (j0 & sft) continue;
          const int j1 = j0 | sft;
          const float4 x = hi ? e[j0] : e[j1];
          float4 y;
          y.x = __shfl_xor_sync(0xffffffffu, x.x, sft);
          y.y = __shfl_xor_sync(0xffffffffu, x.y, sft);
          y.z = __shfl_xor_sync(0xffffffffu, x.z, sft);
          y.w = __shfl_xor_sync(0xffffffffu, x.w, sft);
          if (hi) e[j0] = y;
          else e[j1] = y;
        }
      }
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (rb + j < t.rows && drow[j] >= 0)
          *reinterpret_cast<float4*>(D0 + static_cast<int64_t>(drow[j]) * N + 32 * b) = e[j];
    }
  } else {
    // h = SiLU(gate) * up overwrites the gate accumulators: h[2i], h[2i+1]
    // are acc[i].x, acc[i].y; the up channels are acc[32..63]
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      acc[i].x = silu_mul(acc[i].x, acc[32 + i].x);
      acc[i].y = silu_mul(acc[i].y, acc[32 + i].y);
      amax = fmaxf(amax, fmaxf(fabsf(acc[i].x), fabsf(acc[i].y)));
    }
    // the 1x128 tile amax is shared with the partner thread of the other half
    const int xb = xtile & 1;
    amax_x[(xb * 2 + g) * 128 + r_in] = amax;
    mbar_arrive(&xbar[xb]);
    if (!__all_sync(0xffffffffu, mbar_wait(&xbar[xb], (xtile >> 1) & 1, abort_v, args.dev_err)))
      return false;
    amax = fmaxf(amax_x[(xb * 2 + 0) * 128 + r_in], amax_x[(xb * 2 + 1) * 128 + r_in]);
    ++xtile;
    const float sq = POW2 ? pow2_ceil(quant_scale(amax)) : quant_scale(amax);
    const float rq = __frcp_rn(sq);
    if (row_ok) {
      const int I = N / 2;
      uint8_t* dst = static_cast<uint8_t*>(args.D) + arow * I + t.n_idx * 128 + 64 * g;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2* hp = acc + 8 * i;  // h[16i .. 16i+15]
        uint32_t w4[4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
          w4[j] = e4m3x4(div_by_scale(hp[2 * j].x, sq, rq), div_by_scale(hp[2 * j].y, sq, rq),
                         div_by_scale(hp[2 * j + 1].x, sq, rq), div_by_scale(hp[2 * j + 1].y, sq, rq));
        reinterpret_cast<uint4*>(dst)[i] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
      }
      if (g == 0) args.d_scale[arow * (I / 128) + t.n_idx] = sq;
    }
  }
  return true;
}

// Promotes every K block of one tile into fp32 registers and writes the
// tile.  Returns false if a bounded wait gave up.
template <int EP>
__device__ __forceinline__ bool epilogue_tile(const GemmArgs& args, const Work& t, uint32_t tmem,
                                              int warp, int lane, int KB, int N, int& tit,
                                              int& xtile, uint64_t* tfull, uint64_t* tempty,
                                              uint64_t* xbar, float* amax_x,
                                              volatile int* abort_v) {
  const int g = (warp - 4) >> 2;   // which half of the columns
  const int q = warp & 3;          // TMEM lane quarter this warp may read
  const int r_in = q * 32 + lane;  // row inside the tile
  const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
  // columns of the 256-wide tile this thread accumulates (two runs of 64)
  const int c_lo = (EP == MOE_EP_F32) ? 128 * g : 64 * g;
  const int c_hi = (EP == MOE_EP_F32) ? 128 * g + 64 : 128 + 64 * g;
  // 128 fp32 accumulators as 64 packed pairs (packed fp32x2 FMA)
  float2 acc[64];
#pragma unroll
  for (int i = 0; i < 64; ++i) acc[i] = make_float2(0.f, 0.f);
  const int64_t arow = static_cast<int64_t>(t.row0) + r_in;
  const int64_t arow_c = arow < args.a_rows ? arow : args.a_rows - 1;
  const float* sa_row = args.sa + arow_c * KB;
  const float* sb0 = args.sb + (static_cast<int64_t>(t.e) * (N / 128) + t.n_idx * 2) * KB;
  const float* sb1 = sb0 + KB;
  const float* sb_lo = (EP == MOE_EP_F32) ? (g ? sb1 : sb0) : sb0;
  const float* sb_hi = (EP == MOE_EP_F32) ? (g ? sb1 : sb0) : sb1;
  // the scales of the next two K blocks are in flight while this one is
  // folded in
  float a_n0 = __ldg(sa_row), lo_n0 = __ldg(sb_lo), hi_n0 = __ldg(sb_hi);
  float a_n1 = 0.f, lo_n1 = 0.f, hi_n1 = 0.f;
  if (KB > 1) {
    a_n1 = __ldg(sa_row + 1);
    lo_n1 = __ldg(sb_lo + 1);
    hi_n1 = __ldg(sb_hi + 1);
  }
  for (int kb = 0; kb < KB; ++kb, ++tit) {
    const int p = tit & 1;
    const uint32_t tph = (tit >> 1) & 1;
    const float f_lo = __fmul_rn(a_n0, lo_n0);
    const float f_hi = __fmul_rn(a_n0, hi_n0);
    a_n0 = a_n1;
    lo_n0 = lo_n1;
    hi_n0 = hi_n1;
    if (kb + 2 < KB) {
      a_n1 = __ldg(sa_row + kb + 2);
      lo_n1 = __ldg(sb_lo + kb + 2);
      hi_n1 = __ldg(sb_hi + kb + 2);
    }
    // warp-uniform outcome: the TMEM loads below are warp-collective
    if (!__all_sync(0xffffffffu, mbar_wait(&tfull[p], tph, abort_v, args.dev_err))) return false;
    tc_fence_after();
    const uint32_t ta = tmem + lane_base + static_cast<uint32_t>(p * kBN);
    // two 32-column loads in flight per wait
    float v0[32], v1[32];
    tmem_ld32(ta + c_lo, v0);
    tmem_ld32(ta + c_lo + 32, v1);
    tmem_ld_wait();
    const float2 flo = make_float2(f_lo, f_lo);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      acc[i] = __ffma2_rn(make_float2(v0[2 * i], v0[2 * i + 1]), flo, acc[i]);
      acc[16 + i] = __ffma2_rn(make_float2(v1[2 * i], v1[2 * i + 1]), flo, acc[16 + i]);
    }
    tmem_ld32(ta + c_hi, v0);
    tmem_ld32(ta + c_hi + 32, v1);
    tmem_ld_wait();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&tempty[p]);
    const float2 fhi = make_float2(f_hi, f_hi);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      acc[32 + i] = __ffma2_rn(make_float2(v0[2 * i], v0[2 * i + 1]), fhi, acc[32 + i]);
      acc[48 + i] = __ffma2_rn(make_float2(v1[2 * i], v1[2 * i + 1]), fhi, acc[48 + i]);
    }
  }
  return write_tile<EP, false>(args, t, acc, warp, lane, N, xtile, xbar, amax_x, abort_v);
}

// ------------------------------------------------------- swapped tail tiles
// A tile of at most kTailRows rows wastes most of a 128-row MMA and of the
// promotion.  The swapped path computes its transpose instead: the weight
// tile's two 128-row halves are the MMA's M side and the tail's (up to 32)
// rows its N side (tcgen05 M = 128, N = 32), so each K block costs a quarter
// of the tensor work, and the promotion folds 16 rows x 2 halves per thread:
// TMEM lane = weight row c (32 q + lane of warp quarter q), column = tail row
// m.  Warpgroup g takes rows 16 g .. 16 g + 15.  The factors f = sa * sb of
// every (K block, half, row) are staged once per tile in shared memory, with
// the same single rounding as the 128-row path, so a row's result is the same
// sum of the same products: acc += f * partial per K block, in K order.
struct TailCtl {
  float* f;          // [kTailMaxKB][2][kTailRows]
  float* amax;       // [2 warpgroups][4 quarters][16 rows]
  uint64_t* staged;  // all 256 epilogue threads wrote their share of f
  uint64_t* used;    // all 256 finished the K loop of the tile (f may be rewritten)
  uint64_t* ax;      // [2]: a warpgroup's 4 warps wrote their row amaxes
};

template <int EP>
__device__ __forceinline__ bool epilogue_tail(const GemmArgs& args, const Work& t, uint32_t tmem,
                                              int warp, int lane, int KB, int N, int& tit,
                                              int& ttile, uint64_t* tfull, uint64_t* tempty,
                                              const TailCtl& tc, volatile int* abort_v) {
  const int g = (warp - 4) >> 2;  // rows 16 g .. 16 g + 15 of the tail
  const int q = warp & 3;         // TMEM lane quarter: weight rows 32 q .. 32 q + 31
  const int c = q * 32 + lane;    // this thread's weight row inside a half
  const int tid = threadIdx.x - 128;
  const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
  const uint32_t ph = static_cast<uint32_t>(ttile & 1);
  // the previous tail's K loop is over on every thread before f is rewritten
  if (ttile > 0 &&
      !__all_sync(0xffffffffu, mbar_wait(tc.used, ph ^ 1u, abort_v, args.dev_err)))
    return false;
  {
    const float* sbh = args.sb + (static_cast<int64_t>(t.e) * (N / 128) + t.n_idx * 2) * KB;
    for (int idx = tid; idx < KB * 2 * kTailRows; idx += kEpiThreads) {
      const int kb = idx / (2 * kTailRows), h = (idx / kTailRows) & 1, m = idx % kTailRows;
      float v = 0.f;
      if (m < t.rows)
        v = __fmul_rn(__ldg(args.sa + (static_cast<int64_t>(t.row0) + m) * KB + kb),
                      __ldg(sbh + h * KB + kb));
      tc.f[idx] = v;
    }
  }
  mbar_arrive(tc.staged);
  if (!__all_sync(0xffffffffu, mbar_wait(tc.staged, ph, abort_v, args.dev_err))) return false;
  float acc0[16], acc1[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc0[i] = acc1[i] = 0.f;
  for (int kb = 0; kb < KB; ++kb, ++tit) {
    const int p = tit & 1;
    if (!__all_sync(0xffffffffu, mbar_wait(&tfull[p], (tit >> 1) & 1, abort_v, args.dev_err)))
      return false;
    tc_fence_after();
    const uint32_t ta = tmem + lane_base + static_cast<uint32_t>(p * kBN);
    float v0[16], v1[16];
    tmem_ld16(ta + 16 * g, v0);                  // half 0, rows 16 g ..
    tmem_ld16(ta + kTailRows + 16 * g, v1);      // half 1
    tmem_ld_wait();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&tempty[p]);
    const float4* f0 = reinterpret_cast<const float4*>(tc.f + kb * 2 * kTailRows + 16 * g);
    const float4* f1 = reinterpret_cast<const float4*>(tc.f + kb * 2 * kTailRows + kTailRows + 16 * g);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float4 a = f0[j], b = f1[j];
      acc0[4 * j + 0] = __fmaf_rn(v0[4 * j + 0], a.x, acc0[4 * j + 0]);
      acc0[4 * j + 1] = __fmaf_rn(v0[4 * j + 1], a.y, acc0[4 * j + 1]);
      acc0[4 * j + 2] = __fmaf_rn(v0[4 * j + 2], a.z, acc0[4 * j + 2]);
      acc0[4 * j + 3] = __fmaf_rn(v0[4 * j + 3], a.w, acc0[4 * j + 3]);
      acc1[4 * j + 0] = __fmaf_rn(v1[4 * j + 0], b.x, acc1[4 * j + 0]);
      acc1[4 * j + 1] = __fmaf_rn(v1[4 * j + 1], b.y, acc1[4 * j + 1]);
      acc1[4 * j + 2] = __fmaf_rn(v1[4 * j + 2], b.z, acc1[4 * j + 2]);
      acc1[4 * j + 3] = __fmaf_rn(v1[4 * j + 3], b.w, acc1[4 * j + 3]);
    }
  }
  mbar_arrive(tc.used);
  ++ttile;
  const int m0 = 16 * g;
  if (EP == MOE_EP_F32) {
    // row m of the tail: columns n_idx*256 + c (half 0) and + 128 + c (half 1);
    // each store instruction writes 128 contiguous bytes of one row per warp
    float* D = static_cast<float*>(args.D);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      if (m0 + i >= t.rows) break;
      int64_t row = static_cast<int64_t>(t.row0) + m0 + i;
      if (args.d_rows != nullptr) {
        const int dr = __ldg(args.d_rows + row);
        if (static_cast<uint32_t>(dr) >= static_cast<uint32_t>(args.a_rows)) {
          set_dev_err(args.dev_err, MOE_DEVERR_BAD_TABLE);
          continue;
        }
        row = dr;
      }
      float* out = D + row * N + t.n_idx * kBN + c;
      out[0] = acc0[i];
      out[128] = acc1[i];
    }
  } else {
    // h = SiLU(gate) * up; the row's 1x128 amax runs over the 128 channels c
    // held by the warpgroup's 4 warps: a butterfly over the lanes, then the
    // 4 warp maxima through shared memory
    float hv[16], am[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      hv[i] = silu_mul(acc0[i], acc1[i]);
      float a = fabsf(hv[i]);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
      am[i] = a;
    }
    if (lane < 16) {
      float mine = 0.f;
#pragma unroll
      for (int i = 0; i < 16; ++i)
        if (i == lane) mine = am[i];
      tc.amax[(g * 4 + q) * 16 + lane] = mine;
    }
    mbar_arrive(&tc.ax[g]);
    if (!__all_sync(0xffffffffu, mbar_wait(&tc.ax[g], ph, abort_v, args.dev_err))) return false;
    const int I = N / 2;
    uint8_t* H = static_cast<uint8_t*>(args.D);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float a = fmaxf(fmaxf(tc.amax[(g * 4 + 0) * 16 + i], tc.amax[(g * 4 + 1) * 16 + i]),
                            fmaxf(tc.amax[(g * 4 + 2) * 16 + i], tc.amax[(g * 4 + 3) * 16 + i]));
      const float sq = quant_scale(a);
      const float rq = __frcp_rn(sq);
      if (m0 + i < t.rows) {
        const int64_t row = static_cast<int64_t>(t.row0) + m0 + i;
        H[row * I + t.n_idx * 128 + c] =
            static_cast<uint8_t>(e4m3x2(div_by_scale(hv[i], sq, rq), 0.f) & 0xFFu);
        if (q == 0 && lane == 0) args.d_scale[row * (I / 128) + t.n_idx] = sq;
      }
    }
  }
  return true;
}

// Shared-memory layout after the 1024-aligned ring.
struct Ctl {
  uint64_t* full;
  uint64_t* empty;
  uint64_t* tfull;
  uint64_t* tempty;
  uint64_t* done;
  uint64_t* xbar;
  uint32_t* tmem_slot;
  int* abort_flag;
  int* rstart;
  float* amax_x;  // [2][2][128]
};

template <int STAGES>
__device__ __forceinline__ Ctl carve(uint8_t* base, int ctl_off = kRingBytes) {
  Ctl c;
  c.full = reinterpret_cast<uint64_t*>(base + ctl_off);
  c.empty = c.full + STAGES;
  c.tfull = c.empty + STAGES;
  c.tempty = c.tfull + 2;
  c.done = c.tempty + 2;
  c.xbar = c.done + 1;
  c.tmem_slot = reinterpret_cast<uint32_t*>(c.xbar + 2);
  c.abort_flag = reinterpret_cast<int*>(c.tmem_slot + 1);
  c.rstart = reinterpret_cast<int*>(base + ctl_off + 512);
  c.amax_x = reinterpret_cast<float*>(c.rstart + kMaxGroups + 1);
  return c;
}

// TMA producer (one thread): every K slice of every work item of this CTA,
// A rows and the weight tile into the stage ring; waits for its own copies
// before returning.
template <int STAGES, int SK>
__device__ __forceinline__ void tma_producer(const ATmaps& tmA, const CUtensorMap& tmB,
                                             const GemmArgs& args, const Ctl& c, uint8_t* base,
                                             int total, int nN, int KB, volatile int* abort_v) {
  constexpr int kSub = kBK / SK;
  constexpr int kA = kBM * SK, kStage = kA + kBN * SK;
  const int N = args.N;
  int it = 0;
  bool live = true;
  for (int w = blockIdx.x; w < total && live; w += gridDim.x) {
    const Work t = decode_work<128>(w, nN, c.rstart, args);
    if (!t.ok) {
      set_dev_err(args.dev_err, MOE_DEVERR_BAD_TABLE);
      continue;
    }
    const int brow = t.e * N + t.n_idx * kBN;
    const int ab = a_box(t.rows);
    const uint32_t bytes = static_cast<uint32_t>((ab + 1) * 32 * SK + kBN * SK);
    for (int kk = 0; kk < KB * kSub; ++kk, ++it) {
      const int s = it % STAGES;
      const uint32_t ph = (it / STAGES) & 1;
      if (!mbar_wait(&c.empty[s], ph ^ 1, abort_v, args.dev_err)) {
        live = false;
        break;
      }
      uint8_t* sA = base + s * kStage;
      mbar_arrive_expect_tx(&c.full[s], bytes);
      tma_load_2d(sA, &tmA.box[ab], &c.full[s], kk * SK, t.row0);
      tma_load_2d(sA + kA, &tmB, &c.full[s], kk * SK, brow);
    }
  }
  // every issued copy lands before the CTA can exit
  const int first = it > STAGES ? it - STAGES : 0;
  for (int i = first; i < it; ++i)
    mbar_wait(&c.full[i % STAGES], (i / STAGES) & 1, nullptr, args.dev_err);
}

// =========================================================== 1-SM mainloop
// Work items reach the three roles through a 4-slot queue in shared memory:
// the producer thread takes the next item -- blockIdx.x + i * gridDim.x
// (static), or from the caller's counter with an atomic add (dynamic, so a
// CTA that drew cheap tail tiles takes more work and the grid stays on
// neighbouring items, whose m-tiles share weight tiles in L2) -- publishes it
// and issues its loads; the MMA thread and the epilogue warps read it and
// free the slot when done.  An item >= total ends every role.
struct WorkQueue {
  uint64_t* full;   // [kWQ]
  uint64_t* empty;  // [kWQ], 1 (MMA) + 8 (epilogue warps) arrivals
  int* item;        // [kWQ]
};

template <int EP, int SK>
__global__ void __launch_bounds__(kThreads, 1) gemm1sm_kernel(
    const __grid_constant__ ATmaps tmA, const __grid_constant__ CUtensorMap tmB,
    const GemmArgs args) {
  constexpr int kSub = kBK / SK;                 // stages per K block
  constexpr int kA = kBM * SK, kB = kBN * SK;    // stage bytes of A and B
  constexpr int kStage = kA + kB;
  constexpr int kStages = kRingBytes / kStage;
  constexpr bool kTail = (SK == 128);            // the swapped tail path needs whole K blocks
  static_assert((2 * kStages + 8) * 8 + 8 <= 512, "barrier area");
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const Ctl c = carve<kStages>(base);
  // queue, tail barriers and amax after the amax exchange area, 16-aligned
  uint8_t* qbase = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(c.amax_x + 2 * 2 * 128) + 15) & ~static_cast<uintptr_t>(15));
  WorkQueue wq;
  wq.full = reinterpret_cast<uint64_t*>(qbase);
  wq.empty = wq.full + kWQ;
  TailCtl tc;
  tc.staged = wq.empty + kWQ;
  tc.used = tc.staged + 1;
  tc.ax = tc.used + 1;
  wq.item = reinterpret_cast<int*>(tc.ax + 2);
  tc.amax = reinterpret_cast<float*>(wq.item + kWQ);
  tc.f = reinterpret_cast<float*>(qbase + kTailFactorOffset);  // 16-aligned, after the amax block
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int N = args.N, KB = args.K / kBK, nN = N / kBN;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&c.full[s], 1);
      mbar_init(&c.empty[s], 1);
    }
    for (int p = 0; p < 2; ++p) {
      mbar_init(&c.tfull[p], 1);
      mbar_init(&c.tempty[p], kEpiThreads / 32);
    }
    for (int i = 0; i < kWQ; ++i) {
      mbar_init(&wq.full[i], 1);
      mbar_init(&wq.empty[i], 1 + kEpiThreads / 32);
    }
    mbar_init(tc.staged, kEpiThreads);
    mbar_init(tc.used, kEpiThreads);
    mbar_init(&tc.ax[0], kEpiThreads / 2);
    mbar_init(&tc.ax[1], kEpiThreads / 2);
    mbar_init(c.done, 1);
    mbar_init(&c.xbar[0], kEpiThreads);
    mbar_init(&c.xbar[1], kEpiThreads);
    *c.abort_flag = 0;
    fence_barrier_init();
    for (int b = 0; b < 4; ++b) prefetch_tmap(&tmA.box[b]);
    prefetch_tmap(&tmB);
  }
  if (warp == 2) load_tile_prefix(args, c.rstart, lane);
  if (warp == 1) {
    tmem_alloc(c.tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *c.tmem_slot;
  volatile int* abort_v = c.abort_flag;
  const int total = c.rstart[args.groups] * nN;

  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsCtl));
    if (warp == 0 && lane == 0) {
      // ---------------------------------------------- TMA producer + queue
      int it = 0;
      bool live = true;
      for (int i = 0; live; ++i) {
        const int qs = i % kWQ;
        if (!mbar_wait(&wq.empty[qs], ((i / kWQ) & 1) ^ 1, abort_v, args.dev_err)) break;
        const int w = args.sched ? atomicAdd(args.sched, 1) : blockIdx.x + i * gridDim.x;
        wq.item[qs] = w;
        mbar_arrive(&wq.full[qs]);
        if (w >= total) break;
        const Work t = decode_work<128>(w, nN, c.rstart, args);
        if (!t.ok) {
          set_dev_err(args.dev_err, MOE_DEVERR_BAD_TABLE);
          continue;
        }
        const int brow = t.e * N + t.n_idx * kBN;
        const int ab = a_box(t.rows);
        const uint32_t bytes = static_cast<uint32_t>((ab + 1) * 32 * SK + kB);
        for (int kk = 0; kk < KB * kSub; ++kk, ++it) {
          const int s = it % kStages;
          if (!mbar_wait(&c.empty[s], ((it / kStages) & 1) ^ 1, abort_v, args.dev_err)) {
            live = false;
            break;
          }
          uint8_t* sA = base + s * kStage;
          mbar_arrive_expect_tx(&c.full[s], bytes);
          tma_load_2d(sA, &tmA.box[ab], &c.full[s], kk * SK, t.row0);
          tma_load_2d(sA + kA, &tmB, &c.full[s], kk * SK, brow);
        }
      }
      // every issued copy lands before the CTA can exit
      const int first = it > kStages ? it - kStages : 0;
      for (int i = first; i < it; ++i)
        mbar_wait(&c.full[i % kStages], (i / kStages) & 1, nullptr, args.dev_err);
    } else if (warp == 1 && lane == 0) {
      // ------------------------------------------------------- MMA issuer
      const uint32_t idesc = instr_desc(kFmtE4M3, kFmtE4M3, kBM, kBN);
      // swapped tail: M = the 128 weight rows of one half, N = kTailRows tail rows
      const uint32_t idesc_t = instr_desc(kFmtE4M3, kFmtE4M3, kBM, kTailRows);
      int it = 0, tit = 0;
      bool live = true;
      for (int i = 0; live; ++i) {
        const int qs = i % kWQ;
        if (!mbar_wait(&wq.full[qs], (i / kWQ) & 1, abort_v, args.dev_err)) break;
        const int w = wq.item[qs];
        if (w >= total) {
          mbar_arrive(&wq.empty[qs]);
          break;
        }
        const Work t = decode_work<128>(w, nN, c.rstart, args);
        const bool swp = kTail && t.swp;
        for (int kb = 0; t.ok && kb < KB && live; ++kb, ++tit) {
          const int p = tit & 1;
          if (!mbar_wait(&c.tempty[p], ((tit >> 1) & 1) ^ 1, abort_v, args.dev_err)) {
            live = false;
            break;
          }
          const uint32_t dt = tmem + static_cast<uint32_t>(p * kBN);
          for (int h = 0; h < kSub; ++h, ++it) {
            const int s = it % kStages;
            if (!mbar_wait(&c.full[s], (it / kStages) & 1, abort_v, args.dev_err)) {
              live = false;
              break;
            }
            tc_fence_after();
            const uint32_t sA = smem_u32(base + s * kStage);
            const uint64_t ad = kmajor_desc<SK>(sA);
            const uint64_t bd = kmajor_desc<SK>(sA + kA);
            if (swp) {
              // D_half[c][m] += W_half[c] . X[m]: the weight half is the A
              // operand (128 rows, 16 KB apart), the tail rows the B operand
              const uint64_t wd0 = smem_desc_sw128(sA + kA);
              const uint64_t wd1 = smem_desc_sw128(sA + kA + kBM * SK);
#pragma unroll
              for (int k = 0; k < SK / 32; ++k) {
                mma_f8f6f4(dt, wd0 + 2 * k, ad + 2 * k, idesc_t, k > 0 ? 1u : 0u);
                mma_f8f6f4(dt + kTailRows, wd1 + 2 * k, ad + 2 * k, idesc_t, k > 0 ? 1u : 0u);
              }
            } else {
#pragma unroll
              for (int k = 0; k < SK / 32; ++k)
                mma_f8f6f4(dt, ad + 2 * k, bd + 2 * k, idesc, (h > 0 || k > 0) ? 1u : 0u);
            }
            mma_commit(&c.empty[s]);
          }
          if (live) mma_commit(&c.tfull[p]);
        }
        mbar_arrive(&wq.empty[qs]);
      }
      mma_commit(c.done);
      mbar_wait(c.done, 0, nullptr, args.dev_err);
    }
    __syncwarp();
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsEpi));
    int tit = 0, xtile = 0, ttile = 0;
    for (int i = 0;; ++i) {
      const int qs = i % kWQ;
      if (!__all_sync(0xffffffffu, mbar_wait(&wq.full[qs], (i / kWQ) & 1, abort_v, args.dev_err)))
        break;
      const int w = wq.item[qs];
      bool ok = true;
      if (w < total) {
        const Work t = decode_work<128>(w, nN, c.rstart, args);
        if (t.ok) {
          if (kTail && t.swp)
            ok = epilogue_tail<EP>(args, t, tmem, warp, lane, KB, N, tit, ttile, c.tfull,
                                   c.tempty, tc, abort_v);
          else
            ok = epilogue_tile<EP>(args, t, tmem, warp, lane, KB, N, tit, xtile, c.tfull,
                                   c.tempty, c.xbar, c.amax_x, abort_v);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&wq.empty[qs]);
      if (w >= total || !ok) break;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}


// ================================================ power-of-two scale mainloop
// When every scale is a power of two (UE8M0), the tensor core applies them
// itself: tcgen05.mma kind::mxf8f6f4.block_scale multiplies each 32-element K
// slice of row m of A by 2^SFA[m] and of row n of B by 2^SFB[n] and keeps
// accumulating the whole K extent in TMEM, so no partial sum is promoted and
// no scale touches the epilogue.  A 1x128 (or 128x128) scale covers four
// consecutive 32-element slices, which all read the same exponent.
//
// Per ring stage (one 128-wide K block) the scale-factor warps write three
// 512-byte atoms into shared memory: A's 128 row exponents and B's two 128-row
// blocks.  Atom byte 16 r + 4 j + b holds the exponent of row 32 j + r for the
// K block (4 g + b) of the group g the stage belongs to, so the MMAs of K block
// kb read byte kb % 4.  The MMA thread moves the atoms into TMEM with
// tcgen05.cp (replicated over the four lane quarters) right before the stage's
// MMAs; the tensor core runs a thread's tcgen05 operations in issue order, so
// one TMEM scale region serves every stage.  TMEM: the 256-column accumulator
// at 0, A's exponents at 256..259, B's at 264..271; with one accumulator the
// epilogue releases it as soon as it has loaded the tile into registers.
constexpr int kSfSlot = 1536;       // per stage: A atom + two B atoms
constexpr uint32_t kTmemSfa = 256, kTmemSfb = 264;
constexpr int kStagesMx = kRingBytes / ((kBM + kBN) * kBK);
constexpr size_t kSmemMxBytes = kSmemBytes + kStagesMx * kSfSlot;

// Exponent bytes (UE8M0 = the fp32 biased exponent) of four power-of-two
// scales, byte i from v[i]; anything that is not a positive normal power of
// two sets `bad`.
__device__ __forceinline__ uint32_t ue8m0x4(const float (&v)[4], uint32_t& bad) {
  uint32_t w = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t b = __float_as_uint(v[i]);
    const uint32_t e = b >> 23;  // sign bit included: a negative scale fails below
    bad |= (b & 0x007FFFFFu) | static_cast<uint32_t>(e == 0u || e >= 255u);
    w |= (e & 0xFFu) << (8 * i);
  }
  return w;
}

// The scales of K-block group g (blocks 4g..4g+3) for this lane: A rows
// row0 + lane + 32 j (clamped into the buffer), or the tile's two B blocks.
template <bool IS_A>
__device__ __forceinline__ void sf_load_group(const GemmArgs& a, const Work& t, const float* sb0,
                                              int KB, int g, int lane, float (&v)[4][4]) {
  if (IS_A) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      int64_t r = static_cast<int64_t>(t.row0) + lane + 32 * j;
      r = r < a.a_rows ? r : a.a_rows - 1;
      const float* p = a.sa + r * KB;
#pragma unroll
      for (int i = 0; i < 4; ++i) v[j][i] = (4 * g + i < KB) ? __ldg(p + 4 * g + i) : 1.0f;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const bool in = 4 * g + i < KB;
      v[0][i] = in ? __ldg(sb0 + 4 * g + i) : 1.0f;
      v[1][i] = in ? __ldg(sb0 + KB + 4 * g + i) : 1.0f;
    }
  }
}

// Scale-factor producers (warp 2 for A's atom, warp 3 for B's two atoms):
// per stage, the exponent atoms.  The next group's scales are loaded while
// the current group's four stages are written.
template <int STAGES, bool IS_A>
__device__ __forceinline__ void sf_producer(const GemmArgs& args, const Ctl& c, uint8_t* sf,
                                            int total, int nN, int KB, int lane,
                                            volatile int* abort_v) {
  const int N = args.N;
  int it = 0;
  uint32_t bad = 0;
  bool live = true;
  for (int w = blockIdx.x; w < total && live; w += gridDim.x) {
    const Work t = decode_work<128>(w, nN, c.rstart, args);
    if (!t.ok) continue;
    const float* sb0 = args.sb + (static_cast<int64_t>(t.e) * (N / 128) + t.n_idx * 2) * KB;
    float v[4][4];
    sf_load_group<IS_A>(args, t, sb0, KB, 0, lane, v);
    for (int g = 0; 4 * g < KB && live; ++g) {
      const uint32_t p0 = ue8m0x4(v[0], bad), p1 = ue8m0x4(v[1], bad);
      const uint32_t p2 = IS_A ? ue8m0x4(v[2], bad) : 0u, p3 = IS_A ? ue8m0x4(v[3], bad) : 0u;
      if (4 * (g + 1) < KB) sf_load_group<IS_A>(args, t, sb0, KB, g + 1, lane, v);
      for (int j = 0; j < 4 && 4 * g + j < KB; ++j, ++it) {
        const int s = it % STAGES;
        if (!__all_sync(0xffffffffu, mbar_wait(&c.empty[s], ((it / STAGES) & 1) ^ 1, abort_v,
                                                args.dev_err))) {
          live = false;
          break;
        }
        uint4* slot = reinterpret_cast<uint4*>(sf + s * kSfSlot);
        if (IS_A) {
          slot[lane] = make_uint4(p0, p1, p2, p3);
        } else {
          slot[32 + lane] = make_uint4(p0, p0, p0, p0);
          slot[64 + lane] = make_uint4(p1, p1, p1, p1);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&c.full[s]);
      }
    }
  }
  if (__any_sync(0xffffffffu, bad != 0) && lane == 0) set_dev_err(args.dev_err, MOE_DEVERR_BAD_SCALE);
}

// Epilogue of one tile: load the accumulator into registers, release it to
// the MMA thread, then write the tile.
template <int EP>
__device__ __forceinline__ bool epilogue_mx_tile(const GemmArgs& args, const Work& t, uint32_t tmem,
                                                 int warp, int lane, int N, int& tit, int& xtile,
                                                 uint64_t* tfull, uint64_t* tempty,
                                                 uint64_t* xbar, float* amax_x,
                                                 volatile int* abort_v) {
  const int g = (warp - 4) >> 2;
  const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
  const int c_lo = (EP == MOE_EP_F32) ? 128 * g : 64 * g;
  const int c_hi = (EP == MOE_EP_F32) ? 128 * g + 64 : 128 + 64 * g;
  if (!__all_sync(0xffffffffu, mbar_wait(tfull, tit & 1, abort_v, args.dev_err))) return false;
  ++tit;
  tc_fence_after();
  float2 acc[64];
  {
    const uint32_t ta = tmem + lane_base;
    float v0[32], v1[32], v2[32], v3[32];
    tmem_ld32(ta + c_lo, v0);
    tmem_ld32(ta + c_lo + 32, v1);
    tmem_ld32(ta + c_hi, v2);
    tmem_ld32(ta + c_hi + 32, v3);
    tmem_ld_wait();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(tempty);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      acc[i] = make_float2(v0[2 * i], v0[2 * i + 1]);
      acc[16 + i] = make_float2(v1[2 * i], v1[2 * i + 1]);
      acc[32 + i] = make_float2(v2[2 * i], v2[2 * i + 1]);
      acc[48 + i] = make_float2(v3[2 * i], v3[2 * i + 1]);
    }
  }
  return write_tile<EP, true>(args, t, acc, warp, lane, N, xtile, xbar, amax_x, abort_v);
}

// Warp roles as in gemm1sm_kernel, plus warps 2 and 3 = scale-factor
// producers (A's and B's exponents; warp 2 first stages the tile prefix).
// Stages are whole 128-wide K blocks.
template <int EP>
__global__ void __launch_bounds__(kThreads, 1) gemm_pow2_kernel(
    const __grid_constant__ ATmaps tmA, const __grid_constant__ CUtensorMap tmB,
    const GemmArgs args) {
  constexpr int kA = kBM * kBK, kB = kBN * kBK;
  constexpr int kStage = kA + kB;
  constexpr int kStages = kStagesMx;
  constexpr int kSfBytes = kStages * kSfSlot;
  static_assert((2 * kStages + 8) * 8 + 8 <= 512, "barrier area");
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* sf = base + kRingBytes;
  const Ctl c = carve<kStages>(base, kRingBytes + kSfBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KB = args.K / kBK, nN = args.N / kBN;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&c.full[s], 3);  // TMA bytes + the two scale-factor warps
      mbar_init(&c.empty[s], 1);
    }
    mbar_init(&c.tfull[0], 1);
    mbar_init(&c.tempty[0], kEpiThreads / 32);
    mbar_init(c.done, 1);
    mbar_init(&c.xbar[0], kEpiThreads);
    mbar_init(&c.xbar[1], kEpiThreads);
    *c.abort_flag = 0;
    fence_barrier_init();
    for (int b = 0; b < 4; ++b) prefetch_tmap(&tmA.box[b]);
    prefetch_tmap(&tmB);
  }
  if (warp == 2) load_tile_prefix(args, c.rstart, lane);
  if (warp == 1) {
    tmem_alloc(c.tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *c.tmem_slot;
  volatile int* abort_v = c.abort_flag;
  const int total = c.rstart[args.groups] * nN;

  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsCtl));
    if (warp == 0 && lane == 0) {
      tma_producer<kStages, kBK>(tmA, tmB, args, c, base, total, nN, KB, abort_v);
    } else if (warp == 2) {
      sf_producer<kStages, true>(args, c, sf, total, nN, KB, lane, abort_v);
    } else if (warp == 3) {
      sf_producer<kStages, false>(args, c, sf, total, nN, KB, lane, abort_v);
    } else if (warp == 1 && lane == 0) {
      // ------------------------------------------------------- MMA issuer
      const uint32_t t_sfa = tmem + kTmemSfa, t_sfb = tmem + kTmemSfb;
      const uint32_t sf0 = smem_u32(sf);
      int it = 0, tit = 0;
      bool live = true;
      for (int w = blockIdx.x; w < total && live; w += gridDim.x) {
        const Work t = decode_work<128>(w, nN, c.rstart, args);
        if (!t.ok) continue;
        // the accumulator is free once the epilogue has loaded the last tile
        if (!mbar_wait(&c.tempty[0], (tit & 1) ^ 1, abort_v, args.dev_err)) break;
        tc_fence_after();
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % kStages;
          if (!mbar_wait(&c.full[s], (it / kStages) & 1, abort_v, args.dev_err)) {
            live = false;
            break;
          }
          tc_fence_after();
          const uint32_t sfs = sf0 + s * kSfSlot;
          tmem_cp_32x128b_x4(t_sfa, smem_desc_interleave(sfs, 128));
          tmem_cp_32x128b_x4(t_sfb, smem_desc_interleave(sfs + 512, 128));
          tmem_cp_32x128b_x4(t_sfb + 4, smem_desc_interleave(sfs + 1024, 128));
          const uint32_t sA = smem_u32(base + s * kStage);
          const uint64_t ad = smem_desc_sw128(sA);
          const uint64_t bd = smem_desc_sw128(sA + kA);
          const uint32_t sid = static_cast<uint32_t>(kb & 3);
          const uint32_t idesc = instr_desc_mx(kBM, kBN, sid);
#pragma unroll
          for (int k = 0; k < kBK / 32; ++k)
            mma_mxf8f6f4(tmem, ad + 2 * k, bd + 2 * k, idesc, (kb > 0 || k > 0) ? 1u : 0u,
                         t_sfa | (sid << 30), t_sfb | (sid << 30));
          mma_commit(&c.empty[s]);
        }
        if (!live) break;
        mma_commit(&c.tfull[0]);
        ++tit;
      }
      mma_commit(c.done);
      mbar_wait(c.done, 0, nullptr, args.dev_err);
    }
    __syncwarp();
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsEpi));
    int tit = 0, xtile = 0;
    for (int w = blockIdx.x; w < total; w += gridDim.x) {
      const Work t = decode_work<128>(w, nN, c.rstart, args);
      if (!t.ok) continue;
      if (!epilogue_mx_tile<EP>(args, t, tmem, warp, lane, args.N, tit, xtile, &c.tfull[0],
                                &c.tempty[0], c.xbar, c.amax_x, abort_v))
        break;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}


// ====================================================== Wgrad (K-grouped) GEMM
// dW[g] = At[:, segment g] . Bt[:, segment g]^T for the token-major operands
// of the weight gradients ("Support for Transposed GEMM Operations": 128x1
// tiles, one power-of-two scale per channel row per 128 tokens).  Here the
// groups split K, not M: group g owns the 128-token blocks
// tile_start[g] .. tile_start[g+1] of both operands and a full Ma x Nb
// output.  Both operands carry per-row exponents, which the block-scaled MMA
// takes as they are (B's 256 rows per tile have 256 exponents).  The
// exponents come pre-arranged in 512-byte atoms (channel block cb, token
// blocks 4a..4a+3: byte 16 r + 4 j + b = row 32 j + r, block 4a + b), so the
// producer thread moves them with three bulk copies per stage and no
// scale-factor warps run.  A group without tokens writes a zero gradient.
struct WgradArgs {
  const uint8_t* sfa;
  const uint8_t* sfb;
  const int32_t* tile_start;
  int64_t atoms_per_row;  // ldt / 512
  int groups, Ma, Nb;
  float* D;
  int32_t* dev_err;
};

struct WItem {
  int e, m, n, k0, kb;
};

__device__ __forceinline__ WItem decode_wgrad(int w, const WgradArgs& a) {
  const int mT = a.Ma / kBM, nN = a.Nb / kBN;
  WItem it;
  it.e = w / (mT * nN);
  const int rem = w - it.e * mT * nN;
  it.n = rem / mT;
  it.m = rem - it.n * mT;
  it.k0 = __ldg(a.tile_start + it.e);
  it.kb = __ldg(a.tile_start + it.e + 1) - it.k0;
  if (it.kb < 0) {
    set_dev_err(a.dev_err, MOE_DEVERR_BAD_TABLE);
    it.kb = 0;
  }
  return it;
}

__global__ void __launch_bounds__(kThreads, 1) gemm_wgrad_kernel(
    const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
    const WgradArgs args) {
  constexpr int kA = kBM * kBK, kB = kBN * kBK;
  constexpr int kStage = kA + kB;
  constexpr int kStages = kStagesMx;
  constexpr int kSfBytes = kStages * kSfSlot;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* sf = base + kRingBytes;
  const Ctl c = carve<kStages>(base, kRingBytes + kSfBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int total = args.groups * (args.Ma / kBM) * (args.Nb / kBN);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&c.full[s], 1);
      mbar_init(&c.empty[s], 1);
    }
    mbar_init(&c.tfull[0], 1);
    mbar_init(&c.tempty[0], kEpiThreads / 32);
    mbar_init(c.done, 1);
    mbar_init(&c.xbar[0], kEpiThreads);
    mbar_init(&c.xbar[1], kEpiThreads);
    *c.abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(c.tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *c.tmem_slot;
  volatile int* abort_v = c.abort_flag;

  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsCtl));
    if (warp == 0 && lane == 0) {
      // ------------------------------------------- TMA + exponent atoms
      int it = 0;
      bool live = true;
      for (int w = blockIdx.x; w < total && live; w += gridDim.x) {
        const WItem t = decode_wgrad(w, args);
        for (int kb = 0; kb < t.kb; ++kb, ++it) {
          const int s = it % kStages;
          if (!mbar_wait(&c.empty[s], ((it / kStages) & 1) ^ 1, abort_v, args.dev_err)) {
            live = false;
            break;
          }
          uint8_t* sA = base + s * kStage;
          uint8_t* sfs = sf + s * kSfSlot;
          const int kk = t.k0 + kb;
          const int64_t atom = kk >> 2;
          mbar_arrive_expect_tx(&c.full[s], kStage + 3 * 512);
          tma_load_2d(sA, &tmA, &c.full[s], kk * kBK, t.m * kBM);
          tma_load_2d(sA + kA, &tmB, &c.full[s], kk * kBK, t.n * kBN);
          bulk_load(sfs, args.sfa + (t.m * args.atoms_per_row + atom) * 512, 512, &c.full[s]);
          bulk_load(sfs + 512, args.sfb + ((2 * t.n) * args.atoms_per_row + atom) * 512, 512,
                    &c.full[s]);
          bulk_load(sfs + 1024, args.sfb + ((2 * t.n + 1) * args.atoms_per_row + atom) * 512, 512,
                    &c.full[s]);
        }
      }
      const int first = it > kStages ? it - kStages : 0;
      for (int i = first; i < it; ++i)
        mbar_wait(&c.full[i % kStages], (i / kStages) & 1, nullptr, args.dev_err);
    } else if (warp == 1 && lane == 0) {
      // ------------------------------------------------------- MMA issuer
      const uint32_t t_sfa = tmem + kTmemSfa, t_sfb = tmem + kTmemSfb;
      const uint32_t sf0 = smem_u32(sf);
      int it = 0, tit = 0;
      bool live = true;
      for (int w = blockIdx.x; w < total && live; w += gridDim.x) {
        const WItem t = decode_wgrad(w, args);
        if (t.kb == 0) continue;
        if (!mbar_wait(&c.tempty[0], (tit & 1) ^ 1, abort_v, args.dev_err)) break;
        tc_fence_after();
        for (int kb = 0; kb < t.kb; ++kb, ++it) {
          const int s = it % kStages;
          if (!mbar_wait(&c.full[s], (it / kStages) & 1, abort_v, args.dev_err)) {
            live = false;
            break;
          }
          tc_fence_after();
          const uint32_t sfs = sf0 + s * kSfSlot;
          tmem_cp_32x128b_x4(t_sfa, smem_desc_interleave(sfs, 128));
          tmem_cp_32x128b_x4(t_sfb, smem_desc_interleave(sfs + 512, 128));
          tmem_cp_32x128b_x4(t_sfb + 4, smem_desc_interleave(sfs + 1024, 128));
          const uint32_t sA = smem_u32(base + s * kStage);
          const uint64_t ad = smem_desc_sw128(sA);
          const uint64_t bd = smem_desc_sw128(sA + kA);
          const uint32_t sid = static_cast<uint32_t>((t.k0 + kb) & 3);
          const uint32_t idesc = instr_desc_mx(kBM, kBN, sid);
#pragma unroll
          for (int k = 0; k < kBK / 32; ++k)
            mma_mxf8f6f4(tmem, ad + 2 * k, bd + 2 * k, idesc, (kb > 0 || k > 0) ? 1u : 0u,
                         t_sfa | (sid << 30), t_sfb | (sid << 30));
          mma_commit(&c.empty[s]);
        }
        if (!live) break;
        mma_commit(&c.tfull[0]);
        ++tit;
      }
      mma_commit(c.done);
      mbar_wait(c.done, 0, nullptr, args.dev_err);
    }
    __syncwarp();
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsEpi));
    GemmArgs ga{};
    ga.D = args.D;
    int tit = 0, xtile = 0;
    for (int w = blockIdx.x; w < total; w += gridDim.x) {
      const WItem it = decode_wgrad(w, args);
      Work t;
      t.e = it.e;
      t.n_idx = it.n;
      t.row0 = it.e * args.Ma + it.m * kBM;  // row of dW viewed as [groups * Ma][Nb]
      t.rows = kBM;
      t.ok = true;
      if (it.kb == 0) {
        float2 acc[64];
#pragma unroll
        for (int i = 0; i < 64; ++i) acc[i] = make_float2(0.f, 0.f);
        write_tile<MOE_EP_F32, true>(ga, t, acc, warp, lane, args.Nb, xtile, c.xbar, c.amax_x,
                                     abort_v);
        continue;
      }
      if (!epilogue_mx_tile<MOE_EP_F32>(ga, t, tmem, warp, lane, args.Nb, tit, xtile,
                                        &c.tfull[0], &c.tempty[0], c.xbar, c.amax_x, abort_v))
        break;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

template <int EP>
const void* kernel_ptr() {
  return reinterpret_cast<const void*>(gemm1sm_kernel<EP, MOE_GEMM_SK>);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace moe

namespace {

moe_status gemm_launch(bool pow2, const uint8_t* A, const float* sa, int64_t a_rows,
                       const uint8_t* B, const float* sb, const int32_t* offsets,
                       const int32_t* tile_group, const int32_t* tile_start,
                       const int32_t* n_tiles, int max_tiles, int groups, int N, int K,
                       moe_epilogue ep, void* D, float* d_scale, const int32_t* d_rows,
                       int32_t* sched, int32_t* dev_err, moe_stream_t stream) {
  using namespace moe;
  if (a_rows < 0 || groups <= 0 || N <= 0 || K <= 0 || max_tiles < 0) return MOE_ERR_INVALID_ARG;
  if (K % kBK != 0 || N % kBN != 0) return MOE_ERR_SHAPE;
  if (ep != MOE_EP_F32 && ep != MOE_EP_SWIGLU_QUANT) return MOE_ERR_INVALID_ARG;
  if (d_rows != nullptr && ep != MOE_EP_F32) return MOE_ERR_INVALID_ARG;
  if (a_rows == 0 || max_tiles == 0) return MOE_OK;
  if (!A || !sa || !B || !sb || !offsets || !tile_group || !tile_start || !n_tiles || !D)
    return MOE_ERR_INVALID_ARG;
  if (ep == MOE_EP_SWIGLU_QUANT && !d_scale) return MOE_ERR_INVALID_ARG;
  if (!aligned16(A) || !aligned16(B) || !aligned16(D)) return MOE_ERR_ALIGN;
  if (a_rows > 0x7FFFFFFF || static_cast<int64_t>(groups) * N > 0x7FFFFFFF)
    return MOE_ERR_UNSUPPORTED;
  if (groups > kMaxGroups) return MOE_ERR_UNSUPPORTED;
  // the block-scaled mainloop stages whole 128-byte K blocks
  const int SK = pow2 ? kBK : MOE_GEMM_SK;
  // A: 128-row boxes; B: the 256 weight rows of a tile; boxes are SK bytes
  // wide with an SK-byte swizzle
  ATmaps tmA;
  CUtensorMap tmB;
  for (int b = 0; b < 4; ++b)
    if (!moe_make_tmap_2d(&tmA.box[b], A, CU_TENSOR_MAP_DATA_TYPE_UINT8, K, a_rows, K, SK,
                          32 * (b + 1), SK))
      return MOE_ERR_CUDA;
  if (!moe_make_tmap_2d(&tmB, B, CU_TENSOR_MAP_DATA_TYPE_UINT8, K,
                        static_cast<uint64_t>(groups) * N, K, SK, kBN, SK))
    return MOE_ERR_CUDA;
  GemmArgs a;
  a.sa = sa;
  a.a_rows = a_rows;
  a.sb = sb;
  a.offsets = offsets;
  a.tile_group = tile_group;
  a.tile_start = tile_start;
  a.n_tiles = n_tiles;
  a.max_tiles = max_tiles;
  a.groups = groups;
  a.N = N;
  a.K = K;
  a.D = D;
  a.d_scale = d_scale;
  a.dev_err = dev_err;
  a.d_rows = d_rows;
  a.sched = pow2 ? nullptr : sched;
  static int configured = 0;
  if (!configured) {
    const void* fs[4] = {kernel_ptr<MOE_EP_F32>(), kernel_ptr<MOE_EP_SWIGLU_QUANT>(),
                         reinterpret_cast<const void*>(gemm_pow2_kernel<MOE_EP_F32>),
                         reinterpret_cast<const void*>(gemm_pow2_kernel<MOE_EP_SWIGLU_QUANT>)};
    for (int i = 0; i < 4; ++i) {
      const int bytes = static_cast<int>(i < 2 ? kSmemPromoteBytes : kSmemMxBytes);
      if (cudaFuncSetAttribute(fs[i], cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
          cudaSuccess)
        return MOE_ERR_CUDA;
    }
    configured = 1;
  }
  // persistent: one CTA per SM, no more CTAs than work items
  const int64_t work_max = static_cast<int64_t>(max_tiles) * (N / kBN);
  const int ctas = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(moe_num_sms(), work_max)));
  const void* fn;
  if (pow2)
    fn = ep == MOE_EP_F32 ? reinterpret_cast<const void*>(gemm_pow2_kernel<MOE_EP_F32>)
                          : reinterpret_cast<const void*>(gemm_pow2_kernel<MOE_EP_SWIGLU_QUANT>);
  else
    fn = ep == MOE_EP_F32 ? kernel_ptr<MOE_EP_F32>() : kernel_ptr<MOE_EP_SWIGLU_QUANT>();
  if (a.sched != nullptr &&
      cudaMemsetAsync(a.sched, 0, sizeof(int32_t), static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return MOE_ERR_CUDA;
  void* kargs[3] = {&tmA, &tmB, &a};
  if (cudaLaunchKernel(fn, dim3(ctas), dim3(kThreads), kargs,
                       pow2 ? kSmemMxBytes : kSmemPromoteBytes,
                       static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

}  // namespace

extern "C" moe_status grouped_gemm_fp8_blockscaled(
    const uint8_t* A, const float* sa, int64_t a_rows, const uint8_t* B, const float* sb,
    const int32_t* offsets, const int32_t* tile_group, const int32_t* tile_start,
    const int32_t* n_tiles, int max_tiles, int groups, int N, int K, moe_epilogue ep, void* D,
    float* d_scale, const int32_t* d_rows, int32_t* sched, int32_t* dev_err,
    moe_stream_t stream) {
  return gemm_launch(false, A, sa, a_rows, B, sb, offsets, tile_group, tile_start, n_tiles,
                     max_tiles, groups, N, K, ep, D, d_scale, d_rows, sched, dev_err, stream);
}

extern "C" moe_status grouped_gemm_fp8_pow2(
    const uint8_t* A, const float* sa, int64_t a_rows, const uint8_t* B, const float* sb,
    const int32_t* offsets, const int32_t* tile_group, const int32_t* tile_start,
    const int32_t* n_tiles, int max_tiles, int groups, int N, int K, moe_epilogue ep, void* D,
    float* d_scale, const int32_t* d_rows, int32_t* sched, int32_t* dev_err,
    moe_stream_t stream) {
  return gemm_launch(true, A, sa, a_rows, B, sb, offsets, tile_group, tile_start, n_tiles,
                     max_tiles, groups, N, K, ep, D, d_scale, d_rows, sched, dev_err, stream);
}

extern "C" moe_status grouped_gemm_fp8_wgrad(const uint8_t* At, const uint8_t* sfa_atoms,
                                             const uint8_t* Bt, const uint8_t* sfb_atoms,
                                             int64_t ldt, int Ma, int Nb,
                                             const int32_t* tile_start, int groups, float* dW,
                                             int32_t* dev_err, moe_stream_t stream) {
  using namespace moe;
  if (ldt < 0 || Ma < 0 || Nb < 0 || groups < 0) return MOE_ERR_INVALID_ARG;
  if (Ma % kBM != 0 || Nb % kBN != 0 || ldt % 512 != 0) return MOE_ERR_SHAPE;
  if (groups == 0 || Ma == 0 || Nb == 0) return MOE_OK;
  if (!At || !sfa_atoms || !Bt || !sfb_atoms || !tile_start || !dW) return MOE_ERR_INVALID_ARG;
  if (ldt == 0) return MOE_ERR_SHAPE;
  if (!aligned16(At) || !aligned16(Bt) || !aligned16(sfa_atoms) || !aligned16(sfb_atoms) ||
      !aligned16(dW))
    return MOE_ERR_ALIGN;
  if (static_cast<int64_t>(groups) * Ma > 0x7FFFFFFF || ldt / kBK > 0x7FFFFFFF / kBK)
    return MOE_ERR_UNSUPPORTED;
  const int64_t items = static_cast<int64_t>(groups) * (Ma / kBM) * (Nb / kBN);
  if (items > 0x7FFFFFFF) return MOE_ERR_UNSUPPORTED;
  CUtensorMap tmA, tmB;
  if (!moe_make_tmap_2d(&tmA, At, CU_TENSOR_MAP_DATA_TYPE_UINT8, ldt, Ma, ldt, kBK, kBM, kBK) ||
      !moe_make_tmap_2d(&tmB, Bt, CU_TENSOR_MAP_DATA_TYPE_UINT8, ldt, Nb, ldt, kBK, kBN, kBK))
    return MOE_ERR_CUDA;
  WgradArgs a;
  a.sfa = sfa_atoms;
  a.sfb = sfb_atoms;
  a.tile_start = tile_start;
  a.atoms_per_row = ldt / 512;
  a.groups = groups;
  a.Ma = Ma;
  a.Nb = Nb;
  a.D = dW;
  a.dev_err = dev_err;
  static int configured = 0;
  if (!configured) {
    if (cudaFuncSetAttribute(reinterpret_cast<const void*>(gemm_wgrad_kernel),
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmemMxBytes)) != cudaSuccess)
      return MOE_ERR_CUDA;
    configured = 1;
  }
  const int ctas = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(moe_num_sms(), items)));
  void* kargs[3] = {&tmA, &tmB, &a};
  if (cudaLaunchKernel(reinterpret_cast<const void*>(gemm_wgrad_kernel), dim3(ctas), dim3(kThreads),
                       kargs, kSmemMxBytes, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}
