// Block-scaled FP8 grouped GEMM for sm_100a (tcgen05 + TMEM + TMA).
//
// "DeepSeek_V3_Report：Annotation", "Fine-Grained Quantization" and
// "Increasing Accumulation Precision": activations carry one fp32 scale per
// 1x128 tile, weights one per 128x128 block, so the scales change along the
// inner dimension K every 128 elements; the pages promote the tensor core's
// partial sums to fp32 registers every N_C = 128 elements and apply the
// scales there.  On Blackwell the same contract maps onto:
//
//   * one 128x256x128 block product per K-block = 4 tcgen05.mma (K=32 each)
//     from a TMA-fed, 128-byte-swizzled shared-memory ring into a fresh TMEM
//     accumulator (two 256-column buffers, ping-pong);
//   * two epilogue warpgroups drain each finished buffer with tcgen05.ld and
//     fold it into fp32 register accumulators: acc += (sa[row,kb] *
//     sb[nblk,kb]) * partial, while the tensor core fills the other buffer;
//   * a persistent grid (one CTA per SM) walks the (expert, n-tile, m-tile)
//     work list derived on the device from the segment tile table, so the
//     ragged expert segments need no host synchronisation; the m-tiles of one
//     expert that share a weight tile run next to each other for L2 reuse.
//
// Warp roles (384 threads): warp 0 = TMA producer, warp 1 = MMA issuer and
// TMEM owner, warps 2-3 idle (the first warpgroup gives its registers to the
// other two), warps 4..11 = epilogue (warp w reads TMEM lanes 32*(w%4)..).
// Epilogues: fp32 rows, or SwiGLU + 1x128 E4M3 requantisation of h (the W1
// rows are gate/up block-interleaved so one 256-wide tile holds 128 gate and
// the matching 128 up channels).
#include <algorithm>

#include "epi_math.cuh"
#include "moe_common.cuh"

namespace moe {
namespace {

constexpr int kBM = 128, kBN = 256, kBK = 128;
constexpr int kStages = 4;
constexpr int kABytes = kBM * kBK;
constexpr int kBBytes = kBN * kBK;
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kThreads = 384;       // 3 warpgroups
constexpr int kEpiThreads = 256;    // warpgroups 1 and 2
// Register split (setmaxnreg), checked against the launch budget of
// 384 threads x 168 registers = 64512: 128 x 56 + 256 x 224 = 64512.
constexpr int kRegsCtl = 56;
constexpr int kRegsEpi = 224;
constexpr uint32_t kTmemCols = 512;
constexpr size_t kSmemBytes = 1024 + static_cast<size_t>(kStages) * kStageBytes + 4096;

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
};

struct Work {
  int e, n_idx, row0, rows;
  bool ok;
};

// Work item w -> (expert, n-tile, m-tile).  The items of expert e occupy
// [nN*tile_start[e], nN*tile_start[e+1]); inside, the m-tile varies fastest.
__device__ __forceinline__ Work decode_work(int w, int nN, const GemmArgs& a) {
  Work t{0, 0, 0, 0, false};
  const int j = w / nN;
  const int e = __ldg(a.tile_group + j);
  if (e < 0 || e >= a.groups) return t;
  const int ms = __ldg(a.tile_start + e);
  const int mc = __ldg(a.tile_start + e + 1) - ms;
  if (mc <= 0 || j < ms || j >= ms + mc) return t;
  const int local = w - nN * ms;
  t.n_idx = local / mc;
  const int m_loc = local - t.n_idx * mc;
  const int r0 = __ldg(a.offsets + e) + kBM * m_loc;
  const int r1 = __ldg(a.offsets + e + 1);
  t.rows = min(kBM, r1 - r0);
  if (t.rows <= 0 || r0 < 0 || r1 > a.a_rows || t.n_idx >= nN) return t;
  t.e = e;
  t.row0 = r0;
  t.ok = true;
  return t;
}

template <int EP>
__global__ void __launch_bounds__(kThreads, 1) grouped_gemm_kernel(
    const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
    const GemmArgs args) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(base + kStages * kStageBytes);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* done = tempty + 2;
  uint64_t* xbar = done + 1;  // [2] amax exchange between the two epilogue halves
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(xbar + 2);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  float* amax_x = reinterpret_cast<float*>(base + kStages * kStageBytes + 256);  // [2][2][128]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int N = args.N, KB = args.K / kBK, nN = N / kBN;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int p = 0; p < 2; ++p) {
      mbar_init(&tfull[p], 1);
      mbar_init(&tempty[p], kEpiThreads / 32);
    }
    mbar_init(done, 1);
    mbar_init(&xbar[0], kEpiThreads);
    mbar_init(&xbar[1], kEpiThreads);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  volatile int* abort_v = abort_flag;

  int n_mt = __ldg(args.n_tiles);
  if (n_mt < 0 || n_mt > args.max_tiles) {
    if (threadIdx.x == 0) set_dev_err(args.dev_err, MOE_DEVERR_BAD_TABLE);
    n_mt = 0;
  }
  const int total = n_mt * nN;

  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsCtl));
    if (warp == 0 && lane == 0) {
      // ------------------------------------------------------ TMA producer
      int it = 0;
      bool live = true;
      for (int w = blockIdx.x; w < total && live; w += gridDim.x) {
        const Work t = decode_work(w, nN, args);
        if (!t.ok) {
          set_dev_err(args.dev_err, MOE_DEVERR_BAD_TABLE);
          continue;
        }
        const int brow = t.e * N + t.n_idx * kBN;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (it / kStages) & 1;
          if (!mbar_wait(&empty[s], ph ^ 1, abort_v, args.dev_err)) {
            live = false;
            break;
          }
          uint8_t* sA = base + s * kStageBytes;
          mbar_arrive_expect_tx(&full[s], kStageBytes);
          tma_load_2d(sA, &tmA, &full[s], kb * kBK, t.row0);
          tma_load_2d(sA + kABytes, &tmB, &full[s], kb * kBK, brow);
        }
      }
      // every issued copy lands before the CTA can exit
      const int first = it > kStages ? it - kStages : 0;
      for (int i = first; i < it; ++i)
        mbar_wait(&full[i % kStages], (i / kStages) & 1, nullptr, args.dev_err);
    } else if (warp == 1 && lane == 0) {
      // ------------------------------------------------------- MMA issuer
      const uint32_t idesc = instr_desc(kFmtE4M3, kFmtE4M3, kBM, kBN);
      int it = 0, tit = 0;
      bool live = true;
      for (int w = blockIdx.x; w < total && live; w += gridDim.x) {
        const Work t = decode_work(w, nN, args);
        if (!t.ok) continue;
        for (int kb = 0; kb < KB; ++kb, ++it, ++tit) {
          const int s = it % kStages;
          const uint32_t ph = (it / kStages) & 1;
          const int p = tit & 1;
          const uint32_t tph = (tit >> 1) & 1;
          if (!mbar_wait(&tempty[p], tph ^ 1, abort_v, args.dev_err) ||
              !mbar_wait(&full[s], ph, abort_v, args.dev_err)) {
            live = false;
            break;
          }
          tc_fence_after();
          const uint32_t sA = smem_u32(base + s * kStageBytes);
          const uint64_t ad = smem_desc_sw128(sA);
          const uint64_t bd = smem_desc_sw128(sA + kABytes);
          const uint32_t dt = tmem + static_cast<uint32_t>(p * kBN);
#pragma unroll
          for (int k = 0; k < kBK / 32; ++k) mma_f8f6f4(dt, ad + 2 * k, bd + 2 * k, idesc, k > 0);
          mma_commit(&empty[s]);
          mma_commit(&tfull[p]);
        }
      }
      mma_commit(done);
      mbar_wait(done, 0, nullptr, args.dev_err);
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsEpi));
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 4;
    const int g = ew >> 2;          // which half of the columns
    const int q = warp & 3;         // TMEM lane quarter this warp may read
    const int r_in = q * 32 + lane; // row inside the tile
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    // columns of the 256-wide tile this thread accumulates (two runs of 64)
    const int c_lo = (EP == MOE_EP_F32) ? 128 * g : 64 * g;
    const int c_hi = (EP == MOE_EP_F32) ? 128 * g + 64 : 128 + 64 * g;
    int tit = 0, xtile = 0;
    bool live = true;
    for (int w = blockIdx.x; w < total && live; w += gridDim.x) {
      const Work t = decode_work(w, nN, args);
      if (!t.ok) continue;
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
      // folded in (their global-load latency would otherwise stall every block)
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
        if (!__all_sync(0xffffffffu, mbar_wait(&tfull[p], tph, abort_v, args.dev_err))) {
          live = false;
          break;
        }
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
      if (!live) break;
      const bool row_ok = r_in < t.rows;
      if (EP == MOE_EP_F32) {
        if (row_ok) {
          float* dst = static_cast<float*>(args.D) + arow * N + t.n_idx * kBN + 128 * g;
#pragma unroll
          for (int i = 0; i < 32; ++i)
            reinterpret_cast<float4*>(dst)[i] =
                make_float4(acc[2 * i].x, acc[2 * i].y, acc[2 * i + 1].x, acc[2 * i + 1].y);
        }
      } else {
        // h = SiLU(gate) * up for this thread's 64 channels, then the 1x128
        // tile amax is shared with the partner thread of the other half.
        // gate channels are acc[0..31] (packed pairs), the matching up channels acc[32..63]
        float h[64];
        float amax = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          h[2 * i] = silu_mul(acc[i].x, acc[32 + i].x);
          h[2 * i + 1] = silu_mul(acc[i].y, acc[32 + i].y);
          amax = fmaxf(amax, fmaxf(fabsf(h[2 * i]), fabsf(h[2 * i + 1])));
        }
        const int xb = xtile & 1;
        amax_x[(xb * 2 + g) * 128 + r_in] = amax;
        mbar_arrive(&xbar[xb]);
        if (!__all_sync(0xffffffffu, mbar_wait(&xbar[xb], (xtile >> 1) & 1, abort_v, args.dev_err)))
          break;
        amax = fmaxf(amax_x[(xb * 2 + 0) * 128 + r_in], amax_x[(xb * 2 + 1) * 128 + r_in]);
        ++xtile;
        const float s = quant_scale(amax);
        if (row_ok) {
          const int I = N / 2;
          uint8_t* dst = static_cast<uint8_t*>(args.D) + arow * I + t.n_idx * 128 + 64 * g;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint4 o;
            o.x = e4m3x4(__fdiv_rn(h[16 * i + 0], s), __fdiv_rn(h[16 * i + 1], s),
                         __fdiv_rn(h[16 * i + 2], s), __fdiv_rn(h[16 * i + 3], s));
            o.y = e4m3x4(__fdiv_rn(h[16 * i + 4], s), __fdiv_rn(h[16 * i + 5], s),
                         __fdiv_rn(h[16 * i + 6], s), __fdiv_rn(h[16 * i + 7], s));
            o.z = e4m3x4(__fdiv_rn(h[16 * i + 8], s), __fdiv_rn(h[16 * i + 9], s),
                         __fdiv_rn(h[16 * i + 10], s), __fdiv_rn(h[16 * i + 11], s));
            o.w = e4m3x4(__fdiv_rn(h[16 * i + 12], s), __fdiv_rn(h[16 * i + 13], s),
                         __fdiv_rn(h[16 * i + 14], s), __fdiv_rn(h[16 * i + 15], s));
            reinterpret_cast<uint4*>(dst)[i] = o;
          }
          if (g == 0) args.d_scale[arow * (I / 128) + t.n_idx] = s;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace moe

extern "C" moe_status grouped_gemm_fp8_blockscaled(
    const uint8_t* A, const float* sa, int64_t a_rows, const uint8_t* B, const float* sb,
    const int32_t* offsets, const int32_t* tile_group, const int32_t* tile_start,
    const int32_t* n_tiles, int max_tiles, int groups, int N, int K, moe_epilogue ep, void* D,
    float* d_scale, int32_t* dev_err, moe_stream_t stream) {
  using namespace moe;
  if (a_rows < 0 || groups <= 0 || N <= 0 || K <= 0 || max_tiles < 0) return MOE_ERR_INVALID_ARG;
  if (K % kBK != 0 || N % kBN != 0) return MOE_ERR_SHAPE;
  if (ep != MOE_EP_F32 && ep != MOE_EP_SWIGLU_QUANT) return MOE_ERR_INVALID_ARG;
  if (a_rows == 0 || max_tiles == 0) return MOE_OK;
  if (!A || !sa || !B || !sb || !offsets || !tile_group || !tile_start || !n_tiles || !D)
    return MOE_ERR_INVALID_ARG;
  if (ep == MOE_EP_SWIGLU_QUANT && !d_scale) return MOE_ERR_INVALID_ARG;
  if (!aligned16(A) || !aligned16(B) || !aligned16(D)) return MOE_ERR_ALIGN;
  if (a_rows > 0x7FFFFFFF || static_cast<int64_t>(groups) * N > 0x7FFFFFFF)
    return MOE_ERR_UNSUPPORTED;
  CUtensorMap tmA, tmB;
  if (!moe_make_tmap_2d(&tmA, A, CU_TENSOR_MAP_DATA_TYPE_UINT8, K, a_rows, K, kBK, kBM) ||
      !moe_make_tmap_2d(&tmB, B, CU_TENSOR_MAP_DATA_TYPE_UINT8, K,
                        static_cast<uint64_t>(groups) * N, K, kBK, kBN))
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
  static int configured = 0;
  if (!configured) {
    if (cudaFuncSetAttribute(grouped_gemm_kernel<MOE_EP_F32>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmemBytes)) != cudaSuccess ||
        cudaFuncSetAttribute(grouped_gemm_kernel<MOE_EP_SWIGLU_QUANT>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmemBytes)) != cudaSuccess)
      return MOE_ERR_CUDA;
    configured = 1;
  }
  const int64_t work_max = static_cast<int64_t>(max_tiles) * (N / kBN);
  const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(moe_num_sms(), work_max)));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (ep == MOE_EP_F32)
    grouped_gemm_kernel<MOE_EP_F32><<<grid, kThreads, kSmemBytes, st>>>(tmA, tmB, a);
  else
    grouped_gemm_kernel<MOE_EP_SWIGLU_QUANT><<<grid, kThreads, kSmemBytes, st>>>(tmA, tmB, a);
  MOE_CUDA_CHECK_LAUNCH();
  return MOE_OK;
}
