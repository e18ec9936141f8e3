// Backward of the expert FFNs: the element-wise and layout kernels around
// the FP8 Dgrad and Wgrad GEMMs.
// "DeepSeek_V3_Report：Annotation", "Mixed Precision Framework" (Fprop,
// Dgrad and Wgrad GEMMs take FP8 inputs), "Low-Precision Activation" (the
// SwiGLU input is cached in FP8 and its output recomputed), "Low-Precision
// Communication" (the gradient before the down projection is quantised with
// power-of-two scales) and "Support for Transposed GEMM Operations" (an
// operand reduced over tokens is re-quantised in 128x1 tiles).
//
//   fp8_quant_1x128_f32     1x128 quantisation of fp32 rows (the SwiGLU input cache)
//   moe_combine_backward    dy = gate * dout per routed row, dout per shared row, 1x128 FP8
//   swiglu_backward         dgu from dh and the cached gu, 1x128 FP8; recomputed h
//   fp8_quant_128x1_pow2    token-major 128x1 re-quantisation per expert segment
//   fp8_transpose_128x128   FP8 weights transposed (each block keeps its scale)
//   moe_unpermute_add       du = dout + the token's expert rows of dx
//
// All are HBM-bound streaming kernels; every sum runs in a fixed order.
#include <cuda_fp8.h>

#include "epi_math.cuh"
#include "moe_common.cuh"

namespace moe {
namespace {

constexpr int kMaxKb = 32;

// Four E4M3 bytes (byte i -> f[i]) through two paired conversions (exact:
// every E4M3 value is a half value).
__device__ __forceinline__ void e4m3x4_to_float(uint32_t w, float (&f)[4]) {
  const __half2_raw lo = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w & 0xFFFFu), __NV_E4M3);
  const __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w >> 16), __NV_E4M3);
  const float2 a = __half22float2(__half2(lo));
  const float2 b = __half22float2(__half2(hi));
  f[0] = a.x;
  f[1] = a.y;
  f[2] = b.x;
  f[3] = b.y;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
  return v;
}

template <bool POW2>
__device__ __forceinline__ float tile_scale_of(float amax) {
  return POW2 ? pow2_ceil(quant_scale(amax)) : quant_scale(amax);
}

// One 1x128 tile held as 4 values per lane -> 4 E4M3 bytes per lane; returns the scale.
template <bool POW2>
__device__ __forceinline__ float quant_tile(const float (&v)[4], uint32_t& codes) {
  const float amax = warp_max(fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3]))));
  const float s = tile_scale_of<POW2>(amax);
  const float rs = __frcp_rn(s);
  codes = e4m3x4(div_by_scale(v[0], s, rs), div_by_scale(v[1], s, rs), div_by_scale(v[2], s, rs),
                 div_by_scale(v[3], s, rs));
  return s;
}

// ------------------------------------------------ fp32 rows, 1x128 tiles --
// One warp per tile.
template <bool POW2>
__global__ void __launch_bounds__(256) quant_f32_kernel(const float* __restrict__ x, int64_t ldx,
                                                        int rows, int tpr, uint8_t* __restrict__ q,
                                                        float* __restrict__ scale) {
  const int lane = threadIdx.x & 31;
  const int64_t tile = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (tile >= static_cast<int64_t>(rows) * tpr) return;
  const int64_t r = tile / tpr;
  const int j = static_cast<int>(tile - r * tpr);
  const float4 a = __ldg(reinterpret_cast<const float4*>(x + r * ldx + j * 128) + lane);
  const float v[4] = {a.x, a.y, a.z, a.w};
  uint32_t codes;
  const float s = quant_tile<POW2>(v, codes);
  reinterpret_cast<uint32_t*>(q + r * (static_cast<int64_t>(tpr) * 128) + j * 128)[lane] = codes;
  if (lane == 0) scale[tile] = s;
}

// --------------------------------------------------------- combine backward --
// One CTA per token, one warp per 128-column tile at a time: the token's
// dout tile is read once and gives its K routed rows (gate * dout, one fp32
// product) and its shared row (dout), each quantised 1x128 with a
// power-of-two scale.
__global__ void __launch_bounds__(256) combine_backward_kernel(
    const float* __restrict__ dout, const int32_t* __restrict__ dst_of,
    const float* __restrict__ gate, int T, int K, int d, uint8_t* __restrict__ dyq,
    float* __restrict__ dys, float* __restrict__ dy) {
  __shared__ int64_t rows[kMaxKb + 1];
  __shared__ float gs[kMaxKb + 1];
  const int64_t t = blockIdx.x;
  const int64_t P = static_cast<int64_t>(T) * K;
  if (threadIdx.x <= K) {
    if (threadIdx.x < K) {
      const int32_t r = dst_of[t * K + threadIdx.x];
      rows[threadIdx.x] = r;
      gs[threadIdx.x] = gate[t * K + threadIdx.x];
    } else {
      rows[K] = P + t;
      gs[K] = 1.0f;
    }
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int tiles = d / 128;
  for (int j = warp; j < tiles; j += 8) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(dout + t * d + j * 128) + lane);
    for (int k = 0; k <= K; ++k) {
      const int64_t row = rows[k];
      if (row < 0) continue;
      const float g = gs[k];
      const float v[4] = {__fmul_rn(g, a.x), __fmul_rn(g, a.y), __fmul_rn(g, a.z),
                          __fmul_rn(g, a.w)};
      uint32_t codes;
      const float s = quant_tile<true>(v, codes);
      reinterpret_cast<uint32_t*>(dyq + row * d + j * 128)[lane] = codes;
      if (lane == 0) dys[row * tiles + j] = s;
      if (dy)
        reinterpret_cast<float4*>(dy + row * d + j * 128)[lane] = make_float4(v[0], v[1], v[2], v[3]);
    }
  }
}

// ---------------------------------------------------------- SwiGLU backward --
// One warp per (row, 128-channel block j): lane l takes channels 4l..4l+3 of
// the gate block (columns 256j..) and of the up block (256j+128..) of the
// cached FP8 gu.  sigma = 1/(1+e^-g), SiLU = g sigma, SiLU' = sigma (1 + g
// (1 - sigma)); dg = dh u SiLU'(g), du = dh SiLU(g), h = SiLU(g) u.
__global__ void __launch_bounds__(256) swiglu_backward_kernel(
    const float* __restrict__ dh, const uint8_t* __restrict__ guq, const float* __restrict__ gus,
    int rows, int I, uint8_t* __restrict__ dguq, float* __restrict__ dgus, float* __restrict__ dgu,
    float* __restrict__ h) {
  const int lane = threadIdx.x & 31;
  const int tpr = I / 128;
  const int64_t item = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (item >= static_cast<int64_t>(rows) * tpr) return;
  const int64_t r = item / tpr;
  const int j = static_cast<int>(item - r * tpr);
  const int64_t two_i = 2 * static_cast<int64_t>(I);
  const uint32_t gc = __ldg(reinterpret_cast<const uint32_t*>(guq + r * two_i + 256 * j) + lane);
  const uint32_t uc = __ldg(reinterpret_cast<const uint32_t*>(guq + r * two_i + 256 * j + 128) + lane);
  const float sg = __ldg(gus + r * (2 * tpr) + 2 * j);
  const float su = __ldg(gus + r * (2 * tpr) + 2 * j + 1);
  const float4 dv = __ldg(reinterpret_cast<const float4*>(dh + r * I + 128 * j) + lane);
  const float dhv[4] = {dv.x, dv.y, dv.z, dv.w};
  float dg[4], du[4], hv[4];
  float gf[4], uf[4];
  e4m3x4_to_float(gc, gf);
  e4m3x4_to_float(uc, uf);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float g = __fmul_rn(gf[i], sg);
    const float u = __fmul_rn(uf[i], su);
    const float sig = __fdiv_rn(1.0f, __fadd_rn(1.0f, expf(-g)));
    const float silu = __fmul_rn(g, sig);
    const float dsilu = __fmul_rn(sig, __fadd_rn(1.0f, __fmul_rn(g, __fsub_rn(1.0f, sig))));
    dg[i] = __fmul_rn(__fmul_rn(dhv[i], u), dsilu);
    du[i] = __fmul_rn(dhv[i], silu);
    hv[i] = __fmul_rn(silu, u);
  }
  uint32_t cg, cu;
  const float s_g = quant_tile<true>(dg, cg);
  const float s_u = quant_tile<true>(du, cu);
  reinterpret_cast<uint32_t*>(dguq + r * two_i + 256 * j)[lane] = cg;
  reinterpret_cast<uint32_t*>(dguq + r * two_i + 256 * j + 128)[lane] = cu;
  if (lane == 0) {
    dgus[r * (2 * tpr) + 2 * j] = s_g;
    dgus[r * (2 * tpr) + 2 * j + 1] = s_u;
  }
  if (dgu) {
    reinterpret_cast<float4*>(dgu + r * two_i + 256 * j)[lane] = make_float4(dg[0], dg[1], dg[2], dg[3]);
    reinterpret_cast<float4*>(dgu + r * two_i + 256 * j + 128)[lane] =
        make_float4(du[0], du[1], du[2], du[3]);
  }
  if (h) reinterpret_cast<float4*>(h + r * I + 128 * j)[lane] = make_float4(hv[0], hv[1], hv[2], hv[3]);
}

// ------------------------------------------------- 128x1 re-quantisation --
// CTA (tile i, channel block cb): the segment's 128-token tile i (rows
// offsets[g] + 128 (i - tile_start[g]) .., zero past the segment's end) of
// channels 128 cb .. 128 cb + 127.  Warp w loads rows 16w .. 16w + 15 (lane l:
// channels 4l .. 4l + 3, one coalesced 512-byte row per load), so a thread
// holds 16 consecutive tokens of its 4 channels.  A channel's 128-token amax
// (shared-memory reduction over the 8 warps) gives its power-of-two scale;
// each thread then writes its 16 codes per channel as one 16-byte store into
// the channel's row of qt.  FP8 sources (x) are dequantised first with their
// 1x128 scale.
template <bool FP8_SRC>
__global__ void __launch_bounds__(256) quant_128x1_kernel(
    const float* __restrict__ src, const uint8_t* __restrict__ src_q,
    const float* __restrict__ src_s, int64_t ld_src, const int32_t* __restrict__ offsets,
    const int32_t* __restrict__ tile_group, const int32_t* __restrict__ tile_start,
    const int32_t* __restrict__ n_tiles, int C, uint8_t* __restrict__ qt, int64_t ldt,
    float* __restrict__ st, uint8_t* __restrict__ atoms) {
  __shared__ float red[8][128];
  __shared__ float scl[128];
  const int i = blockIdx.x;
  if (i >= __ldg(n_tiles)) return;
  const int cb = blockIdx.y;
  const int g = __ldg(tile_group + i);
  const int b = i - __ldg(tile_start + g);
  const int64_t r0 = static_cast<int64_t>(__ldg(offsets + g)) + 128 * b;
  const int64_t left = static_cast<int64_t>(__ldg(offsets + g + 1)) - r0;
  const int nr = static_cast<int>(left < 128 ? left : 128);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int c = 4 * lane;  // this thread's 4 channels within the block
  float v[16][4];
  float am[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int m = 0; m < 16; ++m) {
    const int r = 16 * warp + m;
#pragma unroll
    for (int q = 0; q < 4; ++q) v[m][q] = 0.f;
    if (r < nr) {
      if (FP8_SRC) {
        const uint32_t w = __ldg(reinterpret_cast<const uint32_t*>(src_q + (r0 + r) * ld_src + 128 * cb) + lane);
        const float s = __ldg(src_s + (r0 + r) * (ld_src / 128) + cb);
        float f[4];
        e4m3x4_to_float(w, f);
#pragma unroll
        for (int q = 0; q < 4; ++q) v[m][q] = __fmul_rn(f[q], s);
      } else {
        const float4 a = __ldg(reinterpret_cast<const float4*>(src + (r0 + r) * ld_src + 128 * cb) + lane);
        v[m][0] = a.x;
        v[m][1] = a.y;
        v[m][2] = a.z;
        v[m][3] = a.w;
      }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) am[q] = fmaxf(am[q], fabsf(v[m][q]));
  }
#pragma unroll
  for (int q = 0; q < 4; ++q) red[warp][c + q] = am[q];
  __syncthreads();
  if (threadIdx.x < 128) {
    float a = red[0][threadIdx.x];
#pragma unroll
    for (int w = 1; w < 8; ++w) a = fmaxf(a, red[w][threadIdx.x]);
    const float s = pow2_ceil(quant_scale(a));
    scl[threadIdx.x] = s;
    st[(static_cast<int64_t>(128) * cb + threadIdx.x) * (ldt / 128) + i] = s;
    if (atoms) {
      // UE8M0 atom of (channel block cb, token blocks 4a..4a+3): byte
      // 16 r + 4 j + b holds channel 32 j + r of token block 4a + b
      const int ch = threadIdx.x;
      atoms[(static_cast<int64_t>(cb) * (ldt / 512) + (i >> 2)) * 512 + 16 * (ch & 31) +
            4 * (ch >> 5) + (i & 3)] = static_cast<uint8_t>(__float_as_uint(s) >> 23);
    }
  }
  __syncthreads();
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float s = scl[c + q];
    const float rs = __frcp_rn(s);
    uint32_t w4[4];
#pragma unroll
    for (int k = 0; k < 4; ++k)
      w4[k] = e4m3x4(div_by_scale(v[4 * k][q], s, rs), div_by_scale(v[4 * k + 1][q], s, rs),
                     div_by_scale(v[4 * k + 2][q], s, rs), div_by_scale(v[4 * k + 3][q], s, rs));
    *reinterpret_cast<uint4*>(qt + (static_cast<int64_t>(128) * cb + c + q) * ldt +
                              static_cast<int64_t>(128) * i + 16 * warp) =
        make_uint4(w4[0], w4[1], w4[2], w4[3]);
  }
}

// --------------------------------------------------------- weight transpose --
// CTA per 128x128 block (kb, nb, group): 16 KB through shared memory.
__global__ void __launch_bounds__(256) transpose_128x128_kernel(
    const uint8_t* __restrict__ q, const float* __restrict__ s, int N, int K,
    uint8_t* __restrict__ qt, float* __restrict__ st) {
  __shared__ uint8_t tr[128][128 + 16];
  const int kb = blockIdx.x, nb = blockIdx.y;
  const int64_t g = blockIdx.z;
  const uint8_t* src = q + g * N * static_cast<int64_t>(K);
  uint8_t* dst = qt + g * N * static_cast<int64_t>(K);
#pragma unroll
  for (int pass = 0; pass < 4; ++pass) {
    const int row = (threadIdx.x >> 3) + 32 * pass;  // n within the block
    const int chunk = threadIdx.x & 7;
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(
        src + (static_cast<int64_t>(128) * nb + row) * K + 128 * kb + 16 * chunk));
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4)
#pragma unroll
      for (int e = 0; e < 4; ++e)
        tr[16 * chunk + 4 * q4 + e][row] = static_cast<uint8_t>((ws[q4] >> (8 * e)) & 0xFFu);
  }
  __syncthreads();
#pragma unroll
  for (int pass = 0; pass < 4; ++pass) {
    const int row = (threadIdx.x >> 3) + 32 * pass;  // k within the block
    const int chunk = threadIdx.x & 7;
    uint32_t wv[4];
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4)
      wv[q4] = static_cast<uint32_t>(tr[row][16 * chunk + 4 * q4]) |
               (static_cast<uint32_t>(tr[row][16 * chunk + 4 * q4 + 1]) << 8) |
               (static_cast<uint32_t>(tr[row][16 * chunk + 4 * q4 + 2]) << 16) |
               (static_cast<uint32_t>(tr[row][16 * chunk + 4 * q4 + 3]) << 24);
    *reinterpret_cast<uint4*>(dst + (static_cast<int64_t>(128) * kb + row) * N + 128 * nb +
                              16 * chunk) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
  }
  if (threadIdx.x == 0) {
    const int nbk = K / 128, nbn = N / 128;
    st[(g * nbk + kb) * nbn + nb] = s[(g * nbn + nb) * nbk + kb];
  }
}

// ------------------------------------------------------------ unpermute add --
// du_t = dout_t + dx[T*K + t] + sum_k dx[dst_of[t][k]], added in that order.
__global__ void __launch_bounds__(256) unpermute_add_kernel(
    const float* __restrict__ dx, const int32_t* __restrict__ dst_of,
    const float* __restrict__ dout, int T, int K, int d, float* __restrict__ du) {
  __shared__ int64_t rows[kMaxKb];
  const int64_t t = blockIdx.x;
  if (threadIdx.x < K) {
    const int32_t r = dst_of[t * K + threadIdx.x];
    rows[threadIdx.x] = r < 0 ? -1 : static_cast<int64_t>(r) * d;
  }
  __syncthreads();
  const int64_t shared_row = (static_cast<int64_t>(T) * K + t) * d;
  for (int v = threadIdx.x; v < d / 4; v += 256) {
    float4 acc = __ldg(reinterpret_cast<const float4*>(dout + t * d) + v);
    const float4 s = __ldg(reinterpret_cast<const float4*>(dx + shared_row) + v);
    acc.x = __fadd_rn(acc.x, s.x);
    acc.y = __fadd_rn(acc.y, s.y);
    acc.z = __fadd_rn(acc.z, s.z);
    acc.w = __fadd_rn(acc.w, s.w);
    for (int k = 0; k < K; ++k) {
      if (rows[k] < 0) continue;
      const float4 y = __ldg(reinterpret_cast<const float4*>(dx + rows[k]) + v);
      acc.x = __fadd_rn(acc.x, y.x);
      acc.y = __fadd_rn(acc.y, y.y);
      acc.z = __fadd_rn(acc.z, y.z);
      acc.w = __fadd_rn(acc.w, y.w);
    }
    reinterpret_cast<float4*>(du + t * d)[v] = acc;
  }
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

}  // namespace
}  // namespace moe

extern "C" moe_status fp8_quant_1x128_f32(const float* x, int64_t ldx, int rows, int cols, int pow2,
                                          uint8_t* q, float* scale, moe_stream_t stream) {
  using namespace moe;
  if (rows < 0 || cols < 0) return MOE_ERR_INVALID_ARG;
  if (cols % 128 != 0 || ldx < cols) return MOE_ERR_SHAPE;
  if (rows == 0 || cols == 0) return MOE_OK;
  if (!x || !q || !scale) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned4(q) || (ldx % 4) != 0 || !aligned4(scale)) return MOE_ERR_ALIGN;
  const int64_t tiles = static_cast<int64_t>(rows) * (cols / 128);
  const int64_t blocks = (tiles + 7) / 8;
  if (blocks > 0x7FFFFFFF) return MOE_ERR_UNSUPPORTED;
  auto kern = pow2 ? quant_f32_kernel<true> : quant_f32_kernel<false>;
  kern<<<static_cast<unsigned>(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      x, ldx, rows, cols / 128, q, scale);
  MOE_CUDA_CHECK_LAUNCH();
  return MOE_OK;
}

extern "C" moe_status moe_combine_backward(const float* dout, const int32_t* dst_of,
                                           const float* topk_gate, int T, int K, int d,
                                           uint8_t* dyq, float* dys, float* dy,
                                           moe_stream_t stream) {
  using namespace moe;
  if (T < 0 || K < 0 || d <= 0) return MOE_ERR_INVALID_ARG;
  if (d % 128 != 0) return MOE_ERR_SHAPE;
  if (K > kMaxKb) return MOE_ERR_UNSUPPORTED;
  if (T == 0) return MOE_OK;
  if (!dout || !dyq || !dys || (K > 0 && (!dst_of || !topk_gate))) return MOE_ERR_INVALID_ARG;
  if (!aligned16(dout) || !aligned4(dyq) || !aligned4(dys) || (dy && !aligned16(dy)))
    return MOE_ERR_ALIGN;
  combine_backward_kernel<<<T, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      dout, dst_of, topk_gate, T, K, d, dyq, dys, dy);
  MOE_CUDA_CHECK_LAUNCH();
  return MOE_OK;
}

extern "C" moe_status swiglu_backward(const float* dh, const uint8_t* guq, const float* gus,
                                      int rows, int I, uint8_t* dguq, float* dgus, float* dgu,
                                      float* h, moe_stream_t stream) {
  using namespace moe;
  if (rows < 0 || I < 0) return MOE_ERR_INVALID_ARG;
  if (I % 128 != 0) return MOE_ERR_SHAPE;
  if (rows == 0 || I == 0) return MOE_OK;
  if (!dh || !guq || !gus || !dguq || !dgus) return MOE_ERR_INVALID_ARG;
  if (!aligned16(dh) || !aligned4(guq) || !aligned4(gus) || !aligned4(dguq) || !aligned4(dgus) ||
      (dgu && !aligned16(dgu)) || (h && !aligned16(h)))
    return MOE_ERR_ALIGN;
  const int64_t items = static_cast<int64_t>(rows) * (I / 128);
  const int64_t blocks = (items + 7) / 8;
  if (blocks > 0x7FFFFFFF) return MOE_ERR_UNSUPPORTED;
  swiglu_backward_kernel<<<static_cast<unsigned>(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      dh, guq, gus, rows, I, dguq, dgus, dgu, h);
  MOE_CUDA_CHECK_LAUNCH();
  return MOE_OK;
}

namespace {
moe_status quant_128x1_launch(const float* src, const uint8_t* src_q, const float* src_s,
                              int64_t ld_src, const int32_t* offsets, const int32_t* tile_group,
                              const int32_t* tile_start, const int32_t* n_tiles, int max_tiles,
                              int C, uint8_t* qt, int64_t ldt, float* st, uint8_t* atoms,
                              moe_stream_t stream) {
  using namespace moe;
  if (max_tiles < 0 || C < 0 || ld_src < C) return MOE_ERR_INVALID_ARG;
  if (C % 128 != 0 || ldt % 128 != 0 || ldt < static_cast<int64_t>(128) * max_tiles ||
      (atoms && ldt % 512 != 0))
    return MOE_ERR_SHAPE;
  if (max_tiles == 0 || C == 0) return MOE_OK;
  if (!offsets || !tile_group || !tile_start || !n_tiles || !qt || !st) return MOE_ERR_INVALID_ARG;
  if (!aligned16(qt) || (ldt % 16) != 0 || !aligned4(st)) return MOE_ERR_ALIGN;
  if (C / 128 > 65535) return MOE_ERR_UNSUPPORTED;
  dim3 grid(max_tiles, C / 128);
  if (src_q) {
    if (!src_s || !aligned4(src_q) || (ld_src % 128) != 0 || !aligned4(src_s)) return MOE_ERR_ALIGN;
    quant_128x1_kernel<true><<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
        nullptr, src_q, src_s, ld_src, offsets, tile_group, tile_start, n_tiles, C, qt, ldt, st,
        atoms);
  } else {
    if (!src) return MOE_ERR_INVALID_ARG;
    if (!aligned16(src) || (ld_src % 4) != 0) return MOE_ERR_ALIGN;
    quant_128x1_kernel<false><<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
        src, nullptr, nullptr, ld_src, offsets, tile_group, tile_start, n_tiles, C, qt, ldt, st,
        atoms);
  }
  MOE_CUDA_CHECK_LAUNCH();
  return MOE_OK;
}
}  // namespace

extern "C" moe_status fp8_quant_128x1_pow2(const float* src, int64_t ld_src, const int32_t* offsets,
                                           const int32_t* tile_group, const int32_t* tile_start,
                                           const int32_t* n_tiles, int max_tiles, int C,
                                           uint8_t* qt, int64_t ldt, float* st, uint8_t* sf_atoms,
                                           moe_stream_t stream) {
  if (!src) return MOE_ERR_INVALID_ARG;
  return quant_128x1_launch(src, nullptr, nullptr, ld_src, offsets, tile_group, tile_start, n_tiles,
                            max_tiles, C, qt, ldt, st, sf_atoms, stream);
}

extern "C" moe_status fp8_requant_128x1_pow2(const uint8_t* q, const float* scale, int64_t ld_src,
                                             const int32_t* offsets, const int32_t* tile_group,
                                             const int32_t* tile_start, const int32_t* n_tiles,
                                             int max_tiles, int C, uint8_t* qt, int64_t ldt,
                                             float* st, uint8_t* sf_atoms, moe_stream_t stream) {
  if (!q || !scale) return MOE_ERR_INVALID_ARG;
  return quant_128x1_launch(nullptr, q, scale, ld_src, offsets, tile_group, tile_start, n_tiles,
                            max_tiles, C, qt, ldt, st, sf_atoms, stream);
}

extern "C" moe_status fp8_transpose_128x128(const uint8_t* q, const float* scale, int groups, int N,
                                            int K, uint8_t* qt, float* scale_t,
                                            moe_stream_t stream) {
  using namespace moe;
  if (groups < 0 || N < 0 || K < 0) return MOE_ERR_INVALID_ARG;
  if (N % 128 != 0 || K % 128 != 0) return MOE_ERR_SHAPE;
  if (groups == 0 || N == 0 || K == 0) return MOE_OK;
  if (!q || !scale || !qt || !scale_t) return MOE_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(qt) || !aligned4(scale) || !aligned4(scale_t)) return MOE_ERR_ALIGN;
  if (N / 128 > 65535 || groups > 65535) return MOE_ERR_UNSUPPORTED;
  dim3 grid(K / 128, N / 128, groups);
  transpose_128x128_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(q, scale, N, K, qt,
                                                                               scale_t);
  MOE_CUDA_CHECK_LAUNCH();
  return MOE_OK;
}

extern "C" moe_status moe_unpermute_add(const float* dx, const int32_t* dst_of, const float* dout,
                                        int T, int K, int d, float* du, moe_stream_t stream) {
  using namespace moe;
  if (T < 0 || K < 0 || d <= 0) return MOE_ERR_INVALID_ARG;
  if (d % 4 != 0) return MOE_ERR_SHAPE;
  if (K > kMaxKb) return MOE_ERR_UNSUPPORTED;
  if (T == 0) return MOE_OK;
  if (!dx || !dout || !du || (K > 0 && !dst_of)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(dx) || !aligned16(dout) || !aligned16(du)) return MOE_ERR_ALIGN;
  unpermute_add_kernel<<<T, 256, 0, static_cast<cudaStream_t>(stream)>>>(dx, dst_of, dout, T, K, d, du);
  MOE_CUDA_CHECK_LAUNCH();
  return MOE_OK;
}
