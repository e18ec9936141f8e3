// Online FP8 (E4M3) quantisation kernels: 1x128 activation tiles, 128x128
// weight blocks, and SwiGLU followed by 1x128 quantisation.
// "DeepSeek_V3_Report：Annotation", "Fine-Grained Quantization" and "Online
// Quantization": one fp32 scale per tile/block from its own max |x|.
//
// All three are HBM-bound streaming kernels: 16-byte vector loads, the amax
// reduced with warp shuffles, the scale divided out in fp32 and the cast done
// by the hardware's saturating round-to-nearest-even E4M3 conversion.  For
// bf16 inputs the division is one correctly rounded reciprocal per tile plus
// a per-element FMA correction (div_by_scale), which gives the IEEE quotient
// on every input these kernels can see.
#include "epi_math.cuh"
#include "moe_common.cuh"

namespace moe {
namespace {

// The scale of a tile: amax/448 in fp32, or (POW2) that value rounded up to a
// power of two ("Low-Precision Storage and Communication": scaling factors
// that are integral powers of 2).  Dividing by a power of two is exact, so
// div_by_scale returns the plain product x * 2^-e there.
template <bool POW2>
__device__ __forceinline__ float tile_scale(float amax) {
  return POW2 ? pow2_ceil(quant_scale(amax)) : quant_scale(amax);
}

// ----------------------------------------------------------- 1x128 tiles --
// A half-warp owns one tile (16 lanes x 8 bf16 = 256 bytes); each half-warp
// takes kTilesPerHW consecutive tiles, loading all of them before reducing.
constexpr int kQ1Threads = 256;
constexpr int kTilesPerHW = 4;
constexpr int kQ1TilesPerBlock = (kQ1Threads / 16) * kTilesPerHW;

// With SCATTER the tile is also written to the K routed rows of its token
// (dst_of[row][k] >= 0: row of q_perm / s_perm; the permutation's gather
// fused into the quantiser, so each token is read once and its FP8 bytes go
// straight to every destination).  K <= 16: lane k of a half-warp holds the
// row's k-th destination.
template <bool POW2, bool SCATTER>
__global__ void __launch_bounds__(kQ1Threads) quant_1x128_kernel(
    const uint16_t* __restrict__ x, int64_t ldx, int rows, int tiles_per_row,
    uint8_t* __restrict__ q, float* __restrict__ scale, const int32_t* __restrict__ dst_of,
    int K, uint8_t* __restrict__ q_perm, float* __restrict__ s_perm) {
  const int lane16 = threadIdx.x & 15;
  const int hw = threadIdx.x >> 4;
  const int64_t total = static_cast<int64_t>(rows) * tiles_per_row;
  const int64_t first = (static_cast<int64_t>(blockIdx.x) * (kQ1Threads / 16) + hw) * kTilesPerHW;
  const int cols = tiles_per_row * 128;
  // (row, tile-in-row) of the first tile; the next ones step along the row
  // (one division per half-warp, not per tile)
  const int64_t r0 = first / tiles_per_row;
  const int j0 = static_cast<int>(first - r0 * tiles_per_row);

  uint4 v[kTilesPerHW];
  {
    int64_t r = r0;
    int j = j0;
#pragma unroll
    for (int i = 0; i < kTilesPerHW; ++i) {
      v[i] = make_uint4(0, 0, 0, 0);
      if (first + i < total)
        v[i] = __ldg(reinterpret_cast<const uint4*>(x + r * ldx + j * 128 + lane16 * 8));
      if (++j == tiles_per_row) {
        j = 0;
        ++r;
      }
    }
  }
  int64_t r = r0;
  int j = j0;
#pragma unroll
  for (int i = 0; i < kTilesPerHW; ++i) {
    const int64_t t = first + i;
    float f[8];
    const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      f[2 * k] = bf16_bits_to_float(w[k] & 0xFFFFu);
      f[2 * k + 1] = bf16_bits_to_float(w[k] >> 16);
    }
    float amax = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) amax = fmaxf(amax, fabsf(f[k]));
#pragma unroll
    for (int off = 8; off > 0; off >>= 1)
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    const float s = tile_scale<POW2>(amax);
    const float rs = __frcp_rn(s);
    uint2 out;
    out.x = e4m3x4(div_by_scale(f[0], s, rs), div_by_scale(f[1], s, rs),
                   div_by_scale(f[2], s, rs), div_by_scale(f[3], s, rs));
    out.y = e4m3x4(div_by_scale(f[4], s, rs), div_by_scale(f[5], s, rs),
                   div_by_scale(f[6], s, rs), div_by_scale(f[7], s, rs));
    if (t < total) {
      if (q != nullptr) {
        *reinterpret_cast<uint2*>(q + r * cols + j * 128 + lane16 * 8) = out;
        if (lane16 == 0) scale[t] = s;
      }
    }
    if (SCATTER) {
      // every lane of the warp takes part in the exchange (the two half-warps
      // may be at different rows, or one past the end)
      const int64_t rr = t < total ? r : 0;
      const int my_dst = lane16 < K ? __ldg(dst_of + rr * K + lane16) : -1;
      const int hbase = threadIdx.x & 16;
      for (int k = 0; k < K; ++k) {
        const int dr = __shfl_sync(0xffffffffu, my_dst, hbase + k);
        if (t < total && dr >= 0) {
          *reinterpret_cast<uint2*>(q_perm + static_cast<int64_t>(dr) * cols + j * 128 +
                                    lane16 * 8) = out;
          if (lane16 == 0) s_perm[static_cast<int64_t>(dr) * tiles_per_row + j] = s;
        }
      }
    }
    if (++j == tiles_per_row) {
      j = 0;
      ++r;
    }
  }
}

// --------------------------------------------------------- 128x128 blocks --
// One CTA per block: 256 threads x 8 chunks of 8 bf16 = 128 x 128.
constexpr int kQ2Threads = 256;

template <bool POW2>
__global__ void __launch_bounds__(kQ2Threads) quant_128x128_kernel(
    const uint16_t* __restrict__ w, int64_t ldw, int rows, int cols, uint8_t* __restrict__ q,
    float* __restrict__ scale) {
  __shared__ float red[kQ2Threads / 32];
  const int bj = blockIdx.x;  // column block
  const int bi = blockIdx.y;  // row block
  const int tid = threadIdx.x;
  uint4 v[8];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int c = tid + i * kQ2Threads;  // chunk within the block
    const int rr = c >> 4, cc = c & 15;
    const int64_t r = static_cast<int64_t>(bi) * 128 + rr;
    v[i] = make_uint4(0, 0, 0, 0);
    if (r < rows) v[i] = __ldg(reinterpret_cast<const uint4*>(w + r * ldw + bj * 128 + cc * 8));
    const uint32_t ww[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      amax = fmaxf(amax, fabsf(bf16_bits_to_float(ww[k] & 0xFFFFu)));
      amax = fmaxf(amax, fabsf(bf16_bits_to_float(ww[k] >> 16)));
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  if ((tid & 31) == 0) red[tid >> 5] = amax;
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int k = 1; k < kQ2Threads / 32; ++k) amax = fmaxf(amax, red[k]);
  const float s = tile_scale<POW2>(amax);
  const float rs = __frcp_rn(s);
  if (tid == 0) scale[static_cast<int64_t>(bi) * (cols / 128) + bj] = s;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int c = tid + i * kQ2Threads;
    const int rr = c >> 4, cc = c & 15;
    const int64_t r = static_cast<int64_t>(bi) * 128 + rr;
    if (r >= rows) continue;
    const uint32_t ww[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
    float f[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      f[2 * k] = div_by_scale(bf16_bits_to_float(ww[k] & 0xFFFFu), s, rs);
      f[2 * k + 1] = div_by_scale(bf16_bits_to_float(ww[k] >> 16), s, rs);
    }
    uint2 out;
    out.x = e4m3x4(f[0], f[1], f[2], f[3]);
    out.y = e4m3x4(f[4], f[5], f[6], f[7]);
    *reinterpret_cast<uint2*>(q + r * cols + bj * 128 + cc * 8) = out;
  }
}

// ------------------------------------------------------------ SwiGLU+quant --
// One warp per 128-wide output tile: lane l takes gate/up elements 4l..4l+3.
constexpr int kSwThreads = 256;

template <bool POW2>
__global__ void __launch_bounds__(kSwThreads) swiglu_quant_kernel(
    const float* __restrict__ gu, int rows, int I, uint8_t* __restrict__ h,
    float* __restrict__ h_scale) {
  const int lane = threadIdx.x & 31;
  const int64_t tile = static_cast<int64_t>(blockIdx.x) * (kSwThreads / 32) + (threadIdx.x >> 5);
  const int tpr = I / 128;
  if (tile >= static_cast<int64_t>(rows) * tpr) return;
  const int64_t r = tile / tpr;
  const int j = static_cast<int>(tile - r * tpr);
  const float* base = gu + r * (2 * static_cast<int64_t>(I)) + j * 256;
  const float4 g = __ldg(reinterpret_cast<const float4*>(base) + lane);
  const float4 u = __ldg(reinterpret_cast<const float4*>(base + 128) + lane);
  float hv[4] = {silu_mul(g.x, u.x), silu_mul(g.y, u.y), silu_mul(g.z, u.z), silu_mul(g.w, u.w)};
  float amax = fmaxf(fmaxf(fabsf(hv[0]), fabsf(hv[1])), fmaxf(fabsf(hv[2]), fabsf(hv[3])));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  const float s = tile_scale<POW2>(amax);
  const float rs = __frcp_rn(s);
  const uint32_t packed = e4m3x4(div_by_scale(hv[0], s, rs), div_by_scale(hv[1], s, rs),
                                 div_by_scale(hv[2], s, rs), div_by_scale(hv[3], s, rs));
  *reinterpret_cast<uint32_t*>(h + r * I + j * 128 + lane * 4) = packed;
  if (lane == 0) h_scale[tile] = s;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace moe

namespace {

moe_status quant_1x128_launch(bool pow2, const uint16_t* x, int64_t ldx, int rows, int cols,
                              uint8_t* q, float* scale, moe_stream_t stream) {
  using namespace moe;
  if (rows < 0 || cols < 0) return MOE_ERR_INVALID_ARG;
  if (cols % 128 != 0 || ldx < cols) return MOE_ERR_SHAPE;
  if (rows == 0 || cols == 0) return MOE_OK;
  if (!x || !q || !scale) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(q) || (ldx % 8) != 0 || (reinterpret_cast<uintptr_t>(scale) & 3))
    return MOE_ERR_ALIGN;
  const int64_t tiles = static_cast<int64_t>(rows) * (cols / 128);
  const int64_t blocks = (tiles + kQ1TilesPerBlock - 1) / kQ1TilesPerBlock;
  if (blocks > 0x7FFFFFFF) return MOE_ERR_UNSUPPORTED;
  auto kern = pow2 ? quant_1x128_kernel<true, false> : quant_1x128_kernel<false, false>;
  kern<<<static_cast<unsigned>(blocks), kQ1Threads, 0, static_cast<cudaStream_t>(stream)>>>(
      x, ldx, rows, cols / 128, q, scale, nullptr, 0, nullptr, nullptr);
  MOE_CUDA_CHECK_LAUNCH();
  return MOE_OK;
}

moe_status quant_1x128_scatter_launch(bool pow2, const uint16_t* x, int64_t ldx, int rows,
                                      int cols, const int32_t* dst_of, int K, uint8_t* q_tok,
                                      float* s_tok, uint8_t* q_perm, float* s_perm,
                                      moe_stream_t stream) {
  using namespace moe;
  if (rows < 0 || cols < 0 || K <= 0) return MOE_ERR_INVALID_ARG;
  if (cols % 128 != 0 || ldx < cols) return MOE_ERR_SHAPE;
  if (K > 16) return MOE_ERR_UNSUPPORTED;
  if (rows == 0 || cols == 0) return MOE_OK;
  if (!x || !dst_of || !q_perm || !s_perm || (q_tok == nullptr) != (s_tok == nullptr))
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || (q_tok && !aligned16(q_tok)) || !aligned16(q_perm) || (ldx % 8) != 0 ||
      (reinterpret_cast<uintptr_t>(s_tok) & 3) || (reinterpret_cast<uintptr_t>(s_perm) & 3))
    return MOE_ERR_ALIGN;
  const int64_t tiles = static_cast<int64_t>(rows) * (cols / 128);
  const int64_t blocks = (tiles + kQ1TilesPerBlock - 1) / kQ1TilesPerBlock;
  if (blocks > 0x7FFFFFFF) return MOE_ERR_UNSUPPORTED;
  auto kern = pow2 ? quant_1x128_kernel<true, true> : quant_1x128_kernel<false, true>;
  kern<<<static_cast<unsigned>(blocks), kQ1Threads, 0, static_cast<cudaStream_t>(stream)>>>(
      x, ldx, rows, cols / 128, q_tok, s_tok, dst_of, K, q_perm, s_perm);
  MOE_CUDA_CHECK_LAUNCH();
  return MOE_OK;
}

moe_status quant_128x128_launch(bool pow2, const uint16_t* w, int64_t ldw, int rows, int cols,
                                uint8_t* q, float* scale, moe_stream_t stream) {
  using namespace moe;
  if (rows < 0 || cols < 0) return MOE_ERR_INVALID_ARG;
  if (cols % 128 != 0 || ldw < cols) return MOE_ERR_SHAPE;
  if (rows == 0 || cols == 0) return MOE_OK;
  if (!w || !q || !scale) return MOE_ERR_INVALID_ARG;
  if (!aligned16(w) || !aligned16(q) || (ldw % 8) != 0 || (reinterpret_cast<uintptr_t>(scale) & 3))
    return MOE_ERR_ALIGN;
  const int rb = (rows + 127) / 128;
  if (rb > 65535) return MOE_ERR_UNSUPPORTED;
  dim3 grid(cols / 128, rb);
  auto kern = pow2 ? quant_128x128_kernel<true> : quant_128x128_kernel<false>;
  kern<<<grid, kQ2Threads, 0, static_cast<cudaStream_t>(stream)>>>(w, ldw, rows, cols, q, scale);
  MOE_CUDA_CHECK_LAUNCH();
  return MOE_OK;
}

}  // namespace

extern "C" moe_status fp8_quant_1x128(const uint16_t* x, int64_t ldx, int rows, int cols,
                                      uint8_t* q, float* scale, moe_stream_t stream) {
  return quant_1x128_launch(false, x, ldx, rows, cols, q, scale, stream);
}

extern "C" moe_status fp8_quant_1x128_pow2(const uint16_t* x, int64_t ldx, int rows, int cols,
                                           uint8_t* q, float* scale, moe_stream_t stream) {
  return quant_1x128_launch(true, x, ldx, rows, cols, q, scale, stream);
}

extern "C" moe_status fp8_quant_1x128_scatter(const uint16_t* x, int64_t ldx, int rows, int cols,
                                              const int32_t* dst_of, int K, int pow2,
                                              uint8_t* q_tok, float* s_tok, uint8_t* q_perm,
                                              float* s_perm, moe_stream_t stream) {
  return quant_1x128_scatter_launch(pow2 != 0, x, ldx, rows, cols, dst_of, K, q_tok, s_tok,
                                    q_perm, s_perm, stream);
}

extern "C" moe_status fp8_quant_128x128(const uint16_t* w, int64_t ldw, int rows, int cols,
                                        uint8_t* q, float* scale, moe_stream_t stream) {
  return quant_128x128_launch(false, w, ldw, rows, cols, q, scale, stream);
}

extern "C" moe_status fp8_quant_128x128_pow2(const uint16_t* w, int64_t ldw, int rows, int cols,
                                             uint8_t* q, float* scale, moe_stream_t stream) {
  return quant_128x128_launch(true, w, ldw, rows, cols, q, scale, stream);
}

namespace {
moe_status swiglu_quant_launch(bool pow2, const float* gu, int rows, int I, uint8_t* h,
                               float* h_scale, moe_stream_t stream) {
  using namespace moe;
  if (rows < 0 || I < 0) return MOE_ERR_INVALID_ARG;
  if (I % 128 != 0) return MOE_ERR_SHAPE;
  if (rows == 0 || I == 0) return MOE_OK;
  if (!gu || !h || !h_scale) return MOE_ERR_INVALID_ARG;
  if (!aligned16(gu) || (reinterpret_cast<uintptr_t>(h) & 3) ||
      (reinterpret_cast<uintptr_t>(h_scale) & 3))
    return MOE_ERR_ALIGN;
  const int64_t tiles = static_cast<int64_t>(rows) * (I / 128);
  const int64_t blocks = (tiles + (kSwThreads / 32) - 1) / (kSwThreads / 32);
  if (blocks > 0x7FFFFFFF) return MOE_ERR_UNSUPPORTED;
  auto kern = pow2 ? swiglu_quant_kernel<true> : swiglu_quant_kernel<false>;
  kern<<<static_cast<unsigned>(blocks), kSwThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      gu, rows, I, h, h_scale);
  MOE_CUDA_CHECK_LAUNCH();
  return MOE_OK;
}
}  // namespace

extern "C" moe_status swiglu_quant(const float* gu, int rows, int I, uint8_t* h, float* h_scale,
                                   moe_stream_t stream) {
  return swiglu_quant_launch(false, gu, rows, I, h, h_scale, stream);
}

extern "C" moe_status swiglu_quant_pow2(const float* gu, int rows, int I, uint8_t* h,
                                        float* h_scale, moe_stream_t stream) {
  return swiglu_quant_launch(true, gu, rows, I, h, h_scale, stream);
}
