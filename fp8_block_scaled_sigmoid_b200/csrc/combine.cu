// Combine with residual and the auxiliary-loss-free bias update.
// "DeepSeek_V3_Report：Annotation", eq. (12) and "Auxiliary-Loss-Free Load
// Balancing".
//
// moe_combine is HBM-bound: per token it reads K+1 fp32 expert rows and the
// bf16 residual and writes one fp32 row.  One CTA per token, float4 vectors,
// the K gated rows added in k order (no atomics, deterministic).
#include "epi_math.cuh"
#include "moe_common.cuh"

namespace moe {
namespace {

constexpr int kCbThreads = 256;
constexpr int kMaxK = 32;

__global__ void __launch_bounds__(kCbThreads) combine_kernel(
    const float* __restrict__ Y, const int32_t* __restrict__ dst_of,
    const float* __restrict__ gate, const float* __restrict__ Ys, const uint16_t* __restrict__ u,
    int K, int d, float* __restrict__ out) {
  __shared__ int64_t rows[kMaxK];
  __shared__ float gs[kMaxK];
  const int64_t t = blockIdx.x;
  if (threadIdx.x < K) {
    // a negative row (pair rejected upstream) contributes nothing
    const int32_t r = dst_of[t * K + threadIdx.x];
    rows[threadIdx.x] = r < 0 ? 0 : static_cast<int64_t>(r) * d;
    gs[threadIdx.x] = r < 0 ? 0.f : gate[t * K + threadIdx.x];
  }
  __syncthreads();
  const int nv = d / 4;
  for (int v = threadIdx.x; v < nv; v += kCbThreads) {
    const uint2 ub = __ldg(reinterpret_cast<const uint2*>(u + t * d) + v);
    float4 acc = make_float4(bf16_bits_to_float(ub.x & 0xFFFFu), bf16_bits_to_float(ub.x >> 16),
                             bf16_bits_to_float(ub.y & 0xFFFFu), bf16_bits_to_float(ub.y >> 16));
    if (Ys) {
      const float4 s = __ldg(reinterpret_cast<const float4*>(Ys + t * d) + v);
      acc.x += s.x;
      acc.y += s.y;
      acc.z += s.z;
      acc.w += s.w;
    }
    for (int k = 0; k < K; ++k) {
      const float4 y = __ldg(reinterpret_cast<const float4*>(Y + rows[k]) + v);
      const float g = gs[k];
      acc.x = fmaf(g, y.x, acc.x);
      acc.y = fmaf(g, y.y, acc.y);
      acc.z = fmaf(g, y.z, acc.z);
      acc.w = fmaf(g, y.w, acc.w);
    }
    reinterpret_cast<float4*>(out + t * d)[v] = acc;
  }
}

// b_i -= gamma if c_i > T*K/E, += gamma if below, unchanged if equal.  The
// comparison c_i * E vs T * K is exact in 64-bit integers.
__global__ void bias_update_kernel(const int32_t* __restrict__ counts, int E, int64_t TK,
                                   float gamma, float* __restrict__ bias) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= E) return;
  const int64_t c = static_cast<int64_t>(counts[e]) * E;
  const float b = bias[e];
  if (c > TK) bias[e] = __fsub_rn(b, gamma);
  else if (c < TK) bias[e] = __fadd_rn(b, gamma);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace moe

extern "C" moe_status moe_combine(const float* Y, const int32_t* dst_of, const float* topk_gate,
                                  const float* Y_shared, const uint16_t* u, int T, int K, int d,
                                  float* out, moe_stream_t stream) {
  using namespace moe;
  if (T < 0 || K < 0 || d <= 0) return MOE_ERR_INVALID_ARG;
  if (d % 8 != 0) return MOE_ERR_SHAPE;
  if (K > kMaxK) return MOE_ERR_UNSUPPORTED;
  if (T == 0) return MOE_OK;
  if (!u || !out || (K > 0 && (!Y || !dst_of || !topk_gate))) return MOE_ERR_INVALID_ARG;
  if ((Y && !aligned16(Y)) || (Y_shared && !aligned16(Y_shared)) || !aligned16(u) ||
      !aligned16(out))
    return MOE_ERR_ALIGN;
  combine_kernel<<<T, kCbThreads, 0, static_cast<cudaStream_t>(stream)>>>(Y, dst_of, topk_gate,
                                                                          Y_shared, u, K, d, out);
  MOE_CUDA_CHECK_LAUNCH();
  return MOE_OK;
}

extern "C" moe_status moe_bias_update(const int32_t* counts, int E, int64_t T, int K, float gamma,
                                      float* bias, moe_stream_t stream) {
  using namespace moe;
  if (E <= 0 || T < 0 || K <= 0 || !counts || !bias) return MOE_ERR_INVALID_ARG;
  bias_update_kernel<<<(E + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      counts, E, T * K, gamma, bias);
  MOE_CUDA_CHECK_LAUNCH();
  return MOE_OK;
}
