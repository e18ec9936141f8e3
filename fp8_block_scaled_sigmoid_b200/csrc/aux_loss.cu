// Complementary sequence-wise balance loss ("DeepSeek_V3_Report：Annotation",
// "Complementary Sequence-Wise Auxiliary Loss", eqs. (17)-(20)).  For each
// sequence of S consecutive tokens:
//   L = alpha * sum_i f_i P_i,  f_i = E/(K S) * #{t : i in TopK_K(s_t)},
//   P_i = (1/S) sum_t s_{i,t} / sum_j s_{j,t},  s = Sigmoid(z),
// the TopK taken over the raw affinities of all E routed experts (ties to
// the lower index).
//
// This is the unfused form, from logits kept by moe_route (logits_out); the
// fused form runs inside moe_route's selection pass (moe_balance_loss).  The
// token pass spreads a row's experts over the lanes exactly as the selection
// kernel does (same experts per lane, same orders), so the per-token values
// are the same in both.
//
// Three deterministic passes, no atomics:
//  1. token  -- one warp per token: s, its row sum (fixed butterfly), the
//               normalised s' and the raw top-K; writes s' with the sign bit
//               set on the K chosen experts (s' > 0, so the sign carries the
//               membership) -> ws [T][E].
//  2. chunk  -- one CTA per 32-token chunk of a sequence, one thread per
//               expert: sums |s'| and the members over the chunk in token
//               order -> partials [chunks][E] (sum, count).
//  3. final  -- one CTA per sequence: sums its chunks in order, f_i P_i per
//               expert, a fixed-order tree over experts -> loss, f, P.
#include <climits>

#include "moe_common.cuh"

namespace moe {
namespace {

constexpr int kAuxTokThreads = 256;  // 8 tokens per CTA in pass 1
constexpr int kAuxChunk = 32;        // tokens per partial in pass 2

template <int P>
__global__ void __launch_bounds__(kAuxTokThreads) aux_token_kernel(const float* __restrict__ z,
                                                                    int T, int E, int K,
                                                                    float* __restrict__ ws) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (kAuxTokThreads / 32) + (threadIdx.x >> 5);
  if (t >= T) return;
  const int e0 = lane * P;
  float s[P];
  float sum = 0.f;
#pragma unroll
  for (int i = 0; i < P; ++i) {
    s[i] = 0.f;
    if (e0 + i < E) {
      s[i] = __fdiv_rn(1.0f, __fadd_rn(1.0f, expf(-__ldg(z + static_cast<int64_t>(t) * E + e0 + i))));
      sum = __fadd_rn(sum, s[i]);
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sum = __fadd_rn(sum, __shfl_xor_sync(0xffffffffu, sum, off));
  // raw top-K: each lane keeps its best remaining candidate; one packed
  // (order-preserving key, expert) argmax per round
  uint32_t taken = 0;
  int bi = -1;
  float bv = 0.f;
#pragma unroll
  for (int i = 0; i < P; ++i)
    if (e0 + i < E && (bi < 0 || s[i] > bv)) {
      bi = i;
      bv = s[i];
    }
  for (int k = 0; k < K; ++k) {
    // s > 0: its bit pattern orders like its value
    uint32_t key = bi < 0 ? 0u : __float_as_uint(bv);
    int ex = bi < 0 ? INT_MAX : e0 + bi;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const uint32_t ok = __shfl_xor_sync(0xffffffffu, key, off);
      const int oe = __shfl_xor_sync(0xffffffffu, ex, off);
      if (ok > key || (ok == key && oe < ex)) {
        key = ok;
        ex = oe;
      }
    }
    if (ex / P == lane) {
      taken |= 1u << (ex - e0);
      bi = -1;
      bv = 0.f;
#pragma unroll
      for (int i = 0; i < P; ++i)
        if (e0 + i < E && !((taken >> i) & 1u) && (bi < 0 || s[i] > bv)) {
          bi = i;
          bv = s[i];
        }
    }
  }
#pragma unroll
  for (int i = 0; i < P; ++i) {
    if (e0 + i < E) {
      const float v = __fdiv_rn(s[i], sum);
      ws[static_cast<int64_t>(t) * E + e0 + i] = ((taken >> i) & 1u) ? -v : v;
    }
  }
}

// Pass 2: grid = n_seq * chunks_per_seq, one thread per expert.
__global__ void aux_chunk_kernel(const float* __restrict__ ws, int E, int seq_len,
                                 int chunks_per_seq, float* __restrict__ psum,
                                 int32_t* __restrict__ pcnt) {
  const int e = threadIdx.x;
  if (e >= E) return;
  const int q = blockIdx.x / chunks_per_seq, c = blockIdx.x - q * chunks_per_seq;
  const int t0 = q * seq_len + c * kAuxChunk;
  const int t1 = q * seq_len + min(seq_len, (c + 1) * kAuxChunk);
  float acc = 0.f;
  int cnt = 0;
  int t = t0;
  for (; t + 8 <= t1; t += 8) {  // eight loads in flight, summed in token order
    float v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = __ldg(ws + static_cast<int64_t>(t + j) * E + e);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      acc = __fadd_rn(acc, fabsf(v[j]));
      cnt += v[j] < 0.f;
    }
  }
  for (; t < t1; ++t) {
    const float v = __ldg(ws + static_cast<int64_t>(t) * E + e);
    acc = __fadd_rn(acc, fabsf(v));
    cnt += v < 0.f;
  }
  psum[static_cast<int64_t>(blockIdx.x) * E + e] = acc;
  pcnt[static_cast<int64_t>(blockIdx.x) * E + e] = cnt;
}

// Pass 3: one CTA per sequence (blockDim = power of two >= E, <= 1024).
__global__ void aux_final_kernel(const float* __restrict__ psum, const int32_t* __restrict__ pcnt,
                                 int E, int K, int seq_len, int chunks_per_seq, float alpha,
                                 float* __restrict__ loss, float* __restrict__ f_out,
                                 float* __restrict__ p_out) {
  extern __shared__ float red[];
  const int e = threadIdx.x;
  const int q = blockIdx.x;
  float term = 0.f;
  if (e < E) {
    float acc = 0.f;
    int cnt = 0;
    for (int c = 0; c < chunks_per_seq; ++c) {
      const int64_t j = static_cast<int64_t>(q * chunks_per_seq + c) * E + e;
      acc = __fadd_rn(acc, psum[j]);
      cnt += pcnt[j];
    }
    // f_i = E/(K S) * count, P_i = sum / S
    const float f = __fdiv_rn(static_cast<float>(E) * static_cast<float>(cnt),
                              static_cast<float>(K) * static_cast<float>(seq_len));
    const float p = __fdiv_rn(acc, static_cast<float>(seq_len));
    if (f_out) f_out[static_cast<int64_t>(q) * E + e] = f;
    if (p_out) p_out[static_cast<int64_t>(q) * E + e] = p;
    term = __fmul_rn(f, p);
  }
  red[e] = term;
  __syncthreads();
  for (int w = blockDim.x >> 1; w > 0; w >>= 1) {
    if (e < w) red[e] = __fadd_rn(red[e], red[e + w]);
    __syncthreads();
  }
  if (e == 0) loss[q] = __fmul_rn(alpha, red[0]);
}

template <int P>
void launch_token(int T, int E, int K, const float* z, float* ws, cudaStream_t st) {
  aux_token_kernel<P><<<(T + 7) / 8, kAuxTokThreads, 0, st>>>(z, T, E, K, ws);
}

size_t align256(size_t b) { return (b + 255) / 256 * 256; }

}  // namespace
}  // namespace moe

extern "C" moe_status moe_seq_balance_loss_workspace_size(int T, int E, int seq_len,
                                                           size_t* bytes) {
  using namespace moe;
  if (!bytes || T < 0 || E <= 0 || seq_len <= 0) return MOE_ERR_INVALID_ARG;
  const int64_t n_seq = T / seq_len;
  const int64_t chunks = n_seq * ((seq_len + kAuxChunk - 1) / kAuxChunk);
  *bytes = align256(static_cast<size_t>(T) * E * sizeof(float)) +
           align256(static_cast<size_t>(chunks) * E * sizeof(float)) +
           align256(static_cast<size_t>(chunks) * E * sizeof(int32_t));
  return MOE_OK;
}

extern "C" moe_status moe_seq_balance_loss(const float* logits, int T, int E, int K, int seq_len,
                                           float alpha, float* loss, float* f_out, float* p_out,
                                           void* ws, size_t ws_bytes, moe_stream_t stream) {
  using namespace moe;
  if (T < 0 || E <= 0 || K <= 0 || seq_len <= 0) return MOE_ERR_INVALID_ARG;
  if (K > E || K > 32 || T % seq_len != 0) return MOE_ERR_SHAPE;
  if (E > 1024) return MOE_ERR_UNSUPPORTED;
  if (T == 0) return MOE_OK;
  if (!logits || !loss) return MOE_ERR_INVALID_ARG;
  size_t need = 0;
  moe_seq_balance_loss_workspace_size(T, E, seq_len, &need);
  if (!ws || ws_bytes < need) return MOE_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int n_seq = T / seq_len;
  const int cps = (seq_len + kAuxChunk - 1) / kAuxChunk;
  uint8_t* w = static_cast<uint8_t*>(ws);
  float* srow = reinterpret_cast<float*>(w);
  w += align256(static_cast<size_t>(T) * E * sizeof(float));
  float* psum = reinterpret_cast<float*>(w);
  w += align256(static_cast<size_t>(n_seq) * cps * E * sizeof(float));
  int32_t* pcnt = reinterpret_cast<int32_t*>(w);
  const int P = (E + 31) / 32;
  if (P <= 1) launch_token<1>(T, E, K, logits, srow, st);
  else if (P <= 2) launch_token<2>(T, E, K, logits, srow, st);
  else if (P <= 4) launch_token<4>(T, E, K, logits, srow, st);
  else if (P <= 8) launch_token<8>(T, E, K, logits, srow, st);
  else if (P <= 12) launch_token<12>(T, E, K, logits, srow, st);
  else if (P <= 16) launch_token<16>(T, E, K, logits, srow, st);
  else launch_token<32>(T, E, K, logits, srow, st);
  MOE_CUDA_CHECK_LAUNCH();
  const int ethreads = (E + 31) / 32 * 32;
  aux_chunk_kernel<<<n_seq * cps, ethreads, 0, st>>>(srow, E, seq_len, cps, psum, pcnt);
  MOE_CUDA_CHECK_LAUNCH();
  int fthreads = 32;
  while (fthreads < E) fthreads <<= 1;
  aux_final_kernel<<<n_seq, fthreads, fthreads * sizeof(float), st>>>(
      psum, pcnt, E, K, seq_len, cps, alpha, loss, f_out, p_out);
  MOE_CUDA_CHECK_LAUNCH();
  return MOE_OK;
}

namespace moe {
namespace {

}  // namespace
}  // namespace moe
