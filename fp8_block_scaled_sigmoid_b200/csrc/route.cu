// Sigmoid router with bias-based, group-limited top-K selection.
// "DeepSeek_V3_Report：Annotation", eqs. (13)-(16), "Node-Limited Routing" and
// "Auxiliary-Loss-Free Load Balancing".
//
// Two kernels:
//  1. router_logits_kernel -- z = u . e^T as a bf16 x bf16 -> fp32 tcgen05 GEMM
//     (TMA-fed 128-byte-swizzled smem ring, accumulator in TMEM).  The gating
//     stays in high precision, never FP8.  K is split over blockIdx.z so that
//     a T=4096 batch still covers the SMs; the partial sums land in the
//     caller's workspace and are added in split order (deterministic).
//  2. route_select_kernel -- one warp per token, experts spread over lanes,
//     everything in registers and warp shuffles: sigmoid, biased scores,
//     group scores (sum of each group's top K/M), top-M groups, top-K experts
//     within them (ties to the lower index), gates from the raw scores.  With
//     a moe_balance_loss state it also computes the complementary
//     sequence-wise balance loss ("Complementary Sequence-Wise Auxiliary
//     Loss", eqs. (17)-(20)) from the same affinities.
#include <algorithm>
#include <climits>

#include "moe_common.cuh"

namespace moe {
namespace {

constexpr int kRtStages = 4;
constexpr int kRtBK = 64;                 // bf16 elements per stage (128 bytes)
constexpr int kRtABytes = 128 * 128;      // 128 rows x 128 bytes
constexpr int kRtThreads = 128;

struct RouterTiling {
  int m_tiles, n_tiles, BN, KB, splits, kb_per_split;
};

RouterTiling router_tiling(int T, int d, int E) {
  RouterTiling r;
  r.m_tiles = (T + 127) / 128;
  r.n_tiles = (E + 255) / 256;
  r.BN = ((E + r.n_tiles - 1) / r.n_tiles + 15) / 16 * 16;
  r.KB = d / kRtBK;
  const int tiles = std::max(1, r.m_tiles * r.n_tiles);
  // as many K splits as keep every CTA in one wave (a second, partial wave
  // would double the time)
  int splits = std::max(1, moe_num_sms() / tiles);
  splits = std::max(1, std::min(std::min(splits, 16), r.KB));
  r.kb_per_split = (r.KB + splits - 1) / splits;
  r.splits = (r.KB + r.kb_per_split - 1) / r.kb_per_split;  // no empty split
  return r;
}

size_t router_smem_bytes(int BN) {
  return 1024 + static_cast<size_t>(kRtStages) * (kRtABytes + BN * 128) + 256;
}

__global__ void __launch_bounds__(kRtThreads, 1) router_logits_kernel(
    const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
    float* __restrict__ part, int T, int E, int BN, int KB, int kb_per_split,
    int32_t* dev_err) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* sA = base;
  uint8_t* sB = base + kRtStages * kRtABytes;
  const int b_bytes = BN * 128;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + kRtStages * b_bytes);
  uint64_t* empty = full + kRtStages;
  uint64_t* done = empty + kRtStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * 128, n0 = blockIdx.y * BN, split = blockIdx.z;
  const int kb0 = split * kb_per_split;
  const int nkb = min(KB, kb0 + kb_per_split) - kb0;
  const uint32_t ncols = BN <= 32 ? 32u : (BN <= 64 ? 64u : (BN <= 128 ? 128u : 256u));

  if (threadIdx.x == 0) {
    for (int s = 0; s < kRtStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, ncols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  volatile int* abort_v = abort_flag;

  if (warp == 0 && lane == 0) {
    // TMA producer
    for (int i = 0; i < nkb; ++i) {
      const int s = i % kRtStages;
      const uint32_t ph = (i / kRtStages) & 1;
      if (!mbar_wait(&empty[s], ph ^ 1, abort_v, dev_err)) break;
      mbar_arrive_expect_tx(&full[s], kRtABytes + b_bytes);
      tma_load_2d(sA + s * kRtABytes, &tmA, &full[s], (kb0 + i) * kRtBK, m0);
      tma_load_2d(sB + s * b_bytes, &tmB, &full[s], (kb0 + i) * kRtBK, n0);
    }
  } else if (warp == 1 && lane == 0) {
    // single-thread MMA issuer: 4 x (K=16) per 64-element stage
    const uint32_t idesc = instr_desc(kFmtBF16, kFmtBF16, 128, BN);
    for (int i = 0; i < nkb; ++i) {
      const int s = i % kRtStages;
      const uint32_t ph = (i / kRtStages) & 1;
      if (!mbar_wait(&full[s], ph, abort_v, dev_err)) break;
      tc_fence_after();
      const uint64_t ad = smem_desc_sw128(smem_u32(sA + s * kRtABytes));
      const uint64_t bd = smem_desc_sw128(smem_u32(sB + s * b_bytes));
#pragma unroll
      for (int k = 0; k < 4; ++k)
        mma_f16(tmem, ad + 2 * k, bd + 2 * k, idesc, (i > 0 || k > 0) ? 1u : 0u);
      mma_commit(&empty[s]);
    }
    mma_commit(done);
  }
  __syncwarp();
  // warp-uniform outcome: the TMEM loads below are warp-collective
  const bool ok = __all_sync(0xffffffffu, mbar_wait(done, 0, abort_v, dev_err));
  tc_fence_after();
  if (ok && *abort_v == 0) {
    const int row = m0 + warp * 32 + lane;
    float* dst = part + (static_cast<int64_t>(split) * T + row) * E;
    for (int c = 0; c < BN; c += 16) {
      float v[16];
      tmem_ld16(tmem + (static_cast<uint32_t>(warp * 32) << 16) + c, v);
      tmem_ld_wait();
      if (row < T) {
        if (n0 + c + 16 <= E) {
#pragma unroll
          for (int j = 0; j < 4; ++j)
            reinterpret_cast<float4*>(dst + n0 + c)[j] =
                make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (n0 + c + j < E) dst[n0 + c + j] = v[j];
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, ncols);
}

// --------------------------------------------------------------- selection --
struct Cand {
  float v;  // biased score
  int i;    // expert
  float s;  // raw score
};

// Order-preserving unsigned key of a float score (+0 for both zeros): a > b
// as floats iff key(a) > key(b).
__device__ __forceinline__ uint32_t score_key(float v) {
  const uint32_t u = __float_as_uint(v == 0.f ? 0.f : v);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// The lane holding the warp's largest key; among equal keys the lowest lane
// (lanes own ascending experts, so the lowest expert).  One warp max
// (redux.sync) and one ballot.
__device__ __forceinline__ int warp_argmax_lane(uint32_t key) {
  const uint32_t m = __reduce_max_sync(0xffffffffu, key);
  return __ffs(__ballot_sync(0xffffffffu, key == m)) - 1;
}

__device__ __forceinline__ bool better(float v1, int i1, float v2, int i2) {
  return v1 > v2 || (v1 == v2 && i1 < i2);
}

__device__ __forceinline__ Cand warp_best(Cand c) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float v = __shfl_xor_sync(0xffffffffu, c.v, off);
    const int i = __shfl_xor_sync(0xffffffffu, c.i, off);
    const float s = __shfl_xor_sync(0xffffffffu, c.s, off);
    if (better(v, i, c.v, c.i)) {
      c.v = v;
      c.i = i;
      c.s = s;
    }
  }
  return c;
}

// The balance loss's per-token row ("Complementary Sequence-Wise Auxiliary
// Loss", eqs. (17)-(20)) from the raw affinities s this warp already holds:
// s' = s / sum_j s_j (the sum in a fixed order: each lane's experts in turn,
// then a butterfly over the lanes) and the raw top-K of s over all E experts
// (ties to the lower index, no bias, no group limit), as s' and a 0/1
// membership per expert.  The arithmetic and orders are those of
// moe_seq_balance_loss's token pass.
template <int P>
__device__ __forceinline__ void aux_token_row(const float (&s)[P], int E, int K, int lane,
                                              float* __restrict__ s_norm,
                                              uint8_t* __restrict__ member) {
  const int e0 = lane * P;
  float sum = 0.f;
#pragma unroll
  for (int i = 0; i < P; ++i)
    if (e0 + i < E) sum = __fadd_rn(sum, s[i]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sum = __fadd_rn(sum, __shfl_xor_sync(0xffffffffu, sum, off));
  // raw top-K: each lane keeps its best remaining expert (bi); a round takes
  // the warp's best (score descending, then lower expert) and only its owner
  // looks for its next best
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
    const int owner = warp_argmax_lane(bi < 0 ? 0u : score_key(bv));  // s > 0
    if (lane == owner) {
      taken |= 1u << bi;
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
  for (int i = 0; i < P; ++i)
    if (e0 + i < E) {
      s_norm[e0 + i] = __fdiv_rn(s[i], sum);
      member[e0 + i] = static_cast<uint8_t>((taken >> i) & 1u);
    }
}

constexpr int kSelThreads = 256;

// One token per warp; P = experts per lane (lane l owns experts l*P ..
// l*P+P-1).  Leaves the token's raw affinities in sc.
template <int P>
__device__ __forceinline__ void select_token(
    const float* __restrict__ part, int splits, int t, int T, int E, int G, int M, int K,
    const float* __restrict__ bias, int32_t* __restrict__ idx_out, float* __restrict__ gate_out,
    float* __restrict__ logits_out, int lane, float (&sc)[P]) {
  const int e0 = lane * P;
  const int gs = E / G;
  float beta[P], z[P];
  if (P % 4 == 0 && e0 + P <= E) {
    // whole lane in range: 16-byte loads (E % 16 == 0 keeps them aligned)
#pragma unroll
    for (int i = 0; i < P; i += 4) {
      float4 v = __ldg(reinterpret_cast<const float4*>(part + static_cast<int64_t>(t) * E + e0 + i));
      for (int sp = 1; sp < splits; ++sp) {
        const float4 w = __ldg(reinterpret_cast<const float4*>(
            part + (static_cast<int64_t>(sp) * T + t) * E + e0 + i));
        v = make_float4(__fadd_rn(v.x, w.x), __fadd_rn(v.y, w.y), __fadd_rn(v.z, w.z),
                        __fadd_rn(v.w, w.w));
      }
      z[i] = v.x;
      z[i + 1] = v.y;
      z[i + 2] = v.z;
      z[i + 3] = v.w;
      if (logits_out)
        *reinterpret_cast<float4*>(logits_out + static_cast<int64_t>(t) * E + e0 + i) = v;
    }
  } else {
#pragma unroll
    for (int i = 0; i < P; ++i) {
      const int e = e0 + i;
      z[i] = 0.f;
      if (e < E) {
        float v = part[static_cast<int64_t>(t) * E + e];
        for (int sp = 1; sp < splits; ++sp)
          v = __fadd_rn(v, part[(static_cast<int64_t>(sp) * T + t) * E + e]);
        if (logits_out) logits_out[static_cast<int64_t>(t) * E + e] = v;
        z[i] = v;
      }
    }
  }
#pragma unroll
  for (int i = 0; i < P; ++i) {
    const int e = e0 + i;
    beta[i] = -INFINITY;
    sc[i] = 0.f;
    if (e < E) {
      sc[i] = __fdiv_rn(1.0f, __fadd_rn(1.0f, expf(-z[i])));
      beta[i] = __fadd_rn(sc[i], __ldg(bias + e));
    }
  }

  // groups a token may use (bit g set = allowed)
  uint32_t allowed = 0xffffffffu;
  if (M < G) {
    const int n_top = K / M;
    const int L = gs / P;  // lanes per group when a group spans whole lanes
    if (gs % P == 0 && L > 0 && L <= 32 && (L & (L - 1)) == 0) {
      // every group sits on L consecutive lanes: all groups at once with
      // segmented (xor < L) reductions
      uint32_t tk = 0;
      float sum = 0.f;
      for (int r = 0; r < n_top; ++r) {
        Cand c{-INFINITY, INT_MAX, 0.f};
#pragma unroll
        for (int i = 0; i < P; ++i) {
          const int e = e0 + i;
          if (e < E && !((tk >> i) & 1u) && better(beta[i], e, c.v, c.i)) {
            c.v = beta[i];
            c.i = e;
          }
        }
        for (int off = 1; off < L; off <<= 1) {
          const float v = __shfl_xor_sync(0xffffffffu, c.v, off);
          const int i = __shfl_xor_sync(0xffffffffu, c.i, off);
          if (better(v, i, c.v, c.i)) {
            c.v = v;
            c.i = i;
          }
        }
        if (c.i / P == lane) tk |= 1u << (c.i - e0);
        sum = __fadd_rn(sum, c.v);
      }
      const int my_g = lane / L;
      int rank = 0;
      for (int g = 0; g < G; ++g) {
        const float v = __shfl_sync(0xffffffffu, sum, g * L);
        if (better(v, g, sum, my_g)) ++rank;
      }
      const uint32_t lead = __ballot_sync(0xffffffffu, (lane % L) == 0 && my_g < G && rank < M);
      allowed = 0;
      for (int g = 0; g < G; ++g) allowed |= ((lead >> (g * L)) & 1u) << g;
    } else {
      float my_score = -INFINITY;
      for (int g = 0; g < G; ++g) {
        uint32_t tk = 0;
        float sum = 0.f;
        for (int r = 0; r < n_top; ++r) {
          Cand c{-INFINITY, INT_MAX, 0.f};
#pragma unroll
          for (int i = 0; i < P; ++i) {
            const int e = e0 + i;
            if (e < E && e / gs == g && !((tk >> i) & 1u) && better(beta[i], e, c.v, c.i)) {
              c.v = beta[i];
              c.i = e;
            }
          }
          c = warp_best(c);
          if (c.i / P == lane) tk |= 1u << (c.i - e0);
          sum = __fadd_rn(sum, c.v);
        }
        if (lane == g) my_score = sum;
      }
      int rank = 0;
      for (int g = 0; g < G; ++g) {
        const float v = __shfl_sync(0xffffffffu, my_score, g);
        if (better(v, g, my_score, lane)) ++rank;
      }
      allowed = __ballot_sync(0xffffffffu, lane < G && rank < M);
    }
  }

  // experts of groups the token may not use drop out of the selection
#pragma unroll
  for (int i = 0; i < P; ++i)
    if (e0 + i < E && !((allowed >> ((e0 + i) / gs)) & 1u)) beta[i] = -INFINITY;

  // each lane keeps its best remaining candidate (local index bi, biased
  // score bv, raw score bs); a round takes the warp's best (biased score
  // descending, then lower expert): one warp max over the order-preserving
  // keys and a ballot; only the lane that owned it looks for its next best
  uint32_t taken = 0;
  int bi = -1;
  float bv = -INFINITY, bs = 0.f;
#pragma unroll
  for (int i = 0; i < P; ++i)
    if (e0 + i < E && (bi < 0 || beta[i] > bv)) {
      bi = i;
      bv = beta[i];
      bs = sc[i];
    }
  float ssum = 0.f, my_s = 0.f;
  int my_idx = 0;
  for (int k = 0; k < K; ++k) {
    const int owner = warp_argmax_lane(bi < 0 ? 0u : score_key(bv));
    const int ex = owner * P + __shfl_sync(0xffffffffu, bi, owner);
    const float s_win = __shfl_sync(0xffffffffu, bs, owner);
    if (lane == owner) {
      taken |= 1u << bi;
      bi = -1;
      bv = -INFINITY;
#pragma unroll
      for (int i = 0; i < P; ++i)
        if (e0 + i < E && !((taken >> i) & 1u) && (bi < 0 || beta[i] > bv)) {
          bi = i;
          bv = beta[i];
          bs = sc[i];
        }
    }
    ssum = __fadd_rn(ssum, s_win);
    if (lane == k) {
      my_idx = ex;
      my_s = s_win;
    }
  }
  if (lane < K) {
    idx_out[static_cast<int64_t>(t) * K + lane] = my_idx;
    gate_out[static_cast<int64_t>(t) * K + lane] = __fdiv_rn(my_s, ssum);
  }
}

// Selection, and with the balance loss (has_aux) its sums: each warp writes
// its token's s' and raw top-K membership to shared memory; each thread then
// adds one expert's 8 values (s' in fixed point, 2^32 units) and adds them to
// the sequence's sums with integer atomics, so the totals do not depend on
// the order of the CTAs.  The CTA that finds itself last of its sequence
// (a counter taken after a fence) forms f, P and the loss from the totals,
// which it reads and zeroes in one exchange, and resets the counter.
constexpr float kAuxFix = 4294967296.0f;  // 2^32

template <int P>
__global__ void __launch_bounds__(kSelThreads) route_select_kernel(
    const float* __restrict__ part, int splits, int T, int E, int G, int M, int K,
    const float* __restrict__ bias, int32_t* __restrict__ idx_out, float* __restrict__ gate_out,
    float* __restrict__ logits_out, moe_balance_loss aux, int has_aux) {
  extern __shared__ float aux_sm[];  // [8][E] s', then [8][E] membership bytes
  __shared__ float warp_term[kSelThreads / 32];
  __shared__ int is_last;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int t = blockIdx.x * (kSelThreads / 32) + w;
  float sc[P];
  if (t < T)
    select_token<P>(part, splits, t, T, E, G, M, K, bias, idx_out, gate_out, logits_out, lane, sc);
  if (!has_aux) return;  // the same for the whole grid
  float* sp = aux_sm + w * E;
  uint8_t* sm8 = reinterpret_cast<uint8_t*>(aux_sm + (kSelThreads / 32) * E) + w * E;
  if (t < T) {
    aux_token_row<P>(sc, E, K, lane, sp, sm8);
  } else {
    for (int e = lane; e < E; e += 32) {
      sp[e] = 0.f;
      sm8[e] = 0;
    }
  }
  __syncthreads();
  const int S = aux.seq_len;
  const int q = blockIdx.x * (kSelThreads / 32) / S;  // 8 | S: the CTA's tokens share q
  const uint8_t* mem = reinterpret_cast<const uint8_t*>(aux_sm + (kSelThreads / 32) * E);
  unsigned long long* acc = reinterpret_cast<unsigned long long*>(aux.acc) + static_cast<int64_t>(q) * E;
  int32_t* cnt = aux.cnt + static_cast<int64_t>(q) * E;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    unsigned long long a = 0;
    int c = 0;
#pragma unroll
    for (int j = 0; j < kSelThreads / 32; ++j) {
      a += static_cast<unsigned long long>(__float2ll_rn(__fmul_rn(aux_sm[j * E + e], kAuxFix)));
      c += mem[j * E + e];
    }
    if (a) atomicAdd(acc + e, a);
    if (c) atomicAdd(cnt + e, c);
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0)
    is_last = atomicAdd(aux.done + q, 1) == S / (kSelThreads / 32) - 1;
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  // f_i = E/(K S) * count, P_i = sum / S; term over this thread's experts in
  // ascending order, then the warps' butterflies and the warp sums in order
  float term = 0.f;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const unsigned long long a = atomicExch(acc + e, 0ull);
    const int c = atomicExch(cnt + e, 0);
    const float f = __fdiv_rn(static_cast<float>(E) * static_cast<float>(c),
                              static_cast<float>(K) * static_cast<float>(S));
    const float pv = static_cast<float>(static_cast<double>(a) / (4294967296.0 * S));
    if (aux.f) aux.f[static_cast<int64_t>(q) * E + e] = f;
    if (aux.P) aux.P[static_cast<int64_t>(q) * E + e] = pv;
    term = __fadd_rn(term, __fmul_rn(f, pv));
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) term = __fadd_rn(term, __shfl_xor_sync(0xffffffffu, term, off));
  if (lane == 0) warp_term[w] = term;
  __syncthreads();
  if (threadIdx.x == 0) {
    float tot = 0.f;
#pragma unroll
    for (int i = 0; i < kSelThreads / 32; ++i) tot = __fadd_rn(tot, warp_term[i]);
    aux.loss[q] = __fmul_rn(aux.alpha, tot);
    aux.done[q] = 0;
  }
}

template <int P>
void launch_select(int blocks, cudaStream_t st, const float* part, int splits, int T, int E,
                   int G, int M, int K, const float* bias, int32_t* idx, float* gate,
                   float* logits, const moe_balance_loss* aux) {
  // 8 tokens x E x (4 + 1) bytes <= 40 KB for E <= 1024
  const size_t sm = aux ? static_cast<size_t>(kSelThreads / 32) * E * 5 : 0;
  moe_balance_loss a{};
  if (aux) a = *aux;
  route_select_kernel<P><<<blocks, kSelThreads, sm, st>>>(part, splits, T, E, G, M, K, bias, idx,
                                                           gate, logits, a, aux ? 1 : 0);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace moe

extern "C" moe_status moe_route_workspace_size(int T, int d, int E, size_t* bytes) {
  if (!bytes || T < 0 || d <= 0 || E <= 0) return MOE_ERR_INVALID_ARG;
  if (d % 128 != 0) return MOE_ERR_SHAPE;
  const moe::RouterTiling r = moe::router_tiling(T, d, E);
  const size_t b = static_cast<size_t>(r.splits) * T * E * sizeof(float);
  *bytes = (b + 255) / 256 * 256;
  return MOE_OK;
}

extern "C" moe_status moe_route(const uint16_t* u, int64_t ldu, const uint16_t* centroids,
                                const float* bias, int T, int d, int E, int G, int M, int K,
                                int32_t* topk_idx, float* topk_gate, float* logits_out,
                                const moe_balance_loss* aux, void* ws, size_t ws_bytes,
                                int32_t* dev_err, moe_stream_t stream) {
  using namespace moe;
  if (T < 0 || d <= 0 || E <= 0 || G <= 0 || M <= 0 || K <= 0) return MOE_ERR_INVALID_ARG;
  if (d % 128 != 0 || E % 16 != 0 || E % G != 0 || M > G || K > E || ldu < d) return MOE_ERR_SHAPE;
  if (E > 1024 || G > 32 || K > 32) return MOE_ERR_UNSUPPORTED;
  if (M < G && (K % M != 0 || M * (E / G) < K)) return MOE_ERR_SHAPE;
  if (aux) {
    if (aux->seq_len <= 0) return MOE_ERR_INVALID_ARG;
    if (aux->seq_len % 8 != 0 || T % aux->seq_len != 0 || aux->seq_len > (1 << 30))
      return MOE_ERR_SHAPE;
  }
  if (T == 0) return MOE_OK;
  if (!u || !centroids || !bias || !topk_idx || !topk_gate) return MOE_ERR_INVALID_ARG;
  if (aux && (!aux->acc || !aux->cnt || !aux->done || !aux->loss)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(u) || !aligned16(centroids) || ldu % 8 != 0) return MOE_ERR_ALIGN;
  if (aux && (reinterpret_cast<uintptr_t>(aux->acc) & 7u) != 0) return MOE_ERR_ALIGN;
  size_t need = 0;
  moe_route_workspace_size(T, d, E, &need);
  if (ws_bytes < need || (!ws && need)) return MOE_ERR_WORKSPACE;
  if (!aligned16(ws)) return MOE_ERR_ALIGN;

  const RouterTiling r = router_tiling(T, d, E);
  CUtensorMap tmA, tmB;
  if (!moe_make_tmap_2d(&tmA, u, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, d, T, ldu * 2, kRtBK, 128) ||
      !moe_make_tmap_2d(&tmB, centroids, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, d, E, d * 2, kRtBK,
                        r.BN))
    return MOE_ERR_CUDA;
  const size_t smem = router_smem_bytes(r.BN);
  static int configured = 0;
  if (!configured) {
    if (cudaFuncSetAttribute(router_logits_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(router_smem_bytes(256))) != cudaSuccess)
      return MOE_ERR_CUDA;
    configured = 1;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float* part = static_cast<float*>(ws);
  dim3 grid(r.m_tiles, r.n_tiles, r.splits);
  router_logits_kernel<<<grid, kRtThreads, smem, st>>>(tmA, tmB, part, T, E, r.BN, r.KB,
                                                       r.kb_per_split, dev_err);
  MOE_CUDA_CHECK_LAUNCH();

  const int blocks = (T + kSelThreads / 32 - 1) / (kSelThreads / 32);
  const int P = (E + 31) / 32;
  if (P <= 1) launch_select<1>(blocks, st, part, r.splits, T, E, G, M, K, bias, topk_idx, topk_gate, logits_out, aux);
  else if (P <= 2) launch_select<2>(blocks, st, part, r.splits, T, E, G, M, K, bias, topk_idx, topk_gate, logits_out, aux);
  else if (P <= 4) launch_select<4>(blocks, st, part, r.splits, T, E, G, M, K, bias, topk_idx, topk_gate, logits_out, aux);
  else if (P <= 8) launch_select<8>(blocks, st, part, r.splits, T, E, G, M, K, bias, topk_idx, topk_gate, logits_out, aux);
  else if (P <= 12) launch_select<12>(blocks, st, part, r.splits, T, E, G, M, K, bias, topk_idx, topk_gate, logits_out, aux);
  else if (P <= 16) launch_select<16>(blocks, st, part, r.splits, T, E, G, M, K, bias, topk_idx, topk_gate, logits_out, aux);
  else launch_select<32>(blocks, st, part, r.splits, T, E, G, M, K, bias, topk_idx, topk_gate, logits_out, aux);
  MOE_CUDA_CHECK_LAUNCH();
  return MOE_OK;
}
