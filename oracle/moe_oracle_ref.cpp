// CPU oracle of the DeepSeekMoE layer forward with FP8 block-scaled expert
// GEMMs, in plain single-threaded C++ with fp64 accumulation.
//
// TEST INFRASTRUCTURE ONLY.  Nothing on the product path links or loads this
// file: only the tests, the smoke check and the benchmark's CPU-baseline and
// reference legs do (through oracle/cpp_oracle.py).  It shares no code,
// header, table or constant with the CUDA library.
//
// Pages (titles):
//   [ANN] "DeepSeek_V3_Report：Annotation" (annotated translation of the V3
//         report): eqs. (12)-(20), "Node-Limited Routing",
//         "Auxiliary-Loss-Free Load Balancing", "Fine-Grained Quantization",
//         "Online Quantization", "Low-Precision Communication", "No
//         Token-Dropping", the SwiGLU operator notes.
//   [BLOG] "从MLA到MTP，从FP8到DualPipe：DeepSeek-V3——一场关于效率、智能与工程哲学的“全栈式”架构革命",
//         1.2.2 (the bias update's "overloaded" = above the mean load).
//
// Readings where the pages leave a step open (the same as the numpy oracle's):
//   * the stored scale is the fp32 dequantisation multiplier
//     fl32(max(amax, 1e-4) / 448); the code is E4M3(fl32(x / scale)),
//     nearest, ties to the even mantissa, saturating at +-448;
//   * a power-of-two scale is that fp32 scale rounded up to a power of two;
//   * group score = the sum of the K/M largest biased scores of the group;
//   * every top-k breaks ties toward the lower index; the selected experts
//     are listed by biased score descending, then index ascending;
//   * bias update: sign(c_i - T*K/E) with sign(0) = 0, in fp32;
//   * Swish beta = 1; the shared expert has gate 1;
//   * the balance loss's TopK is over the raw affinities of all experts.
//
// Every function is pinned by the tests in tests/test_oracle_*.py, which run
// each pin against this oracle and against the numpy oracle, and cross-check
// the two.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

namespace {

// ------------------------------------------------------------ E4M3 format
// [ANN] "Mantissa over Exponents" (E4M3 everywhere) and "Online
// Quantization" (largest magnitude 448).  A code is sign | exponent field
// (4 bits, bias 7) | mantissa (3 bits); exponent field 0 holds the
// subnormals m * 2^-9; field 15 with mantissa 7 is NaN; there is no
// infinity.
double decode_code(uint8_t c) {
  const int sign = (c >> 7) & 1;
  const int ef = (c >> 3) & 15;
  const int mf = c & 7;
  double v;
  if (ef == 15 && mf == 7) return std::nan("");
  if (ef == 0) v = std::ldexp(static_cast<double>(mf), -9);
  else v = std::ldexp(1.0 + mf / 8.0, ef - 7);
  return sign ? -v : v;
}

// The 127 finite non-negative magnitudes, indexed by code 0x00..0x7E (the
// codes of one sign increase with the magnitude).
struct Magnitudes {
  double v[127];
  Magnitudes() {
    for (int c = 0; c < 127; ++c) v[c] = decode_code(static_cast<uint8_t>(c));
  }
};
const Magnitudes kMag;

// Nearest representable magnitude by search over the code table: between the
// two neighbours the closer one wins; at an exact midpoint the code with the
// even mantissa (even code) wins; anything from 448 up saturates to 0x7E.
uint8_t encode_value(double x) {
  const bool neg = std::signbit(x);
  const double a = std::fabs(x);
  uint8_t code;
  if (a >= kMag.v[126]) {
    code = 126;
  } else {
    int hi = static_cast<int>(std::upper_bound(kMag.v, kMag.v + 127, a) - kMag.v);  // v[hi] > a
    int lo = hi - 1;                                                              // v[lo] <= a
    const double dlo = a - kMag.v[lo], dhi = kMag.v[hi] - a;
    if (dlo < dhi) code = static_cast<uint8_t>(lo);
    else if (dhi < dlo) code = static_cast<uint8_t>(hi);
    else code = static_cast<uint8_t>((lo & 1) == 0 ? lo : hi);
  }
  return neg ? static_cast<uint8_t>(code | 0x80) : code;
}

// ------------------------------------------------------ online quantisation
// [ANN] "Online Quantization": the scale comes from the tile's own max |x|.
float scale_of(float amax) {
  const float eps = 1e-4f;
  const float a = amax > eps ? amax : eps;
  return a / 448.0f;  // IEEE fp32 division
}

float pow2_up(float s) {
  int e = 0;
  const double m = std::frexp(static_cast<double>(s), &e);  // s = m * 2^e, m in [0.5, 1)
  return static_cast<float>(m == 0.5 ? static_cast<double>(s) : std::ldexp(1.0, e));
}

double sigmoid_of(double z) { return 1.0 / (1.0 + std::exp(-z)); }

// Positions 0..n-1 ordered by value descending, then index ascending.
std::vector<int> order_desc(const double* v, const int* ids, int n) {
  std::vector<int> p(n);
  for (int i = 0; i < n; ++i) p[i] = i;
  std::sort(p.begin(), p.end(), [&](int x, int y) {
    if (v[x] != v[y]) return v[x] > v[y];
    return ids[x] < ids[y];
  });
  return p;
}

}  // namespace

extern "C" {

int orc_version() { return 1; }

void orc_e4m3_decode(const uint8_t* codes, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = decode_code(codes[i]);
}

// Returns 1 (and writes nothing more) on a NaN input.
int orc_e4m3_encode(const double* v, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) {
    if (std::isnan(v[i])) return 1;
    out[i] = encode_value(v[i]);
  }
  return 0;
}

void orc_pow2_ceil(const float* s, int64_t n, float* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = pow2_up(s[i]);
}

// 1x128 tiles along the rows of x [rows][cols] (cols % 128 == 0): one scale
// per (row, tile).  [ANN] "Fine-Grained Quantization".
void orc_quant_1x128(const float* x, int64_t rows, int64_t cols, int pow2, uint8_t* q,
                     float* scale) {
  const int64_t tiles = cols / 128;
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t j = 0; j < tiles; ++j) {
      const float* p = x + r * cols + j * 128;
      float amax = 0.0f;
      for (int k = 0; k < 128; ++k) amax = std::max(amax, std::fabs(p[k]));
      float s = scale_of(amax);
      if (pow2) s = pow2_up(s);
      scale[r * tiles + j] = s;
      for (int k = 0; k < 128; ++k) {
        const float y = p[k] / s;  // fp32 division
        q[r * cols + j * 128 + k] = encode_value(static_cast<double>(y));
      }
    }
  }
}

// 128x128 blocks of w [rows][cols] (cols % 128 == 0; a ragged last row block
// is allowed): one scale per block.
void orc_quant_128x128(const float* w, int64_t rows, int64_t cols, int pow2, uint8_t* q,
                       float* scale) {
  const int64_t rb = (rows + 127) / 128, cb = cols / 128;
  for (int64_t bi = 0; bi < rb; ++bi) {
    const int64_t r0 = bi * 128, r1 = std::min(rows, r0 + 128);
    for (int64_t bj = 0; bj < cb; ++bj) {
      float amax = 0.0f;
      for (int64_t r = r0; r < r1; ++r)
        for (int64_t c = bj * 128; c < bj * 128 + 128; ++c)
          amax = std::max(amax, std::fabs(w[r * cols + c]));
      float s = scale_of(amax);
      if (pow2) s = pow2_up(s);
      scale[bi * cb + bj] = s;
      for (int64_t r = r0; r < r1; ++r)
        for (int64_t c = bj * 128; c < bj * 128 + 128; ++c)
          q[r * cols + c] = encode_value(static_cast<double>(w[r * cols + c] / s));
    }
  }
}

// x = decode(q) * scale; block_rows = 1 for 1x128 tiles, 128 for 128x128
// blocks (scale [ceil(rows/block_rows)][cols/128]).
void orc_dequant(const uint8_t* q, const float* scale, int64_t rows, int64_t cols,
                 int block_rows, double* out) {
  const int64_t cb = cols / 128;
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t c = 0; c < cols; ++c)
      out[r * cols + c] =
          decode_code(q[r * cols + c]) * static_cast<double>(scale[(r / block_rows) * cb + c / 128]);
}

// ------------------------------------------------------------------ router
// [ANN] eq. (15): z = u_t . e_i, in fp64 from the (bf16-valued) inputs.
void orc_router_logits(const float* u, const float* cent, int64_t T, int64_t E, int64_t d,
                       double* z) {
  for (int64_t t = 0; t < T; ++t)
    for (int64_t i = 0; i < E; ++i) {
      double acc = 0.0;
      for (int64_t j = 0; j < d; ++j)
        acc += static_cast<double>(u[t * d + j]) * static_cast<double>(cent[i * d + j]);
      z[t * E + i] = acc;
    }
}

void orc_sigmoid(const double* z, int64_t n, double* s) {
  for (int64_t i = 0; i < n; ++i) s[i] = sigmoid_of(z[i]);
}

// [ANN] eqs. (13)-(16) and "Node-Limited Routing": s = Sigmoid(z); beta =
// s + b selects; at most M of the G contiguous expert groups, ranked by the
// sum of their K/M largest beta (raw_group_score ranks them by s instead --
// a variant kept only so the tests can show it differs); the top K of beta
// among the allowed experts; gates = s of the chosen / their sum.
// Returns 1 on inconsistent sizes.
int orc_route_select(const double* z, const double* bias, int64_t T, int E, int G, int M, int K,
                     int raw_group_score, int32_t* idx, double* gate, double* s_out,
                     double* beta_out, double* k_margin, double* g_margin, double* o_margin) {
  if (G <= 0 || E % G != 0 || M <= 0 || M > G || K <= 0 || K > E) return 1;
  const int gs = E / G;
  const bool limited = M < G;
  if (limited && K % M != 0) return 1;
  const int n_top = limited ? K / M : 0;
  std::vector<double> s(E), beta(E), gscore(G), cand_b;
  std::vector<int> gid(G), cand;
  for (int g = 0; g < G; ++g) gid[g] = g;
  for (int64_t t = 0; t < T; ++t) {
    for (int i = 0; i < E; ++i) {
      s[i] = sigmoid_of(z[t * E + i]);
      beta[i] = s[i] + bias[i];
      if (s_out) s_out[t * E + i] = s[i];
      if (beta_out) beta_out[t * E + i] = beta[i];
    }
    std::vector<char> allowed(E, 1);
    double gm = INFINITY;
    if (limited) {
      for (int g = 0; g < G; ++g) {
        std::vector<double> v(gs);
        for (int j = 0; j < gs; ++j) v[j] = raw_group_score ? s[g * gs + j] : beta[g * gs + j];
        std::sort(v.begin(), v.end(), [](double a, double b) { return a > b; });
        double acc = 0.0;
        for (int j = 0; j < n_top; ++j) acc += v[j];
        gscore[g] = acc;
      }
      const std::vector<int> go = order_desc(gscore.data(), gid.data(), G);
      gm = gscore[go[M - 1]] - gscore[go[M]];
      std::fill(allowed.begin(), allowed.end(), 0);
      for (int j = 0; j < M; ++j)
        for (int i = go[j] * gs; i < (go[j] + 1) * gs; ++i) allowed[i] = 1;
    }
    cand.clear();
    cand_b.clear();
    for (int i = 0; i < E; ++i)
      if (allowed[i]) {
        cand.push_back(i);
        cand_b.push_back(beta[i]);
      }
    const int nc = static_cast<int>(cand.size());
    const std::vector<int> co = order_desc(cand_b.data(), cand.data(), nc);
    double ssum = 0.0;
    for (int k = 0; k < K; ++k) ssum += s[cand[co[k]]];
    double om = INFINITY;
    for (int k = 0; k < K; ++k) {
      const int e = cand[co[k]];
      idx[t * K + k] = e;
      gate[t * K + k] = s[e] / ssum;
      if (k > 0) om = std::min(om, cand_b[co[k - 1]] - cand_b[co[k]]);
    }
    if (k_margin) k_margin[t] = nc > K ? cand_b[co[K - 1]] - cand_b[co[K]] : INFINITY;
    if (g_margin) g_margin[t] = gm;
    if (o_margin) o_margin[t] = om;
  }
  return 0;
}

// ------------------------------------------------------------- permutation
// Stands in for the dispatch ([ANN] "Low-Precision Communication": quantise,
// then dispatch; "No Token-Dropping"): pairs (t, k) grouped by expert,
// ascending token inside an expert.  Returns 1 on an index outside [0, E).
int orc_permute(const int32_t* idx, int64_t T, int K, int E, int32_t* counts, int32_t* offsets,
                int32_t* src_row, int32_t* dst_of) {
  for (int e = 0; e < E; ++e) counts[e] = 0;
  for (int64_t p = 0; p < T * K; ++p) {
    if (idx[p] < 0 || idx[p] >= E) return 1;
    ++counts[idx[p]];
  }
  offsets[0] = 0;
  for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
  std::vector<int32_t> next(offsets, offsets + E);
  for (int64_t t = 0; t < T; ++t)          // tokens in order: a stable fill
    for (int k = 0; k < K; ++k) {
      const int32_t slot = next[idx[t * K + k]]++;
      src_row[slot] = static_cast<int32_t>(t);
      dst_of[t * K + k] = slot;
    }
  return 0;
}

// ----------------------------------------------------- block-scaled GEMM
// [ANN] "Fine-Grained Quantization" / "Increasing Accumulation Precision":
// per segment g (rows offsets[g] .. offsets[g+1]) and output column n,
//   D[m][n] = sum_kb (sa[m][kb] * sb[g][n/128][kb]) * sum_{k in kb} deq(a[m][k]) deq(b[g][n][k])
// in fp64, each inner sum in ascending k and the outer in ascending kb.  The
// loops run over the segment's rows innermost (independent sums side by
// side); no sum is reordered.
void orc_grouped_gemm(const uint8_t* aq, const float* sa, int64_t rows, const uint8_t* bq,
                      const float* sb, int groups, int64_t N, int64_t K, const int32_t* offsets,
                      double* out) {
  const int64_t KB = K / 128;
  double dec[256];
  for (int c = 0; c < 256; ++c) dec[c] = decode_code(static_cast<uint8_t>(c));
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t n = 0; n < N; ++n) out[r * N + n] = 0.0;
  for (int g = 0; g < groups; ++g) {
    const int64_t r0 = offsets[g], r1 = offsets[g + 1], m = r1 - r0;
    if (m <= 0) continue;
    std::vector<double> at(static_cast<size_t>(K * m));  // decoded A of the segment, [k][row]
    for (int64_t i = 0; i < m; ++i)
      for (int64_t k = 0; k < K; ++k) at[k * m + i] = dec[aq[(r0 + i) * K + k]];
    std::vector<double> acc(m), part(m);
    const uint8_t* bg = bq + static_cast<int64_t>(g) * N * K;
    const float* sbg = sb + static_cast<int64_t>(g) * (N / 128) * KB;
    for (int64_t n = 0; n < N; ++n) {
      std::fill(acc.begin(), acc.end(), 0.0);
      for (int64_t kb = 0; kb < KB; ++kb) {
        std::fill(part.begin(), part.end(), 0.0);
        for (int64_t k = kb * 128; k < kb * 128 + 128; ++k) {
          const double w = dec[bg[n * K + k]];
          const double* a = at.data() + k * m;
          for (int64_t i = 0; i < m; ++i) part[i] += a[i] * w;
        }
        const double fb = static_cast<double>(sbg[(n / 128) * KB + kb]);
        for (int64_t i = 0; i < m; ++i)
          acc[i] += (static_cast<double>(sa[(r0 + i) * KB + kb]) * fb) * part[i];
      }
      for (int64_t i = 0; i < m; ++i) out[(r0 + i) * N + n] = acc[i];
    }
  }
}

// ------------------------------------------------------------------ SwiGLU
// [ANN] SwiGLU operator notes: h = Swish(gate) * up, Swish(x) = x *
// Sigmoid(x) (beta = 1).  gu [rows][2I] holds 128-wide gate blocks followed
// by the matching up blocks: columns 256j..256j+127 are gate channels
// 128j.., the next 128 the up channels.
void orc_swiglu(const double* gu, int64_t rows, int64_t I, double* h) {
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t c = 0; c < I; ++c) {
      const int64_t j = c / 128, o = c % 128;
      const double g = gu[r * 2 * I + 256 * j + o];
      const double u = gu[r * 2 * I + 256 * j + 128 + o];
      h[r * I + c] = g / (1.0 + std::exp(-g)) * u;
    }
}

// ----------------------------------------------------------------- combine
// [ANN] eq. (12): out_t = u_t + FFN_shared(u_t) + sum_k g_{t,k} FFN_{e_k}(u_t),
// added in that order, k ascending.  Ys may be NULL (no shared expert).
void orc_combine(const double* Y, const int32_t* dst_of, const double* gate, const double* Ys,
                 const double* u, int64_t T, int K, int64_t d, double* out) {
  for (int64_t t = 0; t < T; ++t)
    for (int64_t j = 0; j < d; ++j) {
      double acc = u[t * d + j];
      if (Ys) acc += Ys[t * d + j];
      for (int k = 0; k < K; ++k) acc += gate[t * K + k] * Y[dst_of[t * K + k] * d + j];
      out[t * d + j] = acc;
    }
}

// ------------------------------------------------------------- bias update
// [ANN] "Auxiliary-Loss-Free Load Balancing"; [BLOG] 1.2.2: b_i -= gamma when
// expert i's load is above the batch mean T*K/E, += gamma below it.
void orc_bias_update(const int32_t* counts, int E, int64_t T, int K, float gamma,
                     const float* bias, float* out) {
  const double mean = static_cast<double>(T) * K / E;
  for (int i = 0; i < E; ++i) {
    const double c = counts[i];
    const double sgn = c > mean ? 1.0 : (c < mean ? -1.0 : 0.0);
    out[i] = static_cast<float>(static_cast<double>(bias[i]) - static_cast<double>(gamma) * sgn);
  }
}

// ---------------------------------------------- sequence-wise balance loss
// [ANN] "Complementary Sequence-Wise Auxiliary Loss", eqs. (17)-(20), per
// sequence of seq_len tokens: f_i = E/(K*seq_len) * #{t : s_{i,t} in
// TopK(s_t, K)}, P_i = mean over t of s_{i,t} / sum_j s_{j,t}, loss = alpha
// * sum_i f_i P_i.  Returns 1 on inconsistent sizes.
int orc_seq_balance_loss(const double* z, int64_t T, int E, int K, int64_t seq_len, double alpha,
                         double* loss, double* f, double* P, double* k_margin) {
  if (seq_len <= 0 || T % seq_len != 0 || K <= 0 || K > E) return 1;
  const int64_t n_seq = T / seq_len;
  std::vector<double> s(E);
  std::vector<int> ids(E);
  for (int i = 0; i < E; ++i) ids[i] = i;
  for (int64_t q = 0; q < n_seq; ++q) {
    std::vector<double> cnt(E, 0.0), psum(E, 0.0);
    for (int64_t t = q * seq_len; t < (q + 1) * seq_len; ++t) {
      double tot = 0.0;
      for (int i = 0; i < E; ++i) {
        s[i] = sigmoid_of(z[t * E + i]);
        tot += s[i];
      }
      const std::vector<int> o = order_desc(s.data(), ids.data(), E);
      for (int k = 0; k < K; ++k) cnt[o[k]] += 1.0;
      if (k_margin) k_margin[t] = K < E ? s[o[K - 1]] - s[o[K]] : INFINITY;
      for (int i = 0; i < E; ++i) psum[i] += s[i] / tot;
    }
    double l = 0.0;
    for (int i = 0; i < E; ++i) {
      const double fi = static_cast<double>(E) / (static_cast<double>(K) * seq_len) * cnt[i];
      const double pi = psum[i] / seq_len;
      if (f) f[q * E + i] = fi;
      if (P) P[q * E + i] = pi;
      l += fi * pi;
    }
    loss[q] = alpha * l;
  }
  return 0;
}

}  // extern "C"
