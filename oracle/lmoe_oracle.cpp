// CPU oracle of the LatentMoE layer forward pass.
//
// TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or
// load this file: only the tests, the smoke check and the benchmark's CPU
// baseline use it.  It shares no code, header, table or helper with the CUDA
// library; its only common ground with it is the seeded input generator,
// which produces the bytes both sides read.
//
// What it computes (LatentMoE paper, arXiv 2601.18089, Section 3, Eq. (1)
// and Eq. (2)): for every token x (a row of width d)
//
//   logits   = x . Wg + b                         router on the full-width x
//   S        = the k experts first under the order (logit desc, index asc)
//   w_j      = exp(l_j - l_0) / sum_{j'} exp(l_j' - l_0)   over the k chosen
//              (variants: the softmax over all N logits taken at the chosen
//              experts; a bias that only steers the selection)
//   z        = x . Wdown                          down-projection d -> l
//   y_j      = act(z . W1[e_j]) . W2[e_j]         expert e_j in latent width
//   comb     = sum_j w_j y_j                      gate-weighted sum, slot order
//   u        = comb . Wup                         up-projection l -> d
//   s        = act(x . Ws1) . Ws2                 shared expert in width d
//   out      = x + u + s                          residual add
//
// with act one of SiLU (non-gated), SwiGLU (columns [0,m) of FC1 are the
// SiLU gate, columns [m,2m) the linear half) or squared ReLU (non-gated).
// Under the projection-skip flag (the paper's standard MoE, Table 1 first
// row) l == d and z = x, u = comb.
//
// Precision: every dot product is accumulated in float64, sequentially along
// its reduction index; bf16 and fp32 inputs are widened exactly.  The one
// decision taken on floating point -- which experts are selected -- is taken
// on fp32 logits, the precision the CUDA library decides in: callers pass the
// fp32 logits to oracle_route (the convenience driver rounds its own fp64
// logits to fp32 first).  The gate weights are then computed in float64 from
// those fp32 values.  Results do not depend on the thread count.
//
// Weights use the API layout [in, out] row-major (y = x . W); the expert
// stacks are passed as one pointer per expert so that a caller may supply
// only the experts its tokens reach (the others may be NULL).  Expert weights
// may instead be fp8 E4M3 codes with one fp32 scale per output column (low-
// precision expert weights: the paper's Section 2 models FP4 weights, its
// Section 4.3 measures FP8 quantisation): the oracle widens each code to the
// exact value it denotes and multiplies by its column's scale.  Or they may
// be block-scaled FP4 (MXFP4: E2M1 codes, two per byte, with one power-of-two
// scale per 32 consecutive input elements of each output column), stored
// output-major: the oracle decodes each code and multiplies by its block's
// power of two.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

namespace {

enum { OR_F32 = 0, OR_BF16 = 1, OR_E4M3 = 2 };
enum { OR_ACT_SILU = 0, OR_ACT_SWIGLU = 1, OR_ACT_RELU2 = 2 };
enum { OR_OK = 0, OR_ERR_ARG = 1, OR_ERR_NAN = 2, OR_ERR_MISSING = 3 };
// Routing variants (paper Section 3 and Section 4):
//   OR_ROUTE_FULL_SOFTMAX  gate w_j = p'_{e_j}, the softmax over all N logits
//                          taken at the selected experts (Eq. (1) literally;
//                          the k gates sum to less than 1)
//   OR_ROUTE_BIAS_SELECT   the router bias only steers the selection (the
//                          auxiliary-loss-free balancing of Section 4): experts
//                          are chosen on l + b, the gates use l
enum { OR_ROUTE_FULL_SOFTMAX = 1, OR_ROUTE_BIAS_SELECT = 2 };

// One fp8 E4M3 code (the OCP "E4M3FN" encoding: 1 sign, 4 exponent bits with
// bias 7, 3 mantissa bits; exponent field 0 is subnormal, S.1111.111 is NaN,
// no infinities; largest finite 448) as the exact double it denotes.
inline double e4m3_value(uint8_t c) {
  const int sgn = c >> 7, E = (c >> 3) & 15, m = c & 7;
  double v;
  if (E == 15 && m == 7) v = NAN;
  else if (E == 0) v = std::ldexp((double)m, -9);           // m/8 * 2^-6
  else v = std::ldexp(8.0 + m, E - 10);                    // (1 + m/8) * 2^(E-7)
  return sgn ? -v : v;
}

// One fp4 E2M1 code (the OCP microscaling element format: 1 sign, 2 exponent
// bits with bias 1, 1 mantissa bit; exponent field 0 is subnormal; no
// infinities or NaN; largest 6) as the exact double it denotes.
inline double e2m1_value(int c) {
  const int sgn = (c >> 3) & 1, E = (c >> 1) & 3, m = c & 1;
  const double v = E == 0 ? 0.5 * m : std::ldexp(1.0 + 0.5 * m, E - 1);
  return sgn ? -v : v;
}

// W[i][o] of an MXFP4 matrix with K inputs, stored output-major: codes
// q[o][i / 2] (element i in the low nibble when i is even), block exponents
// e[o][i / 32] (E8M0: the scale is 2^(e - 127)).
inline double mxfp4_value(const uint8_t* q, const uint8_t* e, int K, int o, int i) {
  const uint8_t b = q[(size_t)o * (K / 2) + i / 2];
  const int code = (i & 1) ? (b >> 4) : (b & 15);
  return std::ldexp(e2m1_value(code), (int)e[(size_t)o * (K / 32) + i / 32] - 127);
}

inline double widen(const void* p, int dtype, size_t i) {
  if (dtype == OR_F32) return (double)static_cast<const float*>(p)[i];
  if (dtype == OR_E4M3) return e4m3_value(static_cast<const uint8_t*>(p)[i]);
  uint32_t bits = (uint32_t)static_cast<const uint16_t*>(p)[i] << 16;
  float f;
  std::memcpy(&f, &bits, sizeof f);
  return (double)f;
}

// Runs fn(item) for item in [0, n) on up to nthreads threads.  Each item is
// processed by exactly one thread, so per-item results are independent of the
// thread count.
template <class F>
void parallel_for(long n, int nthreads, F fn) {
  if (n <= 0) return;
  int nt = (int)std::max<long>(1, std::min<long>(nthreads, n));
  if (nt == 1) {
    for (long i = 0; i < n; ++i) fn(i);
    return;
  }
  std::atomic<long> next{0};
  std::vector<std::thread> pool;
  pool.reserve(nt);
  for (int t = 0; t < nt; ++t)
    pool.emplace_back([&] {
      for (long i; (i = next.fetch_add(1)) < n;) fn(i);
    });
  for (auto& th : pool) th.join();
}

inline double silu(double a) { return a / (1.0 + std::exp(-a)); }
inline double relu2(double a) { return a > 0.0 ? a * a : 0.0; }

// act over one row of pre-activations a (width m_in) into h (width m).
void apply_act(int act, const double* a, int m, double* h) {
  if (act == OR_ACT_SWIGLU) {
    for (int o = 0; o < m; ++o) h[o] = silu(a[o]) * a[m + o];
  } else if (act == OR_ACT_RELU2) {
    for (int o = 0; o < m; ++o) h[o] = relu2(a[o]);
  } else {
    for (int o = 0; o < m; ++o) h[o] = silu(a[o]);
  }
}

// acc[p][o] = sum_i in[p][i] * W[i][o] for p in [0, P), sequential in i.
// in: P rows of width K (double); W: [K, O] in dtype; acc: P rows of width O.
// col_scale (fp8 weights): W[i][o] stands for code(i, o) * col_scale[o].
// blk_exp (MXFP4 weights, W holding the output-major codes): W[i][o] stands
// for mxfp4_value(W, blk_exp, K, o, i).
void rows_times_matrix(const double* in, int P, int K, const void* W, int dtype,
                       int O, double* acc, std::vector<double>& wrow,
                       const float* col_scale = nullptr, const uint8_t* blk_exp = nullptr) {
  std::fill(acc, acc + (size_t)P * O, 0.0);
  wrow.resize(O);
  for (int i = 0; i < K; ++i) {
    for (int o = 0; o < O; ++o)
      wrow[o] = blk_exp ? mxfp4_value(static_cast<const uint8_t*>(W), blk_exp, K, o, i)
                        : widen(W, dtype, (size_t)i * O + o) *
                              (col_scale ? (double)col_scale[o] : 1.0);
    for (int p = 0; p < P; ++p) {
      const double zi = in[(size_t)p * K + i];
      double* a = acc + (size_t)p * O;
      for (int o = 0; o < O; ++o) a[o] += zi * wrow[o];
    }
  }
}

}  // namespace

extern "C" {

struct OracleLayer {
  int d, l, N, k, m, act, shared_m, dtype, skip_proj;
  const void* Wg;          // [d, N]
  const float* bias;       // [N] fp32, or NULL
  const void* Wdown;       // [d, l], unused under skip_proj
  const void* Wup;         // [l, d], unused under skip_proj
  const void* const* W1;   // N pointers, each [l, m_in] (NULL: not supplied)
  const void* const* W2;   // N pointers, each [m, l]
  const void* Ws1;         // [d, ms_in] or NULL when shared_m == 0
  const void* Ws2;         // [shared_m, d]
  int route_mode;          // OR_ROUTE_* bits (0: the default routing)
  // fp8 expert weights: W1[e] / W2[e] hold E4M3 codes in the same layouts,
  // W1s[e] [m_in] and W2s[e] [l] one fp32 scale per output column.
  int expert_fp8;
  const float* const* W1s;
  const float* const* W2s;
  // MXFP4 expert weights: W1[e] [m_in, l / 2] and W2[e] [l, m / 2] hold
  // E2M1 code pairs output-major, W1e[e] [m_in, l / 32] and W2e[e]
  // [l, m / 32] one E8M0 block exponent per 32 inputs of each output column.
  int expert_fp4;
  const uint8_t* const* W1e;
  const uint8_t* const* W2e;
};

static int m_in_of(int act, int m) { return act == OR_ACT_SWIGLU ? 2 * m : m; }

static int check_layer(const OracleLayer* L) {
  if (!L || L->d <= 0 || L->l <= 0 || L->N <= 0 || L->k <= 0 || L->k > L->N ||
      L->m <= 0 || L->shared_m < 0 || L->act < 0 || L->act > 2 ||
      (L->dtype != OR_F32 && L->dtype != OR_BF16) || !L->Wg)
    return OR_ERR_ARG;
  if (L->skip_proj && L->l != L->d) return OR_ERR_ARG;
  if (!L->skip_proj && (!L->Wdown || !L->Wup)) return OR_ERR_ARG;
  if (L->shared_m > 0 && (!L->Ws1 || !L->Ws2)) return OR_ERR_ARG;
  if (!L->W1 || !L->W2) return OR_ERR_ARG;
  return OR_OK;
}

// Router logits (paper Section 3, the routing weights after Eq. (1)): for
// each of the S tokens (rows tokens[s] of x, or row s when tokens is NULL)
// logits[s][e] = sum_i x[i] Wg[i][e] + bias[e], accumulated in float64.
int oracle_router_logits(const OracleLayer* L, const void* x, const int* tokens,
                         int S, double* logits, int nthreads) {
  if (check_layer(L) || S < 0 || (S > 0 && (!x || !logits))) return OR_ERR_ARG;
  const int d = L->d, N = L->N;
  parallel_for(S, nthreads, [&](long s) {
    const long t = tokens ? tokens[s] : s;
    double* lg = logits + (size_t)s * N;
    std::fill(lg, lg + N, 0.0);
    for (int i = 0; i < d; ++i) {
      const double xi = widen(x, L->dtype, (size_t)t * d + i);
      for (int e = 0; e < N; ++e) lg[e] += xi * widen(L->Wg, L->dtype, (size_t)i * N + e);
    }
    if (L->bias && !(L->route_mode & OR_ROUTE_BIAS_SELECT))
      for (int e = 0; e < N; ++e) lg[e] += (double)L->bias[e];
  });
  return OR_OK;
}

// Top-k selection and gate weights on fp32 logits, followed by the grouping
// of (token, slot) pairs by expert (paper Section 3: the top-K index set and
// the dispatch after the down-projection).
//   key[t][e]   the selection key: the logit, or with sel_bias the fp32 sum
//               l + b[e] (rounded once, as the CUDA library decides in fp32)
//   idx[t][j]   the j-th expert of token t under (key desc, index asc);
//               +0.0 and -0.0 compare equal.
//   w[t][j]     in float64 from the fp32 logits l (never from the keys):
//               renormalised  exp(l_j - M) / sum_{j' chosen} exp(l_j' - M),
//               full softmax  exp(l_j - M) / sum_{e < N} exp(l_e - M),
//               with M the largest logit of the sum (a shift that cancels).
//   offsets[e]  number of pairs routed to experts < e (offsets[N] = T*k).
//   perm[r]     the pair t*k+j at expert-sorted row r; rows of one expert in
//               ascending token order.
// Any of w/offsets/perm may be NULL.  Returns OR_ERR_NAN on a NaN logit.
int oracle_route_ex(const float* logits32, const float* sel_bias, int T, int N, int k,
                    int full_softmax, int* idx, double* w, int* offsets, int* perm,
                    int nthreads) {
  if (T < 0 || N <= 0 || k <= 0 || k > N || (T > 0 && (!logits32 || !idx)))
    return OR_ERR_ARG;
  std::atomic<int> bad{0};
  parallel_for(T, nthreads, [&](long t) {
    const float* lg = logits32 + (size_t)t * N;
    std::vector<float> key(lg, lg + N);
    if (sel_bias)
      for (int e = 0; e < N; ++e) key[e] = lg[e] + sel_bias[e];  // one fp32 rounding
    std::vector<int> order(N);
    for (int e = 0; e < N; ++e) {
      if (std::isnan(key[e])) bad = 1;
      order[e] = e;
    }
    if (bad) return;
    std::partial_sort(order.begin(), order.begin() + k, order.end(),
                      [&](int a, int b) {
                        if (key[a] != key[b]) return key[a] > key[b];
                        return a < b;
                      });
    for (int j = 0; j < k; ++j) idx[(size_t)t * k + j] = order[j];
    if (w) {
      double M = -INFINITY, den = 0.0;
      if (full_softmax) {
        for (int e = 0; e < N; ++e) M = std::max(M, (double)lg[e]);
        for (int e = 0; e < N; ++e) den += std::exp((double)lg[e] - M);
      } else {
        for (int j = 0; j < k; ++j) M = std::max(M, (double)lg[order[j]]);
        for (int j = 0; j < k; ++j) den += std::exp((double)lg[order[j]] - M);
      }
      for (int j = 0; j < k; ++j)
        w[(size_t)t * k + j] = std::exp((double)lg[order[j]] - M) / den;
    }
  });
  if (bad) return OR_ERR_NAN;
  if (offsets || perm) {
    std::vector<std::vector<int>> bucket(N);
    for (long t = 0; t < T; ++t)
      for (int j = 0; j < k; ++j) bucket[idx[(size_t)t * k + j]].push_back((int)(t * k + j));
    long pos = 0;
    for (int e = 0; e < N; ++e) {
      if (offsets) offsets[e] = (int)pos;
      for (int p : bucket[e]) {
        if (perm) perm[pos] = p;
        ++pos;
      }
    }
    if (offsets) offsets[N] = (int)pos;
  }
  return OR_OK;
}

// The default routing: selection on the logits, renormalised gates.
int oracle_route(const float* logits32, int T, int N, int k, int* idx, double* w,
                 int* offsets, int* perm, int nthreads) {
  return oracle_route_ex(logits32, nullptr, T, N, k, 0, idx, w, offsets, perm, nthreads);
}

// Steps after routing, for S tokens (rows tokens[s] of x, or row s), given
// their selected experts idx[s][j] and gate weights w[s][j]:
//   z = x Wdown; y_j = act(z W1[e]) W2[e]; comb = sum_j w_j y_j (slot order);
//   out = x + comb Wup + act(x Ws1) Ws2.
// The expert stage runs expert-major (all pairs of one expert against its
// weights, in chunks) so that each expert's weights are widened once per
// chunk.  z_out [S,l] and comb_out [S,l] receive the intermediates when not
// NULL.  Returns OR_ERR_MISSING if a needed expert pointer is NULL.
int oracle_forward(const OracleLayer* L, const void* x, const int* tokens, int S,
                   const int* idx, const double* w, double* out, double* z_out,
                   double* comb_out, int nthreads) {
  if (check_layer(L) || S < 0) return OR_ERR_ARG;
  if (S == 0) return OR_OK;
  if (!x || !idx || !w || !out) return OR_ERR_ARG;
  const int d = L->d, l = L->l, N = L->N, k = L->k, m = L->m, dt = L->dtype;
  const int m_in = m_in_of(L->act, m);
  auto trow = [&](long s) -> long { return tokens ? tokens[s] : s; };

  for (long p = 0; p < (long)S * k; ++p) {
    const int e = idx[p];
    if (e < 0 || e >= N) return OR_ERR_ARG;
    if (!L->W1[e] || !L->W2[e]) return OR_ERR_MISSING;
    if (L->expert_fp8 && (!L->W1s || !L->W2s || !L->W1s[e] || !L->W2s[e])) return OR_ERR_MISSING;
    if (L->expert_fp4 && (!L->W1e || !L->W2e || !L->W1e[e] || !L->W2e[e])) return OR_ERR_MISSING;
  }
  if (L->expert_fp4 && (l % 32 != 0 || m % 32 != 0)) return OR_ERR_ARG;
  const int edt = L->expert_fp8 ? OR_E4M3 : dt;  // the expert weights' element type

  // x rows in float64.
  std::vector<double> X((size_t)S * d);
  for (long s = 0; s < S; ++s)
    for (int i = 0; i < d; ++i) X[(size_t)s * d + i] = widen(x, dt, (size_t)trow(s) * d + i);

  // Down-projection (or identity under skip_proj).
  std::vector<double> Z((size_t)S * l);
  if (L->skip_proj) {
    Z = X;
  } else {
    parallel_for(S, nthreads, [&](long s) {
      std::vector<double> wrow;
      rows_times_matrix(&X[(size_t)s * d], 1, d, L->Wdown, dt, l, &Z[(size_t)s * l], wrow);
    });
  }
  if (z_out) std::memcpy(z_out, Z.data(), Z.size() * sizeof(double));

  // Expert stage, expert-major: pairs p = s*k+j grouped by expert, chunked.
  std::vector<std::vector<int>> pairs(N);
  for (long p = 0; p < (long)S * k; ++p) pairs[idx[p]].push_back((int)p);
  const int CH = 64;
  std::vector<std::pair<int, int>> items;  // (expert, first pair in its list)
  for (int e = 0; e < N; ++e)
    for (int q = 0; q < (int)pairs[e].size(); q += CH) items.push_back({e, q});
  std::vector<double> Y((size_t)S * k * l);
  parallel_for((long)items.size(), nthreads, [&](long it) {
    const int e = items[it].first, q0 = items[it].second;
    const int P = std::min<int>(CH, (int)pairs[e].size() - q0);
    std::vector<double> zin((size_t)P * l), a((size_t)P * m_in), h((size_t)P * m),
        y((size_t)P * l), wrow;
    for (int p = 0; p < P; ++p) {
      const int s = pairs[e][q0 + p] / k;
      std::memcpy(&zin[(size_t)p * l], &Z[(size_t)s * l], l * sizeof(double));
    }
    rows_times_matrix(zin.data(), P, l, L->W1[e], edt, m_in, a.data(), wrow,
                      L->expert_fp8 ? L->W1s[e] : nullptr,
                      L->expert_fp4 ? L->W1e[e] : nullptr);
    for (int p = 0; p < P; ++p) apply_act(L->act, &a[(size_t)p * m_in], m, &h[(size_t)p * m]);
    rows_times_matrix(h.data(), P, m, L->W2[e], edt, l, y.data(), wrow,
                      L->expert_fp8 ? L->W2s[e] : nullptr,
                      L->expert_fp4 ? L->W2e[e] : nullptr);
    for (int p = 0; p < P; ++p)
      std::memcpy(&Y[(size_t)pairs[e][q0 + p] * l], &y[(size_t)p * l], l * sizeof(double));
  });

  // Combine, up-projection, shared expert, residual -- per token.
  const int ms = L->shared_m, ms_in = m_in_of(L->act, ms);
  parallel_for(S, nthreads, [&](long s) {
    std::vector<double> comb(l, 0.0), u(d), wrow;
    for (int j = 0; j < k; ++j) {
      const double wj = w[(size_t)s * k + j];
      const double* yj = &Y[((size_t)s * k + j) * l];
      for (int c = 0; c < l; ++c) comb[c] += wj * yj[c];
    }
    if (comb_out) std::memcpy(comb_out + (size_t)s * l, comb.data(), l * sizeof(double));
    if (L->skip_proj)
      u = comb;
    else
      rows_times_matrix(comb.data(), 1, l, L->Wup, dt, d, u.data(), wrow);
    double* o = out + (size_t)s * d;
    const double* xs = &X[(size_t)s * d];
    if (ms > 0) {
      std::vector<double> as(ms_in), hs(ms), sh(d);
      rows_times_matrix(xs, 1, d, L->Ws1, dt, ms_in, as.data(), wrow);
      apply_act(L->act, as.data(), ms, hs.data());
      rows_times_matrix(hs.data(), 1, ms, L->Ws2, dt, d, sh.data(), wrow);
      for (int c = 0; c < d; ++c) o[c] = xs[c] + u[c] + sh[c];
    } else {
      for (int c = 0; c < d; ++c) o[c] = xs[c] + u[c];
    }
  });
  return OR_OK;
}

// The whole layer for S tokens from the inputs alone: fp64 logits, rounded to
// fp32 for the selection, then the routing of the layer's route_mode and
// oracle_forward.  Optional
// outputs: logits32 [S,N], idx [S,k], w [S,k].
int oracle_layer(const OracleLayer* L, const void* x, const int* tokens, int S,
                 double* out, float* logits32, int* idx, double* w, int nthreads) {
  if (check_layer(L) || S < 0) return OR_ERR_ARG;
  if (S == 0) return OR_OK;
  const int N = L->N, k = L->k;
  std::vector<double> lg((size_t)S * N);
  int rc = oracle_router_logits(L, x, tokens, S, lg.data(), nthreads);
  if (rc) return rc;
  std::vector<float> lg32((size_t)S * N);
  for (size_t i = 0; i < lg.size(); ++i) lg32[i] = (float)lg[i];
  std::vector<int> id((size_t)S * k);
  std::vector<double> ww((size_t)S * k);
  const float* sel_bias = (L->route_mode & OR_ROUTE_BIAS_SELECT) ? L->bias : nullptr;
  rc = oracle_route_ex(lg32.data(), sel_bias, S, N, k, L->route_mode & OR_ROUTE_FULL_SOFTMAX,
                       id.data(), ww.data(), nullptr, nullptr, nthreads);
  if (rc) return rc;
  if (logits32) std::memcpy(logits32, lg32.data(), lg32.size() * sizeof(float));
  if (idx) std::memcpy(idx, id.data(), id.size() * sizeof(int));
  if (w) std::memcpy(w, ww.data(), ww.size() * sizeof(double));
  return oracle_forward(L, x, tokens, S, id.data(), ww.data(), out, nullptr, nullptr, nthreads);
}

int oracle_hardware_threads(void) { return (int)std::thread::hardware_concurrency(); }

// The value an fp8 E4M3 code denotes (exposed for its pin).
double oracle_e4m3_value(int code) { return e4m3_value((uint8_t)code); }

// The value an fp4 E2M1 code denotes (exposed for its pin).
double oracle_e2m1_value(int code) { return e2m1_value(code & 15); }

}  // extern "C"
