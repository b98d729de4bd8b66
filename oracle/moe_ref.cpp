// CPU reference of the DeepSeekMoE layer forward, in plain C++17 with OpenMP
// (TEST INFRASTRUCTURE ONLY: the test-suite, the smoke check and the
// benchmark's CPU arm load it; the CUDA library never does, and nothing here
// is shared with it).  Every value is read from its stored form (float32 or
// bfloat16) and computed in float64 with plain loops; no blocking, fusion or
// reordering beyond what the definitions below state.
//
// Source of every formula: "DeepSeek-V3 技術報告" (xyznot.com summary of
// arXiv 2412.19437), section 方法 / 2 "具備無輔助損失平衡機制的 DeepSeekMoE":
//   h'-equation   h'_t = u_t + sum_s FFN_s(u_t) + sum_i g_{i,t} FFN_i(u_t)
//   affinity      s_{i,t} = Sigmoid(u_t^T e_i)
//   g'-equation   g'_{i,t} = s_{i,t} if s_{i,t} + b_i is in Topk({s_{j,t} + b_j}, K), else 0;
//                 g is g' normalised
//   bias rule     overloaded expert -> b_i - gamma, underloaded -> b_i + gamma
// and the FP8 recipe of the same page, section 核心概念 (E4M3, 1x128
// activation tiles, 128x128 weight blocks, promotion every 128 K-elements).
//
// Readings where the page is silent (the same as the Python oracle's):
//   R1 g = g' / sum g' over the selected experts.
//   R2 ties in the top-K go to the lower expert index; outputs are ordered by
//      descending key, lower index first on equal keys.
//   R3 logits in float64 from the stored values, sigmoid in float64, s rounded
//      once to float32; s + b and the comparisons in float32.
//   R4 overloaded / underloaded: counts_i * N_r against T * K, in integers.
//   R5 FFN(x) = W_down (SiLU(W_gate x) * (W_up x)); shared experts have width I.
//   R6 E4M3: max 448, round to nearest even, saturate; scale = amax / 448 in
//      float32 (1 for an all-zero tile); q = E4M3(x / scale) with a float32
//      division; both FFN inputs (x and h) quantised; h formed in float32.
//   R11 group limit: a group's score is its largest s + b; the topk_groups best
//      groups (ties to the lower group index) stay eligible.
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <omp.h>

#include <algorithm>
#include <vector>

namespace {

// A stored value as float64: dt 0 = float32, 1 = bfloat16 (the upper 16 bits
// of a float32).
inline double load(const void* p, int dt, size_t i) {
  if (dt == 0) return (double)static_cast<const float*>(p)[i];
  const uint32_t w = (uint32_t)static_cast<const uint16_t*>(p)[i] << 16;
  float f;
  memcpy(&f, &w, sizeof(f));
  return (double)f;
}

inline double sigmoid(double z) { return 1.0 / (1.0 + exp(-z)); }
inline double silu(double z) { return z / (1.0 + exp(-z)); }

// Row r of a stored [rows, n] matrix as float64.
void load_row(const void* p, int dt, size_t r, int n, double* out) {
  for (int k = 0; k < n; ++k) out[k] = load(p, dt, r * (size_t)n + k);
}

// ---------------------------------------------------------------- FP8 (R6)

// Nearest E4M3 value, ties to even, saturated to +-448.  In the binade
// [2^e, 2^(e+1)) the spacing is 2^(e-3); below the smallest normal 2^-6 it is
// 2^-9 (subnormals).
double e4m3_round(double x) {
  if (x == 0.0 || x != x) return 0.0;
  int ex = 0;
  frexp(x, &ex);                     // |x| = m 2^ex, m in [0.5, 1)
  int e = ex - 1;
  if (e < -6) e = -6;
  const double quantum = ldexp(1.0, e - 3);
  double q = nearbyint(x / quantum) * quantum;   // default rounding: nearest, ties to even
  if (q > 448.0) q = 448.0;
  if (q < -448.0) q = -448.0;
  return q;
}

float tile_scale(float amax) { return amax == 0.0f ? 1.0f : amax / 448.0f; }

// One tile of float32 values -> E4M3 values (as float64) with its scale.
void quant_tile(const float* v, int n, double* q, float* scale) {
  float amax = 0.0f;
  for (int i = 0; i < n; ++i) amax = std::max(amax, fabsf(v[i]));
  const float s = tile_scale(amax);
  for (int i = 0; i < n; ++i) q[i] = e4m3_round((double)(v[i] / s));
  *scale = s;
}

// A [rows, cols] float32 matrix quantised per 128x128 block.
struct QMat {
  int rows = 0, cols = 0;
  std::vector<double> q;      // E4M3 values
  std::vector<float> s;       // [rows/128, cols/128]
};

QMat quant_128x128(const void* w, int dt, int rows, int cols) {
  QMat m;
  m.rows = rows;
  m.cols = cols;
  m.q.assign((size_t)rows * cols, 0.0);
  const int rb = rows / 128, cb = cols / 128;
  m.s.assign((size_t)rb * cb, 1.0f);
#pragma omp parallel for collapse(2) schedule(static)
  for (int bi = 0; bi < rb; ++bi)
    for (int bj = 0; bj < cb; ++bj) {
      float amax = 0.0f;
      for (int i = 0; i < 128; ++i)
        for (int j = 0; j < 128; ++j)
          amax = std::max(amax,
                          fabsf((float)load(w, dt, (size_t)(bi * 128 + i) * cols + bj * 128 + j)));
      const float s = tile_scale(amax);
      m.s[(size_t)bi * cb + bj] = s;
      for (int i = 0; i < 128; ++i)
        for (int j = 0; j < 128; ++j) {
          const size_t at = (size_t)(bi * 128 + i) * cols + bj * 128 + j;
          m.q[at] = e4m3_round((double)((float)load(w, dt, at) / s));
        }
    }
  return m;
}

// sum over 128-wide K blocks of (sum_k qa[k] qw[n, k]) * sa[kb] * sw[n/128, kb].
double promoted_dot(const double* qa, const float* sa, const QMat& w, int n) {
  const int nkb = w.cols / 128;
  double acc = 0.0;
  for (int kb = 0; kb < nkb; ++kb) {
    double part = 0.0;
    const double* wr = &w.q[(size_t)n * w.cols + kb * 128];
    const double* ar = qa + kb * 128;
    for (int k = 0; k < 128; ++k) part += ar[k] * wr[k];
    acc += part * (double)sa[kb] * (double)w.s[(size_t)(n / 128) * nkb + kb];
  }
  return acc;
}

// ---------------------------------------------------------------- expert FFN (R5)

// y[r] += coef[r] * FFN(x_r) for the rows r of one expert, x_r = u[rows[r]].
// W_gate_up [2I, d] (rows [0, I) gate, [I, 2I) up), W_down [d, I], stored dt.
void ffn_accumulate(const void* u, int dt, int d, int I, const std::vector<int>& rows,
                    const std::vector<double>& coef, const void* W_gate_up, const void* W_down,
                    double* out) {
  const int R = (int)rows.size();
  if (R == 0) return;
  std::vector<double> x((size_t)R * d), h((size_t)R * I);
  for (int r = 0; r < R; ++r) load_row(u, dt, (size_t)rows[r], d, &x[(size_t)r * d]);
#pragma omp parallel for schedule(static)
  for (int i = 0; i < I; ++i) {
    std::vector<double> wg(d), wu(d);
    load_row(W_gate_up, dt, (size_t)i, d, wg.data());
    load_row(W_gate_up, dt, (size_t)(I + i), d, wu.data());
    for (int r = 0; r < R; ++r) {
      const double* xr = &x[(size_t)r * d];
      double a = 0.0, b = 0.0;
      for (int k = 0; k < d; ++k) {
        a += xr[k] * wg[k];
        b += xr[k] * wu[k];
      }
      h[(size_t)r * I + i] = silu(a) * b;
    }
  }
#pragma omp parallel for schedule(static)
  for (int j = 0; j < d; ++j) {
    std::vector<double> wd(I);
    load_row(W_down, dt, (size_t)j, I, wd.data());
    for (int r = 0; r < R; ++r) {
      const double* hr = &h[(size_t)r * I];
      double y = 0.0;
      for (int i = 0; i < I; ++i) y += hr[i] * wd[i];
      out[(size_t)rows[r] * d + j] += coef[r] * y;
    }
  }
}

// The same under the FP8 recipe: x quantised 1x128 from its stored value (as
// float32), both GEMMs promoted per 128-deep block, h = SiLU(gate) * up formed
// in float64 and rounded to float32, quantised 1x128, promoted down GEMM.
void ffn_accumulate_fp8(const void* u, int dt, int d, int I, const std::vector<int>& rows,
                        const std::vector<double>& coef, const QMat& Wgu, const QMat& Wd,
                        double* out) {
  const int R = (int)rows.size();
  if (R == 0) return;
  const int nd = d / 128, ni = I / 128;
  std::vector<double> qx((size_t)R * d), qh((size_t)R * I);
  std::vector<float> sx((size_t)R * nd), sh((size_t)R * ni), hf((size_t)R * I);
#pragma omp parallel for schedule(static)
  for (int r = 0; r < R; ++r) {
    std::vector<float> xr(d);
    for (int k = 0; k < d; ++k) xr[k] = (float)load(u, dt, (size_t)rows[r] * d + k);
    for (int t = 0; t < nd; ++t)
      quant_tile(&xr[t * 128], 128, &qx[(size_t)r * d + t * 128], &sx[(size_t)r * nd + t]);
  }
#pragma omp parallel for collapse(2) schedule(static)
  for (int r = 0; r < R; ++r)
    for (int i = 0; i < I; ++i) {
      const double a = promoted_dot(&qx[(size_t)r * d], &sx[(size_t)r * nd], Wgu, i);
      const double b = promoted_dot(&qx[(size_t)r * d], &sx[(size_t)r * nd], Wgu, I + i);
      hf[(size_t)r * I + i] = (float)(silu(a) * b);
    }
  for (int r = 0; r < R; ++r)
    for (int t = 0; t < ni; ++t)
      quant_tile(&hf[(size_t)r * I + t * 128], 128, &qh[(size_t)r * I + t * 128],
                 &sh[(size_t)r * ni + t]);
#pragma omp parallel for schedule(static)
  for (int j = 0; j < d; ++j)
    for (int r = 0; r < R; ++r)
      out[(size_t)rows[r] * d + j] +=
          coef[r] * promoted_dot(&qh[(size_t)r * I], &sh[(size_t)r * ni], Wd, j);
}

}  // namespace

extern "C" {

int moe_ref_version(void) { return 1; }

// OpenMP threads of the following calls (n > 0); returns the count in force.
// Only the timing of the CPU baseline uses it: results do not depend on it.
int ref_set_threads(int n) {
  if (n > 0) omp_set_num_threads(n);
  return omp_get_max_threads();
}

// Router (affinity line, g'-equation, R1-R3, R11).  u [T, d], E [N_r, d]
// stored as dt; b [N_r] float32.  Writes idx [T, K], gate [T, K], counts
// [N_r] and, when not NULL, s [T, N_r] and key [T, N_r] (float32).
// n_groups = topk_groups = 1: no group limit.  Returns 0, or -1 on bad sizes.
int ref_route(const void* u, const void* E, int dt, const float* b, int T, int d, int N_r, int K,
              int n_groups, int topk_groups, int32_t* idx, float* gate, int32_t* counts,
              float* s_out, float* key_out) {
  if (T < 0 || d <= 0 || N_r <= 0 || K <= 0 || K > N_r || n_groups <= 0 || N_r % n_groups ||
      topk_groups <= 0 || topk_groups > n_groups || topk_groups * (N_r / n_groups) < K)
    return -1;
  std::vector<double> Ed((size_t)N_r * d);
  for (int i = 0; i < N_r; ++i) load_row(E, dt, (size_t)i, d, &Ed[(size_t)i * d]);
  const int gs = N_r / n_groups;
#pragma omp parallel for schedule(dynamic, 16)
  for (int t = 0; t < T; ++t) {
    std::vector<double> ut(d);
    load_row(u, dt, (size_t)t, d, ut.data());
    std::vector<float> s(N_r), key(N_r);
    for (int i = 0; i < N_r; ++i) {
      double x = 0.0;
      for (int k = 0; k < d; ++k) x += ut[k] * Ed[(size_t)i * d + k];
      s[i] = (float)sigmoid(x);
      key[i] = s[i] + b[i];                       // float32 addition (R3)
    }
    // group limit: the kept groups' experts stay eligible
    std::vector<char> eligible(N_r, 1);
    if (topk_groups < n_groups) {
      std::vector<float> gscore(n_groups);
      std::vector<int> gorder(n_groups);
      for (int g = 0; g < n_groups; ++g) {
        gscore[g] = key[g * gs];
        for (int j = 1; j < gs; ++j) gscore[g] = std::max(gscore[g], key[g * gs + j]);
        gorder[g] = g;
      }
      std::stable_sort(gorder.begin(), gorder.end(),
                       [&](int a, int c) { return gscore[a] > gscore[c]; });
      std::vector<char> kept(n_groups, 0);
      for (int r = 0; r < topk_groups; ++r) kept[gorder[r]] = 1;
      for (int i = 0; i < N_r; ++i) eligible[i] = kept[i / gs];
    }
    std::vector<int> order;
    for (int i = 0; i < N_r; ++i)
      if (eligible[i]) order.push_back(i);
    // descending key, lower index first on equal keys (stable sort of ascending ids)
    std::stable_sort(order.begin(), order.end(), [&](int a, int c) { return key[a] > key[c]; });
    double sum = 0.0;
    for (int k = 0; k < K; ++k) sum += (double)s[order[k]];
    for (int k = 0; k < K; ++k) {
      idx[(size_t)t * K + k] = order[k];
      gate[(size_t)t * K + k] = (float)((double)s[order[k]] / sum);
    }
    if (s_out) memcpy(s_out + (size_t)t * N_r, s.data(), sizeof(float) * N_r);
    if (key_out) memcpy(key_out + (size_t)t * N_r, key.data(), sizeof(float) * N_r);
  }
  for (int i = 0; i < N_r; ++i) counts[i] = 0;
  for (size_t p = 0; p < (size_t)T * K; ++p) counts[idx[p]] += 1;
  return 0;
}

// Dispatch permutation: pairs grouped by expert, ascending (t, k) inside a
// group.  offsets [N_r+1], perm_src [T*K] (grouped row -> token), inv_row
// [T, K].  An id outside [0, N_r) is left out (inv_row -1).
void ref_permute(const int32_t* idx, int T, int K, int N_r, int32_t* offsets, int32_t* perm_src,
                 int32_t* inv_row) {
  std::vector<int> cnt(N_r, 0);
  for (size_t p = 0; p < (size_t)T * K; ++p)
    if (idx[p] >= 0 && idx[p] < N_r) cnt[idx[p]] += 1;
  offsets[0] = 0;
  for (int e = 0; e < N_r; ++e) offsets[e + 1] = offsets[e] + cnt[e];
  std::vector<int> next(offsets, offsets + N_r);
  for (int t = 0; t < T; ++t)
    for (int k = 0; k < K; ++k) {
      const int e = idx[(size_t)t * K + k];
      if (e < 0 || e >= N_r) {
        inv_row[(size_t)t * K + k] = -1;
        continue;
      }
      const int r = next[e]++;
      perm_src[r] = t;
      inv_row[(size_t)t * K + k] = r;
    }
}

// Bias rule with reading R4, float32 arithmetic in place.
void ref_bias_update(float* b, const int32_t* counts, int N_r, long long T, int K, float gamma) {
  const long long mean = T * (long long)K;
  for (int i = 0; i < N_r; ++i) {
    const long long load_i = (long long)counts[i] * N_r;
    if (load_i > mean) b[i] = b[i] - gamma;
    else if (load_i < mean) b[i] = b[i] + gamma;
  }
}

// h'-equation for T tokens (u [T, d], stored dt) with their routing idx /
// gate [T, K]: out [T, d] float64.  routed_gu[e] / routed_dn[e]: pointers to
// expert e's W_gate_up [2I, d] and W_down [d, I] (stored dt); an expert no
// token selects may be NULL.  shared_gu / shared_dn: N_s pointers.
// Expert-major, so each weight matrix is read once.  fp8 = 1 evaluates every
// expert FFN under the FP8 recipe (weights quantised 128x128 here, from their
// stored values).  Returns 0, or -1 when a selected expert has no weights.
int ref_layer_forward(const void* u, int dt, int T, int d, int I, const int32_t* idx,
                      const float* gate, int K, const void* const* routed_gu,
                      const void* const* routed_dn, int N_r, const void* const* shared_gu,
                      const void* const* shared_dn, int N_s, int fp8, double* out) {
  for (size_t i = 0; i < (size_t)T * d; ++i) out[i] = load(u, dt, i);
  std::vector<int> all(T);
  std::vector<double> ones(T, 1.0);
  for (int t = 0; t < T; ++t) all[t] = t;
  for (int j = 0; j < N_s; ++j) {
    if (fp8) {
      const QMat gu = quant_128x128(shared_gu[j], dt, 2 * I, d);
      const QMat dn = quant_128x128(shared_dn[j], dt, d, I);
      ffn_accumulate_fp8(u, dt, d, I, all, ones, gu, dn, out);
    } else {
      ffn_accumulate(u, dt, d, I, all, ones, shared_gu[j], shared_dn[j], out);
    }
  }
  for (int e = 0; e < N_r; ++e) {
    std::vector<int> rows;
    std::vector<double> coef;
    for (int t = 0; t < T; ++t)
      for (int k = 0; k < K; ++k)
        if (idx[(size_t)t * K + k] == e) {
          rows.push_back(t);
          coef.push_back((double)gate[(size_t)t * K + k]);
        }
    if (rows.empty()) continue;
    if (!routed_gu[e] || !routed_dn[e]) return -1;
    if (fp8) {
      const QMat gu = quant_128x128(routed_gu[e], dt, 2 * I, d);
      const QMat dn = quant_128x128(routed_dn[e], dt, d, I);
      ffn_accumulate_fp8(u, dt, d, I, rows, coef, gu, dn, out);
    } else {
      ffn_accumulate(u, dt, d, I, rows, coef, routed_gu[e], routed_dn[e], out);
    }
  }
  return 0;
}

// One expert's FFN on n rows x [n, d] (stored dt): y [n, d] float64 (for
// comparing a whole expert group of the grouped GEMMs).
void ref_expert_ffn(const void* x, int dt, int n, int d, int I, const void* W_gate_up,
                    const void* W_down, int fp8, double* y) {
  std::vector<int> rows(n);
  std::vector<double> ones(n, 1.0);
  for (int r = 0; r < n; ++r) rows[r] = r;
  for (size_t i = 0; i < (size_t)n * d; ++i) y[i] = 0.0;
  if (fp8) {
    const QMat gu = quant_128x128(W_gate_up, dt, 2 * I, d);
    const QMat dn = quant_128x128(W_down, dt, d, I);
    ffn_accumulate_fp8(x, dt, d, I, rows, ones, gu, dn, y);
  } else {
    ffn_accumulate(x, dt, d, I, rows, ones, W_gate_up, W_down, y);
  }
}

}  // extern "C"
