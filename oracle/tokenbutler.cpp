// Plain fp64 CPU oracle of the TokenButler decode-step hot path, in C++17.
//
// TEST INFRASTRUCTURE.  Only the tests, __graft_entry__.smoke() and the
// cpu_baseline / --impl reference legs of bench.py may load or run this
// library (through oracle/native.py).  It shares no code with the CUDA path
// and restates, step by step, what oracle/tokenbutler.py states in numpy: the
// same functions, readings and step order.  Plain loops in double precision,
// no blocking, fusion or reordering inside a row; OpenMP only spreads
// independent (sequence, head) rows over host threads.
//
// Sources (cited by page title and section):
//   [MC] "Meta-Llama-3.1-8B-Instruct-Butler" model card: section "Method"
//        (producer layers, Q_imp, W_K, K_imp, consumer slot, top-x selection
//        with sink prefix and local window, full KV cache kept) and section
//        "Memory requirements" (fixed_<N>pc, min_sparse_index,
//        sliding_window, layer 0 dense).
//   [AB] "TokenButler: Token Importance is Predictable", abstract.
//   [TS] TokenSelect README, "Per-head Soft Voting Mechanism".
// Readings R1-R19 are those listed in oracle/tokenbutler.py; each function
// below names the ones it follows.  Parity pins: tests/test_oracle_pins.py
// runs every pin on this library as on the numpy oracle.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <vector>

#include <omp.h>

namespace {
const double kInf = std::numeric_limits<double>::infinity();
}

extern "C" {

// ------------------------------------------------------------------ threads
void tbo_set_threads(int n) { omp_set_num_threads(n < 1 ? 1 : n); }
int tbo_get_threads() { return omp_get_max_threads(); }

// ------------------------------------------------------------------ layers
// [MC] Method: producers at layers 0, G, 2G, ...; each predicts for itself
// and the next G - 1 layers (reading R4).
int tbo_producer_of(int layer, int G) { return G * (layer / G); }

// [MC] Method: consumer slot (l - 1) mod G, non-negative mod (reading R4).
int tbo_consumer_slot(int layer, int G) { return ((layer - 1) % G + G) % G; }

// Reading R2: contiguous groups of Hq / Hkv query heads share a KV head.
int tbo_kv_head_of(int h, int Hq, int Hkv) { return h / (Hq / Hkv); }

// [MC] Memory requirements: "fixed_<N>pc" sparsifies N % of the tokens and
// keeps 100 - N %.  Returns -1 for any other policy string.
int tbo_keep_pct_from_policy(const char* policy) {
  const size_t n = std::strlen(policy);
  if (n < 9 || std::strncmp(policy, "fixed_", 6) != 0 || std::strcmp(policy + n - 2, "pc") != 0) return -1;
  int v = 0;
  for (size_t i = 6; i + 2 < n; ++i) {
    if (policy[i] < '0' || policy[i] > '9') return -1;
    v = 10 * v + (policy[i] - '0');
    if (v > 100) return -1;
  }
  return 100 - v;
}

// [MC] Method: Q_imp has shape (B*H) x G x L x d'; the consumer's query of
// (b, h) is Q_imp[b*Hq + h][slot][position][:].  out: [B][Hq][dimp].
void tbo_importance_queries(const double* q_imp, int B, int Hq, int G, int n_pos, int dimp, int layer, int position,
                            double* out) {
  const int slot = tbo_consumer_slot(layer, G);
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < Hq; ++h)
      for (int j = 0; j < dimp; ++j)
        out[((long)b * Hq + h) * dimp + j] =
            q_imp[((((long)b * Hq + h) * G + slot) * n_pos + position) * dimp + j];
}

// Reading R5: k = floor(P * L / 100) in integer arithmetic.
long tbo_token_budget(long L, int keep_pct) { return (keep_pct * L) / 100; }

// ------------------------------------------------------------------ a1: K_imp
// Nearest bfloat16 value of x (8 significant bits, fp32's exponent range),
// ties to the even significand.  Below 2^-126 the quantum is fixed at 2^-133
// (subnormal bfloat16).  For finite |x| below the largest bfloat16.
double tbo_round_to_bf16(double x) {
  if (x == 0.0) return x;
  int e = 0;
  std::frexp(x, &e);                    // x = m * 2^e, 0.5 <= |m| < 1
  if (e < -125) e = -125;
  const double q = std::ldexp(1.0, e - 8);  // one unit in the 8th significant bit
  return std::nearbyint(x / q) * q;        // default rounding: half to even; x / q is exact
}

void tbo_round_to_bf16_array(const double* x, long n, double* out) {
  for (long i = 0; i < n; ++i) out[i] = tbo_round_to_bf16(x[i]);
}

// [MC] Method: K_imp = K . W_K on the post-RoPE cached keys (reading R1: one
// D x d' matrix per layer).  K: [n][D], W: [D][dimp], out: [n][dimp].  With
// bf16 != 0, the bf16 K_imp storage option: each exact value rounded once.
void tbo_project_keys(const double* K, long n, int D, const double* W, int dimp, int bf16, double* out) {
#pragma omp parallel for schedule(static) if (n >= 4096)
  for (long t = 0; t < n; ++t)
    for (int j = 0; j < dimp; ++j) {
      double acc = 0.0;
      for (int d = 0; d < D; ++d) acc += K[t * D + d] * W[(long)d * dimp + j];
      out[t * dimp + j] = bf16 ? tbo_round_to_bf16(acc) : acc;
    }
}

// ------------------------------------------------------------------ a3: scores
// [MC] Method: s[t] = q_hat . K_imp[t] for every cached token (reading R3:
// no scale).  kimp: [L][dimp].
void tbo_importance_scores(const double* qhat, const double* kimp, long L, int dimp, double* out) {
  for (long t = 0; t < L; ++t) {
    double acc = 0.0;
    for (int j = 0; j < dimp; ++j) acc += qhat[j] * kimp[t * dimp + j];
    out[t] = acc;
  }
}

// Per-KV-group option: the group's per-head scores summed in head order.
// qhat_heads: [gs][dimp].
void tbo_group_scores(const double* qhat_heads, int gs, const double* kimp, long L, int dimp, double* out) {
  std::vector<double> s(L > 0 ? L : 1);
  for (long t = 0; t < L; ++t) out[t] = 0.0;
  for (int h = 0; h < gs; ++h) {
    tbo_importance_scores(qhat_heads + (long)h * dimp, kimp, L, dimp, s.data());
    for (long t = 0; t < L; ++t) out[t] += s[t];
  }
}

// ------------------------------------------------------------------ a4/a5: select
// [MC] Method + Memory requirements: the top-k candidates under a fixed
// budget plus the sink prefix and the recent window.  Candidates are
// [sink, L - window) (reading R6); k is clamped to their number (R7); the
// order is score descending, then index ascending (R8: -0.0 == +0.0 in a
// double comparison).  Writes the selected indices ascending into out_idx
// (room for L) and returns their number.
long tbo_select_tokens(const double* scores, long L, int keep_pct, int sink, int window, long* out_idx) {
  std::vector<long> cand;
  for (long t = sink; t < L - window; ++t) cand.push_back(t);
  const long k = std::min(tbo_token_budget(L, keep_pct), (long)cand.size());
  std::sort(cand.begin(), cand.end(), [&](long a, long b) {
    if (scores[a] != scores[b]) return scores[a] > scores[b];
    return a < b;
  });
  std::vector<char> keep(L > 0 ? L : 1, 0);
  for (long t = 0; t < std::min<long>(sink, L); ++t) keep[t] = 1;            // sink prefix
  for (long t = std::max<long>(L - window, 0); t < L; ++t) keep[t] = 1;      // recent window
  for (long i = 0; i < k; ++i) keep[cand[i]] = 1;                            // top-k
  long n = 0;
  for (long t = 0; t < L; ++t)
    if (keep[t]) out_idx[n++] = t;
  return n;
}

// ------------------------------------------------------------------ a6: attention
// [AB] + [MC] Method: exact attention over the selected tokens of the full
// KV cache, o = sum_{t in Sel} softmax_t(scale * q . K[t]) V[t], and the
// natural-log lse = log sum_{t in Sel} exp(scale * q . K[t]) (reading R9:
// scale = 1/sqrt(D)).  K, V: [>=max idx + 1][D].  An empty set gives o = 0,
// lse = -inf.
void tbo_attend(const double* q, const double* K, const double* V, int D, const long* idx, long n, double scale,
                double* out, double* lse) {
  for (int d = 0; d < D; ++d) out[d] = 0.0;
  if (n == 0) {
    *lse = -kInf;
    return;
  }
  std::vector<double> logit(n);
  double m = -kInf;
  for (long i = 0; i < n; ++i) {
    double acc = 0.0;
    for (int d = 0; d < D; ++d) acc += K[idx[i] * D + d] * q[d];
    logit[i] = scale * acc;
    m = std::max(m, logit[i]);
  }
  double z = 0.0;
  for (long i = 0; i < n; ++i) {
    const double w = std::exp(logit[i] - m);
    z += w;
    for (int d = 0; d < D; ++d) out[d] += w * V[idx[i] * D + d];
  }
  for (int d = 0; d < D; ++d) out[d] /= z;
  *lse = m + std::log(z);
}

// ------------------------------------------------------------------ a8: soft voting
// [TS] Per-head Soft Voting (reading R14): a[h][t] = q_h . K[g(h)][t] /
// sqrt(D), normalised by a softmax over all t < L, summed over the heads.
// q: [Hq][D]; K: [Hkv][ld][D] (ld >= L rows per head).  votes: [L].
void tbo_softvote_scores(const double* q, int Hq, const double* K, int Hkv, long ld, long L, int D, double* votes) {
  for (long t = 0; t < L; ++t) votes[t] = 0.0;
  if (L == 0) return;
  std::vector<double> a(L);
  for (int h = 0; h < Hq; ++h) {
    const double* Kg = K + (long)tbo_kv_head_of(h, Hq, Hkv) * ld * D;
    double m = -kInf;
    for (long t = 0; t < L; ++t) {
      double acc = 0.0;
      for (int d = 0; d < D; ++d) acc += Kg[t * D + d] * q[(long)h * D + d];
      a[t] = acc / std::sqrt((double)D);
      m = std::max(m, a[t]);
    }
    double z = 0.0;
    for (long t = 0; t < L; ++t) {
      a[t] = std::exp(a[t] - m);
      z += a[t];
    }
    for (long t = 0; t < L; ++t) votes[t] += a[t] / z;
  }
}

// ------------------------------------------------------------------ amortised selection (R18)
// Whether a row reuses its cached selection this step: it takes a real top-k
// now, the cache holds one chosen at len0 > 0 no more than `interval` tokens
// ago, and the cosine of the current and cached importance queries is >= tau.
int tbo_reuse_decision(const double* q_now, const double* q_cached, int dimp, long L, long len0, long interval,
                       double tau, int keep_pct, int sink, int window) {
  const long cand = L - window > sink ? L - window - sink : 0;
  const long k = std::min(tbo_token_budget(L, keep_pct), cand);
  if (!(0 < k && k < cand)) return 0;
  if (len0 <= 0 || L < len0 || L - len0 > interval) return 0;
  double aa = 0.0, cc = 0.0, ac = 0.0;
  for (int j = 0; j < dimp; ++j) {
    aa += q_now[j] * q_now[j];
    cc += q_cached[j] * q_cached[j];
    ac += q_now[j] * q_cached[j];
  }
  const double na = std::sqrt(aa), nc = std::sqrt(cc);
  if (na == 0.0 || nc == 0.0) return 0;
  return ac / (na * nc) >= tau ? 1 : 0;
}

// The set a reusing row attends to at length L: the cached top-k (the cached
// set inside [sink, len0 - window)) widened by `radius` tokens each side,
// kept inside [sink, L - window), plus the current sink and window.
// out: room for L indices; returns their number (ascending).
long tbo_reused_set(const long* cached, long n, long len0, long L, int sink, int window, int radius, long* out) {
  std::vector<char> keep(L > 0 ? L : 1, 0);
  for (long i = 0; i < n; ++i) {
    const long t = cached[i];
    if (!(t >= sink && t < len0 - window)) continue;
    for (long d = -radius; d <= radius; ++d) {
      const long u = t + d;
      if (u >= sink && u < L - window) keep[u] = 1;
    }
  }
  for (long t = 0; t < std::min<long>(sink, L); ++t) keep[t] = 1;
  for (long t = std::max<long>(L - window, 0); t < L; ++t) keep[t] = 1;
  long m = 0;
  for (long t = 0; t < L; ++t)
    if (keep[t]) out[m++] = t;
  return m;
}

// ------------------------------------------------------------------ sequence sharding (R19)
// Attention over a set split into disjoint parts, from each part's output
// o_r and lse_r: weights exp(lse_r - lse), lse = log sum_r exp(lse_r).
// Empty parts (lse_r = -inf) carry no weight; all empty: zero output and
// lse = -inf.  outs: [n_parts][D].
void tbo_merge_partials(const double* outs, const double* lses, int n_parts, int D, double* out, double* lse) {
  double m = -kInf;
  for (int r = 0; r < n_parts; ++r)
    if (lses[r] != -kInf) m = std::max(m, lses[r]);
  for (int d = 0; d < D; ++d) out[d] = 0.0;
  if (m == -kInf) {
    *lse = -kInf;
    return;
  }
  double total = 0.0;
  for (int r = 0; r < n_parts; ++r) {
    const double w = lses[r] == -kInf ? 0.0 : std::exp(lses[r] - m);
    total += w;
    for (int d = 0; d < D; ++d) out[d] += w * outs[(long)r * D + d];
  }
  for (int d = 0; d < D; ++d) out[d] /= total;
  *lse = m + std::log(total);
}

// ------------------------------------------------------------------ one decode layer
// [MC] Method in order for the rows (b, h) listed in rows[2 * i], rows[2 * i + 1]:
// K_imp = K W_K (or the given K_imp), consumer slot, scores over every
// cached token, top-k + sink + window per query head (or per KV group with
// group != 0), attention over the selected tokens.  dense != 0 (layer 0):
// every token.  Shapes: q [B][Hq][D]; K, V [B][Hkv][ld][D]; W [D][dimp];
// q_imp [(B*Hq)][G][1][dimp]; kimp (optional) [B][Hkv][ld_imp][dimp];
// lens [B].  Outputs per listed row i: idx_out [i][lmax] and count[i],
// out [i][D], lse [i], scores_out [i][lmax] (may be null).
void tbo_decode_layer(const double* q, const double* K, const double* V, const double* W, const double* q_imp,
                      const double* kimp, long ld_imp, int B, int Hq, int Hkv, int D, int dimp, long ld, int G,
                      int layer, const long* lens, int keep_pct, int sink, int window, int dense, int group,
                      int kimp_bf16, const int* rows, int n_rows, long lmax, long* idx_out, long* count,
                      double* out, double* lse, double* scores_out) {
  (void)B;  // the shapes' batch extent; rows name their sequences
  const double scale = 1.0 / std::sqrt((double)D);
  const int gs = Hq / Hkv;
  const int slot = tbo_consumer_slot(layer, G);
#pragma omp parallel for schedule(dynamic, 1)
  for (int i = 0; i < n_rows; ++i) {
    const int b = rows[2 * i], h = rows[2 * i + 1];
    const long L = lens[b];
    const int g = tbo_kv_head_of(h, Hq, Hkv);
    const double* Kbg = K + ((long)b * Hkv + g) * ld * D;
    const double* Vbg = V + ((long)b * Hkv + g) * ld * D;
    long* idx = idx_out + (long)i * lmax;
    if (dense) {
      for (long t = 0; t < L; ++t) idx[t] = t;
      count[i] = L;
    } else {
      std::vector<double> own;
      const double* kb = nullptr;
      if (kimp != nullptr) {
        kb = kimp + ((long)b * Hkv + g) * ld_imp * dimp;
      } else {
        own.resize(L * dimp + 1);
        tbo_project_keys(Kbg, L, D, W, dimp, kimp_bf16, own.data());
        kb = own.data();
      }
      std::vector<double> s(L + 1);
      if (group) {
        std::vector<double> qh((long)gs * dimp);
        for (int hh = 0; hh < gs; ++hh)
          for (int j = 0; j < dimp; ++j)
            qh[(long)hh * dimp + j] = q_imp[(((long)b * Hq + g * gs + hh) * G + slot) * dimp + j];
        tbo_group_scores(qh.data(), gs, kb, L, dimp, s.data());
      } else {
        tbo_importance_scores(q_imp + (((long)b * Hq + h) * G + slot) * dimp, kb, L, dimp, s.data());
      }
      if (scores_out != nullptr)
        for (long t = 0; t < L; ++t) scores_out[(long)i * lmax + t] = s[t];
      count[i] = tbo_select_tokens(s.data(), L, keep_pct, sink, window, idx);
    }
    tbo_attend(q + ((long)b * Hq + h) * D, Kbg, Vbg, D, idx, count[i], scale, out + (long)i * D, lse + i);
  }
}

// ------------------------------------------------------------------ a7: prefill rows
// Reading R13: row p of head h scores its causal prefix
// s_p[t] = q_hat[h][p - row0] . K_imp[g(h)][t], t <= p, and selects with
// L -> p + 1.  q_hat_rows: [Hq][nrows][dimp]; kimp: [Hkv][ld_imp][dimp].
// idx_out: [Hq][nrows][row0 + nrows], count: [Hq][nrows].
void tbo_prefill_select(const double* q_hat_rows, int Hq, int nrows, int dimp, const double* kimp, int Hkv,
                        long ld_imp, long row0, int keep_pct, int sink, int window, long* idx_out, long* count) {
  const long lmax = row0 + nrows;
#pragma omp parallel for schedule(dynamic, 1)
  for (long i = 0; i < (long)Hq * nrows; ++i) {
    const int h = (int)(i / nrows), r = (int)(i % nrows);
    const long p = row0 + r;
    const double* kb = kimp + (long)tbo_kv_head_of(h, Hq, Hkv) * ld_imp * dimp;
    std::vector<double> s(p + 1);
    tbo_importance_scores(q_hat_rows + ((long)h * nrows + r) * dimp, kb, p + 1, dimp, s.data());
    count[i] = tbo_select_tokens(s.data(), p + 1, keep_pct, sink, window, idx_out + i * lmax);
  }
}

}  // extern "C"
