// TEST INFRASTRUCTURE ONLY: a plain, slow, single-threaded CPU reference of the
// forward pass of one Mixture-of-Experts FFN layer (and, at the end of this file,
// of its backward pass). It exists to check the CUDA path; only the tests, the
// smoke check and the benchmark's CPU-baseline leg may load it. It shares no
// code, header or table with the CUDA library.
//
// What it computes is the plain definition of the layer, written out step by step
// with every accumulation in double:
//
//   p(x) = softmax(W_r x)                                   router
//   y    = sum_{e in TopK(p(x), k)} p_e(x) * E_e(x)          gate-weighted experts
//
//   (DeepSpeed MoE and Model Compression, section "DeepSpeed-MoE: capacity growth
//    is not per-token compute growth", the MoE formula and the pipeline listing:
//    route, keep the top k, pack by expert within a capacity, run the experts,
//    combine)
//
// with a per-expert capacity: tokens beyond an expert's capacity skip that
// expert's FFN and reach the output only through the residual
//   (Switch-vs-DeepSpeed comparison article, section "Expert Capacity Overflow":
//    capacity = (tokens in the batch / experts) x capacity factor).
//
// Readings of points the pages leave open:
//   * capacity C = ceil(k * T / E * cf): the article's tokens-over-experts times the
//     capacity factor, with the k choices counted; a product within rounding error above an
//     integer is that integer (the capacity of the decimal factor);
//   * overflow is first-come: slots are handed out in token order (t ascending,
//     then the token's j-th choice), slot >= C is dropped;
//   * gates are the unrenormalised softmax probabilities p_e;
//   * softmax over all E experts first, then top-k; top-k is taken on the fp32
//     logits, ordered by (logit descending, expert index ascending);
//   * an expert is a two-layer FFN with biases and the exact erf GeLU
//     (MoE pruning/quantisation survey notes, section 1.1.2.1 "Replacing the FFN
//     layer": M_i(x) is a two-layer feed-forward network);
//   * for bf16 workloads the hidden activation h is rounded to bf16 (round to
//     nearest even) because that is the storage type of the second GEMM's operand;
//     the expert output y and the dense-branch output are rounded to fp32;
//   * out = [x if add_input_residual] + [DenseMLP(x) if PR-MoE] + sum_j gate_j * y_j,
//     summed in double and rounded once to the output type
//     (DeepSpeed-MoE notes §3.1 PR-MoE: a fixed dense MLP plus a top-1 residual
//      expert; comparison article, "numeric example: residual correction");
//   * load-balance statistics f_i (share of tokens whose top-1 choice is i, before
//     the capacity drop), Q_i (mean router probability of i over all tokens) and
//     aux = alpha * E * sum_i f_i Q_i (survey notes §1.1.4.1, Switch Transformer loss).
#include <cmath>
#include <cstdint>
#include <algorithm>
#include <cstring>
#include <vector>

extern "C" {

// ---------------------------------------------------------------- number formats

// bf16 bit pattern -> exact double (bf16 is the top half of an fp32 word).
double oracle_bf16_to_double(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return (double)f;
}

// Nearest bf16 value to v, ties to even (8 significant bits), returned as bit pattern.
// Written from the definition: scale the significand to [128, 256), round to the
// nearest integer with ties to even, scale back. Overflow goes to +-inf.
uint16_t oracle_round_bf16(double v) {
  if (std::isnan(v)) return 0x7fc0;
  if (v == 0.0 || std::isinf(v)) {
    float f = (float)v;
    uint32_t u;
    std::memcpy(&u, &f, 4);
    return (uint16_t)(u >> 16);
  }
  int e;
  double m = std::frexp(v, &e);          // v = m * 2^e, 0.5 <= |m| < 1
  int q = e - 8;                           // quantum exponent for 8 significant bits
  if (q < -133) q = -133;                  // bf16 subnormal spacing is 2^-133
  double r = std::nearbyint(std::ldexp(v, -q));  // default rounding mode: ties to even
  double rv = std::ldexp(r, q);
  float f = (float)rv;                     // exact: rv has <= 8 significant bits
  if (std::fabs(rv) > 3.3895313892515355e38) f = v > 0 ? INFINITY : -INFINITY;
  uint32_t u;
  std::memcpy(&u, &f, 4);
  return (uint16_t)(u >> 16);
}

static inline double load(const void* p, int bf16, int64_t i) {
  return bf16 ? oracle_bf16_to_double(((const uint16_t*)p)[i]) : (double)((const float*)p)[i];
}

// GeLU, exact erf form: 0.5 * z * (1 + erf(z / sqrt(2))) = z * Phi(z).
double oracle_gelu(double z) { return 0.5 * z * (1.0 + std::erf(z / std::sqrt(2.0))); }

// ---------------------------------------------------------------- router

// Router logits l[t,e] = sum_i x[t,i] * W_r[e,i] (+ b_r[e]), accumulated in double in
// index order, rounded to fp32. W_r is stored [E, d] (row e is expert e's vector), so
// both W_r x (blog formula) and x W_r (comparison article, "Router computation") read
// the same numbers. b_r is the optional per-expert logit bias of the skewed workloads.
void oracle_router_logits(const void* x, int x_bf16, int64_t T, int d, const float* w_r,
                          const float* b_r, int E, float* logits) {
  for (int64_t t = 0; t < T; ++t)
    for (int e = 0; e < E; ++e) {
      double s = 0.0;
      for (int i = 0; i < d; ++i) s += load(x, x_bf16, t * d + i) * (double)w_r[(int64_t)e * d + i];
      if (b_r) s += (double)b_r[e];
      logits[t * E + e] = (float)s;
    }
}

// Softmax over the E fp32 logits of one token, in double.
static void softmax_row(const float* l, int E, double* p) {
  double m = -INFINITY;
  for (int e = 0; e < E; ++e) m = l[e] > m ? (double)l[e] : m;
  double z = 0.0;
  for (int e = 0; e < E; ++e) z += std::exp((double)l[e] - m);
  for (int e = 0; e < E; ++e) p[e] = std::exp((double)l[e] - m) / z;
}

// TopK(p(x), k) and the gates p_e (unrenormalised). Softmax is monotone, so the top-k
// of p is the top-k of the fp32 logits; ties go to the lowest expert index.
// probs (optional) receives the full [T, E] softmax in double.
void oracle_route(const float* logits, int64_t T, int E, int k, int32_t* ids, float* gates,
                  double* probs) {
  std::vector<double> p(E);
  std::vector<char> taken(E);
  for (int64_t t = 0; t < T; ++t) {
    const float* l = logits + t * E;
    softmax_row(l, E, p.data());
    if (probs)
      for (int e = 0; e < E; ++e) probs[t * E + e] = p[e];
    std::fill(taken.begin(), taken.end(), 0);
    for (int j = 0; j < k; ++j) {
      int best = -1;
      for (int e = 0; e < E; ++e)
        if (!taken[e] && (best < 0 || l[e] > l[best])) best = e;
      taken[best] = 1;
      ids[t * k + j] = best;
      gates[t * k + j] = (float)p[best];
    }
  }
}

// Switch-style load-balance statistics: f_i = (1/T) #{t : top-1 choice of t is i},
// Q_i = (1/T) sum_t p_{t,i}, aux = alpha * E * sum_i f_i * Q_i.
void oracle_lb_stats(const float* logits, const int32_t* ids, int64_t T, int E, int k,
                     double alpha, double* f, double* Q, double* aux) {
  std::vector<double> p(E);
  for (int e = 0; e < E; ++e) f[e] = Q[e] = 0.0;
  for (int64_t t = 0; t < T; ++t) {
    f[ids[t * k]] += 1.0;
    softmax_row(logits + t * E, E, p.data());
    for (int e = 0; e < E; ++e) Q[e] += p[e];
  }
  double s = 0.0;
  for (int e = 0; e < E; ++e) {
    f[e] /= (double)T;
    Q[e] /= (double)T;
    s += f[e] * Q[e];
  }
  *aux = alpha * (double)E * s;
}

// ---------------------------------------------------------------- capacity and slots

// Capacity = (tokens in the batch / experts) x capacity factor (comparison article,
// "Expert Capacity Overflow"), with the k choices of each token counted and rounded up:
// C = ceil(k * T / E * cf). The factor is a decimal number held in binary (1.1 is stored a
// little above 1.1), and the two operations round, so a product that lands within a few units
// in the last place above an integer is that integer: the capacity the decimal factor means
// (k = 1, T = 100, E = 10, cf = 1.1 gives 11, not 12).
int64_t oracle_capacity(int64_t T, int E, int k, double capacity_factor) {
  const double share = (double)k * (double)T / (double)E;
  const double v = share * capacity_factor;
  const double below = std::floor(v);
  const double ulp = std::nextafter(v, INFINITY) - v;
  if (v - below <= 8.0 * ulp) return (int64_t)below;
  return (int64_t)std::ceil(v);
}

// First-come slot assignment: walk the (token, choice) pairs in token order and give
// each the next free position of its expert; a position >= C is an overflow (-1).
// counts[e] receives the demand (before the capacity drop).
void oracle_assign_slots(const int32_t* ids, int64_t T, int k, int E, int64_t C, int32_t* slot,
                         int32_t* counts) {
  std::vector<int64_t> cnt(E, 0);
  for (int64_t t = 0; t < T; ++t)
    for (int j = 0; j < k; ++j) {
      const int e = ids[t * k + j];
      const int64_t s = cnt[e]++;
      slot[t * k + j] = s < C ? (int32_t)s : -1;
    }
  for (int e = 0; e < E; ++e) counts[e] = (int32_t)cnt[e];
}

// Priority overflow (a routing variant): inside each expert, the pairs are ranked by router
// probability, highest first (equal probabilities: lower pair index first), and the first C
// ranks are kept. The comparison article's capacity example ranks E0's tokens by their router
// probability (t3 0.859 > t0 0.817 > t1 0.669) and keeps t3, t0, dropping t1. probs are the
// softmax probabilities p of each chosen expert, [T, k] fp32, before any renormalisation of the
// gates: renormalising over a token's k choices changes what multiplies the expert output, not
// how strongly the router prefers that token for the expert (at k = 1 every renormalised gate
// is 1 and would carry no preference at all).
void oracle_assign_slots_priority(const int32_t* ids, const float* probs, int64_t T, int k, int E,
                                  int64_t C, int32_t* slot, int32_t* counts) {
  std::vector<std::vector<int64_t>> members(E);
  for (int64_t p = 0; p < T * k; ++p) members[ids[p]].push_back(p);
  for (int e = 0; e < E; ++e) {
    std::vector<int64_t>& m = members[e];
    std::sort(m.begin(), m.end(), [&](int64_t a, int64_t b) {
      if (probs[a] != probs[b]) return probs[a] > probs[b];
      return a < b;
    });
    for (size_t r = 0; r < m.size(); ++r) slot[m[r]] = (int64_t)r < C ? (int32_t)r : -1;
    counts[e] = (int32_t)m.size();
  }
}

// Renormalised gates (a routing variant): the k chosen probabilities divided by their sum (the
// survey notes §1.1.1.1: taking top-k after the softmax leaves values that need an extra
// normalisation). Computed in double from the given fp32 gates, rounded to fp32.
void oracle_renormalize_gates(float* gates, int64_t T, int k) {
  for (int64_t t = 0; t < T; ++t) {
    double s = 0.0;
    for (int j = 0; j < k; ++j) s += (double)gates[t * k + j];
    for (int j = 0; j < k; ++j) gates[t * k + j] = (float)((double)gates[t * k + j] / s);
  }
}

// Extra router statistics:
//   z-loss L_z = (1/T) sum_t (log sum_e exp(l_te))^2 (comparison article, "Router Z-loss");
//   CoV^2 of Importance_i = sum over choices routed to i of their gate, and of Load_i = number of
//   choices routed to i (survey notes §1.1.4.1, Importance and Load losses; without noise the
//   probability that expert i is selected is the indicator of the selection). CoV = std / mean
//   with the population variance; 0 when the mean is 0.
static double cov2(const std::vector<double>& v) {
  double mean = 0.0;
  for (double a : v) mean += a;
  mean /= (double)v.size();
  if (mean == 0.0) return 0.0;
  double var = 0.0;
  for (double a : v) var += (a - mean) * (a - mean);
  var /= (double)v.size();
  return var / (mean * mean);
}

void oracle_router_losses(const float* logits, const int32_t* ids, const float* gates, int64_t T,
                          int E, int k, double* z_loss, double* cov2_importance,
                          double* cov2_load) {
  double z = 0.0;
  for (int64_t t = 0; t < T; ++t) {
    const float* l = logits + t * E;
    double m = -INFINITY;
    for (int e = 0; e < E; ++e) m = (double)l[e] > m ? (double)l[e] : m;
    double s = 0.0;
    for (int e = 0; e < E; ++e) s += std::exp((double)l[e] - m);
    const double lz = m + std::log(s);
    z += lz * lz;
  }
  *z_loss = T > 0 ? z / (double)T : 0.0;
  std::vector<double> imp(E, 0.0), load(E, 0.0);
  for (int64_t p = 0; p < T * k; ++p) {
    imp[ids[p]] += (double)gates[p];
    load[ids[p]] += 1.0;
  }
  *cov2_importance = cov2(imp);
  *cov2_load = cov2(load);
}

// ---------------------------------------------------------------- expert FFN

// One expert (or the dense MLP) on one token: z = W1 x + b1, h = GeLU(z) (rounded to
// bf16 for bf16 weights), y = W2 h + b2, rounded to fp32. W1 is [d_ff, d], W2 is
// [d, d_ff]; b1/b2 may be NULL.
void oracle_ffn(const void* x_row, int bf16, int d, int d_ff, const void* w1, const void* b1,
                const void* w2, const void* b2, float* y) {
  std::vector<double> h(d_ff);
  for (int j = 0; j < d_ff; ++j) {
    double z = 0.0;
    for (int i = 0; i < d; ++i) z += load(w1, bf16, (int64_t)j * d + i) * load(x_row, bf16, i);
    if (b1) z += load(b1, bf16, j);
    double g = oracle_gelu(z);
    h[j] = bf16 ? oracle_bf16_to_double(oracle_round_bf16(g)) : g;
  }
  for (int o = 0; o < d; ++o) {
    double s = 0.0;
    for (int j = 0; j < d_ff; ++j) s += load(w2, bf16, (int64_t)o * d_ff + j) * h[j];
    if (b2) s += load(b2, bf16, o);
    y[o] = (float)s;
  }
}

// ---------------------------------------------------------------- combine

// out[t] = [residual[t]] + [dense[t]] + sum_{j : slot[t,j] >= 0} gate[t,j] * y[t,j], in
// double. y holds one expert output per (token, choice) pair: [T, k, d] fp32. Dropped
// pairs (slot < 0) contribute nothing, so an overflowed token keeps only its residual.
void oracle_combine(int64_t T, int d, int k, const void* residual, int res_bf16,
                    const float* dense, const float* gates, const int32_t* slot, const float* y,
                    double* out) {
  for (int64_t t = 0; t < T; ++t)
    for (int i = 0; i < d; ++i) {
      double s = 0.0;
      if (residual) s += load(residual, res_bf16, t * d + i);
      if (dense) s += (double)dense[t * d + i];
      for (int j = 0; j < k; ++j)
        if (slot[t * k + j] >= 0) s += (double)gates[t * k + j] * (double)y[(t * k + j) * (int64_t)d + i];
      out[t * d + i] = s;
    }
}

// ---------------------------------------------------------------- whole layer

// The layer, step by step: logits -> route -> statistics -> capacity -> slots -> for each
// requested token: residual + dense MLP + gate-weighted kept experts.
//
// logits_in: if non-NULL these fp32 logits are used instead of computing them (routing
//            decided from the same logits as another implementation).
// probs_in:  if non-NULL, [T, k] fp32 softmax probabilities of the chosen experts (before any
//            renormalisation) used instead of the oracle's own: the priority ranking key and,
//            renormalised when asked, the gates.
// tokens:    the tokens whose output rows are computed (NULL = all T, in order);
//            routing, slots and statistics always cover all T tokens.
// out_exact: [n, d] double before the final rounding; out_rounded: [n, d] in the output
//            type (bf16 bits if out_bf16, else fp32). Either may be NULL.
// Returns the capacity C.
int64_t oracle_layer_forward(int64_t T, int d, int d_ff, int E, int k, double capacity_factor,
                             int bf16, int add_input_residual, const void* x, const float* w_r,
                             const float* b_r, const void* w1, const void* b1, const void* w2,
                             const void* b2, const void* dense_w1, const void* dense_b1,
                             const void* dense_w2, const void* dense_b2, double aux_alpha,
                             const float* logits_in, const int64_t* tokens, int64_t n_tokens,
                             float* logits_out, int32_t* ids, float* gates, int32_t* slot,
                             int32_t* counts, double* lb_stats, double* out_exact,
                             void* out_rounded, int out_bf16, int overflow_priority,
                             int renormalize, const float* probs_in, double* losses) {
  std::vector<float> logits_own;
  const float* logits = logits_in;
  if (!logits) {
    logits_own.resize((size_t)T * E);
    oracle_router_logits(x, bf16, T, d, w_r, b_r, E, logits_own.data());
    logits = logits_own.data();
  }
  if (logits_out && logits_out != logits) std::memcpy(logits_out, logits, sizeof(float) * T * E);
  oracle_route(logits, T, E, k, ids, gates, nullptr);
  // probs_in: the fp32 probabilities of the chosen experts another implementation computed (a
  // priority ranking between two nearly equal probabilities is decided in that implementation's
  // precision); NULL = the oracle's own
  if (probs_in && probs_in != gates) std::memcpy(gates, probs_in, sizeof(float) * T * k);
  const std::vector<float> probs(gates, gates + T * k);  // before any renormalisation
  if (renormalize) oracle_renormalize_gates(gates, T, k);
  if (lb_stats) oracle_lb_stats(logits, ids, T, E, k, aux_alpha, lb_stats, lb_stats + E, lb_stats + 2 * E);
  if (losses) oracle_router_losses(logits, ids, gates, T, E, k, losses, losses + 1, losses + 2);
  const int64_t C = oracle_capacity(T, E, k, capacity_factor);
  if (overflow_priority) oracle_assign_slots_priority(ids, probs.data(), T, k, E, C, slot, counts);
  else oracle_assign_slots(ids, T, k, E, C, slot, counts);

  const int64_t n = tokens ? n_tokens : T;
  const size_t esz = bf16 ? 2 : 4;
  std::vector<float> y((size_t)k * d), dense((size_t)d);
  std::vector<double> row(d);
  for (int64_t r = 0; r < n; ++r) {
    const int64_t t = tokens ? tokens[r] : r;
    const char* xt = (const char*)x + (size_t)t * d * esz;
    for (int j = 0; j < k; ++j) {
      if (slot[t * k + j] < 0) continue;
      const int64_t e = ids[t * k + j];
      oracle_ffn(xt, bf16, d, d_ff, (const char*)w1 + (size_t)e * d_ff * d * esz,
                 b1 ? (const char*)b1 + (size_t)e * d_ff * esz : nullptr,
                 (const char*)w2 + (size_t)e * d * d_ff * esz,
                 b2 ? (const char*)b2 + (size_t)e * d * esz : nullptr, y.data() + (size_t)j * d);
    }
    const bool has_dense = dense_w1 != nullptr;
    if (has_dense) oracle_ffn(xt, bf16, d, d_ff, dense_w1, dense_b1, dense_w2, dense_b2, dense.data());
    oracle_combine(1, d, k, add_input_residual ? xt : nullptr, bf16, has_dense ? dense.data() : nullptr,
                   gates + t * k, slot + t * k, y.data(), row.data());
    for (int i = 0; i < d; ++i) {
      if (out_exact) out_exact[r * d + i] = row[i];
      if (out_rounded) {
        if (out_bf16) ((uint16_t*)out_rounded)[r * d + i] = oracle_round_bf16(row[i]);
        else ((float*)out_rounded)[r * d + i] = (float)row[i];
      }
    }
  }
  return C;
}

// ---------------------------------------------------------------- backward (training)
//
// The gradient of the training objective
//     L = sum_{t,i} dout[t,i] * out[t,i] + aux_weight * aux + z_weight * z_loss
// with respect to x, W_r, b_r, every expert's W1, b1, W2, b2 and the dense MLP's weights, by the
// chain rule through the forward pass above (the pages' headline numbers are training
// throughput; DeepSpeed-MoE notes on training cost; survey notes §1.1.4.1 and the comparison
// article's "Router Z-loss" give the two extra loss terms). Readings:
//   * the routing decisions (top-k ids, slots, the counts f_i) are piecewise constant and carry
//     no gradient; the gates carry it through the softmax (and the renormalisation);
//   * a dropped pair contributes nothing forward, so nothing backward (comparison article,
//     "Expert Capacity Overflow": no gradient for that expert);
//   * the roundings of the forward pass (fp32 logits, bf16 h) are passed straight through, and
//     every gradient uses the forward's own values (y rounded to fp32, h to bf16).

// dGeLU/dz for GeLU(z) = z * Phi(z): Phi(z) + z * phi(z).
double oracle_gelu_grad(double z) {
  const double Phi = 0.5 * (1.0 + std::erf(z / std::sqrt(2.0)));
  const double phi = std::exp(-0.5 * z * z) / std::sqrt(2.0 * M_PI);
  return Phi + z * phi;
}

// One FFN (an expert or the dense MLP) on one token, forward then backward for an output
// gradient dy (d doubles). Accumulates dW1 [d_ff, d], db1 [d_ff], dW2 [d, d_ff], db2 [d] and
// dx_row [d]; y_out (optional) receives the forward output rounded to fp32.
static void ffn_backward(const void* x_row, int bf16, int d, int d_ff, const void* w1,
                         const void* b1, const void* w2, const void* b2, const double* dy,
                         double* dw1, double* db1, double* dw2, double* db2, double* dx_row) {
  std::vector<double> z(d_ff), h(d_ff), dz(d_ff);
  for (int j = 0; j < d_ff; ++j) {
    double a = 0.0;
    for (int i = 0; i < d; ++i) a += load(w1, bf16, (int64_t)j * d + i) * load(x_row, bf16, i);
    if (b1) a += load(b1, bf16, j);
    z[j] = a;
    const double g = oracle_gelu(a);
    h[j] = bf16 ? oracle_bf16_to_double(oracle_round_bf16(g)) : g;
  }
  // y = W2 h + b2: dW2 += dy h^T, db2 += dy, dh = W2^T dy
  for (int o = 0; o < d; ++o) {
    if (db2) db2[o] += dy[o];
    for (int j = 0; j < d_ff; ++j) dw2[(int64_t)o * d_ff + j] += dy[o] * h[j];
  }
  for (int j = 0; j < d_ff; ++j) {
    double dh = 0.0;
    for (int o = 0; o < d; ++o) dh += load(w2, bf16, (int64_t)o * d_ff + j) * dy[o];
    dz[j] = dh * oracle_gelu_grad(z[j]);
  }
  // z = W1 x + b1: dW1 += dz x^T, db1 += dz, dx += W1^T dz
  for (int j = 0; j < d_ff; ++j) {
    if (db1) db1[j] += dz[j];
    for (int i = 0; i < d; ++i) dw1[(int64_t)j * d + i] += dz[j] * load(x_row, bf16, i);
  }
  for (int i = 0; i < d; ++i) {
    double s = 0.0;
    for (int j = 0; j < d_ff; ++j) s += load(w1, bf16, (int64_t)j * d + i) * dz[j];
    dx_row[i] += s;
  }
}

// Gradients of the whole layer. Inputs are those of oracle_layer_forward (logits_in / probs_in
// as there: routing decided on another implementation's fp32 values), plus dout [T, d] and the
// weights of the two extra loss terms. Outputs (double, zeroed here, any may be NULL):
// dx [T, d], dw_r [E, d], db_r [E], dw1 [E, d_ff, d], db1 [E, d_ff], dw2 [E, d, d_ff],
// db2 [E, d], and the dense MLP's ddw1 [d_ff, d], ddb1 [d_ff], ddw2 [d, d_ff], ddb2 [d].
// dgates (optional, [T, k]) receives dL/dgate of each choice; dlogits (optional, [T, E]) dL/dl.
void oracle_layer_backward(int64_t T, int d, int d_ff, int E, int k, double capacity_factor,
                           int bf16, int add_input_residual, const void* x, const float* w_r,
                           const float* b_r, const void* w1, const void* b1, const void* w2,
                           const void* b2, const void* dense_w1, const void* dense_b1,
                           const void* dense_w2, const void* dense_b2, double aux_alpha,
                           int overflow_priority, int renormalize, const float* logits_in,
                           const float* probs_in, const double* dout, double aux_weight,
                           double z_weight, double* dx, double* dw_r, double* db_r, double* dw1,
                           double* db1, double* dw2, double* db2, double* ddw1, double* ddb1,
                           double* ddw2, double* ddb2, double* dgates, double* dlogits) {
  // ---- forward decisions
  std::vector<float> logits((size_t)T * E);
  if (logits_in) std::memcpy(logits.data(), logits_in, sizeof(float) * T * E);
  else oracle_router_logits(x, bf16, T, d, w_r, b_r, E, logits.data());
  std::vector<int32_t> ids((size_t)T * k), slot((size_t)T * k), counts(E);
  std::vector<float> gates((size_t)T * k);
  std::vector<double> probs((size_t)T * E);
  oracle_route(logits.data(), T, E, k, ids.data(), gates.data(), probs.data());
  if (probs_in) std::memcpy(gates.data(), probs_in, sizeof(float) * T * k);
  std::vector<float> raw = gates;  // the chosen p before any renormalisation
  if (renormalize) oracle_renormalize_gates(gates.data(), T, k);
  std::vector<double> f(E), Q(E);
  double aux = 0.0;
  oracle_lb_stats(logits.data(), ids.data(), T, E, k, aux_alpha, f.data(), Q.data(), &aux);
  const int64_t C = oracle_capacity(T, E, k, capacity_factor);
  if (overflow_priority) oracle_assign_slots_priority(ids.data(), raw.data(), T, k, E, C, slot.data(), counts.data());
  else oracle_assign_slots(ids.data(), T, k, E, C, slot.data(), counts.data());

  auto zero = [](double* a, size_t n) { if (a) std::fill(a, a + n, 0.0); };
  zero(dx, (size_t)T * d);
  zero(dw_r, (size_t)E * d);
  zero(db_r, E);
  zero(dw1, (size_t)E * d_ff * d);
  zero(db1, (size_t)E * d_ff);
  zero(dw2, (size_t)E * d * d_ff);
  zero(db2, (size_t)E * d);
  zero(ddw1, (size_t)d_ff * d);
  zero(ddb1, d_ff);
  zero(ddw2, (size_t)d * d_ff);
  zero(ddb2, d);
  const size_t es = bf16 ? 2 : 4;
  std::vector<double> dx_row(d), dy(d), dl(E), dp(E);
  std::vector<float> y(d);
  for (int64_t t = 0; t < T; ++t) {
    const char* xt = (const char*)x + (size_t)t * d * es;
    const double* go = dout + (size_t)t * d;
    std::fill(dx_row.begin(), dx_row.end(), 0.0);
    // residual: out += x
    if (add_input_residual)
      for (int i = 0; i < d; ++i) dx_row[i] += go[i];
    // dense MLP: out += DenseMLP(x)
    if (dense_w1) ffn_backward(xt, bf16, d, d_ff, dense_w1, dense_b1, dense_w2, dense_b2, go, ddw1,
                               dense_b1 ? ddb1 : nullptr, ddw2, dense_b2 ? ddb2 : nullptr,
                               dx_row.data());
    // experts: out += gate_j * y_j over the kept choices
    std::vector<double> dg(k, 0.0);
    for (int j = 0; j < k; ++j) {
      if (slot[t * k + j] < 0) continue;
      const int e = ids[t * k + j];
      const size_t w1o = (size_t)e * d_ff * d * es, w2o = (size_t)e * d * d_ff * es;
      const void* we1 = (const char*)w1 + w1o;
      const void* we2 = (const char*)w2 + w2o;
      const void* be1 = b1 ? (const void*)((const char*)b1 + (size_t)e * d_ff * es) : nullptr;
      const void* be2 = b2 ? (const void*)((const char*)b2 + (size_t)e * d * es) : nullptr;
      oracle_ffn(xt, bf16, d, d_ff, we1, be1, we2, be2, y.data());
      double s = 0.0;
      for (int i = 0; i < d; ++i) s += go[i] * (double)y[i];
      dg[j] = s;  // dL/dgate
      const double g = gates[t * k + j];
      for (int i = 0; i < d; ++i) dy[i] = g * go[i];
      ffn_backward(xt, bf16, d, d_ff, we1, be1, we2, be2, dy.data(), dw1 + (size_t)e * d_ff * d,
                   b1 ? db1 + (size_t)e * d_ff : nullptr, dw2 + (size_t)e * d * d_ff,
                   b2 ? db2 + (size_t)e * d : nullptr, dx_row.data());
    }
    if (dgates)
      for (int j = 0; j < k; ++j) dgates[t * k + j] = dg[j];
    // gates -> p: gate_j = p_{e_j} (or p_{e_j} / S with S = sum of the chosen p)
    const double* pt = probs.data() + (size_t)t * E;
    std::fill(dp.begin(), dp.end(), 0.0);
    if (renormalize) {
      double S = 0.0, gdg = 0.0;
      for (int j = 0; j < k; ++j) S += (double)raw[t * k + j];
      for (int j = 0; j < k; ++j) gdg += dg[j] * ((double)raw[t * k + j] / S);
      for (int j = 0; j < k; ++j) dp[ids[t * k + j]] += (dg[j] - gdg) / S;
    } else {
      for (int j = 0; j < k; ++j) dp[ids[t * k + j]] += dg[j];
    }
    // aux = alpha * E * sum_e f_e * Q_e, Q_e = (1/T) sum_t p_te, f constant
    for (int e = 0; e < E; ++e) dp[e] += aux_weight * aux_alpha * E * f[e] / (double)T;
    // p = softmax(l): dl_e = p_e (dp_e - sum_e' p_e' dp_e')
    double pdp = 0.0;
    for (int e = 0; e < E; ++e) pdp += pt[e] * dp[e];
    for (int e = 0; e < E; ++e) dl[e] = pt[e] * (dp[e] - pdp);
    // z-loss = (1/T) sum_t (log sum_e exp l_te)^2: dl_e += 2 log Z p_e / T
    if (z_weight != 0.0) {
      double m = -INFINITY;
      for (int e = 0; e < E; ++e) m = std::max(m, (double)logits[(size_t)t * E + e]);
      double zs = 0.0;
      for (int e = 0; e < E; ++e) zs += std::exp((double)logits[(size_t)t * E + e] - m);
      const double lz = m + std::log(zs);
      for (int e = 0; e < E; ++e) dl[e] += z_weight * 2.0 * lz * pt[e] / (double)T;
    }
    if (dlogits)
      for (int e = 0; e < E; ++e) dlogits[(size_t)t * E + e] = dl[e];
    // l = W_r x + b_r
    for (int e = 0; e < E; ++e) {
      if (db_r) db_r[e] += dl[e];
      if (dw_r)
        for (int i = 0; i < d; ++i) dw_r[(size_t)e * d + i] += dl[e] * load(xt, bf16, i);
      for (int i = 0; i < d; ++i) dx_row[i] += (double)w_r[(size_t)e * d + i] * dl[e];
    }
    if (dx)
      for (int i = 0; i < d; ++i) dx[(size_t)t * d + i] = dx_row[i];
  }
}

}  // extern "C"
