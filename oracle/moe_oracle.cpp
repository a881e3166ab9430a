// moe_oracle.cpp -- plain fp64 CPU oracle of the sparse Mixture-of-Experts FFN layer forward.
//
// TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's CPU-baseline
// leg load this code.  It shares no source with the CUDA path.  Every function is the plain
// definition, written for a reader to check against the pages by eye:
//
//   * josueisai.com, "Mixture of experts: por que un modelo enorme apenas usa sus parametros",
//     section "El router: la pieza que de verdad decide": the router is a linear projection
//     followed by a softmax; the k best experts are kept, the softmax is normalised only over
//     the chosen k, and the chosen experts' outputs are summed weighted by those scores; the
//     eager per-expert loop printed there is the procedural form (oracle_layer_eager below).
//   * gotburnout.io glossary "MoE (Mixture of Experts)", section 2 (layer diagram):
//     p = Softmax(TopK(W_g x)), y = sum_i p_i Expert_i(x) (+ residual, which the caller adds),
//     shared experts always active; section 3 step 3: the SwiGLU expert FFN.
//   * dev.smart-guide.co.kr deep-dive, section "La Solucion: WeightConverter": the packed
//     gate_up_proj tensor is the per-expert w1 and w3 matrices merged along a new expert dim 0
//     and concatenated along dim 1 (w1 first), so gate_up[e] = [w1_e ; w3_e], shape [2F, D].
//
// Readings taken where the pages are silent or garbled (each is repeated in the design notes):
//   - SiLU goes on rows [0, F) of gate_up[e] (w1, "gate"); rows [F, 2F) (w3, "up") multiply.
//   - The optional per-expert bias (aux-loss-free balancing) enters the selection only; the
//     weights p use the unbiased logits.
//   - top-k order: score descending, ties to the lower expert id.
//   - expert-contiguous order: experts ascending, tokens ascending within an expert.
//   - the shared expert is added with coefficient 1.
//   - no intermediate rounding: bf16 inputs are read as exact doubles and everything after is fp64.

#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>
#include <algorithm>

namespace {

inline double bf16_value(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  std::memcpy(&f, &u, sizeof f);
  return (double)f;
}

template <class Fn>
void for_tokens(int64_t T, int nthreads, Fn fn) {
  if (nthreads <= 1 || T < 2) {
    for (int64_t t = 0; t < T; ++t) fn(t);
    return;
  }
  std::vector<std::thread> pool;
  int n = (int)std::min<int64_t>(nthreads, T);
  for (int w = 0; w < n; ++w)
    pool.emplace_back([=] {
      for (int64_t t = w; t < T; t += n) fn(t);
    });
  for (auto& th : pool) th.join();
}

// logits l[e] = sum_d x[d] * W_g[e, d] for one token (the router's linear projection)
void router_logits(const uint16_t* x_row, const uint16_t* wg, int64_t D, int E, double* l) {
  for (int e = 0; e < E; ++e) {
    double acc = 0.0;
    const uint16_t* w = wg + (int64_t)e * D;
    for (int64_t d = 0; d < D; ++d) acc += bf16_value(x_row[d]) * bf16_value(w[d]);
    l[e] = acc;
  }
}

// Top-k selection on s = l + bias, then p = softmax over the chosen k of the unbiased l.
void select_and_weight(const double* l, const float* bias, int E, int k, int32_t* idx, double* p) {
  std::vector<double> s(E);
  std::vector<char> taken(E, 0);
  for (int e = 0; e < E; ++e) s[e] = l[e] + (bias ? (double)bias[e] : 0.0);
  for (int j = 0; j < k; ++j) {
    int best = -1;
    for (int e = 0; e < E; ++e)
      if (!taken[e] && (best < 0 || s[e] > s[best])) best = e;  // strict '>' keeps the lower id on ties
    taken[best] = 1;
    idx[j] = best;
  }
  double m = l[idx[0]];
  for (int j = 1; j < k; ++j) m = std::max(m, l[idx[j]]);
  double z = 0.0;
  for (int j = 0; j < k; ++j) z += std::exp(l[idx[j]] - m);
  for (int j = 0; j < k; ++j) p[j] = std::exp(l[idx[j]] - m) / z;
}

// One SwiGLU expert on one token: a = silu(G x) * (U x), out = Down a.
// G = gate_up[0:F, :], U = gate_up[F:2F, :], Down = down[D, F]; silu(z) = z / (1 + e^-z).
void expert_ffn(const uint16_t* x_row, const uint16_t* gate_up, const uint16_t* down, int64_t D,
                int64_t F, double* out) {
  std::vector<double> a(F);
  for (int64_t n = 0; n < F; ++n) {
    const uint16_t* grow = gate_up + n * D;
    const uint16_t* urow = gate_up + (F + n) * D;
    double g = 0.0, u = 0.0;
    for (int64_t d = 0; d < D; ++d) {
      double xv = bf16_value(x_row[d]);
      g += bf16_value(grow[d]) * xv;
      u += bf16_value(urow[d]) * xv;
    }
    a[n] = g / (1.0 + std::exp(-g)) * u;
  }
  for (int64_t d = 0; d < D; ++d) {
    const uint16_t* drow = down + d * F;
    double acc = 0.0;
    for (int64_t n = 0; n < F; ++n) acc += bf16_value(drow[n]) * a[n];
    out[d] = acc;
  }
}

}  // namespace

extern "C" {

// Router: idx[T, k] (score-descending) and p[T, k]; logits[T, E] if non-NULL.
// Returns 0, or -1 on invalid sizes.
int oracle_router(const uint16_t* x, const uint16_t* wg, const float* bias, int64_t T, int64_t D,
                  int E, int k, double* logits, int32_t* idx, double* p, int nthreads) {
  if (T < 0 || D < 1 || E < 1 || k < 1 || k > E) return -1;
  for_tokens(T, nthreads, [&](int64_t t) {
    std::vector<double> l(E);
    router_logits(x + t * D, wg, D, E, l.data());
    if (logits) std::copy(l.begin(), l.end(), logits + t * E);
    select_and_weight(l.data(), bias, E, k, idx + t * k, p + t * k);
  });
  return 0;
}

// Top-k by exhaustive search over all k-subsets: the chosen set is the one with the largest
// total score (with distinct scores this is exactly the set of the k largest), listed by
// score descending.  Independent of the selection loop above; for small E only.
int oracle_topk_exhaustive(const double* s, int64_t T, int E, int k, int32_t* idx) {
  if (E > 20 || k < 1 || k > E) return -1;
  for (int64_t t = 0; t < T; ++t) {
    const double* st = s + t * E;
    double best_sum = -INFINITY;
    uint32_t best_mask = 0;
    for (uint32_t mask = 0; mask < (1u << E); ++mask) {
      if (__builtin_popcount(mask) != k) continue;
      double sum = 0.0;
      for (int e = 0; e < E; ++e)
        if (mask >> e & 1u) sum += st[e];
      if (sum > best_sum) best_sum = sum, best_mask = mask;
    }
    std::vector<int> chosen;
    for (int e = 0; e < E; ++e)
      if (best_mask >> e & 1u) chosen.push_back(e);
    std::stable_sort(chosen.begin(), chosen.end(), [&](int a, int b) { return st[a] > st[b]; });
    for (int j = 0; j < k; ++j) idx[t * k + j] = chosen[j];
  }
  return 0;
}

// Dispatch metadata: counts[E], offsets[E+1] (exclusive prefix sum), and the expert-contiguous
// order (experts ascending, tokens ascending within an expert): row r holds the assignment
// (perm_token[r], perm_slot[r]) and inv_perm[t*k + j] = r.  Returns -1 on an expert id
// outside [0, E).
int oracle_permute(const int32_t* idx, int64_t T, int E, int k, int32_t* counts, int32_t* offsets,
                   int32_t* perm_token, int32_t* perm_slot, int32_t* inv_perm) {
  for (int64_t i = 0; i < T * k; ++i)
    if (idx[i] < 0 || idx[i] >= E) return -1;
  for (int e = 0; e < E; ++e) counts[e] = 0;
  for (int64_t i = 0; i < T * k; ++i) counts[idx[i]]++;
  offsets[0] = 0;
  for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
  int64_t r = 0;
  for (int e = 0; e < E; ++e)
    for (int64_t t = 0; t < T; ++t)
      for (int j = 0; j < k; ++j)
        if (idx[t * k + j] == e) {
          perm_token[r] = (int32_t)t;
          perm_slot[r] = j;
          inv_perm[t * k + j] = (int32_t)r;
          ++r;
        }
  return 0;
}

// One expert FFN on one token row (exposed for per-assignment checks).
void oracle_expert_ffn(const uint16_t* x_row, const uint16_t* gate_up, const uint16_t* down, int64_t D,
                       int64_t F, double* out) {
  expert_ffn(x_row, gate_up, down, D, F, out);
}

// Layer forward: y[t] = sum_j p[t,j] * Expert_{idx[t,j]}(x_t) + SharedExpert(x_t).
// gate_up_ptrs[e] -> [2F, D] and down_ptrs[e] -> [D, F] for each expert e (an entry may be NULL
// when no token routes to e).  shared_gate_up [2Fs, D], shared_down [D, Fs] may be NULL (Fs = 0).
// idx_out / p_out (optional) receive the routing.  Returns 0, -1 bad sizes, -2 missing expert.
int oracle_layer(const uint16_t* x, const uint16_t* wg, const float* bias,
                 const uint16_t* const* gate_up_ptrs, const uint16_t* const* down_ptrs,
                 const uint16_t* shared_gate_up, const uint16_t* shared_down, int64_t T, int64_t D,
                 int E, int k, int64_t F, int64_t Fs, double* y, int32_t* idx_out, double* p_out,
                 int nthreads) {
  if (T < 0 || D < 1 || E < 1 || k < 1 || k > E || F < 1 || Fs < 0) return -1;
  std::vector<int> missing(T, 0);
  for_tokens(T, nthreads, [&](int64_t t) {
    std::vector<double> l(E), p(k), o(D), yt(D, 0.0);
    std::vector<int32_t> idx(k);
    router_logits(x + t * D, wg, D, E, l.data());
    select_and_weight(l.data(), bias, E, k, idx.data(), p.data());
    for (int j = 0; j < k; ++j) {
      int e = idx[j];
      if (!gate_up_ptrs[e] || !down_ptrs[e]) { missing[t] = 1; return; }
      expert_ffn(x + t * D, gate_up_ptrs[e], down_ptrs[e], D, F, o.data());
      for (int64_t d = 0; d < D; ++d) yt[d] += p[j] * o[d];
    }
    if (Fs > 0 && shared_gate_up && shared_down) {
      expert_ffn(x + t * D, shared_gate_up, shared_down, D, Fs, o.data());
      for (int64_t d = 0; d < D; ++d) yt[d] += o[d];
    }
    std::copy(yt.begin(), yt.end(), y + t * D);
    if (idx_out) std::copy(idx.begin(), idx.end(), idx_out + t * k);
    if (p_out) std::copy(p.begin(), p.end(), p_out + t * k);
  });
  for (int64_t t = 0; t < T; ++t)
    if (missing[t]) return -2;
  return 0;
}

// The eager form of the same layer: route every token, then for each top-k slot j and each
// expert e, run expert e on exactly the tokens whose j-th choice is e and accumulate
// p[t, j] * Expert_e(x_t) into their output rows; finally add the shared expert.  The top-k here
// sorts all E experts by score (ties to the lower id) instead of the selection loop.
int oracle_layer_eager(const uint16_t* x, const uint16_t* wg, const float* bias,
                       const uint16_t* gate_up, const uint16_t* down, const uint16_t* shared_gate_up,
                       const uint16_t* shared_down, int64_t T, int64_t D, int E, int k, int64_t F,
                       int64_t Fs, double* y) {
  if (T < 0 || D < 1 || E < 1 || k < 1 || k > E) return -1;
  std::vector<double> l(T * E), p(T * k);
  std::vector<int32_t> idx(T * k);
  for (int64_t t = 0; t < T; ++t) {
    router_logits(x + t * D, wg, D, E, &l[t * E]);
    std::vector<int> order(E);
    for (int e = 0; e < E; ++e) order[e] = e;
    auto score = [&](int e) { return l[t * E + e] + (bias ? (double)bias[e] : 0.0); };
    std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return score(a) > score(b); });
    double z = 0.0, m = -INFINITY;
    for (int j = 0; j < k; ++j) m = std::max(m, l[t * E + order[j]]);
    for (int j = 0; j < k; ++j) z += std::exp(l[t * E + order[j]] - m);
    for (int j = 0; j < k; ++j) {
      idx[t * k + j] = order[j];
      p[t * k + j] = std::exp(l[t * E + order[j]] - m) / z;
    }
  }
  std::fill(y, y + T * D, 0.0);
  std::vector<double> o(D);
  for (int j = 0; j < k; ++j)
    for (int e = 0; e < E; ++e)
      for (int64_t t = 0; t < T; ++t) {
        if (idx[t * k + j] != e) continue;
        expert_ffn(x + t * D, gate_up + (int64_t)e * 2 * F * D, down + (int64_t)e * D * F, D, F, o.data());
        for (int64_t d = 0; d < D; ++d) y[t * D + d] += p[t * k + j] * o[d];
      }
  if (Fs > 0 && shared_gate_up && shared_down)
    for (int64_t t = 0; t < T; ++t) {
      expert_ffn(x + t * D, shared_gate_up, shared_down, D, Fs, o.data());
      for (int64_t d = 0; d < D; ++d) y[t * D + d] += o[d];
    }
  return 0;
}

// Aux-loss-free balancing (gotburnout.io glossary "MoE", section 2 item 4: router biases are
// adjusted dynamically so that no expert is overloaded).  The pages give no rule; the reading
// taken: after a batch with per-expert loads c_e (slots routed to e), every bias moves by a fixed
// step gamma towards balance,
//     bias_e <- bias_e + gamma * sign(mean(c) - c_e),
// an underloaded expert gaining score and an overloaded one losing it.  The comparison with the
// mean is done exactly as sign(sum(c) - E * c_e).  Each new bias is the fp32 value of the exact
// sum (the addition of two fp32 numbers rounded once).
void oracle_update_bias(const int32_t* counts, int E, float gamma, const float* bias_in, float* bias_out) {
  long long total = 0;
  for (int e = 0; e < E; ++e) total += counts[e];
  for (int e = 0; e < E; ++e) {
    const long long diff = total - (long long)E * counts[e];
    const double step = diff > 0 ? (double)gamma : (diff < 0 ? -(double)gamma : 0.0);
    bias_out[e] = (float)((double)bias_in[e] + step);
  }
}

// ---- FP8 (E4M3) expert weights -------------------------------------------------------------
// keryc.com "Mixture of Experts optimiza...", section "Resultados practicos": quantising "per
// expert" makes sense once the experts are packed.  Reading taken: each row of a packed weight
// tensor (one output feature of one expert) gets its own fp32 scale s = amax(row) / 448 and the
// codes q = E4M3(w / s), round to nearest even, saturating at +-448.  The row is dequantised as
// q * s.  E4M3 (OCP FP8): 1 sign, 4 exponent (bias 7), 3 mantissa bits; normal values
// 2^(e-7) * (1 + m/8) for e = 1..15 (e = 15 with m = 7 is NaN, so the largest is 448);
// subnormals m * 2^-9.

// Value of an E4M3 code.
double oracle_e4m3_value(uint8_t code) {
  const int sgn = code >> 7, e = (code >> 3) & 15, m = code & 7;
  double v = (e == 0) ? m * std::ldexp(1.0, -9) : std::ldexp(1.0 + m / 8.0, e - 7);
  if (e == 15 && m == 7) v = NAN;
  return sgn ? -v : v;
}

// Nearest E4M3 code to a finite value (ties to the even code), saturating at +-448.  The
// non-negative finite codes 0x00..0x7E have increasing values, so the nearest one is found by
// bisection over their values.
uint8_t oracle_e4m3_encode(double v) {
  static const std::vector<double> table = [] {
    std::vector<double> t(127);
    for (int c = 0; c <= 0x7E; ++c) t[c] = oracle_e4m3_value((uint8_t)c);
    return t;
  }();
  const uint8_t sgn = std::signbit(v) ? 0x80 : 0;
  const double a = std::fabs(v);
  if (a >= table[0x7E]) return sgn | 0x7E;
  int lo = 0, hi = 0x7E;  // table[lo] <= a < table[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) / 2;
    if (table[mid] <= a) lo = mid; else hi = mid;
  }
  const double dlo = a - table[lo], dhi = table[hi] - a;
  const int c = dlo < dhi ? lo : (dhi < dlo ? hi : ((lo & 1) == 0 ? lo : hi));
  return sgn | (uint8_t)c;
}

// Per-row quantisation of a bf16 [rows, K] tensor: scales[r] = amax / 448 (fp32), codes of
// (w / scale) computed in fp32.  All-zero rows get scale 1 and zero codes.
void oracle_quantize_rows_fp8(const uint16_t* w, int64_t rows, int64_t K, uint8_t* q, float* scales,
                              int nthreads) {
  for_tokens(rows, nthreads, [&](int64_t r) {  // rows are independent
    float amax = 0.0f;
    for (int64_t k = 0; k < K; ++k) amax = std::max(amax, (float)std::fabs(bf16_value(w[r * K + k])));
    const float s = amax > 0.0f ? amax / 448.0f : 1.0f;
    scales[r] = s;
    for (int64_t k = 0; k < K; ++k) {
      const float v = (float)bf16_value(w[r * K + k]) / s;
      q[r * K + k] = oracle_e4m3_encode((double)v);
    }
  });
}

// One SwiGLU expert on one token with E4M3 weights: the definition of expert_ffn above on the
// dequantised weights (q * scale, exact in fp64).
void oracle_expert_ffn_fp8(const uint16_t* x_row, const uint8_t* gu_q, const float* gu_s, const uint8_t* dn_q,
                           const float* dn_s, int64_t D, int64_t F, double* out) {
  std::vector<double> a(F);
  for (int64_t n = 0; n < F; ++n) {
    double g = 0.0, u = 0.0;
    for (int64_t d = 0; d < D; ++d) {
      const double xv = bf16_value(x_row[d]);
      g += oracle_e4m3_value(gu_q[n * D + d]) * (double)gu_s[n] * xv;
      u += oracle_e4m3_value(gu_q[(F + n) * D + d]) * (double)gu_s[F + n] * xv;
    }
    a[n] = g / (1.0 + std::exp(-g)) * u;
  }
  for (int64_t d = 0; d < D; ++d) {
    double acc = 0.0;
    for (int64_t n = 0; n < F; ++n) acc += oracle_e4m3_value(dn_q[d * F + n]) * (double)dn_s[d] * a[n];
    out[d] = acc;
  }
}

// ---- backward pass (training) ----------------------------------------------------------------
// keryc.com, section "Entrenamiento: todavia desafiante, pero con avances", and dev.smart-guide.co.kr,
// section "Entrenamiento MoE: 12x Mas Rapido": MoE layers are trained, with grouped-GEMM kernels.
// The pages print no formulas for the backward pass, so it is the chain rule applied to the
// forward defined above, step by step.  With L = sum(dy * y):
//   slot (t, j), expert e = idx[t, j], o = Expert_e(x_t), h = silu(g) * u, g = G_e x_t, u = U_e x_t:
//     dp_j = dy_t . o,           do = p_j dy_t,
//     dh   = Down_e^T do,        dDown_e += do h^T,
//     dg   = dh * u * silu'(g),  du = dh * silu(g),    silu'(z) = s(z) (1 + z (1 - s(z))),
//     dx_t += G_e^T dg + U_e^T du,   dG_e += dg x_t^T,   dU_e += du x_t^T;
//   softmax over the chosen k:  dl_j = p_j (dp_j - sum_i p_i dp_i), and the other logits get 0;
//     dx_t += sum_j dl_j W_g[idx_j],   dW_g[idx_j] += dl_j x_t;
//   the shared expert: the same with p = 1.
// The top-k selection is piecewise constant: neither it nor the selection bias carries a gradient.
// These entry points take fp64 parameters so that the gradient can be checked against finite
// differences of oracle_layer_f64.

namespace {

// x as doubles: logits, g and u of one expert, its output
void router_logits_f64(const double* x, const double* wg, int64_t D, int E, double* l) {
  for (int e = 0; e < E; ++e) {
    double acc = 0.0;
    for (int64_t d = 0; d < D; ++d) acc += x[d] * wg[(int64_t)e * D + d];
    l[e] = acc;
  }
}

struct ExpertFwd {
  std::vector<double> g, u, h, o;
};

void expert_fwd_f64(const double* x, const double* gate_up, const double* down, int64_t D, int64_t F,
                    ExpertFwd& r) {
  r.g.assign(F, 0.0), r.u.assign(F, 0.0), r.h.assign(F, 0.0), r.o.assign(D, 0.0);
  for (int64_t f = 0; f < F; ++f) {
    double g = 0.0, u = 0.0;
    for (int64_t d = 0; d < D; ++d) {
      g += gate_up[f * D + d] * x[d];
      u += gate_up[(F + f) * D + d] * x[d];
    }
    r.g[f] = g, r.u[f] = u, r.h[f] = g / (1.0 + std::exp(-g)) * u;
  }
  for (int64_t d = 0; d < D; ++d) {
    double acc = 0.0;
    for (int64_t f = 0; f < F; ++f) acc += down[d * F + f] * r.h[f];
    r.o[d] = acc;
  }
}

// Backward of one expert applied to one token with output gradient do_ (already scaled by p):
// dg, du [F] and this expert's contribution to dx (added into dx).
void expert_bwd_f64(const double* gate_up, const double* down, int64_t D, int64_t F, const ExpertFwd& r,
                    const double* do_, double* dg, double* du, double* dx) {
  for (int64_t f = 0; f < F; ++f) {
    double dh = 0.0;
    for (int64_t d = 0; d < D; ++d) dh += down[d * F + f] * do_[d];
    const double sg = 1.0 / (1.0 + std::exp(-r.g[f]));
    const double silu = r.g[f] * sg;
    const double dsilu = sg * (1.0 + r.g[f] * (1.0 - sg));
    dg[f] = dh * r.u[f] * dsilu;
    du[f] = dh * silu;
  }
  for (int64_t d = 0; d < D; ++d) {
    double acc = 0.0;
    for (int64_t f = 0; f < F; ++f) acc += gate_up[f * D + d] * dg[f] + gate_up[(F + f) * D + d] * du[f];
    dx[d] += acc;
  }
}

}  // namespace

// fp64-parameter forward: the same definition as oracle_layer.  gate_up [E, 2F, D], down [E, D, F],
// shared_* may be NULL (Fs = 0).  Returns 0, or -1 on invalid sizes.
int oracle_layer_f64(const double* x, const double* wg, const float* bias, const double* gate_up,
                     const double* down, const double* shared_gate_up, const double* shared_down, int64_t T,
                     int64_t D, int E, int k, int64_t F, int64_t Fs, double* y, int nthreads) {
  if (T < 0 || D < 1 || E < 1 || k < 1 || k > E || F < 1 || Fs < 0) return -1;
  for_tokens(T, nthreads, [&](int64_t t) {
    std::vector<double> l(E), p(k), yt(D, 0.0);
    std::vector<int32_t> idx(k);
    ExpertFwd r;
    router_logits_f64(x + t * D, wg, D, E, l.data());
    select_and_weight(l.data(), bias, E, k, idx.data(), p.data());
    for (int j = 0; j < k; ++j) {
      const int e = idx[j];
      expert_fwd_f64(x + t * D, gate_up + (int64_t)e * 2 * F * D, down + (int64_t)e * D * F, D, F, r);
      for (int64_t d = 0; d < D; ++d) yt[d] += p[j] * r.o[d];
    }
    if (Fs > 0 && shared_gate_up && shared_down) {
      expert_fwd_f64(x + t * D, shared_gate_up, shared_down, D, Fs, r);
      for (int64_t d = 0; d < D; ++d) yt[d] += r.o[d];
    }
    std::copy(yt.begin(), yt.end(), y + t * D);
  });
  return 0;
}

// Gradients of L = sum(dy * y) (definitions above).  Outputs (overwritten, fp64): dx [T, D],
// dwg [E, D], dgate_up [E, 2F, D], ddown [E, D, F], dshared_gate_up [2Fs, D], dshared_down [D, Fs]
// (the last two may be NULL when Fs = 0).  Weight gradients are summed over tokens in token
// order.  Returns 0, or -1 on invalid sizes.
int oracle_layer_backward_f64(const double* x, const double* wg, const float* bias, const double* gate_up,
                              const double* down, const double* shared_gate_up, const double* shared_down,
                              const double* dy, int64_t T, int64_t D, int E, int k, int64_t F, int64_t Fs,
                              double* dx, double* dwg, double* dgate_up, double* ddown, double* dshared_gate_up,
                              double* dshared_down, int nthreads) {
  if (T < 0 || D < 1 || E < 1 || k < 1 || k > E || F < 1 || Fs < 0) return -1;
  const bool sh = Fs > 0 && shared_gate_up && shared_down;
  // per slot: expert, dl, do [D], h [F], dg [F], du [F]; per token (shared): do = dy, h, dg, du
  std::vector<int32_t> idx(T * k);
  std::vector<double> dl(T * k), slot_do(T * k * D), slot_h(T * k * F), slot_dg(T * k * F), slot_du(T * k * F);
  std::vector<double> sh_h(sh ? T * Fs : 0), sh_dg(sh ? T * Fs : 0), sh_du(sh ? T * Fs : 0);
  for_tokens(T, nthreads, [&](int64_t t) {
    const double* xt = x + t * D;
    const double* dyt = dy + t * D;
    double* dxt = dx + t * D;
    std::fill(dxt, dxt + D, 0.0);
    std::vector<double> l(E), p(k), dp(k);
    ExpertFwd r;
    router_logits_f64(xt, wg, D, E, l.data());
    select_and_weight(l.data(), bias, E, k, &idx[t * k], p.data());
    for (int j = 0; j < k; ++j) {
      const int64_t slot = t * k + j;
      const int e = idx[slot];
      const double* gu = gate_up + (int64_t)e * 2 * F * D;
      const double* dn = down + (int64_t)e * D * F;
      expert_fwd_f64(xt, gu, dn, D, F, r);
      double dpj = 0.0;
      for (int64_t d = 0; d < D; ++d) dpj += dyt[d] * r.o[d];
      dp[j] = dpj;
      double* dos = &slot_do[slot * D];
      for (int64_t d = 0; d < D; ++d) dos[d] = p[j] * dyt[d];
      std::copy(r.h.begin(), r.h.end(), &slot_h[slot * F]);
      expert_bwd_f64(gu, dn, D, F, r, dos, &slot_dg[slot * F], &slot_du[slot * F], dxt);
    }
    double s = 0.0;
    for (int j = 0; j < k; ++j) s += p[j] * dp[j];
    for (int j = 0; j < k; ++j) {
      const double dlj = p[j] * (dp[j] - s);
      dl[t * k + j] = dlj;
      const double* w = wg + (int64_t)idx[t * k + j] * D;
      for (int64_t d = 0; d < D; ++d) dxt[d] += dlj * w[d];
    }
    if (sh) {
      expert_fwd_f64(xt, shared_gate_up, shared_down, D, Fs, r);
      std::copy(r.h.begin(), r.h.end(), &sh_h[t * Fs]);
      expert_bwd_f64(shared_gate_up, shared_down, D, Fs, r, dyt, &sh_dg[t * Fs], &sh_du[t * Fs], dxt);
    }
  });
  // weight gradients: one expert per task, its slots in token order
  for_tokens(E, nthreads, [&](int64_t e) {
    double* dgu = dgate_up + e * 2 * F * D;
    double* ddn = ddown + e * D * F;
    double* dw = dwg + e * D;
    std::fill(dgu, dgu + 2 * F * D, 0.0);
    std::fill(ddn, ddn + D * F, 0.0);
    std::fill(dw, dw + D, 0.0);
    for (int64_t slot = 0; slot < T * k; ++slot) {
      if (idx[slot] != e) continue;
      const double* xt = x + (slot / k) * D;
      const double* dos = &slot_do[slot * D];
      const double* h = &slot_h[slot * F];
      const double* dg = &slot_dg[slot * F];
      const double* du = &slot_du[slot * F];
      for (int64_t d = 0; d < D; ++d)
        for (int64_t f = 0; f < F; ++f) ddn[d * F + f] += dos[d] * h[f];
      for (int64_t f = 0; f < F; ++f)
        for (int64_t d = 0; d < D; ++d) {
          dgu[f * D + d] += dg[f] * xt[d];
          dgu[(F + f) * D + d] += du[f] * xt[d];
        }
      for (int64_t d = 0; d < D; ++d) dw[d] += dl[slot] * xt[d];
    }
  });
  if (sh) {
    std::fill(dshared_gate_up, dshared_gate_up + 2 * Fs * D, 0.0);
    std::fill(dshared_down, dshared_down + D * Fs, 0.0);
    for (int64_t t = 0; t < T; ++t) {
      const double* xt = x + t * D;
      const double* dyt = dy + t * D;
      for (int64_t d = 0; d < D; ++d)
        for (int64_t f = 0; f < Fs; ++f) dshared_down[d * Fs + f] += dyt[d] * sh_h[t * Fs + f];
      for (int64_t f = 0; f < Fs; ++f)
        for (int64_t d = 0; d < D; ++d) {
          dshared_gate_up[f * D + d] += sh_dg[t * Fs + f] * xt[d];
          dshared_gate_up[(Fs + f) * D + d] += sh_du[t * Fs + f] * xt[d];
        }
    }
  }
  return 0;
}

// ---------------------------------------------------------------------------------------------
// Load-balancing auxiliary loss of the router (training).  The pages say only that training adds
// an auxiliary loss that penalises the router for spreading tokens unevenly and pushes it to use
// all experts alike (josueisai.com, "El coste que la cifra bonita esconde"; dev.smart-guide.co.kr,
// "Limitaciones y Cuidados": router collapse without a load-balancing loss).  They print no
// formula; the reading taken is the product form of expert load and router probability:
//   f_e = (number of the T*k routed slots that chose e) / (T*k)     (top-k of l + bias)
//   P_e = (1/T) sum_t softmax(l_t)_e                               (all E, unbiased logits)
//   L   = alpha * E * sum_e f_e P_e                                (= alpha when both are uniform)
// f is piecewise constant in the parameters (it counts a selection), so only P carries a gradient:
//   dL/dl_{t,e} = (alpha E / T) s_{t,e} (f_e - sum_j f_j s_{t,j}),   s_t = softmax(l_t),
//   dW_g[e] = sum_t dL/dl_{t,e} x_t,   dx_t = sum_e dL/dl_{t,e} W_g[e].
// fp64 parameters; outputs (overwritten): loss [1], dwg [E, D], dx [T, D].  Returns 0, or -1 on
// invalid sizes.  T = 0 gives loss 0 and zero gradients.
int oracle_router_aux_loss_f64(const double* x, const double* wg, const float* bias, int64_t T, int64_t D, int E,
                               int k, double alpha, double* loss, double* dwg, double* dx, int nthreads) {
  if (T < 0 || D < 1 || E < 1 || k < 1 || k > E) return -1;
  std::fill(dwg, dwg + (int64_t)E * D, 0.0);
  *loss = 0.0;
  if (T == 0) return 0;
  std::vector<double> l((size_t)T * E), s((size_t)T * E), dl((size_t)T * E);
  std::vector<int32_t> idx((size_t)T * k);
  for_tokens(T, nthreads, [&](int64_t t) {
    std::vector<double> p(k);
    router_logits_f64(x + t * D, wg, D, E, &l[t * E]);
    select_and_weight(&l[t * E], bias, E, k, &idx[t * k], p.data());
    double m = l[t * E];
    for (int e = 1; e < E; ++e) m = std::max(m, l[t * E + e]);
    double z = 0.0;
    for (int e = 0; e < E; ++e) z += std::exp(l[t * E + e] - m);
    for (int e = 0; e < E; ++e) s[t * E + e] = std::exp(l[t * E + e] - m) / z;
  });
  std::vector<double> f(E, 0.0), P(E, 0.0);
  for (int64_t i = 0; i < T * k; ++i) f[idx[i]] += 1.0;
  for (int e = 0; e < E; ++e) f[e] /= (double)(T * k);
  for (int64_t t = 0; t < T; ++t)
    for (int e = 0; e < E; ++e) P[e] += s[t * E + e];
  double acc = 0.0;
  for (int e = 0; e < E; ++e) acc += f[e] * (P[e] / (double)T);
  *loss = alpha * (double)E * acc;
  const double scale = alpha * (double)E / (double)T;
  for_tokens(T, nthreads, [&](int64_t t) {
    double c = 0.0;
    for (int e = 0; e < E; ++e) c += f[e] * s[t * E + e];
    double* dxt = dx + t * D;
    std::fill(dxt, dxt + D, 0.0);
    for (int e = 0; e < E; ++e) {
      const double g = scale * s[t * E + e] * (f[e] - c);
      dl[t * E + e] = g;
      for (int64_t d = 0; d < D; ++d) dxt[d] += g * wg[(int64_t)e * D + d];
    }
  });
  for_tokens(E, nthreads, [&](int64_t e) {
    double* dw = dwg + e * D;
    for (int64_t t = 0; t < T; ++t)
      for (int64_t d = 0; d < D; ++d) dw[d] += dl[t * E + e] * x[t * D + d];
  });
  return 0;
}

}  // extern "C"
