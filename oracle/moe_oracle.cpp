// Oracle: a plain, slow, FP64 CPU statement of the dots.llm1 fine-grained MoE
// FFN layer, forward and backward.
//
// TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
// benchmark's CPU-baseline leg load this library.  It shares no code, header,
// table or helper with the CUDA path.
//
// What it follows (dots.llm1 Technical Report):
//   * §Architecture, "Mixture of Experts layer": 128 routed + 2 shared experts,
//     each a fine-grained two-layer SwiGLU FFN; the router picks the top-6
//     routed experts per token and the shared experts see every token; the
//     gating layer is computed in FP32 rather than BF16.
//   * §Architecture, "Load balancing": auxiliary-loss-free balancing: a
//     per-expert bias is added to the affinity scores only to decide the
//     top-k routing; no token is dropped.
//   * §3.2 "Efficient implementation of Grouped GEMM": each expert's token
//     segment M_i is padded to a fixed block so a thread block's tile belongs
//     to one expert.
// Readings where the pages are silent (the affinity is a softmax over all
// routed logits; ties go to the lower expert index; combine weights are the
// unbiased affinities renormalised over the chosen k; shared experts are added
// with weight 1; segments are in expert order and ascending token order; pad
// rows are zero; H and Y are stored in bf16 with round-to-nearest-even) are the
// ones this library states in its design notes.
//
// Everything accumulates in double.  bf16 inputs are widened exactly.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>
#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

inline double bf(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return (double)f;
}
// The FFN and gradient code below is written once for two input types: bf16
// bit patterns (the layer's real inputs) and double (used only so that finite
// differences can perturb inputs continuously).
inline double bf(double v) { return v; }

// Round a double to the nearest bf16 value (ties to even), returned as a
// double.  bf16 keeps 8 significant bits: scale the significand to [128, 256),
// round to an integer with ties to even, scale back.
inline double round_bf16(double v) {
  if (v == 0.0 || !std::isfinite(v)) return v;
  int e;
  double m = std::frexp(v, &e);             // v = m * 2^e, 0.5 <= |m| < 1
  if (e - 8 < -133) e = -133 + 8;           // below the smallest subnormal step
  double scaled = std::ldexp(v, 8 - e);     // |scaled| < 256
  double r = std::nearbyint(scaled);        // default rounding mode: ties to even
  (void)m;
  return std::ldexp(r, e - 8);
}

template <class W>
inline double dot_bf16(const double* a, const W* w, int n) {
  double s = 0.0;
#pragma omp simd reduction(+ : s)
  for (int c = 0; c < n; ++c) s += a[c] * bf(w[c]);
  return s;
}

inline double silu(double g) { return g / (1.0 + std::exp(-g)); }
inline double sigmoid(double g) { return 1.0 / (1.0 + std::exp(-g)); }

// One expert's SwiGLU FFN on one row a[d] (already widened):
//   G = W1[0:I] a, U = W1[I:2I] a, H = silu(G) * U, Y = W2 H.
// W1 is [2I, d] (gate rows, then up rows); W2 is [d, I].
template <class W>
void expert_row_fwd(const double* a, const W* w1, const W* w2, int d, int I, bool rnd,
                    double* g, double* u, double* h, double* y) {
  for (int i = 0; i < I; ++i) {
    g[i] = dot_bf16(a, w1 + (size_t)i * d, d);
    u[i] = dot_bf16(a, w1 + (size_t)(I + i) * d, d);
    double hv = silu(g[i]) * u[i];
    h[i] = rnd ? round_bf16(hv) : hv;
  }
  for (int r = 0; r < d; ++r) {
    double yv = dot_bf16(h, w2 + (size_t)r * I, I);
    y[r] = rnd ? round_bf16(yv) : yv;
  }
}

// Backward of one expert for one row, given dY[d].  Accumulates W1^T dA into
// dx[d] (if dx != nullptr).  Straight-through for the bf16 rounding points.
//   dH = W2^T dY;  dG = dH * U * s (1 + G (1 - s)), s = sigmoid(G);  dU = dH * silu(G)
//   dA = [dG | dU];  dx += W1^T dA
template <class W>
void expert_row_bwd(const double* g, const double* u, const double* dy, const W* w1,
                    const W* w2, int d, int I, double* dh, double* da, double* dx) {
  for (int i = 0; i < I; ++i) dh[i] = 0.0;
  for (int r = 0; r < d; ++r) {
    const W* row = w2 + (size_t)r * I;
    double dyr = dy[r];
    for (int i = 0; i < I; ++i) dh[i] += dyr * bf(row[i]);
  }
  for (int i = 0; i < I; ++i) {
    double s = sigmoid(g[i]);
    da[i] = dh[i] * u[i] * s * (1.0 + g[i] * (1.0 - s));
    da[I + i] = dh[i] * silu(g[i]);
  }
  if (dx) {
    for (int i = 0; i < 2 * I; ++i) {
      const W* row = w1 + (size_t)i * d;
      double a = da[i];
      for (int c = 0; c < d; ++c) dx[c] += a * bf(row[c]);
    }
  }
}

}  // namespace

extern "C" {

int oracle_num_threads() {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

double oracle_round_bf16(double v) { return round_bf16(v); }

// Gate: logit[t, e] = sum_j X[t, j] * Wg[e, j]  (X bf16 widened, Wg f32 widened).
void oracle_gate_logits(const uint16_t* x, const float* wg, int64_t T, int d, int E,
                        double* logits) {
#pragma omp parallel
  {
    std::vector<double> xt(d);
#pragma omp for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
      for (int c = 0; c < d; ++c) xt[c] = bf(x[t * d + c]);
      for (int e = 0; e < E; ++e) {
        const float* w = wg + (size_t)e * d;
        double s = 0.0;
#pragma omp simd reduction(+ : s)
        for (int c = 0; c < d; ++c) s += xt[c] * (double)w[c];
        logits[t * E + e] = s;
      }
    }
  }
}

// Router.  p = softmax(logit) over the E routed experts; s = p + bias (for
// selection only); the k experts with the largest s, in descending s, equal s
// going to the lower index; w_j = p_{e_j} / sum_j' p_{e_j'}.
// margin[t] = s of the k-th pick minus the best s left out (+inf when k == E).
void oracle_route(const double* logits, const float* bias, int64_t T, int E, int k,
                  double* probs, int32_t* idx, double* w, double* margin) {
#pragma omp parallel
  {
    std::vector<double> p(E), s(E);
    std::vector<char> taken(E);
#pragma omp for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
      const double* l = logits + t * E;
      double m = l[0];
      for (int e = 1; e < E; ++e) m = std::max(m, l[e]);
      double z = 0.0;
      for (int e = 0; e < E; ++e) {
        p[e] = std::exp(l[e] - m);
        z += p[e];
      }
      for (int e = 0; e < E; ++e) {
        p[e] /= z;
        s[e] = p[e] + (double)bias[e];
        taken[e] = 0;
        if (probs) probs[t * E + e] = p[e];
      }
      double psum = 0.0;
      for (int j = 0; j < k; ++j) {
        int best = -1;
        for (int e = 0; e < E; ++e)
          if (!taken[e] && (best < 0 || s[e] > s[best])) best = e;
        taken[best] = 1;
        idx[t * k + j] = best;
        psum += p[best];
      }
      for (int j = 0; j < k; ++j) w[t * k + j] = p[idx[t * k + j]] / psum;
      if (margin) {
        int next = -1;
        for (int e = 0; e < E; ++e)
          if (!taken[e] && (next < 0 || s[e] > s[next])) next = e;
        margin[t] = next < 0 ? INFINITY : s[idx[t * k + k - 1]] - s[next];
      }
    }
  }
}

// Router backward: the gradient of the combine weights w[t, j] through the
// renormalisation over the chosen set C and the softmax, then into the gate's
// input and weights.  The selection (made on p + bias) is piecewise constant and
// carries no gradient; the bias gets none.  With Z = sum_{j in C} p_j:
//   w_j = p_j / Z        =>  dp_i = (dw_i - sum_j dw_j w_j) / Z   (i in C; 0 elsewhere)
//   p = softmax(logit)   =>  dlogit_e = p_e (dp_e - sum_i p_i dp_i)
//   logit = X Wg^T       =>  dX = dlogit Wg,   dWg = dlogit^T X
// Logits and p are recomputed in FP64 from x and wg.  Any of the outputs may be null.
// dl_extra [T, E] (nullable) is a further dL/dlogit term (the sequence-wise balance
// loss's) added before dX and dWg are formed.
void oracle_router_bwd(const uint16_t* x, const float* wg, const int32_t* idx, const double* dw,
                       int64_t T, int d, int E, int k, const double* dl_extra, double* dlogits,
                       double* dx, double* dwg) {
  std::vector<double> dl((size_t)T * E);
#pragma omp parallel
  {
    std::vector<double> xt(d), p(E), dp(E);
#pragma omp for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
      for (int c = 0; c < d; ++c) xt[c] = bf(x[t * d + c]);
      double m = -INFINITY;
      for (int e = 0; e < E; ++e) {
        const float* w = wg + (size_t)e * d;
        double s = 0.0;
        for (int c = 0; c < d; ++c) s += xt[c] * (double)w[c];
        p[e] = s;
        m = std::max(m, s);
      }
      double z = 0.0;
      for (int e = 0; e < E; ++e) {
        p[e] = std::exp(p[e] - m);
        z += p[e];
      }
      for (int e = 0; e < E; ++e) {
        p[e] /= z;
        dp[e] = 0.0;
      }
      double zc = 0.0, dot = 0.0;
      for (int j = 0; j < k; ++j) zc += p[idx[t * k + j]];
      for (int j = 0; j < k; ++j) dot += dw[t * k + j] * (p[idx[t * k + j]] / zc);
      for (int j = 0; j < k; ++j) dp[idx[t * k + j]] = (dw[t * k + j] - dot) / zc;
      double pdp = 0.0;
      for (int e = 0; e < E; ++e) pdp += p[e] * dp[e];
      for (int e = 0; e < E; ++e) dl[(size_t)t * E + e] = p[e] * (dp[e] - pdp);
    }
  }
  if (dl_extra)
    for (size_t i = 0; i < dl.size(); ++i) dl[i] += dl_extra[i];
  if (dlogits) std::copy(dl.begin(), dl.end(), dlogits);
  if (dx) {
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t)
      for (int c = 0; c < d; ++c) {
        double s = 0.0;
        for (int e = 0; e < E; ++e) s += dl[(size_t)t * E + e] * (double)wg[(size_t)e * d + c];
        dx[t * d + c] = s;
      }
  }
  if (dwg) {
#pragma omp parallel for schedule(static)
    for (int e = 0; e < E; ++e)
      for (int c = 0; c < d; ++c) {
        double s = 0.0;
        for (int64_t t = 0; t < T; ++t) s += dl[(size_t)t * E + e] * bf(x[t * d + c]);
        dwg[(size_t)e * d + c] = s;
      }
  }
}

// Sequence-wise balance loss and its gradient with respect to the logits.
// The pages add a sequence-wise balance loss to the aux-loss-free method without
// stating it; the method they cite (the DeepSeek-V3 report) defines one, taken
// here with this layer's softmax affinities.  The batch's T tokens form
// sequences of L tokens (the last one may be shorter); for sequence s with L_s
// tokens:
//   p_t   = softmax(logit_t),   q_t = p_t / sum_e p_t,e      (normalised affinities)
//   f_s,i = E / (k L_s) * #{(t in s, j) : idx[t, j] = i}     (load fraction, x E)
//   P_s,i = (1 / L_s) * sum_{t in s} q_t,i                   (mean affinity)
//   loss  = (1 / n_seq) * sum_s alpha * sum_i f_s,i P_s,i     (mean over sequences)
// The selection is piecewise constant, so the gradient runs through P only:
//   dloss/dq_t,i = alpha f_s,i / (n_seq L_s)
//   dloss/dp_t,j = sum_i dloss/dq_t,i (delta_ij / z - p_t,i / z^2),  z = sum_e p_t,e
//   dloss/dlogit_t,e = p_t,e (dloss/dp_t,e - sum_j p_t,j dloss/dp_t,j)
// Returns the loss; dlogits [T, E] may be null.
double oracle_seq_balance(const double* logits, const int32_t* idx, int64_t T, int E, int k,
                          int64_t L, double alpha, double* dlogits) {
  if (T <= 0 || L <= 0) return 0.0;
  const int64_t nseq = (T + L - 1) / L;
  std::vector<double> p((size_t)T * E), q((size_t)T * E), z(T);
  for (int64_t t = 0; t < T; ++t) {
    const double* lg = logits + t * E;
    double m = -INFINITY;
    for (int e = 0; e < E; ++e) m = std::max(m, lg[e]);
    double sum = 0.0;
    for (int e = 0; e < E; ++e) sum += (p[t * E + e] = std::exp(lg[e] - m));
    for (int e = 0; e < E; ++e) p[t * E + e] /= sum;
    z[t] = 0.0;
    for (int e = 0; e < E; ++e) z[t] += p[t * E + e];
    for (int e = 0; e < E; ++e) q[t * E + e] = p[t * E + e] / z[t];
  }
  double loss = 0.0;
  std::vector<double> f(E), P(E), g(E), dp(E);
  for (int64_t s = 0; s < nseq; ++s) {
    const int64_t t0 = s * L, t1 = std::min(T, t0 + L), Ls = t1 - t0;
    std::fill(f.begin(), f.end(), 0.0);
    std::fill(P.begin(), P.end(), 0.0);
    for (int64_t t = t0; t < t1; ++t) {
      for (int j = 0; j < k; ++j) f[idx[t * k + j]] += 1.0;
      for (int e = 0; e < E; ++e) P[e] += q[t * E + e];
    }
    double ls = 0.0;
    for (int e = 0; e < E; ++e) {
      f[e] *= (double)E / ((double)k * (double)Ls);
      P[e] /= (double)Ls;
      ls += f[e] * P[e];
    }
    loss += alpha * ls / (double)nseq;
    if (!dlogits) continue;
    for (int e = 0; e < E; ++e) g[e] = alpha * f[e] / ((double)nseq * (double)Ls);
    for (int64_t t = t0; t < t1; ++t) {
      const double* pt = p.data() + t * E;
      double gp = 0.0;
      for (int i = 0; i < E; ++i) gp += g[i] * pt[i];
      for (int j = 0; j < E; ++j) dp[j] = g[j] / z[t] - gp / (z[t] * z[t]);
      double pdp = 0.0;
      for (int e = 0; e < E; ++e) pdp += pt[e] * dp[e];
      for (int e = 0; e < E; ++e) dlogits[t * E + e] = pt[e] * (dp[e] - pdp);
    }
  }
  return loss;
}

// Aux-loss-free bias update, one step (the pages say the bias is adjusted during
// training to keep the expert loads balanced; this is the plainest rule of that
// kind): load_e = number of (token, pick) pairs routed to e in the batch, mean =
// T k / E, bias_e += gamma * sign(mean - load_e) with sign(0) = 0.  The sum of two
// f32 values is exact in double.
void oracle_bias_update(const int32_t* idx, int64_t T, int E, int k, const float* bias,
                        float gamma, double* out) {
  std::vector<int64_t> load(E, 0);
  for (int64_t i = 0; i < T * k; ++i) load[idx[i]] += 1;
  for (int e = 0; e < E; ++e) {
    const double diff = (double)T * k - (double)load[e] * E;  // E * (mean - load_e)
    const double sgn = diff > 0 ? 1.0 : diff < 0 ? -1.0 : 0.0;
    out[e] = (double)bias[e] + (double)gamma * sgn;
  }
}

// Permutation into padded per-expert segments.
//   c_e = #{(t, j) : idx[t, j] = e};  off_0 = 0, off_{e+1} = off_e + roundup(c_e, P)
//   segment e lists its tokens in ascending order; pad rows hold -1.
// Returns the padded total off_E, or -1 if it exceeds rows_cap.
int64_t oracle_permute(const int32_t* idx, int64_t T, int E, int k, int P, int64_t rows_cap,
                       int32_t* counts, int32_t* offsets, int32_t* sorted_ids, int32_t* row_of) {
  for (int e = 0; e < E; ++e) counts[e] = 0;
  for (int64_t f = 0; f < T * k; ++f) counts[idx[f]] += 1;
  offsets[0] = 0;
  for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + (counts[e] + P - 1) / P * P;
  if (offsets[E] > rows_cap) return -1;
  for (int64_t r = 0; r < rows_cap; ++r) sorted_ids[r] = -1;
  std::vector<int32_t> fill(E, 0);
  for (int64_t t = 0; t < T; ++t)
    for (int j = 0; j < k; ++j) {
      int e = idx[t * k + j];
      int32_t pos = offsets[e] + fill[e]++;
      sorted_ids[pos] = (int32_t)t;
      row_of[t * k + j] = pos;
    }
  return offsets[E];
}

}  // extern "C"

namespace {

// Forward of one expert on M rows A[M, d].  Outputs may be null.
template <class W>
void expert_fwd_impl(const W* a, int64_t M, const W* w1, const W* w2, int d, int I, int rnd,
                     double* g, double* u, double* h, double* y) {
#pragma omp parallel
  {
    std::vector<double> ar(d), gr(I), ur(I), hr(I), yr(d);
#pragma omp for schedule(dynamic, 1)
    for (int64_t m = 0; m < M; ++m) {
      for (int c = 0; c < d; ++c) ar[c] = bf(a[m * d + c]);
      expert_row_fwd(ar.data(), w1, w2, d, I, rnd != 0, gr.data(), ur.data(), hr.data(),
                     yr.data());
      if (g) std::copy(gr.begin(), gr.end(), g + m * I);
      if (u) std::copy(ur.begin(), ur.end(), u + m * I);
      if (h) std::copy(hr.begin(), hr.end(), h + m * I);
      if (y) std::copy(yr.begin(), yr.end(), y + m * d);
    }
  }
}

// Layer forward for a list of tokens, straight from the definition (no
// permutation): out[t] = sum_j w[t, j] * Y_{idx[t, j]}(x_t) + sum_s Y_{E+s}(x_t).
// W1 is [E+S, 2I, d], W2 is [E+S, d, I]; routed experts first, shared after.
// y_routed [n, k, d] and y_shared [n, S, d] may be null.
template <class W>
void layer_fwd_impl(const W* x, const int32_t* idx, const double* w, const W* w1, const W* w2,
                    int d, int E, int k, int S, int I, const int64_t* tokens, int64_t n, int rnd,
                    double* out, double* y_routed, double* y_shared) {
  const size_t w1s = (size_t)2 * I * d, w2s = (size_t)d * I;
#pragma omp parallel
  {
    std::vector<double> a(d), g(I), u(I), h(I), y(d), acc(d);
#pragma omp for schedule(dynamic, 1)
    for (int64_t q = 0; q < n; ++q) {
      int64_t t = tokens[q];
      for (int c = 0; c < d; ++c) {
        a[c] = bf(x[t * d + c]);
        acc[c] = 0.0;
      }
      for (int j = 0; j < k + S; ++j) {
        int e = j < k ? idx[t * k + j] : E + (j - k);
        double wt = j < k ? w[t * k + j] : 1.0;
        expert_row_fwd(a.data(), w1 + e * w1s, w2 + e * w2s, d, I, rnd != 0, g.data(), u.data(),
                       h.data(), y.data());
        for (int c = 0; c < d; ++c) acc[c] += wt * y[c];
        if (j < k && y_routed) std::copy(y.begin(), y.end(), y_routed + (q * k + j) * d);
        if (j >= k && y_shared) std::copy(y.begin(), y.end(), y_shared + (q * S + (j - k)) * d);
      }
      std::copy(acc.begin(), acc.end(), out + q * d);
    }
  }
}

// Layer backward for a list of tokens: given dOut, the gradient with respect
// to x through the experts (the router's own gradient is not included) and to
// the combine weights:
//   dY_j = w_j dOut (routed), dY_s = dOut (shared);  dw_j = <dOut, Y_j>;
//   dx = sum over the token's experts of W1^T dA.
template <class W>
void layer_bwd_impl(const W* x, const int32_t* idx, const double* w, const W* w1, const W* w2,
                    const W* dout, int d, int E, int k, int S, int I, const int64_t* tokens,
                    int64_t n, int rnd, double* dx, double* dw) {
  const size_t w1s = (size_t)2 * I * d, w2s = (size_t)d * I;
#pragma omp parallel
  {
    std::vector<double> a(d), g(I), u(I), h(I), y(d), dy(d), dh(I), da(2 * I), gx(d), go(d);
#pragma omp for schedule(dynamic, 1)
    for (int64_t q = 0; q < n; ++q) {
      int64_t t = tokens[q];
      for (int c = 0; c < d; ++c) {
        a[c] = bf(x[t * d + c]);
        go[c] = bf(dout[t * d + c]);
        gx[c] = 0.0;
      }
      for (int j = 0; j < k + S; ++j) {
        int e = j < k ? idx[t * k + j] : E + (j - k);
        double wt = j < k ? w[t * k + j] : 1.0;
        expert_row_fwd(a.data(), w1 + e * w1s, w2 + e * w2s, d, I, rnd != 0, g.data(), u.data(),
                       h.data(), y.data());
        if (j < k) {
          double s = 0.0;
          for (int c = 0; c < d; ++c) s += go[c] * y[c];
          dw[q * k + j] = s;
        }
        for (int c = 0; c < d; ++c) dy[c] = wt * go[c];
        expert_row_bwd(g.data(), u.data(), dy.data(), w1 + e * w1s, w2 + e * w2s, d, I,
                       dh.data(), da.data(), gx.data());
      }
      std::copy(gx.begin(), gx.end(), dx + q * d);
    }
  }
}

// Weight gradients of one group g (routed g < E, shared g >= E), selected
// entries only, summed over every token the group sees:
//   dW1_g[i, :] = sum_t dA_t[i] x_t          for i in w1_rows (rows of [2I, d])
//   dW2_g[:, c] = sum_t dY_t H_t[c]          for c in w2_cols (columns of [d, I])
// dw1 is [n1, d], dw2 is [d, n2] (column c of dW2 stored as dw2[:, q]).
// Each entry needs only a few dot products per token, so whole groups of a
// full-size layer stay cheap.
template <class W>
void group_dw_impl(const W* x, const int32_t* idx, const double* w, const W* w1, const W* w2,
                   const W* dout, int64_t T, int d, int E, int k, int I, int grp, int rnd,
                   const int32_t* w1_rows, int n1, const int32_t* w2_cols, int n2, double* dw1,
                   double* dw2) {
  const W* W1 = w1 + (size_t)grp * 2 * I * d;
  const W* W2 = w2 + (size_t)grp * d * I;
  // tokens of the group and their combine weight
  std::vector<int64_t> toks;
  std::vector<double> wts;
  for (int64_t t = 0; t < T; ++t) {
    if (grp >= E) {
      toks.push_back(t);
      wts.push_back(1.0);
    } else {
      for (int j = 0; j < k; ++j)
        if (idx[t * k + j] == grp) {
          toks.push_back(t);
          wts.push_back(w[t * k + j]);
        }
    }
  }
  // the intermediate columns i' that are needed
  std::vector<int> need;
  for (int q = 0; q < n1; ++q) need.push_back(w1_rows[q] % I);
  for (int q = 0; q < n2; ++q) need.push_back(w2_cols[q]);
  std::sort(need.begin(), need.end());
  need.erase(std::unique(need.begin(), need.end()), need.end());
  const int nn = (int)need.size();
  std::vector<int> pos(I, -1);
  for (int q = 0; q < nn; ++q) pos[need[q]] = q;

  const int64_t nt = (int64_t)toks.size();
  // per token: G, U, dH at the needed columns
  std::vector<double> G(nt * nn), U(nt * nn), DH(nt * nn);
#pragma omp parallel
  {
    std::vector<double> a(d), dy(d);
#pragma omp for schedule(dynamic, 4)
    for (int64_t q = 0; q < nt; ++q) {
      int64_t t = toks[q];
      for (int c = 0; c < d; ++c) {
        a[c] = bf(x[t * d + c]);
        dy[c] = wts[q] * bf(dout[t * d + c]);
      }
      for (int z = 0; z < nn; ++z) {
        int i = need[z];
        G[q * nn + z] = dot_bf16(a.data(), W1 + (size_t)i * d, d);
        U[q * nn + z] = dot_bf16(a.data(), W1 + (size_t)(I + i) * d, d);
        double s = 0.0;
        for (int r = 0; r < d; ++r) s += dy[r] * bf(W2[(size_t)r * I + i]);
        DH[q * nn + z] = s;
      }
    }
  }
  // dW1 rows
#pragma omp parallel for schedule(dynamic, 1)
  for (int q1 = 0; q1 < n1; ++q1) {
    int i = w1_rows[q1];
    int z = pos[i % I];
    double* out = dw1 + (size_t)q1 * d;
    for (int c = 0; c < d; ++c) out[c] = 0.0;
    for (int64_t q = 0; q < nt; ++q) {
      double g = G[q * nn + z], u = U[q * nn + z], dh = DH[q * nn + z];
      double s = sigmoid(g);
      double da = i < I ? dh * u * s * (1.0 + g * (1.0 - s)) : dh * silu(g);
      const W* xr = x + toks[q] * d;
      for (int c = 0; c < d; ++c) out[c] += da * bf(xr[c]);
    }
  }
  // dW2 columns: H_t[c] = silu(G) * U (stored bf16 in the forward when rnd)
  std::vector<double> H(nt * nn);
  for (int64_t q = 0; q < nt * nn; ++q) {
    double hv = silu(G[q]) * U[q];
    H[q] = rnd ? round_bf16(hv) : hv;
  }
  for (int64_t r = 0; r < (int64_t)d * n2; ++r) dw2[r] = 0.0;
#pragma omp parallel
  {
    int nth = 1, me = 0;
#ifdef _OPENMP
    nth = omp_get_num_threads();
    me = omp_get_thread_num();
#endif
    int r0 = (int)((int64_t)d * me / nth), r1 = (int)((int64_t)d * (me + 1) / nth);
    for (int64_t q = 0; q < nt; ++q) {
      const W* gr = dout + toks[q] * d;
      for (int q2 = 0; q2 < n2; ++q2) {
        double sc = wts[q] * H[q * nn + pos[w2_cols[q2]]];
        for (int r = r0; r < r1; ++r) dw2[(size_t)r * n2 + q2] += sc * bf(gr[r]);
      }
    }
  }
}

}  // namespace

extern "C" {

// Exported forms.  *_bf16 take the layer's real inputs (bf16 bit patterns);
// *_f64 take doubles and exist for finite-difference checks of the gradients.
#define ORACLE_EXPORTS(SUFFIX, W)                                                              \
  void oracle_expert_fwd##SUFFIX(const W* a, int64_t M, const W* w1, const W* w2, int d,      \
                                 int I, int rnd, double* g, double* u, double* h, double* y) { \
    expert_fwd_impl<W>(a, M, w1, w2, d, I, rnd, g, u, h, y);                                   \
  }                                                                                            \
  void oracle_layer_fwd##SUFFIX(const W* x, const int32_t* idx, const double* w, const W* w1,  \
                                const W* w2, int d, int E, int k, int S, int I,                \
                                const int64_t* tokens, int64_t n, int rnd, double* out,        \
                                double* y_routed, double* y_shared) {                          \
    layer_fwd_impl<W>(x, idx, w, w1, w2, d, E, k, S, I, tokens, n, rnd, out, y_routed,         \
                      y_shared);                                                               \
  }                                                                                            \
  void oracle_layer_bwd##SUFFIX(const W* x, const int32_t* idx, const double* w, const W* w1,  \
                                const W* w2, const W* dout, int d, int E, int k, int S, int I, \
                                const int64_t* tokens, int64_t n, int rnd, double* dx,         \
                                double* dw) {                                                  \
    layer_bwd_impl<W>(x, idx, w, w1, w2, dout, d, E, k, S, I, tokens, n, rnd, dx, dw);         \
  }                                                                                            \
  void oracle_group_dw##SUFFIX(const W* x, const int32_t* idx, const double* w, const W* w1,   \
                               const W* w2, const W* dout, int64_t T, int d, int E, int k,     \
                               int I, int grp, int rnd, const int32_t* w1_rows, int n1,        \
                               const int32_t* w2_cols, int n2, double* dw1, double* dw2) {     \
    group_dw_impl<W>(x, idx, w, w1, w2, dout, T, d, E, k, I, grp, rnd, w1_rows, n1, w2_cols,   \
                     n2, dw1, dw2);                                                            \
  }

ORACLE_EXPORTS(_bf16, uint16_t)
ORACLE_EXPORTS(_f64, double)

}  // extern "C"
