/*
 * moe_oracle.c — plain, slow fp64 CPU oracle for the forward pass of the
 * sparse top-k Mixture-of-Experts layer.
 *
 * TEST INFRASTRUCTURE. Only tests/, __graft_entry__.smoke() and bench.py's
 * cpu_baseline leg (and its `--impl reference` arm) may load or call this
 * library. It shares no code, header, table or helper with the CUDA path, and
 * the CUDA path never links or imports it.
 *
 * Every step is the plain definition from the pages, written out in fp64:
 *
 *   router        logits[t,e] = sum_c x[t,c] * Wr[e,c] (+ b[e])
 *                 axonml-nn layers/moe.rs, MoERouter::route (gate Linear,
 *                 no bias); the optional per-expert bias is the skewed-load
 *                 workload's "router logit bias", added before the softmax.
 *   softmax       p = exp(l - max l) / sum exp(l - max l)
 *                 axonml-nn moe.rs, MoERouter::route (softmax(-1));
 *                 Mixtral MoE Block, "The PyTorch it exports" (_moe_forward).
 *   top-k         the k largest p, ordered by (p descending, index ascending):
 *                 axonml-nn moe.rs, MoERouter::route sorts (index, prob) pairs
 *                 with a stable descending sort, so equal probabilities keep
 *                 the lower expert index first.
 *   gates         renorm: g_j = p_j / sum_j p_j (1/k each if that sum is <= 0),
 *                 axonml-nn moe.rs, MoERouter::route ("Normalize top-k
 *                 weights"); Mixtral MoE Block, _moe_forward (top_w / sum).
 *                 no renorm: g_j = p_j, Model Architecture Patterns,
 *                 "Top-K Router" (TopKRouter returns the raw top-k softmax).
 *   statistics    counts[e] = #{(t,j) : idx[t,j] = e}, axonml-nn moe.rs,
 *                 MoELayer::forward ("Track expert utilization") and
 *                 expert_utilization(); P[e] = mean_t p[t,e] and
 *                 aux = E * sum_e f_e * P_e, load_balancing_loss().
 *                 f_e is read as counts_e / (T*k), the fraction of the T*k
 *                 routed assignments, so that sum_e f_e = 1 and the statistic
 *                 equals 1 under uniform routing; the page's own code divides
 *                 by T only, which is k times this value.
 *   dispatch      for e ascending, for t ascending, every (t,j) with
 *                 idx[t,j] = e takes the next row: axonml-nn moe.rs,
 *                 MoELayer::forward ("Process each expert: gather tokens").
 *   expert        y = down(SiLU(gate(x)) * up(x)), SiLU(z) = z / (1 + e^-z),
 *                 axonml-nn moe.rs, Expert::forward; Model Architecture
 *                 Patterns, "SwiGLU FFN". Weights are nn.Linear layout
 *                 [out, in], stacked per expert: gate/up [E, I, d],
 *                 down [E, d, I].
 *   combine       out[t] = sum_j g[t,j] * y_{idx[t,j]}(x[t]), each expert's
 *                 output weighted by its own gate: axonml-nn moe.rs,
 *                 MoELayer::forward ("Scatter weighted outputs back");
 *                 Mixtral MoE Block markdown, _moe_forward.
 *
 * Inputs are read as stored (fp32, or bf16 bit patterns widened exactly to
 * fp64). All arithmetic is fp64. OpenMP parallelises over independent tokens
 * or rows only; no step is blocked, fused or reordered beyond the definition.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORACLE_F32 = 0, ORACLE_BF16 = 1 };

/* Exact widening of one stored element to fp64. */
static double load_elem(const void* base, int dtype, int64_t i) {
  if (dtype == ORACLE_F32) return (double)((const float*)base)[i];
  uint32_t bits = ((uint32_t)((const uint16_t*)base)[i]) << 16;
  float f;
  memcpy(&f, &bits, sizeof f);
  return (double)f;
}

/* Round an fp32 value to the nearest bf16, ties to even (for the diagnostic
 * mode that mimics an intermediate stored in bf16). NaN is kept quiet. */
static double round_to_bf16(double v) {
  float f = (float)v;
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu)) {
    u |= 0x00400000u;
  } else {
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
  }
  u &= 0xffff0000u;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

void oracle_set_num_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

/* ---- router: logits and softmax ------------------------------------------ */

/* probs[t*E + e] for every token. */
void oracle_router_probs(const void* x, const void* w_router, const float* b_router,
                         int dtype, int64_t T, int64_t d, int E, double* probs) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t) {
    double* p = probs + t * E;
    for (int e = 0; e < E; ++e) {
      double acc = 0.0;
      for (int64_t c = 0; c < d; ++c)
        acc += load_elem(x, dtype, t * d + c) * load_elem(w_router, dtype, (int64_t)e * d + c);
      if (b_router) acc += (double)b_router[e];
      p[e] = acc; /* logit for now */
    }
    double m = p[0];
    for (int e = 1; e < E; ++e)
      if (p[e] > m) m = p[e];
    double s = 0.0;
    for (int e = 0; e < E; ++e) {
      p[e] = exp(p[e] - m);
      s += p[e];
    }
    for (int e = 0; e < E; ++e) p[e] /= s;
  }
}

/* ---- top-k ---------------------------------------------------------------- */

typedef struct {
  double p;
  int e;
} ranked_t;

/* Descending by probability, ascending by index among equal probabilities. */
static int cmp_ranked(const void* a, const void* b) {
  const ranked_t* ra = (const ranked_t*)a;
  const ranked_t* rb = (const ranked_t*)b;
  if (ra->p > rb->p) return -1;
  if (ra->p < rb->p) return 1;
  return (ra->e > rb->e) - (ra->e < rb->e);
}

/* Gates for a given set of chosen experts per token (used both for the
 * oracle's own choice and to evaluate another valid choice of a near tie). */
void oracle_gates(const double* probs, int64_t T, int E, int k, const int32_t* idx,
                  int renorm, double* gate) {
  for (int64_t t = 0; t < T; ++t) {
    double s = 0.0;
    for (int j = 0; j < k; ++j) s += probs[t * E + idx[t * k + j]];
    for (int j = 0; j < k; ++j) {
      double pj = probs[t * E + idx[t * k + j]];
      if (!renorm)
        gate[t * k + j] = pj;
      else if (s > 0.0)
        gate[t * k + j] = pj / s;
      else
        gate[t * k + j] = 1.0 / (double)k;
    }
  }
}

/* Top-k experts per token; gap[t] = p_(k) - p_(k+1) (+inf when k == E). */
void oracle_topk(const double* probs, int64_t T, int E, int k, int renorm,
                 int32_t* topk_idx, double* topk_gate, double* gap) {
#pragma omp parallel
  {
    ranked_t* r = (ranked_t*)malloc(sizeof(ranked_t) * (size_t)E);
#pragma omp for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
      for (int e = 0; e < E; ++e) {
        r[e].p = probs[t * E + e];
        r[e].e = e;
      }
      qsort(r, (size_t)E, sizeof(ranked_t), cmp_ranked);
      for (int j = 0; j < k; ++j) topk_idx[t * k + j] = r[j].e;
      if (gap) gap[t] = (k < E) ? r[k - 1].p - r[k].p : INFINITY;
    }
    free(r);
  }
  oracle_gates(probs, T, E, k, topk_idx, renorm, topk_gate);
}

/* ---- statistics: histogram, mean probability, load-balancing statistic ---- */

void oracle_stats(const double* probs, const int32_t* topk_idx, int64_t T, int E, int k,
                  int64_t* counts, double* mean_prob, double* aux) {
  for (int e = 0; e < E; ++e) {
    counts[e] = 0;
    mean_prob[e] = 0.0;
  }
  if (T == 0) {
    *aux = 0.0;
    return;
  }
  for (int64_t t = 0; t < T; ++t)
    for (int j = 0; j < k; ++j) counts[topk_idx[t * k + j]] += 1;
  for (int64_t t = 0; t < T; ++t)
    for (int e = 0; e < E; ++e) mean_prob[e] += probs[t * E + e];
  for (int e = 0; e < E; ++e) mean_prob[e] /= (double)T;
  double s = 0.0;
  for (int e = 0; e < E; ++e) s += ((double)counts[e] / ((double)T * (double)k)) * mean_prob[e];
  *aux = (double)E * s;
}

/* ---- dispatch order ------------------------------------------------------- */

/* offsets[E+1]; perm_tok[R] = token of each dispatched row; inv[T*k] = row of
 * each (token, slot). Rows are expert-contiguous, tokens ascending within an
 * expert. */
void oracle_dispatch(const int32_t* topk_idx, int64_t T, int k, int E, int64_t* offsets,
                     int32_t* perm_tok, int32_t* inv) {
  int64_t row = 0;
  for (int e = 0; e < E; ++e) {
    offsets[e] = row;
    for (int64_t t = 0; t < T; ++t)
      for (int j = 0; j < k; ++j)
        if (topk_idx[t * k + j] == e) {
          perm_tok[row] = (int32_t)t;
          inv[t * k + j] = (int32_t)row;
          ++row;
        }
  }
  offsets[E] = row;
}

/* ---- expert SwiGLU MLP ---------------------------------------------------- */

/* y[r, :] = down_e(SiLU(gate_e(x_t)) * up_e(x_t)) for each requested row
 * (t = tok[r], e = expert[r]). h_round = 1 rounds the hidden activation to
 * bf16 (a diagnostic mode; parity is judged with h_round = 0). */
void oracle_expert_rows(const void* x, const void* w_gate, const void* w_up, const void* w_down,
                        int dtype, int64_t d, int64_t I, int64_t n, const int32_t* tok,
                        const int32_t* expert, int h_round, double* y) {
#pragma omp parallel
  {
    double* xv = (double*)malloc(sizeof(double) * (size_t)d);
    double* h = (double*)malloc(sizeof(double) * (size_t)I);
#pragma omp for schedule(dynamic, 1)
    for (int64_t r = 0; r < n; ++r) {
      const int64_t t = tok[r];
      const int64_t e = expert[r];
      for (int64_t c = 0; c < d; ++c) xv[c] = load_elem(x, dtype, t * d + c);
      for (int64_t i = 0; i < I; ++i) {
        const int64_t wrow = (e * I + i) * d;
        double g = 0.0, u = 0.0;
        for (int64_t c = 0; c < d; ++c) {
          g += xv[c] * load_elem(w_gate, dtype, wrow + c);
          u += xv[c] * load_elem(w_up, dtype, wrow + c);
        }
        double silu = g / (1.0 + exp(-g));
        h[i] = silu * u;
        if (h_round) h[i] = round_to_bf16(h[i]);
      }
      for (int64_t o = 0; o < d; ++o) {
        const int64_t wrow = (e * d + o) * I;
        double acc = 0.0;
        for (int64_t i = 0; i < I; ++i) acc += h[i] * load_elem(w_down, dtype, wrow + i);
        y[r * d + o] = acc;
      }
    }
    free(xv);
    free(h);
  }
}

/* ---- combine -------------------------------------------------------------- */

/* out[i, :] = sum_j gate[i,j] * expert_{idx[i,j]}(x[tok[i]]) for a list of
 * tokens with their chosen experts and gates. */
void oracle_moe_tokens(const void* x, const void* w_gate, const void* w_up, const void* w_down,
                       int dtype, int64_t d, int64_t I, int k, int64_t ntok, const int32_t* tok,
                       const int32_t* idx, const double* gate, int h_round, double* out) {
  const int64_t n = ntok * k;
  int32_t* rtok = (int32_t*)malloc(sizeof(int32_t) * (size_t)(n > 0 ? n : 1));
  double* y = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n * d : 1));
  for (int64_t i = 0; i < ntok; ++i)
    for (int j = 0; j < k; ++j) rtok[i * k + j] = tok[i];
  oracle_expert_rows(x, w_gate, w_up, w_down, dtype, d, I, n, rtok, idx, h_round, y);
  for (int64_t i = 0; i < ntok; ++i)
    for (int64_t c = 0; c < d; ++c) {
      double acc = 0.0;
      for (int j = 0; j < k; ++j) acc += gate[i * k + j] * y[(i * k + j) * d + c];
      out[i * d + c] = acc;
    }
  free(rtok);
  free(y);
}
