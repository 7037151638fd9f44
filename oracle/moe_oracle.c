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
 *                 workload's per-expert bias on the router logits, added before
 *                 the softmax.
 *   softmax       p = exp(l - max l) / sum exp(l - max l)
 *                 axonml-nn moe.rs, MoERouter::route (softmax(-1));
 *                 Mixtral MoE Block, the exported PyTorch (_moe_forward).
 *   top-k         the k largest p, ordered by (p descending, index ascending):
 *                 axonml-nn moe.rs, MoERouter::route sorts (index, prob) pairs
 *                 with a stable descending sort, so equal probabilities keep
 *                 the lower expert index first.
 *   gates         renorm: g_j = p_j / sum_j p_j (1/k each if that sum is <= 0),
 *                 axonml-nn moe.rs, MoERouter::route (its renormalisation of
 *                 the k weights); Mixtral MoE Block, _moe_forward (top_w / sum).
 *                 no renorm: g_j = p_j, Model Architecture Patterns,
 *                 "Top-K Router" (TopKRouter returns the raw top-k softmax).
 *   statistics    counts[e] = #{(t,j) : idx[t,j] = e}, axonml-nn moe.rs,
 *                 MoELayer::forward (its utilization counts) and
 *                 expert_utilization(); P[e] = mean_t p[t,e] and
 *                 aux = E * sum_e f_e * P_e, load_balancing_loss().
 *                 f_e is read as counts_e / (T*k), the fraction of the T*k
 *                 routed assignments, so that sum_e f_e = 1 and the statistic
 *                 equals 1 under uniform routing; the page's own code divides
 *                 by T only, which is k times this value.
 *   dispatch      for e ascending, for t ascending, every (t,j) with
 *                 idx[t,j] = e takes the next row: axonml-nn moe.rs,
 *                 MoELayer::forward (its loop over experts collecting their tokens).
 *   expert        y = down(SiLU(gate(x)) * up(x)), SiLU(z) = z / (1 + e^-z),
 *                 axonml-nn moe.rs, Expert::forward; Model Architecture
 *                 Patterns, "SwiGLU FFN". Weights are nn.Linear layout
 *                 [out, in], stacked per expert: gate/up [E, I, d],
 *                 down [E, d, I].
 *   combine       out[t] = sum_j g[t,j] * y_{idx[t,j]}(x[t]), each expert's
 *                 output weighted by its own gate: axonml-nn moe.rs,
 *                 MoELayer::forward (its weighted scatter back to token order);
 *                 Mixtral MoE Block markdown, _moe_forward.
 *
 * Options of the layer that the pages name as configuration knobs:
 *
 *   RMSNorm       the block applies RMSNorm before the MoE layer (Mixtral MoE
 *                 Block, layer table "post_attn_norm", nn.RMSNorm). Form 1 is
 *                 torch's nn.RMSNorm, x / sqrt(mean(x^2) + eps) * w; form 2 is
 *                 the one printed under Model Architecture Patterns, "RMSNorm
 *                 (no bias, no mean centering)": w * x / (||x|| / sqrt(d) + eps).
 *                 The router and every expert then see the normalised x.
 *   z-loss        the router z-loss statistic of ST-MoE that the training
 *                 config enables ("moe_router_z_loss_weight"; the Mixtral
 *                 page's note on the router z-loss): mean over tokens of
 *                 (logsumexp_e logits[t,e])^2, on the logits with their bias.
 *   capacity      KempnerForge ModelConfig, moe_capacity_factor (zero keeps
 *                 every assignment, a positive factor limits the tokens an
 *                 expert takes): capacity C = ceil(cf * T * k / E) assignments per
 *                 expert; an expert keeps its first C assignments in dispatch
 *                 order (tokens ascending) and drops the rest, whose slots
 *                 then contribute nothing to the output. Routing, gates,
 *                 counts and the balance statistic are those before dropping.
 *   shared        KempnerForge ModelConfig, moe_shared_experts (experts that
 *                 every token passes through), each the same SwiGLU MLP as a
 *                 routed expert
 *                 (the parameter count adds n_shared * expert_mlp); their
 *                 outputs are added to every token with weight 1.
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

enum { ORACLE_F32 = 0, ORACLE_BF16 = 1, ORACLE_F64 = 2 };

/* Exact widening of one stored element to fp64. */
static double load_elem(const void* base, int dtype, int64_t i) {
  if (dtype == ORACLE_F64) return ((const double*)base)[i];
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

/* out[i] = in[i] rounded to fp32 and then to the nearest bf16 (ties to even):
 * how a value computed in fp32 is stored in bf16 (diagnostic comparisons). */
void oracle_round_bf16(const double* in, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = round_to_bf16(in[i]);
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

/* ---- pre-MoE RMSNorm ------------------------------------------------------ */

/* xhat[t*d + c] = x[t,c] * r_t * w[c] with r_t = 1 / sqrt(mean_c x^2 + eps)
 * (form 1) or 1 / (sqrt(mean_c x^2) + eps) (form 2); w = 1 when NULL. */
void oracle_rmsnorm(const void* x, int x_dtype, const void* weight, int w_dtype, int64_t T, int64_t d,
                    double eps, int form, double* xhat) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t) {
    double ss = 0.0;
    for (int64_t c = 0; c < d; ++c) {
      const double v = load_elem(x, x_dtype, t * d + c);
      ss += v * v;
    }
    const double ms = ss / (double)d;
    const double r = form == 1 ? 1.0 / sqrt(ms + eps) : 1.0 / (sqrt(ms) + eps);
    for (int64_t c = 0; c < d; ++c) {
      const double w = weight ? load_elem(weight, w_dtype, c) : 1.0;
      xhat[t * d + c] = load_elem(x, x_dtype, t * d + c) * r * w;
    }
  }
}

/* ---- router: logits, softmax, z-loss ---------------------------------------- */

/* logits[t*E + e] = sum_c x[t,c] * Wr[e,c] (+ b[e]). */
void oracle_router_logits(const void* x, int x_dtype, const void* w_router, int w_dtype, const float* b_router,
                          int64_t T, int64_t d, int E, double* logits) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t) {
    for (int e = 0; e < E; ++e) {
      double acc = 0.0;
      for (int64_t c = 0; c < d; ++c)
        acc += load_elem(x, x_dtype, t * d + c) * load_elem(w_router, w_dtype, (int64_t)e * d + c);
      if (b_router) acc += (double)b_router[e];
      logits[t * E + e] = acc;
    }
  }
}

/* probs[t*E + e] = exp(l - max l) / sum exp(l - max l), per token. */
void oracle_softmax(const double* logits, int64_t T, int E, double* probs) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t) {
    const double* l = logits + t * E;
    double* p = probs + t * E;
    double m = l[0];
    for (int e = 1; e < E; ++e)
      if (l[e] > m) m = l[e];
    double s = 0.0;
    for (int e = 0; e < E; ++e) {
      p[e] = exp(l[e] - m);
      s += p[e];
    }
    for (int e = 0; e < E; ++e) p[e] /= s;
  }
}

/* mean_t (log sum_e exp logits[t,e])^2; 0 when T = 0. */
double oracle_z_loss(const double* logits, int64_t T, int E) {
  if (T == 0) return 0.0;
  double acc = 0.0;
  for (int64_t t = 0; t < T; ++t) {
    const double* l = logits + t * E;
    double m = l[0];
    for (int e = 1; e < E; ++e)
      if (l[e] > m) m = l[e];
    double s = 0.0;
    for (int e = 0; e < E; ++e) s += exp(l[e] - m);
    const double lse = m + log(s);
    acc += lse * lse;
  }
  return acc / (double)T;
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

/* ---- dispatch order and capacity ------------------------------------------- */

/* Assignments an expert may keep: ceil(cf * T * k / E), or -1 (no limit) when
 * cf <= 0. */
int64_t oracle_capacity(double cf, int64_t T, int k, int E) {
  if (!(cf > 0.0)) return -1;
  return (int64_t)ceil(cf * (double)T * (double)k / (double)E);
}

/* offsets[E+1]; perm_tok[R] = token of each dispatched row; inv[T*k] = row of
 * each (token, slot), or -1 when the slot was dropped. Rows are
 * expert-contiguous, tokens ascending within an expert; with capacity >= 0 an
 * expert keeps only its first `capacity` assignments in that order. Returns
 * the number of dropped assignments. */
int64_t oracle_dispatch(const int32_t* topk_idx, int64_t T, int k, int E, int64_t capacity, int64_t* offsets,
                        int32_t* perm_tok, int32_t* inv) {
  int64_t row = 0, dropped = 0;
  for (int e = 0; e < E; ++e) {
    offsets[e] = row;
    int64_t taken = 0;
    for (int64_t t = 0; t < T; ++t)
      for (int j = 0; j < k; ++j)
        if (topk_idx[t * k + j] == e) {
          if (capacity >= 0 && taken >= capacity) {
            inv[t * k + j] = -1;
            ++dropped;
            continue;
          }
          perm_tok[row] = (int32_t)t;
          inv[t * k + j] = (int32_t)row;
          ++row;
          ++taken;
        }
  }
  offsets[E] = row;
  return dropped;
}

/* ---- expert SwiGLU MLP ---------------------------------------------------- */

/* y[r, :] = down_e(SiLU(gate_e(x_t)) * up_e(x_t)) for each requested row
 * (t = tok[r], e = expert[r]); x is read as x_dtype, the weights as dtype. */
void oracle_expert_rows(const void* x, int x_dtype, const void* w_gate, const void* w_up, const void* w_down,
                        int dtype, int64_t d, int64_t I, int64_t n, const int32_t* tok,
                        const int32_t* expert, double* y) {
#pragma omp parallel
  {
    double* xv = (double*)malloc(sizeof(double) * (size_t)d);
    double* h = (double*)malloc(sizeof(double) * (size_t)I);
#pragma omp for schedule(dynamic, 1)
    for (int64_t r = 0; r < n; ++r) {
      const int64_t t = tok[r];
      const int64_t e = expert[r];
      for (int64_t c = 0; c < d; ++c) xv[c] = load_elem(x, x_dtype, t * d + c);
      for (int64_t i = 0; i < I; ++i) {
        const int64_t wrow = (e * I + i) * d;
        double g = 0.0, u = 0.0;
        for (int64_t c = 0; c < d; ++c) {
          g += xv[c] * load_elem(w_gate, dtype, wrow + c);
          u += xv[c] * load_elem(w_up, dtype, wrow + c);
        }
        double silu = g / (1.0 + exp(-g));
        h[i] = silu * u;
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

/* out[i, :] = sum_j keep[i,j] * gate[i,j] * expert_{idx[i,j]}(x[tok[i]])
 *           + sum_s shared_s(x[tok[i]])
 * for a list of tokens with their chosen experts and gates. keep == NULL keeps
 * every slot; n_shared shared experts (weights [n_shared, I, d] and
 * [n_shared, d, I]) are added with weight 1. */
void oracle_moe_tokens(const void* x, int x_dtype, const void* w_gate, const void* w_up, const void* w_down,
                       int dtype, int64_t d, int64_t I, int k, int64_t ntok, const int32_t* tok,
                       const int32_t* idx, const double* gate, const int8_t* keep, int n_shared,
                       const void* s_gate, const void* s_up, const void* s_down, double* out) {
  const int64_t n = ntok * k;
  const int64_t ns = ntok * n_shared;
  int32_t* rtok = (int32_t*)malloc(sizeof(int32_t) * (size_t)(n > 0 ? n : 1));
  double* y = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n * d : 1));
  int32_t* stok = (int32_t*)malloc(sizeof(int32_t) * (size_t)(ns > 0 ? ns : 1));
  int32_t* sexp = (int32_t*)malloc(sizeof(int32_t) * (size_t)(ns > 0 ? ns : 1));
  double* ys = (double*)malloc(sizeof(double) * (size_t)(ns > 0 ? ns * d : 1));
  for (int64_t i = 0; i < ntok; ++i)
    for (int j = 0; j < k; ++j) rtok[i * k + j] = tok[i];
  oracle_expert_rows(x, x_dtype, w_gate, w_up, w_down, dtype, d, I, n, rtok, idx, y);
  for (int64_t i = 0; i < ntok; ++i)
    for (int s = 0; s < n_shared; ++s) {
      stok[i * n_shared + s] = tok[i];
      sexp[i * n_shared + s] = s;
    }
  if (ns > 0) oracle_expert_rows(x, x_dtype, s_gate, s_up, s_down, dtype, d, I, ns, stok, sexp, ys);
  for (int64_t i = 0; i < ntok; ++i)
    for (int64_t c = 0; c < d; ++c) {
      double acc = 0.0;
      for (int j = 0; j < k; ++j)
        if (!keep || keep[i * k + j]) acc += gate[i * k + j] * y[(i * k + j) * d + c];
      for (int s = 0; s < n_shared; ++s) acc += ys[(i * n_shared + s) * d + c];
      out[i * d + c] = acc;
    }
  free(rtok);
  free(y);
  free(stok);
  free(sexp);
  free(ys);
}
