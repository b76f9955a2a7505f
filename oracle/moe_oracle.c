/*
 * fp64 CPU oracle for the forward pass of a sparse top-k Mixture-of-Experts layer.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, obviously correct statement of what the
 * layer computes.  Only the tests, the package's smoke check and the bench's CPU-baseline leg may
 * load it; the CUDA library never links, includes or calls it, and it shares no code with it.
 *
 * Sources (web pages on MoE; cited by page title and section):
 *  [SKILL]  "MoE Training: Mixture of Experts" (moe-training SKILL.md of the @r1z4x/tezgah package)
 *           - Quick Start, "Basic MoE Architecture": class MoELayer -- gate = Linear(H, E) with bias,
 *             softmax over experts, torch.topk(k), division of the k scores by their sum, per-slot /
 *             per-expert dispatch, expert = Linear(H, 4H) -> GELU -> Linear(4H, H), output[mask] +=
 *             score * expert_output.
 *           - Core Concepts 2, "Routing Mechanisms": top-1 by argmax of the logits; top-2 with
 *             renormalised scores.
 *           - Core Concepts 3, "Load Balancing": load_balancing_loss = E * sum_e f_e * P_e with
 *             f = bincount(top-k indices) / numel and P = mean softmax; router_z_loss =
 *             mean(logsumexp(logits)^2).
 *           - Core Concepts 4, "Expert Parallelism" and Best Practices 2, "Capacity Factor Tuning":
 *             capacity ~ tokens * capacity_factor / num_experts, tokens over capacity are dropped.
 *           - Advanced Patterns, "Mixtral 8x7B Architecture": expert-major gather
 *             (where(selected == e)), scaling by the routing weight, index_add_ back to token order.
 *  [CSDN]   "MOE- Mixture of Experts Explained" (CSDN article), section 8 "capacity factor and
 *           communication cost": CF 1.25 with top-2 as a starting point.
 *
 * Readings taken where the pages are silent or disagree (each is listed in the design notes):
 *  - selection is done on the logits (softmax is monotone, so the chosen set equals the set chosen
 *    on the probabilities); ties go to the lower expert index; slot s = rank s in that order;
 *  - renormalisation is always applied (k = 1 gives weight 1 exactly);
 *  - aux loss uses pre-drop counts divided by T*k and P averaged over all T tokens;
 *  - capacity = ceil(CF * T * k / E) evaluated in double, or unlimited when CF is +infinity;
 *  - assignments are visited slot-major then in token order (slot 0 of every token first); an
 *    assignment is kept iff its rank among earlier assignments to the same expert is < capacity,
 *    and that rank is also its row inside the expert's segment of the permuted buffer;
 *  - a dropped assignment contributes nothing and the kept weights are not renormalised again;
 *  - GELU is the exact erf form 0.5*u*(1 + erf(u/sqrt(2))) (nn.GELU() default); the Mixtral block's
 *    variant uses SiLU u*sigmoid(u) and bias-free Linear layers (a NULL bias pointer means zeros);
 *  - for T = 0 both losses are defined as 0.
 *
 * Inputs are passed in their storage type (fp32 or bf16 bit patterns) and widened to double element
 * by element (both widenings are exact), so the oracle never needs a double copy of the weights.
 */
#define _USE_MATH_DEFINES
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORACLE_F32 = 0, ORACLE_BF16 = 1 };

/* exact widening of one stored element to double */
static double load(const void* base, int dtype, size_t i) {
  if (dtype == ORACLE_F32) return (double)((const float*)base)[i];
  uint32_t bits = (uint32_t)((const uint16_t*)base)[i] << 16;
  float f;
  memcpy(&f, &bits, sizeof f);
  return (double)f;
}

/* GELU, exact erf form (nn.GELU() default) -- [SKILL] Quick Start expert FFN */
double oracle_gelu(double u) { return 0.5 * u * (1.0 + erf(u / sqrt(2.0))); }

/* SiLU, u * sigmoid(u) (nn.SiLU()) -- [SKILL] Advanced Patterns, "Mixtral 8x7B Architecture" experts */
double oracle_silu(double u) { return u / (1.0 + exp(-u)); }

enum { ORACLE_ACT_GELU = 0, ORACLE_ACT_SILU = 1 };
static double activation(int act, double u) { return act == ORACLE_ACT_SILU ? oracle_silu(u) : oracle_gelu(u); }

/* a bias pointer may be NULL: the Mixtral block's Linear layers have bias=False */
static double load_bias(const void* base, int dtype, size_t i) { return base ? load(base, dtype, i) : 0.0; }

/* capacity of one expert: max(ceil(CF * T * k / E), min_capacity), or -1 for "unlimited" (CF = +inf).
 * [SKILL] Core Concepts 4 / Best Practices 2; the k factor and the ceiling follow the workload
 * statement (the pages' formulas differ only in rounding and in whether k appears); the lower
 * bound is the "min_capacity" of the Core Concepts 4 configuration (0 = none). */
int64_t oracle_capacity(double cf, int64_t T, int64_t k, int64_t E, int64_t min_capacity) {
  if (isinf(cf) && cf > 0) return -1;
  const int64_t c = (int64_t)ceil(cf * (double)T * (double)k / (double)E);
  return c > min_capacity ? c : min_capacity;
}

/*
 * Router for all tokens -- [SKILL] Quick Start (gate, softmax, topk, renormalise) and Core
 * Concepts 2.
 *   logits[t,e] = bg[e] + sum_h x[t,h] * Wg[h,e]
 *   lse[t]      = log sum_e exp(logits[t,e])            (max-shifted)
 *   p[t,e]      = exp(logits[t,e] - lse[t])
 *   topk_idx[t,s], s < k : experts in order (logit descending, index ascending)
 *   topk_w[t,s] = p[t, topk_idx[t,s]] / sum_s' p[t, topk_idx[t,s']]
 *   margin[t]   = smallest gap between consecutive logits among the first k+1 in that order
 *                 (the k-th vs (k+1)-th gap included when k < E); +inf when k == E and k == 1
 * Any output pointer may be NULL except topk_idx.
 */
void oracle_route(int64_t T, int64_t H, int64_t E, int64_t k, int dtype, const void* x, const void* Wg,
                  const void* bg, double* logits_out, double* lse_out, double* p_out, int32_t* topk_idx,
                  double* topk_w, double* margin_out) {
#pragma omp parallel
  {
    double* logit = (double*)malloc(sizeof(double) * (size_t)E);
    char* taken = (char*)malloc((size_t)E);
    int32_t* order = (int32_t*)malloc(sizeof(int32_t) * (size_t)(k + 1));
#pragma omp for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
      for (int64_t e = 0; e < E; ++e) {
        double acc = load_bias(bg, dtype, (size_t)e);
        for (int64_t h = 0; h < H; ++h) acc += load(x, dtype, (size_t)(t * H + h)) * load(Wg, dtype, (size_t)(h * E + e));
        logit[e] = acc;
      }
      double m = logit[0];
      for (int64_t e = 1; e < E; ++e)
        if (logit[e] > m) m = logit[e];
      double s = 0.0;
      for (int64_t e = 0; e < E; ++e) s += exp(logit[e] - m);
      double lse = m + log(s);

      /* selection: repeatedly take the best remaining expert (logit desc, index asc) */
      memset(taken, 0, (size_t)E);
      int64_t nsel = (k < E) ? k + 1 : k;
      for (int64_t r = 0; r < nsel; ++r) {
        int64_t best = -1;
        for (int64_t e = 0; e < E; ++e) {
          if (taken[e]) continue;
          if (best < 0 || logit[e] > logit[best]) best = e; /* strict '>' keeps the lower index on ties */
        }
        taken[best] = 1;
        order[r] = (int32_t)best;
      }
      double psum = 0.0;
      for (int64_t r = 0; r < k; ++r) psum += exp(logit[order[r]] - lse);
      for (int64_t r = 0; r < k; ++r) {
        topk_idx[t * k + r] = order[r];
        if (topk_w) topk_w[t * k + r] = exp(logit[order[r]] - lse) / psum;
      }
      if (margin_out) {
        double mg = INFINITY;
        for (int64_t r = 0; r + 1 < nsel; ++r) {
          double g = logit[order[r]] - logit[order[r + 1]];
          if (g < mg) mg = g;
        }
        margin_out[t] = mg;
      }
      if (lse_out) lse_out[t] = lse;
      for (int64_t e = 0; e < E; ++e) {
        if (logits_out) logits_out[t * E + e] = logit[e];
        if (p_out) p_out[t * E + e] = exp(logit[e] - lse);
      }
    }
    free(logit);
    free(taken);
    free(order);
  }
}

/*
 * Switch load-balancing loss and router z-loss -- [SKILL] Core Concepts 3, "Load Balancing".
 *   f_e = #{(t,s): topk_idx[t,s] = e} / (T*k)        (pre-drop counts)
 *   P_e = (1/T) sum_t p[t,e]
 *   aux = E * sum_e f_e * P_e
 *   z   = (1/T) sum_t lse[t]^2
 */
void oracle_losses(int64_t T, int64_t E, int64_t k, const double* p, const double* lse, const int32_t* topk_idx,
                   double* aux, double* z) {
  if (T == 0) {
    *aux = 0.0;
    *z = 0.0;
    return;
  }
  double* cnt = (double*)calloc((size_t)E, sizeof(double));
  for (int64_t i = 0; i < T * k; ++i) cnt[topk_idx[i]] += 1.0;
  double a = 0.0;
  for (int64_t e = 0; e < E; ++e) {
    double P = 0.0;
    for (int64_t t = 0; t < T; ++t) P += p[t * E + e];
    a += (cnt[e] / (double)(T * k)) * (P / (double)T);
  }
  *aux = (double)E * a;
  double zz = 0.0;
  for (int64_t t = 0; t < T; ++t) zz += lse[t] * lse[t];
  *z = zz / (double)T;
  free(cnt);
}

/*
 * Capacity-aware dispatch -- [SKILL] Core Concepts 4 and Best Practices 2 (capacity, drop_tokens);
 * [SKILL] Advanced Patterns, Mixtral block (expert-major gather).
 * cap < 0 means unlimited.  Outputs:
 *   cnt_pre[E]       assignments per expert before dropping
 *   expert_counts[E] kept assignments per expert = min(cnt_pre, cap)
 *   offsets[E+1]     exclusive prefix sum of expert_counts (offsets[E] = kept total)
 *   dropped[T*k]     1 if assignment (t,s) is over capacity
 *   row_of[T*k]      row of (t,s) in the permuted buffer, -1 if dropped
 *   row_token[kept]  token of each row; row_slot[kept] its slot
 * Returns the number of kept assignments.
 */
int64_t oracle_dispatch(int64_t T, int64_t E, int64_t k, int64_t cap, const int32_t* topk_idx, int32_t* cnt_pre,
                        int32_t* expert_counts, int32_t* offsets, uint8_t* dropped, int32_t* row_of,
                        int32_t* row_token, int32_t* row_slot) {
  int64_t* seen = (int64_t*)calloc((size_t)E, sizeof(int64_t));
  int64_t* rank = (int64_t*)malloc(sizeof(int64_t) * (size_t)(T * k > 0 ? T * k : 1));
  for (int64_t s = 0; s < k; ++s)     /* slot-major ... */
    for (int64_t t = 0; t < T; ++t) { /* ... then token order */
      int32_t e = topk_idx[t * k + s];
      rank[t * k + s] = seen[e]++;
    }
  for (int64_t e = 0; e < E; ++e) {
    cnt_pre[e] = (int32_t)seen[e];
    expert_counts[e] = (int32_t)((cap >= 0 && seen[e] > cap) ? cap : seen[e]);
  }
  offsets[0] = 0;
  for (int64_t e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + expert_counts[e];
  for (int64_t t = 0; t < T; ++t)
    for (int64_t s = 0; s < k; ++s) {
      int64_t i = t * k + s;
      int32_t e = topk_idx[i];
      int keep = (cap < 0) || (rank[i] < cap);
      dropped[i] = (uint8_t)!keep;
      if (keep) {
        int32_t r = (int32_t)(offsets[e] + rank[i]);
        row_of[i] = r;
        row_token[r] = (int32_t)t;
        row_slot[r] = (int32_t)s;
      } else {
        row_of[i] = -1;
      }
    }
  int64_t kept = offsets[E];
  free(seen);
  free(rank);
  return kept;
}

/*
 * One expert's FFN on one input row -- [SKILL] Quick Start expert: Linear(H, F) -> GELU -> Linear(F, H);
 * Advanced Patterns, Mixtral block: Linear(H, F, bias=False) -> SiLU -> Linear(F, H, bias=False).
 *   u[f] = b1[e,f] + sum_h xrow[h] * W1[e,h,f]        (b1 = 0 when absent)
 *   g[f] = act(u[f])                                   (GELU or SiLU)
 *   y[h] = b2[e,h] + sum_f g[f] * W2[e,f,h]            (b2 = 0 when absent)
 * xrow is already double; u is scratch of length F.
 */
static void expert_ffn_row(int64_t H, int64_t F, int dtype, int act, const double* xrow, int32_t e, const void* W1,
                           const void* b1, const void* W2, const void* b2, double* u, double* y) {
  for (int64_t f = 0; f < F; ++f) u[f] = load_bias(b1, dtype, (size_t)(e * F + f));
  for (int64_t h = 0; h < H; ++h) {
    double xh = xrow[h];
    size_t base = (size_t)((e * H + h) * F);
    for (int64_t f = 0; f < F; ++f) u[f] += xh * load(W1, dtype, base + (size_t)f);
  }
  for (int64_t f = 0; f < F; ++f) u[f] = activation(act, u[f]);
  for (int64_t h = 0; h < H; ++h) y[h] = load_bias(b2, dtype, (size_t)(e * H + h));
  for (int64_t f = 0; f < F; ++f) {
    double gf = u[f];
    size_t base = (size_t)((e * F + f) * H);
    for (int64_t h = 0; h < H; ++h) y[h] += gf * load(W2, dtype, base + (size_t)h);
  }
}

/*
 * Expert FFN for a list of (token, expert) pairs: y[i,:] = FFN_{experts[i]}(x[tokens[i],:]).
 * Used to check the grouped GEMM stage on its own, fed any dispatch.
 */
void oracle_expert_rows(int64_t H, int64_t F, int dtype, int act, const void* x, const void* W1, const void* b1,
                        const void* W2, const void* b2, int64_t n, const int32_t* tokens, const int32_t* experts,
                        double* y, int nthreads) {
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
#pragma omp parallel
  {
    double* xrow = (double*)malloc(sizeof(double) * (size_t)H);
    double* u = (double*)malloc(sizeof(double) * (size_t)F);
#pragma omp for schedule(dynamic, 1)
    for (int64_t i = 0; i < n; ++i) {
      for (int64_t h = 0; h < H; ++h) xrow[h] = load(x, dtype, (size_t)(tokens[i] * H + h));
      expert_ffn_row(H, F, dtype, act, xrow, experts[i], W1, b1, W2, b2, u, y + i * H);
    }
    free(xrow);
    free(u);
  }
}

/*
 * Weighted combine for a list of tokens -- [SKILL] Quick Start (output[mask] += score * expert_output)
 * and Advanced Patterns, Mixtral block (index_add_ of weighted expert outputs):
 *   out[t,:] = sum over kept slots s (slot order) of topk_w[t,s] * FFN_{topk_idx[t,s]}(x[t,:])
 * A token whose every slot was dropped gets zeros.
 */
void oracle_forward_tokens(int64_t H, int64_t F, int64_t k, int dtype, int act, const void* x, const void* W1,
                           const void* b1, const void* W2, const void* b2, const int32_t* topk_idx,
                           const double* topk_w, const uint8_t* dropped, int64_t n, const int32_t* tokens,
                           double* out, int nthreads) {
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
#pragma omp parallel
  {
    double* xrow = (double*)malloc(sizeof(double) * (size_t)H);
    double* u = (double*)malloc(sizeof(double) * (size_t)F);
    double* y = (double*)malloc(sizeof(double) * (size_t)H);
#pragma omp for schedule(dynamic, 1)
    for (int64_t i = 0; i < n; ++i) {
      int64_t t = tokens[i];
      double* o = out + i * H;
      for (int64_t h = 0; h < H; ++h) o[h] = 0.0;
      for (int64_t h = 0; h < H; ++h) xrow[h] = load(x, dtype, (size_t)(t * H + h));
      for (int64_t s = 0; s < k; ++s) {
        if (dropped && dropped[t * k + s]) continue;
        expert_ffn_row(H, F, dtype, act, xrow, topk_idx[t * k + s], W1, b1, W2, b2, u, y);
        double w = topk_w[t * k + s];
        for (int64_t h = 0; h < H; ++h) o[h] += w * y[h];
      }
    }
    free(xrow);
    free(u);
    free(y);
  }
}

/* ----------------------------------------------------------------------------------------------
 * Expert-choice routing -- [SKILL] Core Concepts 2, "Expert Choice Routing": the router scores
 * are transposed to (experts, tokens) and every expert takes the top capacity_per_expert tokens
 * of its row ("guarantees perfect load balancing").  Readings (listed in the design notes):
 *  - the scores are the router's logits, as printed (no softmax before the per-expert top-k);
 *  - capacity_per_expert C = min(T, max(ceil(CF * T * k / E), min_capacity)), k being the average number of experts
 *    per token; CF = +inf gives C = T (every expert sees every token);
 *  - ties go to the lower token index; an expert's chosen tokens are listed in ascending token
 *    order, which is also their row order inside the expert's segment;
 *  - a chosen (token, expert) pair is weighted by the token's softmax probability p[t,e] over the
 *    experts, without renormalisation; a token chosen by no expert gets out = 0.
 * ---------------------------------------------------------------------------------------------- */
int64_t oracle_ec_capacity(double cf, int64_t T, int64_t k, int64_t E, int64_t min_capacity) {
  if (isinf(cf) && cf > 0) return T;
  int64_t c = (int64_t)ceil(cf * (double)T * (double)k / (double)E);
  if (c < min_capacity) c = min_capacity;
  return c < T ? c : T;
}

typedef struct {
  double v;
  int32_t t;
} scored_token;

/* score descending, token index ascending */
static int by_score_then_token(const void* pa, const void* pb) {
  const scored_token* a = (const scored_token*)pa;
  const scored_token* b = (const scored_token*)pb;
  if (a->v > b->v) return -1;
  if (a->v < b->v) return 1;
  return (a->t > b->t) - (a->t < b->t);
}

/*
 * chosen[e*C + j], j < C: the C tokens of expert e in ascending token order.
 * margin[e]: logits gap between the C-th and (C+1)-th token of expert e in score order
 *            (+inf when C == T).  margin may be NULL.
 */
void oracle_expert_choice(int64_t T, int64_t E, int64_t C, const double* logits, int32_t* chosen, double* margin) {
#pragma omp parallel
  {
    scored_token* order = (scored_token*)malloc(sizeof(scored_token) * (size_t)(T > 0 ? T : 1));
    char* mark = (char*)malloc((size_t)(T > 0 ? T : 1));
#pragma omp for schedule(dynamic, 1)
    for (int64_t e = 0; e < E; ++e) {
      for (int64_t t = 0; t < T; ++t) {
        order[t].v = logits[t * E + e];
        order[t].t = (int32_t)t;
      }
      qsort(order, (size_t)T, sizeof(scored_token), by_score_then_token);
      for (int64_t t = 0; t < T; ++t) mark[t] = 0;
      for (int64_t j = 0; j < C; ++j) mark[order[j].t] = 1;
      int64_t j = 0;
      for (int64_t t = 0; t < T; ++t)
        if (mark[t]) chosen[e * C + j++] = (int32_t)t;
      if (margin) margin[e] = (C < T && C > 0) ? order[C - 1].v - order[C].v : INFINITY;
    }
    free(order);
    free(mark);
  }
}

/* Losses under expert choice: every expert holds C of the E*C assignments, so f_e = 1/E and
 * aux = E * sum_e f_e * P_e = sum_e P_e; z = mean_t lse_t^2 as for token choice (Core Concepts 3). */
void oracle_ec_losses(int64_t T, int64_t E, int64_t C, const double* p, const double* lse, double* aux, double* z) {
  if (T == 0) {
    *aux = 0.0;
    *z = 0.0;
    return;
  }
  double a = 0.0;
  for (int64_t e = 0; e < E; ++e) {
    double P = 0.0;
    for (int64_t t = 0; t < T; ++t) P += p[t * E + e];
    P /= (double)T;
    const double f = (double)C / ((double)E * (double)C);
    a += f * P;
  }
  *aux = (double)E * a;
  double zz = 0.0;
  for (int64_t t = 0; t < T; ++t) zz += lse[t] * lse[t];
  *z = zz / (double)T;
}

/* ----------------------------------------------------------------------------------------------
 * Backward pass.  The pages train MoE layers (the skill's subject; Core Concepts 3 adds the two
 * losses to the training loss), so the layer's gradients are the chain rule through the forward
 * definition above.  Given dout[t,:] = dL/dout[t,:], d_aux = dL/daux and d_z = dL/dz:
 *
 * every kept slot (t, s) with expert e and weight w = topk_w[t,s]:
 *   u = x_t.W1[e] + b1[e],  g = act(u),  y = g.W2[e] + b2[e]
 *   dY = w dout_t                dw[t,s] = dout_t . y
 *   dW2[e] += g^T dY             db2[e] += dY
 *   du = (W2[e] dY) * act'(u)    dW1[e] += x_t^T du      db1[e] += du      dx_t += W1[e] du
 * a dropped slot has dw = 0 and adds nothing;
 *
 * the router, per token (p = softmax(logits), lse, chosen experts e_s, S = sum_s p[e_s]):
 *   dp[e_s]  = (dw[t,s] - sum_s' dw[t,s'] w[t,s']) / S          renormalisation w_s = p[e_s] / S
 *   dp[e]   += d_aux * E * f_e / T                              aux = E sum_e f_e P_e (f fixed)
 *   dlogit[e] = p[e] (dp[e] - sum_e' p[e'] dp[e']) + d_z * 2 lse p[e] / T
 *   dWg += x_t^T dlogit          dbg += dlogit                  dx_t += Wg dlogit
 * The top-k choice and the capacity drops are piecewise constant and carry no gradient.
 * ---------------------------------------------------------------------------------------------- */

/* d act / du: GELU' = Phi(u) + u phi(u); SiLU' = s(u) (1 + u (1 - s(u))) with s the logistic */
double oracle_act_grad(int act, double u) {
  if (act == ORACLE_ACT_SILU) {
    const double sg = 1.0 / (1.0 + exp(-u));
    return sg * (1.0 + u * (1.0 - sg));
  }
  return 0.5 * (1.0 + erf(u / sqrt(2.0))) + u * exp(-0.5 * u * u) / sqrt(2.0 * M_PI);
}

/*
 * One kept slot: dx_part[H] = W1[e] du and dw = dout_t . y; du_out[F] (may be NULL) receives du.
 * dout_t is the token's output gradient row (double, length H).
 */
void oracle_bwd_slot(int64_t H, int64_t F, int dtype, int act, const void* x, int64_t t, int32_t e, const void* W1,
                     const void* b1, const void* W2, const void* b2, const double* dout_t, double w, double* dx_part,
                     double* dw, double* du_out) {
  double* u = (double*)malloc(sizeof(double) * (size_t)F);
  double* du = (double*)malloc(sizeof(double) * (size_t)F);
  for (int64_t f = 0; f < F; ++f) u[f] = load_bias(b1, dtype, (size_t)(e * F + f));
  for (int64_t h = 0; h < H; ++h) {
    const double xv = load(x, dtype, (size_t)(t * H + h));
    const size_t base = (size_t)((e * H + h) * F);
    for (int64_t f = 0; f < F; ++f) u[f] += xv * load(W1, dtype, base + (size_t)f);
  }
  /* dout . y = dout . b2[e] + sum_f g[f] (W2[e][f,:] . dout);  dg[f] = w (W2[e][f,:] . dout) */
  double acc = 0.0;
  for (int64_t h = 0; h < H; ++h) acc += dout_t[h] * load_bias(b2, dtype, (size_t)(e * H + h));
  for (int64_t f = 0; f < F; ++f) {
    const size_t base = (size_t)((e * F + f) * H);
    double wd = 0.0;
    for (int64_t h = 0; h < H; ++h) wd += load(W2, dtype, base + (size_t)h) * dout_t[h];
    acc += activation(act, u[f]) * wd;
    du[f] = w * wd * oracle_act_grad(act, u[f]);
  }
  *dw = acc;
  for (int64_t h = 0; h < H; ++h) {
    const size_t base = (size_t)((e * H + h) * F);
    double s = 0.0;
    for (int64_t f = 0; f < F; ++f) s += load(W1, dtype, base + (size_t)f) * du[f];
    dx_part[h] = s;
  }
  if (du_out)
    for (int64_t f = 0; f < F; ++f) du_out[f] = du[f];
  free(u);
  free(du);
}

/*
 * Weight gradients of expert e from its kept rows (tokens[i], weight w[i]), restricted to the
 * listed FFN columns fcols[j] (all F of them for the full gradient):
 *   dW2_rows[j, :] = dW2[e][fcols[j], :]      dW1_cols[j, :] = dW1[e][:, fcols[j]]
 *   db1_sel[j]     = db1[e][fcols[j]]          db2_e[:]       = db2[e][:]
 * dout is [T,H] double.  Rows are visited in the order given.
 */
void oracle_bwd_expert_weights(int64_t H, int64_t F, int dtype, int act, const void* x, int32_t e, const void* W1,
                               const void* b1, const void* W2, int64_t n, const int32_t* tokens, const double* w,
                               const double* dout, int64_t nf, const int32_t* fcols, double* dW2_rows,
                               double* dW1_cols, double* db1_sel, double* db2_e, int nthreads) {
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
  for (int64_t h = 0; h < H; ++h) db2_e[h] = 0.0;
  for (int64_t i = 0; i < n; ++i)
    for (int64_t h = 0; h < H; ++h) db2_e[h] += w[i] * dout[tokens[i] * H + h];
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t j = 0; j < nf; ++j) {
    const int64_t f = fcols[j];
    double* r2 = dW2_rows + j * H;
    double* c1 = dW1_cols + j * H;
    for (int64_t h = 0; h < H; ++h) r2[h] = c1[h] = 0.0;
    double db1 = 0.0;
    for (int64_t i = 0; i < n; ++i) {
      const int64_t t = tokens[i];
      double u = load_bias(b1, dtype, (size_t)(e * F + f));
      for (int64_t h = 0; h < H; ++h) u += load(x, dtype, (size_t)(t * H + h)) * load(W1, dtype, (size_t)((e * H + h) * F + f));
      const double g = activation(act, u);
      double wd = 0.0;
      for (int64_t h = 0; h < H; ++h) wd += load(W2, dtype, (size_t)((e * F + f) * H + h)) * dout[t * H + h];
      const double du = w[i] * wd * oracle_act_grad(act, u);
      for (int64_t h = 0; h < H; ++h) {
        r2[h] += g * w[i] * dout[t * H + h];
        c1[h] += load(x, dtype, (size_t)(t * H + h)) * du;
      }
      db1 += du;
    }
    db1_sel[j] = db1;
  }
}

/*
 * Router backward for all tokens, given dw[T,k] (zero for dropped slots) and the pre-drop counts
 * cnt_pre[E].  Outputs dlogits[T,E], dWg[H,E], dbg[E] and dx_router[T,H] (the gate's part of dx).
 */
void oracle_bwd_router(int64_t T, int64_t H, int64_t E, int64_t k, int dtype, const void* x, const void* Wg,
                       const void* bg, const int32_t* topk_idx, const int32_t* cnt_pre, const double* dw,
                       double d_aux, double d_z, double* dlogits, double* dWg, double* dbg, double* dx_router) {
  double* lg = (double*)malloc(sizeof(double) * (size_t)E);
  double* p = (double*)malloc(sizeof(double) * (size_t)E);
  double* dp = (double*)malloc(sizeof(double) * (size_t)E);
  for (int64_t i = 0; i < H * E; ++i) dWg[i] = 0.0;
  for (int64_t e = 0; e < E; ++e) dbg[e] = 0.0;
  for (int64_t t = 0; t < T; ++t) {
    for (int64_t e = 0; e < E; ++e) {
      double acc = load_bias(bg, dtype, (size_t)e);
      for (int64_t h = 0; h < H; ++h) acc += load(x, dtype, (size_t)(t * H + h)) * load(Wg, dtype, (size_t)(h * E + e));
      lg[e] = acc;
    }
    double m = lg[0];
    for (int64_t e = 1; e < E; ++e)
      if (lg[e] > m) m = lg[e];
    double se = 0.0;
    for (int64_t e = 0; e < E; ++e) se += exp(lg[e] - m);
    const double lse = m + log(se);
    for (int64_t e = 0; e < E; ++e) p[e] = exp(lg[e] - lse);
    double S = 0.0;
    for (int64_t s = 0; s < k; ++s) S += p[topk_idx[t * k + s]];
    double dww = 0.0;
    for (int64_t s = 0; s < k; ++s) dww += dw[t * k + s] * p[topk_idx[t * k + s]] / S;
    for (int64_t e = 0; e < E; ++e) dp[e] = d_aux * (double)E * ((double)cnt_pre[e] / ((double)T * (double)k)) / (double)T;
    for (int64_t s = 0; s < k; ++s) dp[topk_idx[t * k + s]] += (dw[t * k + s] - dww) / S;
    double pdp = 0.0;
    for (int64_t e = 0; e < E; ++e) pdp += p[e] * dp[e];
    double* dl = dlogits + t * E;
    for (int64_t e = 0; e < E; ++e) dl[e] = p[e] * (dp[e] - pdp) + d_z * 2.0 * lse * p[e] / (double)T;
    for (int64_t e = 0; e < E; ++e) dbg[e] += dl[e];
    for (int64_t h = 0; h < H; ++h) {
      const double xv = load(x, dtype, (size_t)(t * H + h));
      double s = 0.0;
      for (int64_t e = 0; e < E; ++e) {
        dWg[h * E + e] += xv * dl[e];
        s += load(Wg, dtype, (size_t)(h * E + e)) * dl[e];
      }
      dx_router[t * H + h] = s;
    }
  }
  free(lg);
  free(p);
  free(dp);
}

/*
 * Router backward under expert choice (Core Concepts 2): the weight of a chosen pair (t, e) is the
 * token's softmax probability itself, so dp[t,e] = dw[t,e] for chosen pairs (0 elsewhere), plus the
 * aux-loss term d_aux / T (f_e = 1/E is fixed), which the softmax backward cancels because the
 * probabilities of a token sum to 1:
 *   dlogit[e] = p[e] (dp[e] - sum_e' p[e'] dp[e']) + d_z * 2 lse p[e] / T
 * dw[T,E] holds dout_t . y for every chosen pair.  Outputs as for oracle_bwd_router.
 */
void oracle_bwd_router_ec(int64_t T, int64_t H, int64_t E, int dtype, const void* x, const void* Wg, const void* bg,
                          const double* dw, double d_aux, double d_z, double* dlogits, double* dWg, double* dbg,
                          double* dx_router) {
  double* lg = (double*)malloc(sizeof(double) * (size_t)E);
  double* p = (double*)malloc(sizeof(double) * (size_t)E);
  double* dp = (double*)malloc(sizeof(double) * (size_t)E);
  for (int64_t i = 0; i < H * E; ++i) dWg[i] = 0.0;
  for (int64_t e = 0; e < E; ++e) dbg[e] = 0.0;
  for (int64_t t = 0; t < T; ++t) {
    for (int64_t e = 0; e < E; ++e) {
      double acc = load_bias(bg, dtype, (size_t)e);
      for (int64_t h = 0; h < H; ++h) acc += load(x, dtype, (size_t)(t * H + h)) * load(Wg, dtype, (size_t)(h * E + e));
      lg[e] = acc;
    }
    double m = lg[0];
    for (int64_t e = 1; e < E; ++e)
      if (lg[e] > m) m = lg[e];
    double se = 0.0;
    for (int64_t e = 0; e < E; ++e) se += exp(lg[e] - m);
    const double lse = m + log(se);
    for (int64_t e = 0; e < E; ++e) p[e] = exp(lg[e] - lse);
    for (int64_t e = 0; e < E; ++e) dp[e] = dw[t * E + e] + d_aux / (double)T;
    double pdp = 0.0;
    for (int64_t e = 0; e < E; ++e) pdp += p[e] * dp[e];
    double* dl = dlogits + t * E;
    for (int64_t e = 0; e < E; ++e) dl[e] = p[e] * (dp[e] - pdp) + d_z * 2.0 * lse * p[e] / (double)T;
    for (int64_t e = 0; e < E; ++e) dbg[e] += dl[e];
    for (int64_t h = 0; h < H; ++h) {
      const double xv = load(x, dtype, (size_t)(t * H + h));
      double s = 0.0;
      for (int64_t e = 0; e < E; ++e) {
        dWg[h * E + e] += xv * dl[e];
        s += load(Wg, dtype, (size_t)(h * E + e)) * dl[e];
      }
      dx_router[t * H + h] = s;
    }
  }
  free(lg);
  free(p);
  free(dp);
}

/* threads the OpenMP runtime will use for a parallel region (for reporting) */
int oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

void oracle_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}
