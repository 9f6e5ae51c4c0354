/*
 * moe_oracle.c -- plain fp64 CPU oracle of the sparse-MoE FFN layer forward.
 *
 * TEST INFRASTRUCTURE: only the tests, the package smoke check and the
 * benchmark's CPU-baseline leg may call it. It shares no code with the CUDA
 * library. Every step is the plain definition written out in binary64; loops
 * over tokens are independent and may run on several OpenMP threads, which
 * does not change any result.
 *
 * Readings taken where the pages are silent (each one also listed in the
 * design notes of the repository):
 *  - softmax routing selects on the logits (softmax is strictly increasing);
 *  - ties go to the lower expert index, and between groups to the lower group
 *    index; output slots are in descending selection score;
 *  - SiLU(z) = z * sigmoid(z);
 *  - capacity: "excess" tokens are the later ones in token order; a token
 *    whose preferred expert is full walks further down its own ranking; slots
 *    left without a non-full eligible expert are dropped (index -1, weight 0);
 *  - gates of a capacity-redirected slot are the redirected expert's own
 *    probability (or score), renormalised over the kept slots when asked.
 */
#include "moe_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ---- element access: exact widening of binary32 / bf16 to binary64 ------- */

static double elem(const void* p, int32_t dt, int64_t i) {
  if (dt == 0) return (double)((const float*)p)[i];
  union { uint32_t u; float f; } c;
  c.u = (uint32_t)((const uint16_t*)p)[i] << 16;
  return (double)c.f;
}

static int near_tie(double a, double b) {
  double m = fabs(a) > fabs(b) ? fabs(a) : fabs(b);
  return a == b || fabs(a - b) < ORACLE_TIE_REL * m;
}

static double sigmoid(double z) { return 1.0 / (1.0 + exp(-z)); }

/* sqrt(softplus(z)), softplus(z) = log(1 + e^z) written without overflow. */
static double sqrtsoftplus(double z) {
  double sp = (z > 0 ? z : 0.0) + log1p(exp(-fabs(z)));
  return sqrt(sp);
}

/* Raw score of the biased-score routers: sigmoid ([DS] V3) or sqrtsoftplus ([DS] V4). */
static double raw_score(int32_t score_fn, double z) { return score_fn == 2 ? sqrtsoftplus(z) : sigmoid(z); }

/* ---- router logits ([DS] router listing; [MoE] 3.1 linear router) --------- */

void oracle_router_logits(int64_t n, int32_t d, int32_t E, const void* x, int32_t x_dt,
                          const void* w_r, int32_t w_dt, double* logits) {
#pragma omp parallel for schedule(dynamic, 16)
  for (int64_t t = 0; t < n; ++t)
    for (int32_t e = 0; e < E; ++e) {
      double acc = 0.0;
      for (int32_t i = 0; i < d; ++i)
        acc += elem(x, x_dt, t * (int64_t)d + i) * elem(w_r, w_dt, (int64_t)e * d + i);
      logits[t * (int64_t)E + e] = acc;
    }
}

/* ---- per-token scoring and selection -------------------------------------- */

typedef struct {
  double v;   /* selection value */
  int32_t e;  /* expert (or group) index */
} keyed;

/* Descending value; equal values: ascending index. */
static int cmp_keyed(const void* pa, const void* pb) {
  const keyed* a = (const keyed*)pa;
  const keyed* b = (const keyed*)pb;
  if (a->v > b->v) return -1;
  if (a->v < b->v) return 1;
  return (a->e > b->e) - (a->e < b->e);
}

/*
 * Selection values and the eligible ranking of one token.
 *   softmax:  v_e = l_e (same order as the softmax probabilities)
 *   sigmoid:  s_e = sigmoid(l_e), v_e = s_e + b_e        (bias: selection only)
 * Group limit ([DS]): the E experts form n_group consecutive groups; a group's
 * score is the sum of its two largest v; the topk_group best groups stay
 * eligible and every other expert is excluded.
 * Writes rank[0..n_elig) and returns n_elig; *exempt |= near-tied group cut.
 */
static int32_t token_ranking(const oracle_cfg* cfg, const double* l, const float* bias, double* v,
                             int32_t* rank, int* exempt) {
  const int32_t E = cfg->n_routed;
  for (int32_t e = 0; e < E; ++e) {
    if (cfg->score_fn != 0)
      v[e] = raw_score(cfg->score_fn, l[e]) + (bias ? (double)bias[e] : 0.0);
    else
      v[e] = l[e];
  }
  keyed* ks = (keyed*)malloc(sizeof(keyed) * (size_t)E);
  uint8_t* eligible = (uint8_t*)malloc((size_t)E);
  memset(eligible, 1, (size_t)E);
  if (cfg->n_group > 1) {
    const int32_t G = cfg->n_group, per = E / G;
    keyed* gs = (keyed*)malloc(sizeof(keyed) * (size_t)G);
    for (int32_t g = 0; g < G; ++g) {
      double top1 = -INFINITY, top2 = -INFINITY;
      for (int32_t j = 0; j < per; ++j) {
        double x = v[g * per + j];
        if (x > top1) {
          top2 = top1;
          top1 = x;
        } else if (x > top2) {
          top2 = x;
        }
      }
      gs[g].v = top1 + top2;
      gs[g].e = g;
    }
    qsort(gs, (size_t)G, sizeof(keyed), cmp_keyed);
    if (cfg->topk_group < G && near_tie(gs[cfg->topk_group - 1].v, gs[cfg->topk_group].v))
      *exempt = 1;
    memset(eligible, 0, (size_t)E);
    for (int32_t r = 0; r < cfg->topk_group; ++r)
      for (int32_t j = 0; j < per; ++j) eligible[gs[r].e * per + j] = 1;
    free(gs);
  }
  int32_t m = 0;
  for (int32_t e = 0; e < E; ++e)
    if (eligible[e]) {
      ks[m].v = v[e];
      ks[m].e = e;
      ++m;
    }
  qsort(ks, (size_t)m, sizeof(keyed), cmp_keyed);
  for (int32_t r = 0; r < m; ++r) rank[r] = ks[r].e;
  free(ks);
  free(eligible);
  return m;
}

/*
 * Gate weights of the kept slots of one token ([DS] gates from raw scores and
 * routed_scaling_factor; [MoE] 4.1 softmax probabilities of the top-k;
 * [1.8T] 4.1 softmax over the selected logits = renormalised probabilities).
 */
static void token_gates(const oracle_cfg* cfg, const double* l, const int32_t* idx, double* w) {
  const int32_t E = cfg->n_routed, k = cfg->top_k;
  double denom = 1.0;
  double* p = (double*)malloc(sizeof(double) * (size_t)E);
  if (cfg->score_fn != 0) {
    for (int32_t e = 0; e < E; ++e) p[e] = raw_score(cfg->score_fn, l[e]);
  } else {
    double mx = -INFINITY, z = 0.0;
    for (int32_t e = 0; e < E; ++e) mx = l[e] > mx ? l[e] : mx;
    for (int32_t e = 0; e < E; ++e) z += exp(l[e] - mx);
    for (int32_t e = 0; e < E; ++e) p[e] = exp(l[e] - mx) / z;
  }
  if (cfg->renormalize) {
    denom = 0.0;
    for (int32_t j = 0; j < k; ++j)
      if (idx[j] >= 0) denom += p[idx[j]];
  }
  for (int32_t j = 0; j < k; ++j)
    w[j] = idx[j] >= 0 ? p[idx[j]] / denom * cfg->routed_scaling_factor : 0.0;
  free(p);
}

/* Exemption: k-th vs (k+1)-th and every adjacent pair of the kept order. */
static int order_exempt(const double* v, const int32_t* order, int32_t count, int32_t k) {
  int ex = 0;
  for (int32_t r = 0; r + 1 < count && r < k; ++r)
    if (near_tie(v[order[r]], v[order[r + 1]])) ex = 1;
  return ex;
}

void oracle_route(const oracle_cfg* cfg, int64_t n, const double* logits, const float* bias,
                  int32_t* topk_idx, double* topk_w, uint8_t* exempt, int32_t* ranking,
                  oracle_stats* stats) {
  const int32_t E = cfg->n_routed, k = cfg->top_k;
  int64_t n_exempt = 0;
#pragma omp parallel for schedule(dynamic, 16) reduction(+ : n_exempt)
  for (int64_t t = 0; t < n; ++t) {
    double* v = (double*)malloc(sizeof(double) * (size_t)E);
    int32_t* rank = (int32_t*)malloc(sizeof(int32_t) * (size_t)E);
    int ex = 0;
    const double* l = logits + t * (int64_t)E;
    int32_t m = token_ranking(cfg, l, bias, v, rank, &ex);
    if (order_exempt(v, rank, m, k)) ex = 1;
    for (int32_t j = 0; j < k; ++j) topk_idx[t * k + j] = j < m ? rank[j] : -1;
    token_gates(cfg, l, topk_idx + t * k, topk_w + t * k);
    if (ranking)
      for (int32_t r = 0; r < E; ++r) ranking[t * (int64_t)E + r] = r < m ? rank[r] : -1;
    if (exempt) exempt[t] = (uint8_t)ex;
    n_exempt += ex;
    free(v);
    free(rank);
  }
  if (stats) {
    stats->overflowed = 0;
    stats->dropped = 0;
    stats->exempt_tokens = n_exempt;
    stats->capacity = 0;
  }
}

int64_t oracle_capacity_value(const oracle_cfg* cfg, int64_t n) {
  if (cfg->capacity > 0) return cfg->capacity;
  return (int64_t)ceil(cfg->capacity_factor * (double)n * (double)cfg->top_k / (double)cfg->n_routed);
}

/*
 * Expert capacity ([1.8T] 2.2): each expert takes at most C slots per batch;
 * when a token's choice is already full, the token is forced to its
 * next-best expert. Tokens are served first come, first served in token
 * order: token t walks its own ranking and takes the first k experts whose
 * count is still below C. Drop policy ([1.8T] 4.2, drop_tokens): the token
 * keeps its top-k and a slot whose expert is full is dropped instead.
 */
void oracle_route_capacity(const oracle_cfg* cfg, int64_t n, const double* logits,
                           const float* bias, int32_t* topk_idx, double* topk_w, uint8_t* exempt,
                           oracle_stats* stats) {
  if (cfg->cap_policy == 0) {
    oracle_route(cfg, n, logits, bias, topk_idx, topk_w, exempt, NULL, stats);
    return;
  }
  const int32_t E = cfg->n_routed, k = cfg->top_k;
  const int64_t C = oracle_capacity_value(cfg, n);
  int32_t* ranking = (int32_t*)malloc(sizeof(int32_t) * (size_t)(n * E));
  uint8_t* group_exempt = (uint8_t*)calloc((size_t)n, 1);
  double* vals = (double*)malloc(sizeof(double) * (size_t)(n * E));
#pragma omp parallel for schedule(dynamic, 16)
  for (int64_t t = 0; t < n; ++t) {
    int ex = 0;
    int32_t m = token_ranking(cfg, logits + t * (int64_t)E, bias, vals + t * (int64_t)E,
                              ranking + t * (int64_t)E, &ex);
    for (int32_t r = m; r < E; ++r) ranking[t * (int64_t)E + r] = -1;
    group_exempt[t] = (uint8_t)ex;
  }
  int64_t* count = (int64_t*)calloc((size_t)E, sizeof(int64_t));
  int64_t overflowed = 0, dropped = 0, n_exempt = 0;
  int32_t* walk = (int32_t*)malloc(sizeof(int32_t) * (size_t)(E + 1));
  for (int64_t t = 0; t < n; ++t) {
    const int32_t* rank = ranking + t * (int64_t)E;
    const double* v = vals + t * (int64_t)E;
    int32_t* idx = topk_idx + t * k;
    int ex = group_exempt[t];
    if (cfg->cap_policy == 1) {
      /* Non-full eligible experts in ranking order; the first k are taken. */
      int32_t avail = 0, taken = 0;
      for (int32_t r = 0; r < E && rank[r] >= 0 && avail <= k; ++r)
        if (count[rank[r]] < C) {
          walk[avail++] = rank[r];
          if (taken < k) {
            idx[taken++] = rank[r];
            if (r >= k) ++overflowed;
          }
        }
      if (order_exempt(v, walk, avail, k)) ex = 1;
      for (int32_t j = taken; j < k; ++j) {
        idx[j] = -1;
        ++dropped;
      }
      for (int32_t j = 0; j < taken; ++j) ++count[idx[j]];
    } else {
      int32_t m = 0;
      while (m < E && rank[m] >= 0) ++m;
      if (order_exempt(v, rank, m, k)) ex = 1;
      for (int32_t j = 0; j < k; ++j) {
        int32_t e = j < m ? rank[j] : -1;
        if (e >= 0 && count[e] < C) {
          idx[j] = e;
          ++count[e];
        } else {
          idx[j] = -1;
          ++dropped;
        }
      }
    }
    token_gates(cfg, logits + t * (int64_t)E, idx, topk_w + t * k);
    if (exempt) exempt[t] = (uint8_t)ex;
    n_exempt += ex;
  }
  if (stats) {
    stats->overflowed = overflowed;
    stats->dropped = dropped;
    stats->exempt_tokens = n_exempt;
    stats->capacity = C;
  }
  free(walk);
  free(count);
  free(vals);
  free(group_exempt);
  free(ranking);
}

/*
 * Hash routing ([DS] section V4: the first layers choose experts by a fixed
 * table indexed by token id; the router only weights the chosen experts).
 * topk_idx[t, j] = tid2eid[token_id[t], j]; gates as token_gates().
 */
void oracle_route_hash(const oracle_cfg* cfg, int64_t n, const double* logits, const int32_t* token_ids,
                       const int32_t* tid2eid, int32_t* topk_idx, double* topk_w) {
  const int32_t E = cfg->n_routed, k = cfg->top_k;
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < n; ++t) {
    for (int32_t j = 0; j < k; ++j) topk_idx[t * k + j] = tid2eid[(int64_t)token_ids[t] * k + j];
    token_gates(cfg, logits + t * (int64_t)E, topk_idx + t * k, topk_w + t * k);
  }
}

/*
 * Auxiliary-loss-free balancing step ([DS] V3: after each step the bias of an
 * over-loaded expert is decreased by gamma and that of an under-loaded one
 * increased by gamma). Load is compared with the mean load sum(counts) / E;
 * an expert exactly at the mean keeps its bias.
 */
void oracle_bias_update(int32_t E, const int32_t* counts, const float* bias, double gamma, double* out) {
  double total = 0.0;
  for (int32_t e = 0; e < E; ++e) total += counts[e];
  const double mean = total / E;
  for (int32_t e = 0; e < E; ++e) {
    double b = (double)bias[e];
    if (counts[e] > mean) b -= gamma;
    else if (counts[e] < mean) b += gamma;
    out[e] = b;
  }
}

/* ---- dispatch: histogram, exclusive scan, stable permutation -------------- */

int64_t oracle_dispatch(int64_t n, int32_t k, int32_t E, const int32_t* topk_idx, int32_t* counts,
                        int32_t* offsets, int32_t* perm_token, int32_t* slot_dest) {
  for (int32_t e = 0; e < E; ++e) counts[e] = 0;
  for (int64_t a = 0; a < n * k; ++a)
    if (topk_idx[a] >= 0) ++counts[topk_idx[a]];
  offsets[0] = 0;
  for (int32_t e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
  int32_t* next = (int32_t*)malloc(sizeof(int32_t) * (size_t)E);
  for (int32_t e = 0; e < E; ++e) next[e] = offsets[e];
  for (int64_t t = 0; t < n; ++t)
    for (int32_t j = 0; j < k; ++j) {
      int32_t e = topk_idx[t * k + j];
      if (e < 0) {
        slot_dest[t * k + j] = -1;
        continue;
      }
      int32_t pos = next[e]++;
      perm_token[pos] = (int32_t)t;
      slot_dest[t * k + j] = pos;
    }
  free(next);
  return offsets[E];
}

/* ---- SwiGLU expert ([DS] ledger: gate, up, down; [KL] SwiGLU) ------------- */

void oracle_swiglu(int32_t d, int32_t I, int64_t m, const double* x, const void* w_gate,
                   const void* w_up, const void* w_down, int32_t w_dt, double* out) {
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t r = 0; r < m; ++r) {
    const double* xr = x + r * (int64_t)d;
    double* h = (double*)malloc(sizeof(double) * (size_t)I);
    for (int32_t i = 0; i < I; ++i) {
      double g = 0.0, u = 0.0;
      for (int32_t j = 0; j < d; ++j) {
        g += xr[j] * elem(w_gate, w_dt, (int64_t)i * d + j);
        u += xr[j] * elem(w_up, w_dt, (int64_t)i * d + j);
      }
      h[i] = g * sigmoid(g) * u;
    }
    for (int32_t c = 0; c < d; ++c) {
      double acc = 0.0;
      for (int32_t i = 0; i < I; ++i) acc += h[i] * elem(w_down, w_dt, (int64_t)c * I + i);
      out[r * (int64_t)d + c] = acc;
    }
    free(h);
  }
}

/* ---- combine ([DS]: y = sum_k w_k expert_k(x) + shared_expert(x)) --------- */

void oracle_combine(int64_t n, int32_t k, int32_t d, const double* eo, const int32_t* slot_dest,
                    const double* topk_w, const double* sh, double* y) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < n; ++t)
    for (int32_t c = 0; c < d; ++c) {
      double acc = 0.0;
      for (int32_t j = 0; j < k; ++j) {
        int32_t pos = slot_dest[t * k + j];
        if (pos >= 0) acc += topk_w[t * k + j] * eo[(int64_t)pos * d + c];
      }
      if (sh) acc += sh[t * (int64_t)d + c];
      y[t * (int64_t)d + c] = acc;
    }
}

/* ---- whole layer ---------------------------------------------------------- */

void oracle_layer(const oracle_cfg* cfg, int64_t n, const void* x, const void* w_r,
                  const float* bias, const void* w_gate, const void* w_up, const void* w_down,
                  const void* ws_gate, const void* ws_up, const void* ws_down, int32_t dt,
                  double* y, int32_t* topk_idx, double* topk_w, int32_t* counts,
                  uint8_t* exempt, oracle_stats* stats) {
  const int32_t d = cfg->d_model, E = cfg->n_routed, k = cfg->top_k, I = cfg->inter;
  const int64_t nk = n * k;
  double* logits = (double*)malloc(sizeof(double) * (size_t)(n * E));
  int32_t* idx = topk_idx ? topk_idx : (int32_t*)malloc(sizeof(int32_t) * (size_t)nk);
  double* w = topk_w ? topk_w : (double*)malloc(sizeof(double) * (size_t)nk);
  int32_t* cnt = counts ? counts : (int32_t*)malloc(sizeof(int32_t) * (size_t)E);
  int32_t* offsets = (int32_t*)malloc(sizeof(int32_t) * (size_t)(E + 1));
  int32_t* perm = (int32_t*)malloc(sizeof(int32_t) * (size_t)(nk > 0 ? nk : 1));
  int32_t* dest = (int32_t*)malloc(sizeof(int32_t) * (size_t)(nk > 0 ? nk : 1));

  oracle_router_logits(n, d, E, x, dt, w_r, dt, logits);
  oracle_route_capacity(cfg, n, logits, bias, idx, w, exempt, stats);
  int64_t kept = oracle_dispatch(n, k, E, idx, cnt, offsets, perm, dest);

  /* Gathered expert inputs, one expert at a time, then the expert outputs. */
  double* eo = (double*)malloc(sizeof(double) * (size_t)((kept > 0 ? kept : 1) * d));
  double* xe = (double*)malloc(sizeof(double) * (size_t)((kept > 0 ? kept : 1) * d));
  for (int64_t p = 0; p < kept; ++p)
    for (int32_t c = 0; c < d; ++c) xe[p * d + c] = elem(x, dt, (int64_t)perm[p] * d + c);
  const int64_t esz = (int64_t)I * d;
  const size_t bytes = dt == 0 ? 4 : 2;
  for (int32_t e = 0; e < E; ++e) {
    int64_t m = offsets[e + 1] - offsets[e];
    if (m == 0) continue;
    oracle_swiglu(d, I, m, xe + (int64_t)offsets[e] * d,
                  (const char*)w_gate + (size_t)(e * esz) * bytes,
                  (const char*)w_up + (size_t)(e * esz) * bytes,
                  (const char*)w_down + (size_t)(e * esz) * bytes, dt,
                  eo + (int64_t)offsets[e] * d);
  }
  double* sh = NULL;
  if (cfg->n_shared > 0 && n > 0) {
    double* xs = (double*)malloc(sizeof(double) * (size_t)(n * d));
    for (int64_t i = 0; i < n * d; ++i) xs[i] = elem(x, dt, i);
    sh = (double*)malloc(sizeof(double) * (size_t)(n * d));
    oracle_swiglu(d, cfg->n_shared * I, n, xs, ws_gate, ws_up, ws_down, dt, sh);
    free(xs);
  }
  oracle_combine(n, k, d, eo, dest, w, sh, y);

  free(sh);
  free(xe);
  free(eo);
  free(dest);
  free(perm);
  free(offsets);
  if (!counts) free(cnt);
  if (!topk_w) free(w);
  if (!topk_idx) free(idx);
  free(logits);
}

/* ---- parameter ledger ([DS] "671B and 37B") ------------------------------- */

void oracle_ds_params(const oracle_ds_arch* a, int64_t* total, int64_t* active) {
  const int64_t d = a->d_model, H = a->n_heads;
  /* MLA: q_a, q_b, kv_a (latent + shared rope part), kv_b, o, two small norms. */
  const int64_t mla = d * a->q_lora_rank + a->q_lora_rank * H * (a->qk_nope_dim + a->qk_rope_dim) +
                      d * (a->kv_lora_rank + a->qk_rope_dim) +
                      a->kv_lora_rank * H * (a->qk_nope_dim + a->v_head_dim) +
                      H * a->v_head_dim * d + a->q_lora_rank + a->kv_lora_rank;
  const int64_t expert = 3 * d * a->moe_inter;  /* gate, up, down */
  const int64_t dense = 3 * d * a->dense_inter;
  const int64_t router = a->n_routed * d;
  const int64_t embed = a->vocab * d;
  const int64_t norms = a->n_layers * 2 * d + d;
  const int64_t moe_layers = a->n_layers - a->first_k_dense;
  *total = a->n_layers * mla + a->first_k_dense * dense +
           moe_layers * (router + (a->n_routed + a->n_shared) * expert) + 2 * embed + norms;
  *active = a->n_layers * mla + a->first_k_dense * dense +
            moe_layers * (router + (a->top_k + a->n_shared) * expert) + 2 * embed + norms;
}

/* ---- FP8 E4M3 codes and UE8M0 block scales ([DS] FP8 section) -------------- */

double oracle_e4m3_value(uint8_t code) {
  const int sign = code >> 7, ex = (code >> 3) & 15, man = code & 7;
  double mag;
  if (ex == 15 && man == 7) return NAN;
  if (ex == 0)
    mag = ldexp((double)man, -9);                  /* subnormal: man/8 * 2^-6   */
  else
    mag = ldexp(1.0 + man / 8.0, ex - 7);          /* normal: 1.man * 2^(ex-7) */
  return sign ? -mag : mag;
}

uint8_t oracle_e4m3_encode(double v) {
  if (isnan(v)) return 0x7F;
  const uint8_t sign = signbit(v) ? 0x80 : 0x00;
  const double a = fabs(v);
  if (a >= 448.0) return sign | 0x7E;
  if (a < ldexp(1.0, -6)) {
    /* subnormal range: multiples of 2^-9; 8 * 2^-9 is the smallest normal, code 0x08 */
    const double q = nearbyint(ldexp(a, 9));       /* round half to even */
    return sign | (uint8_t)q;
  }
  int x;
  const double f = frexp(a, &x);                   /* a = f * 2^x, f in [0.5, 1) */
  int ex = x - 1;                                  /* a = (2f) * 2^ex, 2f in [1, 2) */
  double m = nearbyint((2.0 * f - 1.0) * 8.0);     /* three mantissa bits, half to even */
  if (m == 8.0) {
    m = 0.0;
    ++ex;
  }
  const int field = ex + 7;
  if (field > 15 || (field == 15 && m > 6.0)) return sign | 0x7E;
  return sign | (uint8_t)((field << 3) | (int)m);
}

int32_t oracle_ue8m0_exponent(double amax) {
  if (!(amax > 0.0)) return 0;
  int x;
  const double f = frexp(amax, &x);                /* amax = f * 2^x, f in [0.5, 1) */
  /* amax <= 448 * 2^e  <=>  f * 2^(x - 8 - e) <= 1.75 (448 = 1.75 * 2^8):
   * e = x - 8 always holds; e = x - 9 holds iff f <= 0.875; e = x - 10 never. */
  int32_t e = f <= 0.875 ? x - 9 : x - 8;
  if (e < -127) e = -127;
  if (e > 127) e = 127;
  return e;
}

void oracle_quantize_rows(int64_t rows, int32_t cols, const void* src, int32_t src_dt, uint8_t* codes,
                          uint8_t* scale_byte) {
  const int32_t tiles = cols / 128;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    for (int32_t t = 0; t < tiles; ++t) {
      double amax = 0.0;
      for (int32_t c = 0; c < 128; ++c) {
        const int64_t i = r * cols + t * 128 + c;
        const double v = src_dt == 2 ? ((const double*)src)[i] : elem(src, src_dt, i);
        if (fabs(v) > amax) amax = fabs(v);
      }
      const int32_t e = oracle_ue8m0_exponent(amax);
      scale_byte[r * tiles + t] = (uint8_t)(e + 127);
      for (int32_t c = 0; c < 128; ++c) {
        const int64_t i = r * cols + t * 128 + c;
        const double v = src_dt == 2 ? ((const double*)src)[i] : elem(src, src_dt, i);
        codes[i] = oracle_e4m3_encode(ldexp(v, -e));
      }
    }
  }
}
