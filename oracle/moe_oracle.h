/*
 * moe_oracle.h -- plain, slow, fp64 CPU oracle of the sparse Mixture-of-Experts
 * FFN layer forward pass (router -> dispatch -> per-expert SwiGLU -> shared
 * experts -> gate-weighted combine).
 *
 * TEST INFRASTRUCTURE. Only the tests, the package smoke check and the
 * benchmark's CPU-baseline leg may load or call this code. It shares no code,
 * header or table with the CUDA library and includes none of its files.
 *
 * Sources (page title, then section):
 *   [DS]  "15. DeepSeek: MLA, MoE and MTP", section "V3 MoE: how 8 of 256
 *         experts are chosen" (router listing, sigmoid scores, bias, groups,
 *         gate weights, routed_scaling_factor, shared expert) and section
 *         "671B and 37B parameter ledger" (three matrices per expert).
 *         Section "V2" gives 160 routed + 2 shared experts, top-6, softmax.
 *         Section "V4": sqrtsoftplus scores with the bias and no group limit;
 *         hash routing of the first layers through a token-id table.
 *   [MoE] "MoE architecture revealed", section 3.1 (linear router, softmax,
 *         top-k) and section 4.1 (router logits -> softmax -> topk probs).
 *   [1.8T] "1.8T parameters / 2% per token", section 2.2 (expert capacity:
 *         tokens beyond an expert's capacity are forced to the next-best
 *         expert), section 4.1 (softmax over the top-k logits as gates) and
 *         section 4.2 (capacity config with drop_tokens).
 *   [KL]  "MoE" tag feed, section on activation functions (SwiGLU FFN).
 *
 * Element types: every tensor argument is (pointer, dtype) with dtype 0 =
 * IEEE binary32 and 1 = bf16 stored as its 16 raw bits. Values are widened to
 * binary64 exactly and all arithmetic is binary64.
 */
#ifndef MOE_ORACLE_H_
#define MOE_ORACLE_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct {
  int32_t d_model;       /* d                                                    */
  int32_t n_routed;      /* E                                                    */
  int32_t n_shared;      /* shared experts, concatenated to width n_shared * I   */
  int32_t top_k;         /* k                                                    */
  int32_t n_group;       /* expert groups (1 = no group limit)                   */
  int32_t topk_group;    /* groups kept per token                                */
  int32_t inter;         /* I = moe_intermediate_size                            */
  int32_t score_fn;      /* 0 = softmax, 1 = sigmoid, 2 = sqrtsoftplus (+ bias)  */
  int32_t renormalize;   /* gates normalised over the selected experts           */
  double routed_scaling_factor;
  int32_t cap_policy;    /* 0 = none, 1 = overflow to next-best, 2 = drop        */
  double capacity_factor;
  int32_t capacity;      /* > 0 overrides capacity_factor                        */
} oracle_cfg;

typedef struct {
  int64_t overflowed;    /* slots that went to an expert ranked below the k-th   */
  int64_t dropped;       /* slots left empty (expert index -1)                   */
  int64_t exempt_tokens; /* tokens with a near-tied decision boundary            */
  int64_t capacity;      /* C used (0 when capacity is off)                      */
} oracle_stats;

/* Relative near-tie threshold of the exemption rule. */
#define ORACLE_TIE_REL 1e-6

/* logits[t, e] = sum_i x[t, i] * W_r[e, i]                         ([DS], [MoE] 3.1) */
void oracle_router_logits(int64_t n, int32_t d, int32_t E, const void* x, int32_t x_dt,
                          const void* w_r, int32_t w_dt, double* logits);

/*
 * Routing without capacity, token by token: scores, group limit, top-k, gates.
 * topk_idx[n, k] (slots in descending selection score, ties to the lower
 * expert index), topk_w[n, k], exempt[n] (1 when a decision boundary is a
 * near-tie), ranking[n, E] (optional: eligible experts in selection order,
 * padded with -1). bias may be NULL (= 0).               ([DS] router listing)
 */
void oracle_route(const oracle_cfg* cfg, int64_t n, const double* logits, const float* bias,
                  int32_t* topk_idx, double* topk_w, uint8_t* exempt, int32_t* ranking,
                  oracle_stats* stats);

/*
 * Routing with the expert-capacity rule of [1.8T] 2.2 / 4.2, applied in token
 * order. Without a capacity policy it equals oracle_route.
 */
void oracle_route_capacity(const oracle_cfg* cfg, int64_t n, const double* logits,
                           const float* bias, int32_t* topk_idx, double* topk_w, uint8_t* exempt,
                           oracle_stats* stats);

/* Hash routing: topk_idx[t] = tid2eid[token_ids[t]] ([DS] V4), gates from the scores. */
void oracle_route_hash(const oracle_cfg* cfg, int64_t n, const double* logits, const int32_t* token_ids,
                       const int32_t* tid2eid, int32_t* topk_idx, double* topk_w);

/* Bias update of the auxiliary-loss-free balancing ([DS] V3): out = bias -/+ gamma. */
void oracle_bias_update(int32_t E, const int32_t* counts, const float* bias, double gamma, double* out);

/* Capacity C = capacity if > 0, else ceil(capacity_factor * n * k / E). */
int64_t oracle_capacity_value(const oracle_cfg* cfg, int64_t n);

/*
 * Histogram, exclusive scan and stable (token-ordered) permutation.
 * counts[E], offsets[E + 1], perm_token[total], slot_dest[n * k] (-1 for a
 * dropped slot). Returns the number of kept slots.
 */
int64_t oracle_dispatch(int64_t n, int32_t k, int32_t E, const int32_t* topk_idx, int32_t* counts,
                        int32_t* offsets, int32_t* perm_token, int32_t* slot_dest);

/*
 * SwiGLU expert on m rows: out = (silu(x W_g^T) * (x W_u^T)) W_d^T with
 * W_g, W_u of shape [I, d] and W_d of shape [d, I].     ([DS] ledger, [KL])
 */
void oracle_swiglu(int32_t d, int32_t I, int64_t m, const double* x, const void* w_gate,
                   const void* w_up, const void* w_down, int32_t w_dt, double* out);

/* y[t] = sum_j w[t, j] * eo[slot_dest[t, j]] + sh[t]    ([DS] last line of listing) */
void oracle_combine(int64_t n, int32_t k, int32_t d, const double* eo, const int32_t* slot_dest,
                    const double* topk_w, const double* sh, double* y);

/*
 * Whole layer. Weights: w_gate/w_up [E, I, d], w_down [E, d, I], shared
 * ws_gate/ws_up [n_shared * I, d], ws_down [d, n_shared * I] (NULL when
 * n_shared = 0). y[n, d] in binary64; topk_idx/topk_w/counts optional.
 */
void oracle_layer(const oracle_cfg* cfg, int64_t n, const void* x, const void* w_r,
                  const float* bias, const void* w_gate, const void* w_up, const void* w_down,
                  const void* ws_gate, const void* ws_up, const void* ws_down, int32_t dt,
                  double* y, int32_t* topk_idx, double* topk_w, int32_t* counts,
                  uint8_t* exempt, oracle_stats* stats);

/*
 * FP8 experts ([DS] section "FP8 training is a recipe, not the architecture"):
 * matrix inputs in E4M3, one scale per 1 x 128 tile of activations and per
 * 128 x 128 block of weights; V3.1 stores the scales as UE8M0 (an 8-bit
 * exponent: scale = 2^(byte - 127)).
 *
 * E4M3: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits, no infinities,
 * S.1111.111 is NaN, largest finite magnitude 448, subnormals m/8 * 2^-6.
 */
double oracle_e4m3_value(uint8_t code);
/* Nearest E4M3 value, ties to the even mantissa; |v| > 448 saturates to +-448. */
uint8_t oracle_e4m3_encode(double v);
/* UE8M0 scale of a block whose largest magnitude is amax: the smallest power of
 * two 2^e with amax <= 448 * 2^e (e = 0 when amax = 0). Returns e. */
int32_t oracle_ue8m0_exponent(double amax);
/* Rows of `cols` values (cols a multiple of 128) quantised in 1 x 128 tiles:
 * scale_byte[r, t] = e + 127 for tile t, codes[r, c] = encode(v * 2^-e).
 * src dtype: 0 = binary32, 1 = bf16 bits, 2 = binary64. */
void oracle_quantize_rows(int64_t rows, int32_t cols, const void* src, int32_t src_dt, uint8_t* codes,
                          uint8_t* scale_byte);

/* DeepSeek-style architecture fields for the parameter ledger of [DS]. */
typedef struct {
  int64_t n_layers, d_model, q_lora_rank, kv_lora_rank, n_heads, qk_nope_dim, qk_rope_dim,
      v_head_dim, vocab, first_k_dense, dense_inter, n_routed, n_shared, top_k, moe_inter;
} oracle_ds_arch;

/* Total and per-token active parameters, summed as in [DS] "671B and 37B". */
void oracle_ds_params(const oracle_ds_arch* a, int64_t* total, int64_t* active);

#ifdef __cplusplus
}
#endif

#endif /* MOE_ORACLE_H_ */
