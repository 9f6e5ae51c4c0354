/*
 * moe.h -- C ABI of the B200 (sm_100a) sparse Mixture-of-Experts FFN layer,
 * forward pass: router -> dispatch -> per-expert SwiGLU -> shared experts ->
 * gate-weighted combine.
 *
 * Where each operation is defined (page title, then section):
 *   [DS]   "15. DeepSeek: MLA, MoE and MTP" -- section "V3 MoE: how 8 of 256
 *          experts are chosen": x @ W^T with W [E, d]; sigmoid scores; bias
 *          (e_score_correction_bias) added for selection only; E experts viewed
 *          as n_group groups, a group scored by the sum of its two best biased
 *          scores, topk_group groups kept, the rest masked; top-k; gates taken
 *          from the raw scores, divided by their sum and multiplied by
 *          routed_scaling_factor; y = sum_k w_k expert_k(x) + shared_expert(x).
 *          Section "V2": softmax scoring, 160 routed + 2 shared experts, top-6.
 *          Section "671B and 37B": an expert is three matrices gate, up, down.
 *   [MoE]  "MoE architecture revealed", section 3.1: a linear router maps x to
 *          E logits, softmax turns them into probabilities, the top-k experts
 *          are chosen; section 4.1: top-k of the probabilities as gates.
 *   [1.8T] "1.8T parameters / 2% per token", section 2.2: each expert has a
 *          capacity per batch and tokens beyond it are forced to the
 *          next-best expert; section 4.1: gates as the softmax of the top-k
 *          logits (renormalised); section 4.2: capacity_factor and
 *          drop_tokens.
 *   [KL]   "MoE" tag feed, section on activation functions: SwiGLU FFN.
 *   [DS4]  "15. DeepSeek: MLA, MoE and MTP", section "V4": scores are
 *          sqrt(softplus(l)) with the selection bias and no group limit; the
 *          first layers choose experts by a fixed token-id table (tid2eid) and
 *          the router only weights them.
 *
 * Conventions for every entry point:
 *   - Pointers named x, w_*, y, topk_*, offsets, perm_token, slot_dest,
 *     x_perm, expert_out, expert_counts, diag and ws are DEVICE pointers
 *     (one GPU); cfg, the moe_weights struct itself and bytes are HOST
 *     pointers. The caller owns all memory; the library allocates no device
 *     memory and keeps no data between calls. Scratch space comes only from
 *     the workspace ws of at least moe_workspace_size() bytes. The one
 *     runtime resource it keeps is, per device, a non-blocking stream and two
 *     events created on the first moe_layer_forward with shared experts: the
 *     shared experts run there, joined back to `stream` before the combine.
 *   - Arrays are dense row-major. Weights use the out x in (nn.Linear)
 *     convention: W_r [E, d]; w_gate, w_up [E, I, d]; w_down [E, d, I];
 *     shared experts concatenated along I: ws_gate, ws_up [n_shared*I, d],
 *     ws_down [d, n_shared*I]. Activations and weights share cfg->dtype
 *     (MOE_F32 or MOE_BF16); gates are binary32; indices are int32.
 *   - MOE_FP8 ([DS] FP8 section: E4M3 matrix inputs, one scale per 1 x 128
 *     activation tile and per 128 x 128 weight block, scales stored as UE8M0):
 *     x, y, x_perm, expert_out and w_router are bf16; every expert matrix
 *     (w_gate, w_up, w_down, ws_*) holds E4M3 codes (one byte per element) with
 *     its UE8M0 scale bytes (scale = 2^(byte - 127)) in the matching *_scale
 *     array, [E, ceil(rows/128), cols/128] (shared: [ceil(rows/128), cols/128]).
 *     Activations entering an expert matrix (x, and h between gate/up and
 *     down) are quantised to E4M3 in 1 x 128 tiles by the library:
 *     e = the smallest integer with max|tile| <= 448 * 2^e, code = E4M3 of
 *     v * 2^-e, round to nearest even. d and I must be multiples of 128.
 *   - Every device pointer must be 16-byte aligned; ws must be 256-byte
 *     aligned.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream). Results are deterministic run to run (fixed reduction
 *     orders, no floating-point atomics).
 *   - Argument and shape errors are returned synchronously before anything
 *     is enqueued. A failed launch returns MOE_ERR_CUDA. Errors that only the
 *     device can see (a bounded wait that ran out, an internal check) are
 *     written to the status word in the workspace and are returned by
 *     moe_sync_status(). n = 0 is a valid no-op.
 *   - Expert order and tie rule: output slots are ordered by descending
 *     selection score (logit for softmax, score + bias for sigmoid); equal
 *     scores go to the lower expert index, equal group scores to the lower
 *     group index. Dropped slots carry index -1, weight 0 and slot_dest -1.
 *   - Environment variables, read at each call (none is needed):
 *     MOE_TC_MODE=1sm|2sm forces the one-SM or SM-pair bf16 expert GEMM;
 *     MOE_TC_WIDE=1|gate|0 gives the SM-pair bf16 GEMMs (all, the gate/up one
 *     only, or none) 256 x 512 tiles instead of 256 x 256; unset, the gate/up
 *     GEMM takes them when its groups average at most 768 rows, and both GEMMs
 *     of one group (the shared experts) do;
 *     MOE_CAP_MODE=1cta runs the capacity rule on one CTA instead of the
 *     cooperative grid;
 *     MOE_FP8_BN=128|256|pair|s128|s256 forces an FP8 expert GEMM tile shape
 *     (one-SM 128-row tiles of that width, SM-pair tiles, or 32-row tiles where
 *     the rows per expert allow them); these exist for tuning and tests, and
 *     results are identical up to floating-point summation order.
 *     MOE_EP_TIMEOUT_MS bounds the expert-parallel barrier wait (see below).
 *     MOE_TEST_STALL=1 withholds one pipeline stage of the bf16 expert GEMM so
 *     that its bounded wait runs out and MOE_ERR_TIMEOUT is reported (a test of
 *     the failure path; never set it otherwise).
 *     MOE_TEST_NO_TENSOR_MAPS=1 makes the bf16 tensor-core GEMMs report every
 *     shape as unsupported (a test of that path; never set it otherwise).
 *   - bf16 matrix products run on the tcgen05 tensor cores only: a shape or
 *     pointer alignment they cannot take (or a missing tensor-map entry point
 *     in the driver) is MOE_ERR_UNSUPPORTED, never a slower fallback. binary32
 *     layers run on the CUDA cores (FFMA), the precision their tolerance needs.
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
typedef struct CUstream_st* moe_stream_t; /* same object as cudaStream_t */

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size or field     */
  MOE_ERR_UNSUPPORTED = 2, /* valid but outside what the kernels handle      */
  MOE_ERR_WORKSPACE = 3,   /* ws_bytes below moe_workspace_size()            */
  MOE_ERR_CUDA = 4,        /* a CUDA runtime call or launch failed           */
  MOE_ERR_TIMEOUT = 5,     /* a bounded device wait gave up                  */
  MOE_ERR_INTERNAL = 6     /* a device-side consistency check failed         */
} moe_status;

typedef enum { MOE_SCORE_SOFTMAX = 0, MOE_SCORE_SIGMOID = 1, MOE_SCORE_SQRTSOFTPLUS = 2 } moe_score_fn;
typedef enum { MOE_CAP_NONE = 0, MOE_CAP_OVERFLOW_NEXT = 1, MOE_CAP_DROP = 2 } moe_cap_policy;
typedef enum { MOE_F32 = 0, MOE_BF16 = 1, MOE_FP8 = 2 } moe_dtype;

/* Layer configuration, in the field names of [DS] and [1.8T] 4.2. */
typedef struct {
  int32_t d_model;               /* d                                              */
  int32_t n_routed;              /* E, 1..256                                      */
  int32_t n_shared;              /* shared experts (0 = none)                      */
  int32_t top_k;                 /* k, 1..min(E, 32)                               */
  int32_t n_group;               /* expert groups; 1 = no group limit              */
  int32_t topk_group;            /* groups kept per token                          */
  int32_t moe_intermediate_size; /* I                                              */
  int32_t score_fn;              /* moe_score_fn; SIGMOID and SQRTSOFTPLUS add bias */
  int32_t renormalize;           /* 1: gates normalised over the kept slots        */
  float routed_scaling_factor;   /* multiplies every gate ([DS]: 2.5 for V3)       */
  int32_t cap_policy;            /* moe_cap_policy                                 */
  float capacity_factor;         /* C = ceil(capacity_factor * n * k / E)          */
  int32_t capacity;              /* > 0 overrides capacity_factor                  */
  int32_t dtype;                 /* moe_dtype of activations and weights           */
} moe_config;

/* Caller-owned device weights. bias may be NULL (= 0); ws_* NULL when n_shared = 0. */
typedef struct {
  const void* w_router; /* [E, d]                */
  const void* w_gate;   /* [E, I, d]             */
  const void* w_up;     /* [E, I, d]             */
  const void* w_down;   /* [E, d, I]             */
  const void* ws_gate;  /* [n_shared*I, d]       */
  const void* ws_up;    /* [n_shared*I, d]       */
  const void* ws_down;  /* [d, n_shared*I]       */
  const float* bias;    /* [E] selection bias    */
  /* MOE_FP8 only: UE8M0 block-scale bytes of the expert matrices (NULL otherwise). */
  const uint8_t* w_gate_scale;   /* [E, ceil(I/128), d/128]  */
  const uint8_t* w_up_scale;     /* [E, ceil(I/128), d/128]  */
  const uint8_t* w_down_scale;   /* [E, d/128, I/128]        */
  const uint8_t* ws_gate_scale;  /* [ceil(I_s/128), d/128]   */
  const uint8_t* ws_up_scale;    /* [ceil(I_s/128), d/128]   */
  const uint8_t* ws_down_scale;  /* [d/128, I_s/128]         */
} moe_weights;

/* Device-resident diagnostics written by moe_route / moe_layer_forward. */
typedef struct {
  int32_t overflowed;     /* slots sent to an expert ranked below the k-th       */
  int32_t dropped;        /* slots left empty                                     */
  int32_t refined_tokens; /* tokens whose decision was re-taken in binary64       */
  int32_t max_load;       /* largest per-expert slot count                        */
  int32_t refined_logits; /* router logits recomputed in binary64 (all tokens)    */
  int32_t status;         /* moe_status seen on the device                        */
  int32_t reserved[2];
} moe_diag;

/*
 * Workspace bytes needed by any entry point for this cfg and token count n.
 * Returns MOE_ERR_INVALID_ARG / MOE_ERR_UNSUPPORTED for a bad cfg.
 */
moe_status moe_workspace_size(const moe_config* cfg, int64_t n, size_t* bytes);

/*
 * Router ([DS] router; [MoE] 3.1; capacity: [1.8T] 2.2, 4.2).
 *   in : x [n, d]; weights->w_router, weights->bias.
 *   out: topk_idx [n, k] int32, topk_w [n, k] float, expert_counts [E] int32
 *        (slots per expert after capacity; may be NULL), diag (may be NULL).
 * Logits are accumulated in binary32 on tensor cores; a token whose decision
 * (group cut, k-th/(k+1)-th expert, order of the kept experts, and under a
 * capacity every rank cut) is closer than the binary32 error bound is
 * re-decided from binary64 logits, so indices equal the binary64 definition.
 */
moe_status moe_route(const moe_config* cfg, int64_t n, const void* x, const moe_weights* weights,
                     int32_t* topk_idx, float* topk_w, int32_t* expert_counts, moe_diag* diag,
                     void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * Dispatch: per-expert histogram, exclusive scan and stable permutation
 * (token order within an expert), plus the row copy x_perm[slot_dest[t, j]] = x[t]
 * (each token row read once and written to its kept slots).
 *   in : x [n, d], topk_idx [n, k] (-1 = dropped).
 *   out: offsets [E + 1] (offsets[E] = kept slots), perm_token [n * k]
 *        (first offsets[E] entries valid: source token of each permuted row),
 *        slot_dest [n, k] (permuted row of each slot, -1 if dropped),
 *        x_perm [n * k, d] (first offsets[E] rows valid).
 */
moe_status moe_permute(const moe_config* cfg, int64_t n, const void* x, const int32_t* topk_idx,
                       int32_t* offsets, int32_t* perm_token, int32_t* slot_dest, void* x_perm,
                       void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * Routed experts ([DS] three matrices; [KL] SwiGLU): for every expert e and
 * every permuted row r in [offsets[e], offsets[e+1]):
 *   expert_out[r] = (silu(x_perm[r] W_gate[e]^T) * (x_perm[r] W_up[e]^T)) W_down[e]^T
 * with silu(z) = z * sigmoid(z), binary32 accumulation, the intermediate
 * rounded to cfg->dtype. n bounds the rows: offsets[E] <= n * k.
 */
moe_status moe_expert_ffn(const moe_config* cfg, int64_t n, const void* x_perm, const int32_t* offsets,
                          const moe_weights* weights, void* expert_out, void* ws, size_t ws_bytes,
                          moe_stream_t stream);

/*
 * Combine ([DS] last line of the router listing):
 *   y[t] = sum_{j<k, slot kept} topk_w[t, j] * expert_out[slot_dest[t, j]] + shared(x[t])
 * summed in binary32 in slot order, the shared experts' SwiGLU (computed here
 * from x and weights->ws_*) added last with weight 1. y [n, d].
 */
moe_status moe_combine(const moe_config* cfg, int64_t n, const void* expert_out, const int32_t* slot_dest,
                       const float* topk_w, const void* x, const moe_weights* weights, void* y, void* ws,
                       size_t ws_bytes, moe_stream_t stream);

/*
 * Whole layer: moe_route -> moe_permute -> moe_expert_ffn -> moe_combine with
 * all intermediates in the workspace. y [n, d]. topk_idx_opt, topk_w_opt,
 * counts_opt and diag_opt may be NULL; when given they receive the routing.
 */
moe_status moe_layer_forward(const moe_config* cfg, int64_t n, const void* x, const moe_weights* weights,
                             void* y, int32_t* topk_idx_opt, float* topk_w_opt, int32_t* counts_opt,
                             moe_diag* diag_opt, void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * E4M3 quantisation of bf16 rows in 1 x 128 tiles, the activation format of
 * the MOE_FP8 experts ([DS] FP8 section): for row r and tile t,
 * e = the smallest integer with max|x[r, 128t .. 128t+127]| <= 448 * 2^e
 * (0 for an all-zero tile), scale_bytes[r, t] = e + 127 (UE8M0) and
 * codes[r, c] = E4M3 of x[r, c] * 2^-e, round to nearest even.
 *   in : x [rows, cols] bf16 (device), cols a multiple of 128.
 *   out: codes [rows, cols] and scale_bytes [rows, cols / 128] (device bytes).
 * No workspace; MOE_ERR_INVALID_ARG for bad pointers or shapes.
 */
moe_status moe_quantize_fp8(const void* x, int64_t rows, int32_t cols, uint8_t* codes, uint8_t* scale_bytes,
                            moe_stream_t stream);

/*
 * Hash routing ([DS4]): the experts of token t are row token_ids[t] of the
 * fixed table tid2eid (device int32 [vocab, k], row-major); the gates come
 * from the router scores of those experts exactly as in moe_route (score_fn,
 * renormalize, routed_scaling_factor; cap_policy must be MOE_CAP_NONE).
 *   in : x [n, d], token_ids [n] (device int32), tid2eid, vocab, weights->w_router.
 *   out: topk_idx [n, k] in table order, topk_w [n, k], expert_counts [E]
 *        (may be NULL), diag (may be NULL).
 * A token id outside [0, vocab) or a table entry outside [0, E) leaves that
 * slot empty (-1, weight 0) and sets MOE_ERR_INVALID_ARG in the status word
 * (moe_sync_status).
 */
moe_status moe_route_hash(const moe_config* cfg, int64_t n, const void* x, const int32_t* token_ids,
                          const int32_t* tid2eid, int32_t vocab, const moe_weights* weights, int32_t* topk_idx,
                          float* topk_w, int32_t* expert_counts, moe_diag* diag, void* ws, size_t ws_bytes,
                          moe_stream_t stream);

/*
 * One step of the auxiliary-loss-free balancing ([DS] V3): with counts the
 * per-expert slot counts of a batch (device int32 [E], e.g. expert_counts of
 * moe_route) and mean = sum(counts) / E, bias[e] (device float [E], updated in
 * place) is decreased by gamma where counts[e] > mean, increased by gamma where
 * counts[e] < mean, and kept where equal. Computed in binary64, stored binary32.
 */
moe_status moe_bias_update(const moe_config* cfg, const int32_t* counts, float* bias, float gamma,
                           moe_stream_t stream);

/*
 * Bytes of the device array behind moe_route_static_scratch (8 MiB).
 */
#define MOE_STATIC_SCRATCH_BYTES (8u << 20)

/*
 * moe_route for callers that cannot allocate device memory. The pages have no
 * counterpart to this entry point; it exists for deployment. Some callers only
 * ever receive their input and output buffers: a plug-in running inside a
 * serving engine whose memory planner owns every device allocation, or code on
 * a latency-critical path where a cudaMalloc would synchronise the device. They
 * cannot provide a workspace, so this variant keeps the router's scratch (the
 * binary32 logits, the capacity ranking, per-block counts, the count scan and
 * the status word) in one array of MOE_STATIC_SCRATCH_BYTES in device memory
 * that is part of this library. It calls no cudaMalloc, cudaFree or
 * allocating routine. The array lives in the library's device code, which the
 * CUDA runtime loads on a device when it is first needed there (lazy module
 * loading): the first call on each device loads it and reserves its 8 MiB on
 * that device, which then holds it until the process exits; later calls
 * reserve nothing.
 *   Arguments and outputs are those of moe_route, without ws/ws_bytes; diag
 *   is required here (see below). `stream` must belong to the current device.
 *   Returns MOE_ERR_WORKSPACE when this cfg and n need more scratch than the
 *   array holds (E * 4 bytes of logits per token dominate, plus E * 2 bytes of
 *   ranking under a capacity, or about 0.5 KB for the queue of tokens re-decided
 *   in binary64 when bf16 batches of n >= 2048 route without a capacity; e.g.
 *   E = 256 fits about 5400 tokens, E = 8 about 200000),
 *   MOE_ERR_INVALID_ARG for a NULL diag or a stream of another device,
 *   MOE_ERR_CUDA if the array's device address cannot be found, and the errors
 *   of moe_route otherwise.
 *   The first call on each device performs a one-time set-up that looks up the
 *   array's device address with that device current; make this first call
 *   before any stream capture begins.
 *   All calls on a device share the one array and it keeps the contents of the
 *   last call (everything that must start at zero is cleared by each call).
 *   Calls that overlap on the GPU, e.g. on two streams at once, race on it and
 *   produce undefined results; order them on one stream. The status word that
 *   moe_sync_status reads lives in the array, so that call does not apply here:
 *   the call copies its device status word (a moe_status value, 0 = MOE_OK)
 *   into diag->status on `stream`.
 */
moe_status moe_route_static_scratch(const moe_config* cfg, int64_t n, const void* x, const moe_weights* weights,
                                    int32_t* topk_idx, float* topk_w, int32_t* expert_counts, moe_diag* diag,
                                    moe_stream_t stream);

/*
 * ---- Expert parallelism -----------------------------------------------------
 * [DS] section "V3 MoE: how 8 of 256 experts are chosen" places one expert
 * group per node and limits each token to topk_group of them; [MoE] 4.2
 * spreads the experts evenly over the GPUs with the routing decision known to
 * every GPU. Here R ranks (one GPU each) share a layer: rank q owns the routed
 * experts [q E/R, (q+1) E/R) and holds only their matrices; every rank holds
 * the router, the bias and the shared experts, and routes its own tokens.
 * One layer step per rank:
 *   1. route its n tokens; write its per-expert slot counts into row `rank` of
 *      every rank's count table;
 *   2. push every kept slot's token row into the owner's receive buffer;
 *   3. run the owned experts over the rows it received;
 *   4. y[t] = sum_j topk_w[t, j] * (owner's output row of slot j) + shared(x[t]),
 *      pulling the rows from the owners' output buffers, binary32 in slot order
 *      then the shared experts, as in moe_combine.
 * A flag barrier separates the steps (and ends the call), so the buffers may
 * be reused by the next call. Receive layout at owner q: its experts in order,
 * inside an expert the source ranks in order, inside a source its tokens in
 * order. With the ranks' batches concatenated in rank order this is the
 * stable permutation of moe_permute restricted to q's experts, so a layer
 * split over R ranks computes what moe_layer_forward computes on the
 * concatenated batch. cfg->cap_policy must be MOE_CAP_NONE (a capacity is a
 * property of one batch in one token order) and E must be a multiple of R.
 */
#define MOE_EP_MAX_RANKS 8

/*
 * The exchange buffers of a group of `world` ranks as seen from the calling
 * device: entry q is rank q's buffer (device memory of the calling GPU for
 * q = the caller's rank, a peer mapping -- moe_ep_open_handle -- otherwise).
 * Every rank allocates the same buffers:
 *   recv_x[q], recv_out[q]: [recv_rows, d] activations (cfg->dtype; bf16 for
 *     MOE_FP8), the rows owner q receives and its experts' outputs;
 *   counts[q]: [world, E] int32 count table;
 *   flags[q]:  [world + 1] uint32 barrier words, zeroed once before the first
 *     call and then left to the library.
 * recv_rows bounds the rows an owner receives: the sum over ranks of
 * n_r * min(k, E / world) can never be exceeded. More rows than that set
 * MOE_ERR_WORKSPACE in the status word and the excess slots are skipped.
 */
typedef struct {
  int32_t world;
  int32_t reserved;
  int64_t recv_rows;
  void* recv_x[MOE_EP_MAX_RANKS];
  void* recv_out[MOE_EP_MAX_RANKS];
  int32_t* counts[MOE_EP_MAX_RANKS];
  uint32_t* flags[MOE_EP_MAX_RANKS];
} moe_ep_group;

/*
 * One rank's inputs and outputs. x [n, d], y [n, d] device; weights (host
 * struct): w_router [E, d] and bias [E] of the whole layer, w_gate/w_up/w_down
 * (and their FP8 scales) holding only this rank's E / world experts in order,
 * ws_* the shared experts. topk_idx_opt [n, k] and topk_w_opt [n, k] may be
 * NULL. ws: at least moe_ep_workspace_size() bytes, 256-byte aligned; its
 * status word (moe_sync_status) reports this rank's device errors.
 */
typedef struct {
  int64_t n;
  const void* x;
  const moe_weights* weights;
  void* y;
  int32_t* topk_idx_opt;
  float* topk_w_opt;
  void* ws;
  size_t ws_bytes;
} moe_ep_rank;

/* Workspace bytes of one rank with n tokens in a group of `world` ranks. */
moe_status moe_ep_workspace_size(const moe_config* cfg, int32_t world, int64_t n, int64_t recv_rows, size_t* bytes);

/*
 * One MoE layer step of ranks [first_rank, first_rank + num_ranks) of the
 * group, ranks[i] describing rank first_rank + i, all on `stream`.
 *   num_ranks == 1: the call of one process driving one rank; the steps are
 *     separated by the flag barrier, whose wait is bounded (MOE_EP_TIMEOUT_MS
 *     in the environment, default 5000 ms): past it the rank records
 *     MOE_ERR_TIMEOUT in its status word and does not wait at later barriers
 *     of the call. Every rank of the group must make the call.
 *   num_ranks == world: one process drives every rank on one device (all
 *     buffers local); the steps of all ranks run in stream order, no barrier.
 * Returns MOE_ERR_INVALID_ARG for a bad group, rank range or buffer,
 * MOE_ERR_UNSUPPORTED for a capacity policy or world > MOE_EP_MAX_RANKS.
 */
moe_status moe_ep_layer_forward(const moe_config* cfg, const moe_ep_group* group, int32_t first_rank,
                                int32_t num_ranks, const moe_ep_rank* ranks, moe_stream_t stream);

/*
 * Peer mappings for moe_ep_group: an opaque 72-byte record of a device
 * allocation (a CUDA IPC handle of the allocation holding ptr, and ptr's
 * offset inside it), made by the process owning it and opened by the others
 * (one per GPU of the same node, peer access between the GPUs). open returns
 * the address of the same byte in the calling process; close releases a
 * mapping made by open (pass the address open returned).
 */
#define MOE_EP_HANDLE_BYTES 72
moe_status moe_ep_export_handle(const void* ptr, void* handle);
moe_status moe_ep_open_handle(const void* handle, void** ptr);
moe_status moe_ep_close_handle(void* ptr);

/*
 * Synchronises `stream`, then returns the device status word kept in the
 * workspace (MOE_OK, MOE_ERR_TIMEOUT or MOE_ERR_INTERNAL) and clears it. Every
 * entry point clears the word when it starts, so it reports the most recent
 * call made on this workspace.
 */
moe_status moe_sync_status(void* ws, moe_stream_t stream);

/* Static text for a status code. */
const char* moe_status_string(moe_status status);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H_ */
