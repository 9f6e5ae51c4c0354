// api.cu -- the C ABI entry points declared in moe.h: argument checks,
// workspace carving and the launch sequence of each stage on the caller's
// stream. No allocation, no host synchronisation (except moe_sync_status).
#include <cuda.h>
#include <math.h>
#include <stddef.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Workspace layout; every region starts on a 256-byte boundary.
struct Plan {
  size_t diag, logits, rq, rc, ranking, capg, blk, idx, w, counts, offsets, perm, dest, xperm, h, eo, shh, sh, shoff, sched;
  size_t xq, sfx, hq, sfh, xsq, sfxs, hsq, sfhs;  // FP8 experts: E4M3 activations and their scale blocks
  size_t sfb, sfbs;  // FP8 SM-pair GEMMs: B scale blocks (routed, shared experts)
  size_t ep_off;  // expert parallelism: receive offsets of the rank's own experts
  size_t total;
  bool batched;   // the two-kernel router queues its undecided tokens for launch_refine (rq, rc reserved)
};

// 512-byte scale blocks of the FP8 activations entering a matrix with k columns: one per row tile
// and four 128-wide k blocks.
int64_t fp8_sf_blocks(int64_t rows, int32_t G, int64_t k) { return fp8_sf_tiles_bound(rows, G) * ceil_div(k / 128, 4); }

// Element type of the activations (x, y, x_perm, expert_out) and of the router
// weight: bf16 for the FP8 experts, whose matrices alone are E4M3.
int act_dtype(const moe_config& c) { return c.dtype == MOE_FP8 ? MOE_BF16 : c.dtype; }

// Row stride of the binary32 logits: E rounded up to four floats, so that every row
// starts on a 16-byte boundary for the tensor-core GEMM's vector stores.
int64_t logits_ld(const moe_config& c) { return align_up(c.n_routed, 4); }

// Split-K factor of the router GEMM: small token counts leave most SMs idle
// (one 128-row tile per 128 tokens), so the k range is split and the route
// kernel sums the partial logits in a fixed order. Capped at 4 MiB of partials
// and at 32 splits: every logit's sum is a chain through all of them.
int router_splits(const moe_config& c, int64_t n) {
  if (act_dtype(c) != MOE_BF16 || n <= 0) return 1;
  const int64_t tiles = ceil_div(n, 128) * ceil_div(c.n_routed, 256);
  if (tiles >= 74) return 1;
  const int64_t num_kb = ceil_div(c.d_model, 64);
  int64_t s = 148 / tiles;
  const int64_t cap = ((int64_t)4 << 20) / (n * logits_ld(c) * 4);
  if (s > cap) s = cap;
  if (s > 32) s = 32;
  if (s > num_kb) s = num_kb;
  if (s < 1) s = 1;
  const int64_t kb_per = ceil_div(num_kb, s);
  return (int)ceil_div(num_kb, kb_per);
}

// Batches from this many tokens route in one pass (route_tc.cu) when the configuration allows;
// smaller ones keep the split-K logits GEMM, which spreads a few token tiles over every SM.
constexpr int64_t kOnePassMinTokens = 2048;

// Whether the one-pass router may take this configuration (its kernel checks the rest).
bool one_pass_possible(const moe_config& c, int64_t n) {
  return act_dtype(c) == MOE_BF16 && c.cap_policy == MOE_CAP_NONE && n >= kOnePassMinTokens && c.top_k <= 8;
}

// Whether undecided tokens are refined in one batch (launch_refine over a queue) rather than one
// warp at a time: bf16 rows of a whole number of 16-byte chunks.
bool batched_refine_possible(const moe_config& c) { return act_dtype(c) == MOE_BF16 && c.d_model % 8 == 0; }

// The candidate region of n queued tokens: 16 bytes of counters, the candidate table
// [n][kRouteCandMax + 1] int32, their binary64 logits (same shape, 16-byte aligned whatever n),
// then the pair list [n * kRouteCandMax] int32.
size_t cand_val_offset(int64_t n) { return (size_t)align_up(16 + n * (kRouteCandMax + 1) * 4, 16); }
size_t pairs_offset(int64_t n) { return cand_val_offset(n) + (size_t)n * (kRouteCandMax + 1) * 8; }
size_t cand_region_bytes(int64_t n) { return pairs_offset(n) + (size_t)n * kRouteCandMax * 4; }

// ep_world > 0: the layout of one expert-parallel rank. The routed experts run over the
// ep_recv_rows rows of the group's receive buffer in E / ep_world groups, so h and the FP8
// activations are sized for those; the permuted rows and expert outputs live in the group's
// buffers, not here.
// batched: reserve the token queue for the two-kernel router too (the router-only scratch layout
// leaves it out and refines those tokens warp by warp).
Plan make_plan(const moe_config& c, int64_t n, int32_t ep_world = 0, int64_t ep_recv_rows = 0, bool batched = true) {
  const size_t b = act_dtype(c) == MOE_BF16 ? 2 : 4;
  const int64_t nk = n * c.top_k;
  const bool ep = ep_world > 0;
  const int64_t fr = ep ? ep_recv_rows : nk;             // rows through the routed experts
  const int32_t fg = ep ? c.n_routed / ep_world : c.n_routed;  // their groups
  const int64_t Is = (int64_t)c.n_shared * c.moe_intermediate_size;
  Plan p{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off += (size_t)align_up((int64_t)(bytes > 0 ? bytes : 1), 256);
    return at;
  };
  p.diag = take(sizeof(moe_diag));
  p.logits = take((size_t)router_splits(c, n) * n * logits_ld(c) * 4);
  // the queue of tokens left to the binary64 router (one-pass router, or the first pass of the
  // two-kernel router), and their candidate experts: four counters, the candidate table, its
  // binary64 logits, the list of pairs to refine
  p.batched = batched && batched_refine_possible(c);
  const bool queued = one_pass_possible(c, n) || p.batched;
  p.rq = take(queued ? (size_t)2 * n * 4 : 0);  // the one-pass router's queue, then the refinement queue
  p.rc = take(queued ? cand_region_bytes(n) : 0);
  p.ranking = take(c.cap_policy != MOE_CAP_NONE ? (size_t)n * c.n_routed * 2 : 0);
  p.capg = take(c.cap_policy != MOE_CAP_NONE ? (size_t)capacity_grid_scratch_bytes(n, c.n_routed) : 0);
  p.blk = take((size_t)dispatch_blocks(n, c.top_k) * c.n_routed * 4);
  p.idx = take((size_t)nk * 4);
  p.w = take((size_t)nk * 4);
  p.counts = take((size_t)c.n_routed * 4);
  p.offsets = take((size_t)(c.n_routed + 1) * 4);
  p.perm = take((size_t)nk * 4);
  p.dest = take((size_t)nk * 4);
  p.xperm = take(ep ? 0 : (size_t)nk * c.d_model * b);
  p.h = take((size_t)fr * c.moe_intermediate_size * b);
  p.eo = take(ep ? 0 : (size_t)nk * c.d_model * b);
  p.shh = take((size_t)(Is > 0 ? n * Is : 0) * b);
  p.sh = take((size_t)(Is > 0 ? n * c.d_model : 0) * b);
  p.shoff = take(2 * 4);
  p.sched = take(4 * 4);  // tile counters of the SM-pair GEMM launches (routed GEMM1/2, shared GEMM1/2)
  const bool fp8 = c.dtype == MOE_FP8;
  const int64_t I = c.moe_intermediate_size, d = c.d_model;
  p.xq = take(fp8 ? (size_t)fr * d : 0);
  // scale blocks: 512 bytes per row tile and four 128-wide k blocks
  auto sf_bytes = [](int64_t rows, int32_t G, int64_t k) { return (size_t)fp8_sf_blocks(rows, G, k) * 512; };
  p.sfx = take(fp8 ? sf_bytes(fr, fg, d) : 0);
  p.hq = take(fp8 ? (size_t)fr * I : 0);
  p.sfh = take(fp8 ? sf_bytes(fr, fg, I) : 0);
  p.xsq = take(fp8 && Is > 0 ? (size_t)n * d : 0);
  p.sfxs = take(fp8 && Is > 0 ? sf_bytes(n, 1, d) : 0);
  p.hsq = take(fp8 && Is > 0 ? (size_t)n * Is : 0);
  p.sfhs = take(fp8 && Is > 0 ? sf_bytes(n, 1, Is) : 0);
  auto sfb_bytes = [](int32_t G, int64_t I_, int64_t d_) {
    const int64_t a = fp8_pair_sfb_bytes(G, (int32_t)I_, (int32_t)d_, true);
    const int64_t b = fp8_pair_sfb_bytes(G, (int32_t)d_, (int32_t)I_, false);
    return (size_t)(a > b ? a : b);
  };
  p.sfb = take(fp8 ? sfb_bytes(fg, I, d) : 0);
  p.sfbs = take(fp8 && Is > 0 ? sfb_bytes(1, Is, d) : 0);
  p.ep_off = take(ep ? (size_t)(fg + 1) * 4 : 0);
  p.total = off;
  return p;
}

moe_status check_cfg(const moe_config* c, int64_t n) {
  if (!c || n < 0) return MOE_ERR_INVALID_ARG;
  if (c->dtype != MOE_F32 && c->dtype != MOE_BF16 && c->dtype != MOE_FP8) return MOE_ERR_INVALID_ARG;
  if (c->score_fn != MOE_SCORE_SOFTMAX && c->score_fn != MOE_SCORE_SIGMOID && c->score_fn != MOE_SCORE_SQRTSOFTPLUS)
    return MOE_ERR_INVALID_ARG;
  if (c->cap_policy < MOE_CAP_NONE || c->cap_policy > MOE_CAP_DROP) return MOE_ERR_INVALID_ARG;
  if (c->d_model <= 0 || c->n_routed <= 0 || c->top_k <= 0 || c->moe_intermediate_size <= 0 || c->n_shared < 0 ||
      c->n_group <= 0 || c->topk_group <= 0)
    return MOE_ERR_INVALID_ARG;
  if (c->top_k > c->n_routed || c->topk_group > c->n_group || c->n_routed % c->n_group != 0)
    return MOE_ERR_INVALID_ARG;
  if ((int64_t)c->topk_group * (c->n_routed / c->n_group) < c->top_k) return MOE_ERR_INVALID_ARG;
  if (c->cap_policy != MOE_CAP_NONE && c->capacity <= 0 && !(c->capacity_factor > 0.0f)) return MOE_ERR_INVALID_ARG;
  if (!isfinite(c->routed_scaling_factor)) return MOE_ERR_INVALID_ARG;
  if (c->n_routed > kMaxExperts || c->top_k > kMaxTopK || c->n_group > kMaxGroups) return MOE_ERR_UNSUPPORTED;
  if (c->n_group > 1 && c->score_fn == MOE_SCORE_SOFTMAX) return MOE_ERR_UNSUPPORTED;
  if (c->d_model % 8 != 0 || c->moe_intermediate_size % 8 != 0) return MOE_ERR_UNSUPPORTED;
  // FP8 experts: 128-wide scale tiles along every matrix dimension, at most 128 of them along k
  if (c->dtype == MOE_FP8 && (c->d_model % 128 != 0 || c->moe_intermediate_size % 128 != 0 ||
                              c->d_model > 128 * 128 || (int64_t)c->n_shared * c->moe_intermediate_size > 128 * 128 ||
                              c->moe_intermediate_size > 128 * 128))
    return MOE_ERR_UNSUPPORTED;
  if (n * c->top_k >= (int64_t)1 << 31 || n * (int64_t)c->n_routed >= (int64_t)1 << 40) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

int64_t capacity_of(const moe_config& c, int64_t n) {
  if (c.capacity > 0) return c.capacity;
  return (int64_t)ceil((double)c.capacity_factor * (double)n * (double)c.top_k / (double)c.n_routed);
}

moe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

#define MOE_TRY(expr)                         \
  do {                                        \
    const moe_status st_ = (expr);            \
    if (st_ != MOE_OK) return st_;            \
  } while (0)
#define MOE_CUDA(expr) MOE_TRY(cuda_status(expr))

struct Ctx {
  moe_config c;
  int64_t n;
  Plan p;
  char* ws;
  cudaStream_t s;
  template <typename T>
  T* at(size_t off) const {
    return reinterpret_cast<T*>(ws + off);
  }
  moe_diag* status() const { return at<moe_diag>(p.diag); }
};

moe_status begin(const moe_config* cfg, int64_t n, void* ws, size_t ws_bytes, moe_stream_t stream, Ctx* ctx) {
  MOE_TRY(check_cfg(cfg, n));
  if (!ws || !aligned(ws, 256)) return MOE_ERR_INVALID_ARG;
  ctx->c = *cfg;
  ctx->n = n;
  ctx->p = make_plan(*cfg, n);
  if (ws_bytes < ctx->p.total) return MOE_ERR_WORKSPACE;
  ctx->ws = static_cast<char*>(ws);
  ctx->s = reinterpret_cast<cudaStream_t>(stream);
  return MOE_OK;
}

// First enqueued work of every entry point, after all argument checks: the
// status word reports the most recent entry point on this workspace.
moe_status clear_status(const Ctx& ctx) {
  return cuda_status(cudaMemsetAsync(&ctx.status()->status, 0, sizeof(int32_t), ctx.s));
}

bool ptr_ok(const void* p) { return p && aligned(p, 16); }
// Per-token buffers may be null (zero-size tensors) when there are no tokens.
bool tok_ok(const void* p, int64_t n) { return n == 0 ? (!p || aligned(p, 16)) : ptr_ok(p); }

moe_status check_weights(const moe_config& c, const moe_weights* w, bool routed, bool shared) {
  if (!w) return MOE_ERR_INVALID_ARG;
  if (routed && (!ptr_ok(w->w_gate) || !ptr_ok(w->w_up) || !ptr_ok(w->w_down))) return MOE_ERR_INVALID_ARG;
  if (shared && c.n_shared > 0 && (!ptr_ok(w->ws_gate) || !ptr_ok(w->ws_up) || !ptr_ok(w->ws_down)))
    return MOE_ERR_INVALID_ARG;
  if (w->bias && !aligned(w->bias, 4)) return MOE_ERR_INVALID_ARG;
  if (c.dtype == MOE_FP8) {
    if (routed && (!w->w_gate_scale || !w->w_up_scale || !w->w_down_scale)) return MOE_ERR_INVALID_ARG;
    if (shared && c.n_shared > 0 && (!w->ws_gate_scale || !w->ws_up_scale || !w->ws_down_scale))
      return MOE_ERR_INVALID_ARG;
  }
  return MOE_OK;
}

// Grouped GEMM dispatch: bf16 runs on the tcgen05 tensor cores only (a shape or
// alignment they cannot take is MOE_ERR_UNSUPPORTED, never a slower path);
// binary32 layers run on the CUDA cores, whose FFMA meets their 1e-4 tolerance.
moe_status gemm(const Ctx& x, const GemmArgs& a, bool swiglu, bool out_f32) {
  if (act_dtype(x.c) == MOE_BF16) {
    if (!gemm_tc_supported(a, swiglu, out_f32)) return MOE_ERR_UNSUPPORTED;
    return cuda_status(launch_gemm_tc(a, swiglu, out_f32, x.status(), x.s));
  }
  return cuda_status(launch_gemm_simt(a, act_dtype(x.c), out_f32, swiglu, x.s));
}

// Arguments of the warp-per-token router over the logits buffer (splits partial sums).
RouteArgs route_args(const Ctx& x, const void* X, const moe_weights* w, int32_t* idx, float* tw, moe_diag* d,
                     int splits) {
  const moe_config& c = x.c;
  const int64_t ld = logits_ld(c);
  RouteArgs r{};
  r.logits = x.at<float>(x.p.logits);
  r.splits = splits;
  r.split_stride = x.n * ld;
  r.ldl = ld;
  r.x = X;
  r.w_r = w->w_router;
  r.bias = c.score_fn != MOE_SCORE_SOFTMAX ? w->bias : nullptr;
  r.dtype = act_dtype(c);
  r.d = c.d_model;
  r.n = x.n;
  r.E = c.n_routed;
  r.k = c.top_k;
  r.G = c.n_group;
  r.topk_group = c.topk_group;
  r.score_fn = c.score_fn;
  r.renorm = c.renormalize;
  r.rsf = c.routed_scaling_factor;
  r.topk_idx = idx;
  r.topk_w = tw;
  r.diag = d;
  r.ranking = nullptr;
  return r;
}

// Router logits (binary32; small batches split K and sum the partials into one row per token)
// and the route arguments.
moe_status router_logits(const Ctx& x, const void* X, const moe_weights* w, int32_t* idx, float* tw, moe_diag* d,
                         RouteArgs* out) {
  const moe_config& c = x.c;
  const int splits = router_splits(c, x.n);
  const int64_t ld = logits_ld(c);
  GemmArgs g{X, c.d_model, w->w_router, nullptr, 0, x.at<float>(x.p.logits), ld, nullptr, 1, x.n, c.n_routed,
             c.d_model, splits, x.n * ld};
  MOE_TRY(gemm(x, g, false, true));
  // the partials summed once, so every later reader takes one row per token
  MOE_CUDA(launch_sum_splits(x.at<float>(x.p.logits), splits, x.n * ld, x.n, ld, c.n_routed, x.s));
  *out = route_args(x, X, w, idx, tw, d, 1);
  return MOE_OK;
}

// The token queue and candidate region: queue length in the workspace's diag block; four counters
// (pairs listed, refine cursor, second-pass cursor, length of the one-pass router's refinement
// queue), then the candidate table, their binary64 logits, the pair list.
void queue_args(const Ctx& x, RouteTcArgs* a) {
  a->queue = x.at<int32_t>(x.p.rq);
  a->queue_len = &x.status()->reserved[1];
  a->pair_count = x.at<int32_t>(x.p.rc);
  a->cand = x.at<int32_t>(x.p.rc + 16);
  a->cand_val = reinterpret_cast<double*>(x.ws + x.p.rc + cand_val_offset(x.n));
  a->pairs = reinterpret_cast<int32_t*>(x.ws + x.p.rc + pairs_offset(x.n));
}

// The one-pass router's arguments; false when this configuration takes the two-kernel path.
bool one_pass_args(const Ctx& x, const void* X, const moe_weights* w, int32_t* idx, float* tw, RouteTcArgs* ra) {
  const moe_config& c = x.c;
  if (!one_pass_possible(c, x.n)) return false;
  RouteTcArgs a{};
  a.x = X;
  a.w_r = w->w_router;
  a.bias = c.score_fn != MOE_SCORE_SOFTMAX ? w->bias : nullptr;
  a.n = x.n;
  a.d = c.d_model;
  a.E = c.n_routed;
  a.k = c.top_k;
  a.G = c.n_group;
  a.topk_group = c.topk_group;
  a.score_fn = c.score_fn;
  a.renorm = c.renormalize;
  a.rsf = c.routed_scaling_factor;
  a.topk_idx = idx;
  a.topk_w = tw;
  a.logits = x.at<float>(x.p.logits);
  a.ldl = logits_ld(c);
  queue_args(x, &a);
  a.status = x.status();
  if (!route_tc_supported(a)) return false;
  *ra = a;
  return true;
}

// The batched refinement's arguments for the two-kernel router; false when its tokens are refined
// one warp at a time.
bool refine_args(const Ctx& x, const void* X, const moe_weights* w, RouteTcArgs* ra) {
  const moe_config& c = x.c;
  if (!x.p.batched || reinterpret_cast<uintptr_t>(X) % 16 ||
      reinterpret_cast<uintptr_t>(w->w_router) % 16)
    return false;
  RouteTcArgs a{};
  a.x = X;
  a.w_r = w->w_router;
  a.n = x.n;
  a.d = c.d_model;
  a.E = c.n_routed;
  queue_args(x, &a);
  a.status = x.status();
  *ra = a;
  return true;
}

moe_status route_impl(const Ctx& x, const void* X, const moe_weights* w, int32_t* idx, float* tw, int32_t* counts,
                      moe_diag* diag) {
  const moe_config& c = x.c;
  moe_diag* d = diag ? diag : x.status();
  static_assert(offsetof(moe_diag, status) == 5 * sizeof(int32_t), "the counters precede the status word");
  MOE_CUDA(cudaMemsetAsync(d, 0, 5 * sizeof(int32_t), x.s));  // the counters, not the status word
  if (x.n == 0) {
    if (counts) MOE_CUDA(launch_fill_i32(counts, c.n_routed, 0, x.s));
    return MOE_OK;
  }
  // token cursor of the router's warps and the one-pass router's queue length, in the workspace's
  // own diag block
  int32_t* cursor = &x.status()->reserved[0];
  MOE_CUDA(cudaMemsetAsync(cursor, 0, 2 * sizeof(int32_t), x.s));
  RouteTcArgs ra;
  RouteArgs r;
  if (one_pass_args(x, X, w, idx, tw, &ra)) {
    // Decisions in the tensor-core epilogue. The tokens it could not certify (their logits rows
    // written, their indices queued) go through the batched binary64 refinement: a first pass
    // decides what binary64 certifies from the rows and queues the rest with the experts to
    // refine, refine_kernel computes those, and a second pass decides the tokens it queued.
    MOE_CUDA(cudaMemsetAsync(ra.pair_count, 0, 4 * sizeof(int32_t), x.s));
    MOE_CUDA(launch_route_tc(ra, x.s));
    int32_t* queue2 = ra.queue + x.n;
    int32_t* queue2_len = ra.pair_count + 3;
    r = route_args(x, X, w, idx, tw, d, 1);
    r.cursor = cursor;
    r.queue = ra.queue;
    r.queue_len = ra.queue_len;
    r.defer_queue = queue2;
    r.defer_len = queue2_len;
    r.defer_cand = ra.cand;
    r.defer_cand_val = ra.cand_val;
    r.defer_pairs = ra.pairs;
    r.defer_pair_count = ra.pair_count;
    MOE_CUDA(launch_route(r, x.s));
    RouteTcArgs rb = ra;
    rb.queue = queue2;
    MOE_CUDA(launch_refine(rb, x.s));
    RouteArgs r2 = r;
    r2.defer_queue = r2.defer_len = r2.defer_cand = r2.defer_pairs = r2.defer_pair_count = nullptr;
    r2.defer_cand_val = nullptr;
    r2.cursor = ra.pair_count + 2;
    r2.queue = queue2;
    r2.queue_len = queue2_len;
    r2.cand = ra.cand;
    r2.cand_val = ra.cand_val;
    MOE_CUDA(launch_route(r2, x.s));
  } else {
    MOE_TRY(router_logits(x, X, w, idx, tw, d, &r));
    r.cursor = cursor;
    if (c.cap_policy != MOE_CAP_NONE) r.ranking = x.at<uint16_t>(x.p.ranking);
    if (refine_args(x, X, w, &ra)) {
      // first pass decides what binary32 certifies and queues the rest with the experts to refine;
      // those are refined all at once, then the second pass decides the queued tokens
      MOE_CUDA(cudaMemsetAsync(ra.pair_count, 0, 4 * sizeof(int32_t), x.s));
      r.defer_queue = ra.queue;
      r.defer_len = ra.queue_len;
      r.defer_cand = ra.cand;
      r.defer_cand_val = ra.cand_val;
      r.defer_pairs = ra.pairs;
      r.defer_pair_count = ra.pair_count;
      MOE_CUDA(launch_route(r, x.s));
      MOE_CUDA(launch_refine(ra, x.s));
      RouteArgs r2 = r;
      r2.defer_queue = r2.defer_len = r2.defer_cand = r2.defer_pairs = r2.defer_pair_count = nullptr;
      r2.defer_cand_val = nullptr;
      r2.cursor = ra.pair_count + 2;
      r2.queue = ra.queue;
      r2.queue_len = ra.queue_len;
      r2.cand = ra.cand;
      r2.cand_val = ra.cand_val;
      MOE_CUDA(launch_route(r2, x.s));
    } else {
      MOE_CUDA(launch_route(r, x.s));
    }
  }
  if (c.cap_policy != MOE_CAP_NONE) {
    // the capacity rule on many SMs when its grid fits on the device at once (MOE_CAP_MODE=1cta
    // forces the one-CTA kernel: tuning and tests)
    const char* cm = getenv("MOE_CAP_MODE");
    const bool one_cta = cm && strcmp(cm, "1cta") == 0;
    if (!one_cta && capacity_grid_fits(x.n, c.n_routed)) {
      CapacityArgs ca{r.ranking, x.n, c.n_routed, c.top_k, capacity_of(c, x.n), c.cap_policy, idx, d, nullptr,
                      x.status()};
      const cudaError_t e = launch_capacity_grid(ca, x.ws + x.p.capg, x.s);
      if (e == cudaErrorCooperativeLaunchTooLarge) {
        // the grid did not fit beside other resident work after all: the one-CTA kernel
        cudaGetLastError();
        MOE_CUDA(launch_capacity(r.ranking, x.n, c.n_routed, c.top_k, capacity_of(c, x.n), c.cap_policy, idx, d, x.s));
      } else {
        MOE_CUDA(e);
      }
    } else {
      MOE_CUDA(launch_capacity(r.ranking, x.n, c.n_routed, c.top_k, capacity_of(c, x.n), c.cap_policy, idx, d, x.s));
    }
    MOE_CUDA(launch_gates(r, x.s));
  }
  // per-expert slot counts and the largest load (histogram + scan, no scatter)
  MOE_CUDA(launch_dispatch(idx, x.n, c.top_k, c.n_routed, x.at<int32_t>(x.p.blk), counts,
                           x.at<int32_t>(x.p.offsets), nullptr, nullptr, false, d, x.s));
  return MOE_OK;
}

// counted: route_impl's histogram and scan over the same idx already left the per-block bases and
// offsets in the workspace, so only the permutation runs.
moe_status permute_impl(const Ctx& x, const void* X, const int32_t* idx, int32_t* offsets, int32_t* perm,
                        int32_t* dest, void* xperm, bool counted = false) {
  const moe_config& c = x.c;
  if (x.n == 0) {
    MOE_CUDA(launch_fill_i32(offsets, c.n_routed + 1, 0, x.s));
    return MOE_OK;
  }
  if (counted)
    MOE_CUDA(launch_scatter(idx, x.n, c.top_k, c.n_routed, x.at<int32_t>(x.p.blk), offsets, perm, dest, x.s));
  else
    MOE_CUDA(launch_dispatch(idx, x.n, c.top_k, c.n_routed, x.at<int32_t>(x.p.blk), nullptr, offsets, perm, dest,
                             true, nullptr, x.s));
  if (!xperm) return MOE_OK;  // the FP8 quantiser gathers the rows itself
  const int64_t row_bytes = (int64_t)c.d_model * (act_dtype(c) == MOE_BF16 ? 2 : 4);
  MOE_CUDA(launch_permute_rows(X, dest, x.n, c.top_k, row_bytes, xperm, x.s));
  return MOE_OK;
}

// FP8 experts: quantise the rows (gathered through a_rows when given), gate/up GEMM with the
// SwiGLU epilogue, quantise h, down GEMM; the scale blocks follow the same row groups.
moe_status ffn_fp8(const Ctx& x, const void* A, const int32_t* a_rows, const int32_t* offsets, const moe_weights* w,
                   void* eo) {
  const moe_config& c = x.c;
  const int64_t I = c.moe_intermediate_size, d = c.d_model, nk = x.n * c.top_k;
  uint8_t* xq = x.at<uint8_t>(x.p.xq);
  uint32_t* sfx = x.at<uint32_t>(x.p.sfx);
  uint8_t* hq = x.at<uint8_t>(x.p.hq);
  uint32_t* sfh = x.at<uint32_t>(x.p.sfh);
  void* h = x.ws + x.p.h;
  const int32_t tr = fp8_tile_rows(nk, c.n_routed);
  int32_t* sched = x.at<int32_t>(x.p.sched);
  MOE_CUDA(launch_quantize_rows(A, a_rows, offsets, c.n_routed, nk, (int32_t)d, tr, xq, sfx, x.s));
  GemmFp8Args g1{xq, w->w_gate, w->w_up, sfx, w->w_gate_scale, w->w_up_scale, h, I, offsets, c.n_routed, nk,
                 (int32_t)I, (int32_t)d, tr, sched, fp8_sf_blocks(nk, c.n_routed, d), x.at<uint32_t>(x.p.sfb),
                 fp8_pair_sfb_bytes(c.n_routed, (int32_t)I, (int32_t)d, true)};
  MOE_CUDA(launch_gemm_fp8(g1, true, x.status(), x.s));
  MOE_CUDA(launch_quantize_rows(h, nullptr, offsets, c.n_routed, nk, (int32_t)I, tr, hq, sfh, x.s));
  GemmFp8Args g2{hq, w->w_down, nullptr, sfh, w->w_down_scale, nullptr, eo, d, offsets, c.n_routed, nk,
                 (int32_t)d, (int32_t)I, tr, sched + 1, fp8_sf_blocks(nk, c.n_routed, I), x.at<uint32_t>(x.p.sfb),
                 fp8_pair_sfb_bytes(c.n_routed, (int32_t)d, (int32_t)I, false)};
  MOE_CUDA(launch_gemm_fp8(g2, false, x.status(), x.s));
  return MOE_OK;
}

moe_status ffn_impl(const Ctx& x, const void* xperm, const int32_t* offsets, const moe_weights* w, void* eo) {
  const moe_config& c = x.c;
  if (x.n == 0) return MOE_OK;
  if (c.dtype == MOE_FP8) return ffn_fp8(x, xperm, nullptr, offsets, w, eo);
  const int64_t I = c.moe_intermediate_size, d = c.d_model, nk = x.n * c.top_k;
  void* h = x.ws + x.p.h;
  int32_t* sched = x.at<int32_t>(x.p.sched);
  GemmArgs g1{xperm, d, w->w_gate, w->w_up, I * d, h, I, offsets, c.n_routed, nk, (int32_t)I, (int32_t)d};
  g1.tile_counter = sched;
  MOE_TRY(gemm(x, g1, true, false));
  GemmArgs g2{h, I, w->w_down, nullptr, d * I, eo, d, offsets, c.n_routed, nk, (int32_t)d, (int32_t)I};
  g2.tile_counter = sched + 1;
  MOE_TRY(gemm(x, g2, false, false));
  return MOE_OK;
}

moe_status shared_impl(const Ctx& x, const void* X, const moe_weights* w, void** sh_out) {
  const moe_config& c = x.c;
  *sh_out = nullptr;
  if (c.n_shared == 0 || x.n == 0) return MOE_OK;
  const int64_t Is = (int64_t)c.n_shared * c.moe_intermediate_size, d = c.d_model;
  void* shh = x.ws + x.p.shh;
  void* sh = x.ws + x.p.sh;
  if (c.dtype == MOE_FP8) {
    uint8_t* xq = x.at<uint8_t>(x.p.xsq);
    uint32_t* sfx = x.at<uint32_t>(x.p.sfxs);
    uint8_t* hq = x.at<uint8_t>(x.p.hsq);
    uint32_t* sfh = x.at<uint32_t>(x.p.sfhs);
    const int32_t tr = fp8_tile_rows(x.n, 1);
    int32_t* sched = x.at<int32_t>(x.p.sched);
    MOE_CUDA(launch_quantize_rows(X, nullptr, nullptr, 1, x.n, (int32_t)d, tr, xq, sfx, x.s));
    GemmFp8Args g1{xq, w->ws_gate, w->ws_up, sfx, w->ws_gate_scale, w->ws_up_scale, shh, Is, nullptr, 1, x.n,
                   (int32_t)Is, (int32_t)d, tr, sched + 2, fp8_sf_blocks(x.n, 1, d), x.at<uint32_t>(x.p.sfbs),
                   fp8_pair_sfb_bytes(1, (int32_t)Is, (int32_t)d, true)};
    MOE_CUDA(launch_gemm_fp8(g1, true, x.status(), x.s));
    MOE_CUDA(launch_quantize_rows(shh, nullptr, nullptr, 1, x.n, (int32_t)Is, tr, hq, sfh, x.s));
    GemmFp8Args g2{hq, w->ws_down, nullptr, sfh, w->ws_down_scale, nullptr, sh, d, nullptr, 1, x.n, (int32_t)d,
                   (int32_t)Is, tr, sched + 3, fp8_sf_blocks(x.n, 1, Is), x.at<uint32_t>(x.p.sfbs),
                   fp8_pair_sfb_bytes(1, (int32_t)d, (int32_t)Is, false)};
    MOE_CUDA(launch_gemm_fp8(g2, false, x.status(), x.s));
    *sh_out = sh;
    return MOE_OK;
  }
  int32_t* sched = x.at<int32_t>(x.p.sched);
  GemmArgs g1{X, d, w->ws_gate, w->ws_up, 0, shh, Is, nullptr, 1, x.n, (int32_t)Is, (int32_t)d};
  g1.tile_counter = sched + 2;
  MOE_TRY(gemm(x, g1, true, false));
  GemmArgs g2{shh, Is, w->ws_down, nullptr, 0, sh, d, nullptr, 1, x.n, (int32_t)d, (int32_t)Is};
  g2.tile_counter = sched + 3;
  MOE_TRY(gemm(x, g2, false, false));
  *sh_out = sh;
  return MOE_OK;
}

// Per-device side stream with fork/join events: the shared experts depend only
// on x, so their GEMMs run there while routing and dispatch (CUDA-core and HBM
// bound) run on the caller's stream. Created on first use, kept until exit.
struct SideStream {
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};

SideStream* side_stream() {
  constexpr int kMaxDevices = 64;
  static SideStream table[kMaxDevices];
  static std::mutex lock;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> g(lock);
  SideStream& ss = table[dev];
  if (!ss.s) {
    if (cudaStreamCreateWithFlags(&ss.s, cudaStreamNonBlocking) != cudaSuccess) return nullptr;
    if (cudaEventCreateWithFlags(&ss.fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&ss.join, cudaEventDisableTiming) != cudaSuccess) {
      ss.s = nullptr;
      return nullptr;
    }
  }
  return &ss;
}

// ---- expert parallelism ------------------------------------------------------------

// Limit of one barrier wait: MOE_EP_TIMEOUT_MS from the environment, default 5 s.
uint64_t ep_timeout_ns() {
  const char* v = getenv("MOE_EP_TIMEOUT_MS");
  long ms = v ? atol(v) : 0;
  if (ms <= 0) ms = 5000;
  return (uint64_t)ms * 1000000ull;
}

moe_status check_ep(const moe_config* cfg, const moe_ep_group* g, int32_t first, int32_t num,
                    const moe_ep_rank* ranks) {
  if (!cfg || !g || !ranks) return MOE_ERR_INVALID_ARG;
  if (g->world < 1) return MOE_ERR_INVALID_ARG;
  if (g->world > MOE_EP_MAX_RANKS) return MOE_ERR_UNSUPPORTED;
  if (cfg->n_routed <= 0 || cfg->n_routed % g->world != 0) return MOE_ERR_INVALID_ARG;
  if (cfg->cap_policy != MOE_CAP_NONE) return MOE_ERR_UNSUPPORTED;
  if (g->recv_rows <= 0 || g->recv_rows >= ((int64_t)1 << 31)) return MOE_ERR_INVALID_ARG;
  if (!(num == 1 || num == g->world) || first < 0 || first + num > g->world) return MOE_ERR_INVALID_ARG;
  for (int q = 0; q < g->world; ++q) {
    if (!ptr_ok(g->recv_x[q]) || !ptr_ok(g->recv_out[q]) || !g->counts[q] || !aligned(g->counts[q], 4))
      return MOE_ERR_INVALID_ARG;
    if (num == 1 && g->world > 1 && (!g->flags[q] || !aligned(g->flags[q], 4))) return MOE_ERR_INVALID_ARG;
  }
  return MOE_OK;
}

moe_status begin_ep(const moe_config* cfg, const moe_ep_group* g, const moe_ep_rank& r, cudaStream_t s, Ctx* ctx) {
  MOE_TRY(check_cfg(cfg, r.n));
  if (!r.ws || !aligned(r.ws, 256)) return MOE_ERR_INVALID_ARG;
  ctx->c = *cfg;
  ctx->n = r.n;
  ctx->p = make_plan(*cfg, r.n, g->world, g->recv_rows);
  if (r.ws_bytes < ctx->p.total) return MOE_ERR_WORKSPACE;
  ctx->ws = static_cast<char*>(r.ws);
  ctx->s = s;
  if (!tok_ok(r.x, r.n) || !tok_ok(r.y, r.n) || !r.weights || !ptr_ok(r.weights->w_router))
    return MOE_ERR_INVALID_ARG;
  if ((r.topk_idx_opt && !tok_ok(r.topk_idx_opt, r.n)) || (r.topk_w_opt && !tok_ok(r.topk_w_opt, r.n)))
    return MOE_ERR_INVALID_ARG;
  return check_weights(ctx->c, r.weights, true, true);
}

// The routed experts of one rank: its E / world experts over the receive buffer's rows.
Ctx ep_expert_ctx(const Ctx& c, int32_t world, int64_t recv_rows) {
  Ctx f = c;
  f.c.n_routed = c.c.n_routed / world;
  f.c.top_k = 1;
  f.c.n_group = 1;
  f.c.topk_group = 1;
  f.n = recv_rows;
  return f;
}

moe_status ep_forward(const moe_config* cfg, const moe_ep_group* g, int32_t first, int32_t num,
                      const moe_ep_rank* ranks, cudaStream_t s) {
  MOE_TRY(check_ep(cfg, g, first, num, ranks));
  const int R = g->world;
  const bool barriers = num == 1 && R > 1;
  EpPeers peers{};
  for (int q = 0; q < R; ++q) {
    peers.recv_x[q] = g->recv_x[q];
    peers.recv_out[q] = g->recv_out[q];
    peers.counts[q] = g->counts[q];
    peers.flags[q] = g->flags[q];
  }
  Ctx cx[kMaxEpRanks];
  for (int i = 0; i < num; ++i) MOE_TRY(begin_ep(cfg, g, ranks[i], s, &cx[i]));
  for (int i = 0; i < num; ++i) MOE_TRY(clear_status(cx[i]));
  const moe_config& c = *cfg;
  const uint64_t timeout = ep_timeout_ns();
  auto barrier = [&]() -> moe_status {
    if (!barriers) return MOE_OK;
    return cuda_status(launch_ep_barrier(peers, R, first, timeout, cx[0].status(), s));
  };
  int32_t* idx[kMaxEpRanks];
  float* tw[kMaxEpRanks];
  void* sh[kMaxEpRanks] = {};
  bool any_shared = false;
  for (int i = 0; i < num; ++i) {
    const moe_ep_rank& r = ranks[i];
    idx[i] = r.topk_idx_opt && r.n > 0 ? r.topk_idx_opt : cx[i].at<int32_t>(cx[i].p.idx);
    tw[i] = r.topk_w_opt && r.n > 0 ? r.topk_w_opt : cx[i].at<float>(cx[i].p.w);
    any_shared |= r.n > 0 && c.n_shared > 0;
  }
  // Shared experts of every rank on the side stream, overlapping the exchange.
  SideStream* side = any_shared ? side_stream() : nullptr;
  if (side) {
    MOE_CUDA(cudaEventRecord(side->fork, s));
    MOE_CUDA(cudaStreamWaitEvent(side->s, side->fork, 0));
    for (int i = 0; i < num; ++i) {
      Ctx cs = cx[i];
      cs.s = side->s;
      MOE_TRY(shared_impl(cs, ranks[i].x, ranks[i].weights, &sh[i]));
    }
    MOE_CUDA(cudaEventRecord(side->join, side->s));
  }
  // 1. route, local stable permutation, counts into every rank's table
  for (int i = 0; i < num; ++i) {
    const Ctx& x = cx[i];
    int32_t* counts = x.at<int32_t>(x.p.counts);
    MOE_TRY(route_impl(x, ranks[i].x, ranks[i].weights, idx[i], tw[i], counts, nullptr));
    MOE_TRY(permute_impl(x, ranks[i].x, idx[i], x.at<int32_t>(x.p.offsets), x.at<int32_t>(x.p.perm),
                         x.at<int32_t>(x.p.dest), nullptr));
    MOE_CUDA(launch_ep_publish(peers, R, c.n_routed, first + i, counts, s));
  }
  MOE_TRY(barrier());
  // 2. token rows into the owners' receive buffers
  const int64_t row_bytes = (int64_t)c.d_model * (act_dtype(c) == MOE_BF16 ? 2 : 4);
  for (int i = 0; i < num; ++i) {
    const Ctx& x = cx[i];
    const int rank = first + i;
    MOE_CUDA(launch_ep_dispatch(peers, R, c.n_routed, rank, g->recv_rows, g->counts[rank],
                                x.at<int32_t>(x.p.offsets), x.at<int32_t>(x.p.perm), ranks[i].x, x.n * c.top_k,
                                row_bytes, x.at<int32_t>(x.p.ep_off), x.status(), s));
  }
  MOE_TRY(barrier());
  // 3. each rank's experts over the rows it received
  for (int i = 0; i < num; ++i) {
    const int rank = first + i;
    const Ctx f = ep_expert_ctx(cx[i], R, g->recv_rows);
    MOE_TRY(ffn_impl(f, g->recv_x[rank], cx[i].at<int32_t>(cx[i].p.ep_off), ranks[i].weights, g->recv_out[rank]));
  }
  MOE_TRY(barrier());
  // 4. gate-weighted sum of the owners' output rows, plus the shared experts
  if (side) MOE_CUDA(cudaStreamWaitEvent(s, side->join, 0));
  for (int i = 0; i < num; ++i) {
    const Ctx& x = cx[i];
    const int rank = first + i;
    if (!side && c.n_shared > 0) MOE_TRY(shared_impl(x, ranks[i].x, ranks[i].weights, &sh[i]));
    MOE_CUDA(launch_ep_combine(peers, R, c.n_routed, rank, g->recv_rows, g->counts[rank],
                               x.at<int32_t>(x.p.offsets), idx[i], x.at<int32_t>(x.p.dest), tw[i], sh[i], x.n,
                               c.top_k, c.d_model, act_dtype(c), ranks[i].y, s));
  }
  return barrier();
}

// Driver API entry for the base of the allocation holding a device address.
typedef CUresult (*AddressRangeFn)(CUdeviceptr*, size_t*, CUdeviceptr);
AddressRangeFn address_range_fn() {
  static AddressRangeFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<AddressRangeFn>(p);
  });
  return fn;
}

moe_status allocation_base(const void* ptr, char** base) {
  AddressRangeFn fn = address_range_fn();
  if (!fn) return MOE_ERR_CUDA;
  CUdeviceptr b = 0;
  size_t size = 0;
  if (fn(&b, &size, reinterpret_cast<CUdeviceptr>(ptr)) != CUDA_SUCCESS) return MOE_ERR_INVALID_ARG;
  *base = reinterpret_cast<char*>(b);
  return MOE_OK;
}

static_assert(sizeof(cudaIpcMemHandle_t) + sizeof(uint64_t) == MOE_EP_HANDLE_BYTES, "handle record size");

}  // namespace
}  // namespace moe

namespace moe {

// Router-only layout inside a fixed scratch region: the status word, the logits, the capacity
// ranking, the per-block counts and the offsets of the count scan. The caller's own buffers hold
// the indices, gates and counts, so the full layout's regions for those are left out.
Plan route_plan(const moe_config& c, int64_t n) {
  Plan p = make_plan(c, n, 0, 0, false);
  p.offsets = p.idx;
  p.total = p.offsets + (size_t)align_up((int64_t)(c.n_routed + 1) * 4, 256);
  return p;
}

size_t route_scratch_bytes(const moe_config& c, int64_t n) { return route_plan(c, n).total; }

// moe_route over a scratch region that only needs route_scratch_bytes() bytes.
moe_status route_in_scratch(const moe_config* cfg, int64_t n, const void* x, const moe_weights* weights,
                            int32_t* topk_idx, float* topk_w, int32_t* expert_counts, moe_diag* diag, void* scratch,
                            size_t scratch_bytes, moe_stream_t stream) {
  MOE_TRY(check_cfg(cfg, n));
  if (!scratch || !aligned(scratch, 256)) return MOE_ERR_INVALID_ARG;
  if (scratch_bytes < route_scratch_bytes(*cfg, n)) return MOE_ERR_WORKSPACE;
  Ctx c;
  c.c = *cfg;
  c.n = n;
  c.p = route_plan(*cfg, n);
  c.ws = static_cast<char*>(scratch);
  c.s = reinterpret_cast<cudaStream_t>(stream);
  if (!weights || !ptr_ok(weights->w_router) || !tok_ok(x, n) || !tok_ok(topk_idx, n) || !tok_ok(topk_w, n))
    return MOE_ERR_INVALID_ARG;
  // diag carries the device status word out of the shared scratch, so it is required here
  if (!diag || !aligned(diag, 16) || (expert_counts && !aligned(expert_counts, 4))) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_weights(c.c, weights, false, false));
  MOE_TRY(clear_status(c));
  MOE_TRY(route_impl(c, x, weights, topk_idx, topk_w, expert_counts, diag));
  // The scratch is not the caller's, so hand the device status word over in diag.
  MOE_CUDA(cudaMemcpyAsync(&diag->status, &c.status()->status, sizeof(int32_t), cudaMemcpyDeviceToDevice, c.s));
  return MOE_OK;
}

}  // namespace moe

using namespace moe;

extern "C" {

moe_status moe_workspace_size(const moe_config* cfg, int64_t n, size_t* bytes) {
  MOE_TRY(check_cfg(cfg, n));
  if (!bytes) return MOE_ERR_INVALID_ARG;
  *bytes = make_plan(*cfg, n).total;
  return MOE_OK;
}

moe_status moe_route(const moe_config* cfg, int64_t n, const void* x, const moe_weights* weights,
                     int32_t* topk_idx, float* topk_w, int32_t* expert_counts, moe_diag* diag, void* ws,
                     size_t ws_bytes, moe_stream_t stream) {
  Ctx c;
  MOE_TRY(begin(cfg, n, ws, ws_bytes, stream, &c));
  if (!weights || !ptr_ok(weights->w_router) || !tok_ok(x, n) || !tok_ok(topk_idx, n) || !tok_ok(topk_w, n))
    return MOE_ERR_INVALID_ARG;
  if ((expert_counts && !aligned(expert_counts, 4)) || (diag && !aligned(diag, 16))) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_weights(c.c, weights, false, false));
  MOE_TRY(clear_status(c));
  return route_impl(c, x, weights, topk_idx, topk_w, expert_counts, diag);
}

moe_status moe_route_hash(const moe_config* cfg, int64_t n, const void* x, const int32_t* token_ids,
                          const int32_t* tid2eid, int32_t vocab, const moe_weights* weights, int32_t* topk_idx,
                          float* topk_w, int32_t* expert_counts, moe_diag* diag, void* ws, size_t ws_bytes,
                          moe_stream_t stream) {
  Ctx c;
  MOE_TRY(begin(cfg, n, ws, ws_bytes, stream, &c));
  if (cfg->cap_policy != MOE_CAP_NONE || vocab <= 0) return MOE_ERR_INVALID_ARG;
  if (!weights || !ptr_ok(weights->w_router) || !tok_ok(x, n) || !tok_ok(topk_idx, n) || !tok_ok(topk_w, n) ||
      (n > 0 && (!token_ids || !aligned(token_ids, 4))) || !tid2eid || !aligned(tid2eid, 4))
    return MOE_ERR_INVALID_ARG;
  if ((expert_counts && !aligned(expert_counts, 4)) || (diag && !aligned(diag, 16))) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_weights(c.c, weights, false, false));
  MOE_TRY(clear_status(c));
  moe_diag* d = diag ? diag : c.status();
  MOE_CUDA(cudaMemsetAsync(d, 0, 5 * sizeof(int32_t), c.s));
  if (n == 0) {
    if (expert_counts) MOE_CUDA(launch_fill_i32(expert_counts, c.c.n_routed, 0, c.s));
    return MOE_OK;
  }
  RouteArgs r;
  MOE_TRY(router_logits(c, x, weights, topk_idx, topk_w, d, &r));
  MOE_CUDA(launch_hash_select(token_ids, tid2eid, vocab, n, c.c.top_k, c.c.n_routed, topk_idx, c.status(), c.s));
  MOE_CUDA(launch_gates(r, c.s));
  MOE_CUDA(launch_dispatch(topk_idx, n, c.c.top_k, c.c.n_routed, c.at<int32_t>(c.p.blk), expert_counts,
                           c.at<int32_t>(c.p.offsets), nullptr, nullptr, false, d, c.s));
  return MOE_OK;
}

moe_status moe_bias_update(const moe_config* cfg, const int32_t* counts, float* bias, float gamma,
                           moe_stream_t stream) {
  MOE_TRY(check_cfg(cfg, 0));
  if (!counts || !bias || !aligned(counts, 4) || !aligned(bias, 4) || !isfinite(gamma)) return MOE_ERR_INVALID_ARG;
  return cuda_status(
      launch_bias_update(counts, cfg->n_routed, gamma, bias, reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_permute(const moe_config* cfg, int64_t n, const void* x, const int32_t* topk_idx, int32_t* offsets,
                       int32_t* perm_token, int32_t* slot_dest, void* x_perm, void* ws, size_t ws_bytes,
                       moe_stream_t stream) {
  Ctx c;
  MOE_TRY(begin(cfg, n, ws, ws_bytes, stream, &c));
  if (!tok_ok(x, n) || !tok_ok(topk_idx, n) || !ptr_ok(offsets) || !tok_ok(perm_token, n) ||
      !tok_ok(slot_dest, n) || !tok_ok(x_perm, n))
    return MOE_ERR_INVALID_ARG;
  MOE_TRY(clear_status(c));
  return permute_impl(c, x, topk_idx, offsets, perm_token, slot_dest, x_perm);
}

moe_status moe_expert_ffn(const moe_config* cfg, int64_t n, const void* x_perm, const int32_t* offsets,
                          const moe_weights* weights, void* expert_out, void* ws, size_t ws_bytes,
                          moe_stream_t stream) {
  Ctx c;
  MOE_TRY(begin(cfg, n, ws, ws_bytes, stream, &c));
  if (!tok_ok(x_perm, n) || !ptr_ok(offsets) || !tok_ok(expert_out, n)) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_weights(c.c, weights, true, false));
  MOE_TRY(clear_status(c));
  return ffn_impl(c, x_perm, offsets, weights, expert_out);
}

moe_status moe_combine(const moe_config* cfg, int64_t n, const void* expert_out, const int32_t* slot_dest,
                       const float* topk_w, const void* x, const moe_weights* weights, void* y, void* ws,
                       size_t ws_bytes, moe_stream_t stream) {
  Ctx c;
  MOE_TRY(begin(cfg, n, ws, ws_bytes, stream, &c));
  if (!tok_ok(expert_out, n) || !tok_ok(slot_dest, n) || !tok_ok(topk_w, n) || !tok_ok(y, n))
    return MOE_ERR_INVALID_ARG;
  if (c.c.n_shared > 0 && !tok_ok(x, n)) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_weights(c.c, weights, false, true));
  MOE_TRY(clear_status(c));
  void* sh = nullptr;
  MOE_TRY(shared_impl(c, x, weights, &sh));
  if (n == 0) return MOE_OK;
  return cuda_status(launch_combine(expert_out, slot_dest, topk_w, sh, n, c.c.top_k, c.c.d_model, act_dtype(c.c), y, c.s));
}

moe_status moe_layer_forward(const moe_config* cfg, int64_t n, const void* x, const moe_weights* weights, void* y,
                             int32_t* topk_idx_opt, float* topk_w_opt, int32_t* counts_opt, moe_diag* diag_opt,
                             void* ws, size_t ws_bytes, moe_stream_t stream) {
  Ctx c;
  MOE_TRY(begin(cfg, n, ws, ws_bytes, stream, &c));
  if (!tok_ok(x, n) || !tok_ok(y, n) || !weights || !ptr_ok(weights->w_router)) return MOE_ERR_INVALID_ARG;
  if ((topk_idx_opt && !tok_ok(topk_idx_opt, n)) || (topk_w_opt && !tok_ok(topk_w_opt, n)) ||
      (counts_opt && !aligned(counts_opt, 4)) || (diag_opt && !aligned(diag_opt, 16)))
    return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_weights(c.c, weights, true, true));
  MOE_TRY(clear_status(c));
  int32_t* idx = topk_idx_opt && n > 0 ? topk_idx_opt : c.at<int32_t>(c.p.idx);
  float* tw = topk_w_opt && n > 0 ? topk_w_opt : c.at<float>(c.p.w);
  int32_t* counts = counts_opt ? counts_opt : c.at<int32_t>(c.p.counts);
  int32_t* offsets = c.at<int32_t>(c.p.offsets);
  int32_t* perm = c.at<int32_t>(c.p.perm);
  int32_t* dest = c.at<int32_t>(c.p.dest);
  void* xperm = c.ws + c.p.xperm;
  void* eo = c.ws + c.p.eo;
  // Routing first: the one-pass router needs a whole SM's shared memory per CTA, so it runs before
  // the shared experts take the SMs. The shared experts' GEMMs then run on the side stream next to
  // the permutation, whose HBM-bound kernels fit on the SMs beside the GEMM's CTAs.
  MOE_TRY(route_impl(c, x, weights, idx, tw, counts, diag_opt));
  if (n == 0) return MOE_OK;
  void* sh = nullptr;
  SideStream* side = c.c.n_shared > 0 ? side_stream() : nullptr;
  if (side) {
    MOE_CUDA(cudaEventRecord(side->fork, c.s));
    MOE_CUDA(cudaStreamWaitEvent(side->s, side->fork, 0));
    Ctx cs = c;
    cs.s = side->s;
    MOE_TRY(shared_impl(cs, x, weights, &sh));
    MOE_CUDA(cudaEventRecord(side->join, side->s));
  }
  // route_impl left the histogram's per-block bases and the offsets of idx in the workspace
  if (c.c.dtype == MOE_FP8) {
    // the quantiser gathers the token rows itself: no bf16 permuted copy
    MOE_TRY(permute_impl(c, x, idx, offsets, perm, dest, nullptr, true));
    MOE_TRY(ffn_fp8(c, x, perm, offsets, weights, eo));
  } else {
    MOE_TRY(permute_impl(c, x, idx, offsets, perm, dest, xperm, true));
    MOE_TRY(ffn_impl(c, xperm, offsets, weights, eo));
  }
  if (side)
    MOE_CUDA(cudaStreamWaitEvent(c.s, side->join, 0));
  else
    MOE_TRY(shared_impl(c, x, weights, &sh));
  return cuda_status(launch_combine(eo, dest, tw, sh, n, c.c.top_k, c.c.d_model, act_dtype(c.c), y, c.s));
}

moe_status moe_quantize_fp8(const void* x, int64_t rows, int32_t cols, uint8_t* codes, uint8_t* scale_bytes,
                            moe_stream_t stream) {
  if (rows < 0 || cols <= 0 || cols % 128 != 0 || rows * (int64_t)cols >= (int64_t)1 << 40) return MOE_ERR_INVALID_ARG;
  if (rows == 0) return MOE_OK;
  if (!ptr_ok(x) || !ptr_ok(codes) || !scale_bytes) return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_quantize_rows(x, nullptr, nullptr, 1, rows, cols, 128, codes, nullptr,
                                          reinterpret_cast<cudaStream_t>(stream), scale_bytes));
}

moe_status moe_ep_workspace_size(const moe_config* cfg, int32_t world, int64_t n, int64_t recv_rows, size_t* bytes) {
  MOE_TRY(check_cfg(cfg, n));
  if (!bytes || world < 1 || recv_rows <= 0 || recv_rows >= ((int64_t)1 << 31)) return MOE_ERR_INVALID_ARG;
  if (world > MOE_EP_MAX_RANKS) return MOE_ERR_UNSUPPORTED;
  if (cfg->n_routed % world != 0) return MOE_ERR_INVALID_ARG;
  *bytes = make_plan(*cfg, n, world, recv_rows).total;
  return MOE_OK;
}

moe_status moe_ep_layer_forward(const moe_config* cfg, const moe_ep_group* group, int32_t first_rank,
                                int32_t num_ranks, const moe_ep_rank* ranks, moe_stream_t stream) {
  return ep_forward(cfg, group, first_rank, num_ranks, ranks, reinterpret_cast<cudaStream_t>(stream));
}

moe_status moe_ep_export_handle(const void* ptr, void* handle) {
  if (!ptr || !handle) return MOE_ERR_INVALID_ARG;
  char* base = nullptr;
  MOE_TRY(allocation_base(ptr, &base));
  cudaIpcMemHandle_t h;
  MOE_CUDA(cudaIpcGetMemHandle(&h, base));
  const uint64_t off = (uint64_t)(static_cast<const char*>(ptr) - base);
  memcpy(handle, &h, sizeof(h));
  memcpy(static_cast<char*>(handle) + sizeof(h), &off, sizeof(off));
  return MOE_OK;
}

moe_status moe_ep_open_handle(const void* handle, void** ptr) {
  if (!handle || !ptr) return MOE_ERR_INVALID_ARG;
  cudaIpcMemHandle_t h;
  uint64_t off = 0;
  memcpy(&h, handle, sizeof(h));
  memcpy(&off, static_cast<const char*>(handle) + sizeof(h), sizeof(off));
  void* base = nullptr;
  MOE_CUDA(cudaIpcOpenMemHandle(&base, h, cudaIpcMemLazyEnablePeerAccess));
  *ptr = static_cast<char*>(base) + off;
  return MOE_OK;
}

moe_status moe_ep_close_handle(void* ptr) {
  if (!ptr) return MOE_ERR_INVALID_ARG;
  char* base = nullptr;
  MOE_TRY(allocation_base(ptr, &base));
  return cuda_status(cudaIpcCloseMemHandle(base));
}

moe_status moe_sync_status(void* ws, moe_stream_t stream) {
  if (!ws || !aligned(ws, 256)) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  moe_diag* d = reinterpret_cast<moe_diag*>(ws);  // the diag region is first in the workspace
  int32_t code = 0;
  if (cudaMemcpy(&code, &d->status, sizeof(code), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  if (code != 0 && cudaMemset(&d->status, 0, sizeof(code)) != cudaSuccess) return MOE_ERR_CUDA;
  return (moe_status)code;
}

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported configuration";
    case MOE_ERR_WORKSPACE: return "workspace too small";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_TIMEOUT: return "device wait timed out";
    case MOE_ERR_INTERNAL: return "device-side check failed";
  }
  return "unknown status";
}

}  // extern "C"
