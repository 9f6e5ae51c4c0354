// kernels.h -- internal launch interface between the host entry points and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "moe.h"

namespace moe {

// Grouped GEMM problem. Rows of group g are [offsets[g], offsets[g+1]) of A and
// C (offsets == nullptr: one group of M rows). B holds G consecutive [N, K]
// matrices (out x in) b_group_stride elements apart; B2 likewise (SwiGLU up).
struct GemmArgs {
  const void* A;
  int64_t lda;
  const void* B;
  const void* B2;
  int64_t b_group_stride;
  void* C;
  int64_t ldc;
  const int32_t* offsets;
  int32_t G;
  int64_t M;  // upper bound on the total rows (exact when offsets == nullptr)
  int32_t N;
  int32_t K;
  int32_t k_splits = 1;         // > 1: split-K, partial results written k_splits times
  int64_t c_split_stride = 0;   // elements between the partial result matrices
  int32_t* tile_counter = nullptr;  // device int32 the SM-pair kernel hands out tiles from (zeroed per launch)
};

cudaError_t launch_gemm_simt(const GemmArgs& a, int dtype, bool out_f32, bool swiglu, cudaStream_t s);

// tcgen05 grouped GEMM (bf16 in, fp32 accumulate in TMEM). Returns
// cudaErrorNotSupported when the shape is outside what it handles.
cudaError_t launch_gemm_tc(const GemmArgs& a, bool swiglu, bool out_f32, moe_diag* status, cudaStream_t s);
bool gemm_tc_supported(const GemmArgs& a, bool swiglu, bool out_f32);

// FP8 experts: E4M3 A (quantised rows, scale-factor blocks from launch_quantize_rows)
// times E4M3 B with UE8M0 128 x 128 block-scale bytes, bf16 C; grouped like GemmArgs.
struct GemmFp8Args {
  const void* A;          // [rows, K] E4M3 codes
  const void* B;          // [G * N, K] E4M3 codes
  const void* B2;         // SwiGLU up matrix, like B
  const uint32_t* sfa;    // A scale-factor blocks (512 bytes per 128-row tile and 128-wide k block)
  const uint8_t* sb;      // [G, ceil(N/128), K/128] UE8M0 bytes of B
  const uint8_t* sb2;     // same for B2
  void* C;
  int64_t ldc;
  const int32_t* offsets; // [G + 1] or nullptr (one group of M rows)
  int32_t G;
  int64_t M;
  int32_t N;
  int32_t K;
  int32_t tile_rows;      // rows per A tile and scale block: fp8_tile_rows(M, G)
  int32_t* tile_counter = nullptr;  // SM-pair kernel: device int32 it hands out tiles from
  int64_t sf_blocks = 0;            // 512-byte scale blocks the sfa buffer holds
  uint32_t* sfb = nullptr;          // SM-pair kernel: scratch for B's scale blocks
  int64_t sfb_bytes = 0;            // at least fp8_pair_sfb_bytes(G, N, K, swiglu)
};
int64_t fp8_pair_sfb_bytes(int32_t G, int32_t N, int32_t K, bool swiglu);
cudaError_t launch_gemm_fp8(const GemmFp8Args& a, bool swiglu, moe_diag* status, cudaStream_t s);
// The SM-pair kernel (cta_group::2, 256 x 256 tiles); launch_gemm_fp8 calls it for groups of at
// least 128 rows on average.
cudaError_t launch_gemm_fp8_pair(const GemmFp8Args& a, bool swiglu, moe_diag* status, cudaStream_t s);
// Rows per A tile of the FP8 GEMM (32 for groups of a few rows, else 128); the quantiser lays the
// scale blocks out for the same tiles.
int fp8_tile_rows(int64_t M, int32_t G);

// E4M3 quantisation of bf16 rows in 1 x 128 tiles (row r reads src[src_row[r]] when
// src_row is given); scale words go to the GEMM's scale-factor blocks of the groups, one per
// tile_rows-row tile. fp8_sf_tiles_bound: scale blocks per 128-wide k block for any tile choice.
int64_t fp8_sf_tiles_bound(int64_t rows, int32_t G);
// sf_plain given: scale bytes [rows, cols/128] instead of the GEMM's blocks.
cudaError_t launch_quantize_rows(const void* src, const int32_t* src_row, const int32_t* offsets, int32_t G,
                                 int64_t rows_bound, int32_t cols, int32_t tile_rows, uint8_t* q, uint32_t* sf,
                                 cudaStream_t s, uint8_t* sf_plain = nullptr);

// Router: scoring, group limit, top-k, certification / binary64 refinement, gates.
struct RouteArgs {
  const float* logits;  // [splits][n, ldl] partial logits (first E columns), summed in order
  int32_t splits;
  int64_t split_stride;
  int64_t ldl;          // row stride of the logits (>= E)
  const void* x;        // [n, d] for the binary64 refinement
  const void* w_r;      // [E, d]
  const float* bias;    // [E] or nullptr
  int dtype;
  int32_t d;
  int64_t n;
  int32_t E, k, G, topk_group, score_fn, renorm;
  float rsf;
  uint16_t* ranking;    // [n, E] eligible experts in selection order (capacity), or nullptr
  int32_t* topk_idx;    // [n, k] (written when ranking == nullptr)
  float* topk_w;        // [n, k]
  moe_diag* diag;       // refined_tokens / refined_logits counters
  int32_t* cursor;      // zeroed before the launch: a warp's tokens after its first come from it
  const int32_t* queue = nullptr;      // when set: route only the tokens queue[0 .. *queue_len)
  const int32_t* queue_len = nullptr;
  const int32_t* cand = nullptr;       // with queue: candidate experts and their binary64 logits
  const double* cand_val = nullptr;    // (RouteTcArgs::cand, cand_val)
  // When defer_queue is set, a token whose first decision is not certain is not refined here: it
  // is appended to defer_queue with the experts the decision marked (defer_cand, same layout as
  // RouteTcArgs::cand) and their pairs (defer_pairs), for launch_refine and a second launch_route
  // over that queue.
  int32_t* defer_queue = nullptr;
  int32_t* defer_len = nullptr;        // zeroed before the launch
  int32_t* defer_cand = nullptr;
  double* defer_cand_val = nullptr;    // zeroed for every listed candidate (launch_refine adds into it)
  int32_t* defer_pairs = nullptr;
  int32_t* defer_pair_count = nullptr; // zeroed before the launch
};
cudaError_t launch_route(const RouteArgs& a, cudaStream_t s);
// Sums the split-K partial logits [splits][n, ld] into split 0's rows, in split order (binary64
// sum rounded to binary32), for the first E columns.
cudaError_t launch_sum_splits(float* logits, int32_t splits, int64_t split_stride, int64_t n, int64_t ld, int32_t E,
                              cudaStream_t s);

constexpr int kRouteCandMax = 32;

// Router in one pass (route_tc.cu): logits on the tensor cores and the routing decision of each
// token in the epilogue, in binary32; tokens whose decision is not certain get their logits row
// written and their index queued for launch_route (RouteArgs::queue) to re-decide.
struct RouteTcArgs {
  const void* x;        // [n, d] bf16
  const void* w_r;      // [E, d] bf16
  const float* bias;    // [E] or nullptr
  int64_t n;
  int32_t d, E, k, G, topk_group, score_fn, renorm;
  float rsf;
  int32_t* topk_idx;    // [n, k]
  float* topk_w;        // [n, k]
  float* logits;        // [n, ldl]: rows of the queued tokens
  int64_t ldl;
  int32_t* queue;       // [n] tokens left to the binary64 router (launch_refine: the refinement queue)
  int32_t* queue_len;   // zeroed before the launch
  // launch_refine only (written by a deferring launch_route):
  int32_t* cand;        // [n][kRouteCandMax + 1] per queued token: count (-1: too many), then the experts
                        // an uncertain comparison involves
  double* cand_val;     // [n][kRouteCandMax + 1] binary64 logits of those experts (same slots as cand;
                        // zero before launch_refine, which adds two partial sums into each)
  int32_t* pairs;       // [n * kRouteCandMax] candidate slots to refine: one run per token, padded
                        // with -1 to a multiple of four (a warp refines four pairs of one token)
  int32_t* pair_count;  // [4] zeroed before the launch: pairs listed, the refinement's cursor, the
                        // second route pass's cursor, the second queue's length
  moe_diag* status;
};
bool route_tc_supported(const RouteTcArgs& a);
cudaError_t launch_route_tc(const RouteTcArgs& a, cudaStream_t s);
// Binary64 logits of every listed (queued token, candidate expert) pair, one warp each: the refine
// step of launch_route_tc on its own, for the tokens a deferring launch_route queued. Uses x, w_r,
// d (bf16 rows, d % 8 == 0, 16-byte aligned), queue, cand, cand_val, pairs and pair_count.
cudaError_t launch_refine(const RouteTcArgs& a, cudaStream_t s);

// Capacity rule over the ranking on many SMs (capacity.cu): a cooperative grid, one token per
// thread, one round per fill event. Needs capacity_grid_scratch_bytes of scratch (16-byte aligned)
// and every CTA resident at once (capacity_grid_fits); launch_capacity is the one-CTA form.
struct CapacityArgs {
  const uint16_t* ranking;  // [n, E] eligible experts in selection order, 0xFFFF after the last
  int64_t n;
  int32_t E, k;
  int64_t C;
  int32_t policy;
  int32_t* topk_idx;        // [n, k]
  moe_diag* diag;           // overflowed / dropped counters (added to)
  int32_t* hist;            // set by launch_capacity_grid (inside the scratch)
  moe_diag* status;         // MOE_ERR_TIMEOUT if a grid barrier wait runs out
};
int64_t capacity_grid_scratch_bytes(int64_t n, int32_t E);
bool capacity_grid_fits(int64_t n, int32_t E);
cudaError_t launch_capacity_grid(const CapacityArgs& a, void* scratch, cudaStream_t s);
// Capacity rule over the ranking; writes topk_idx and the overflow/drop counts.
cudaError_t launch_capacity(const uint16_t* ranking, int64_t n, int32_t E, int32_t k, int64_t C, int policy,
                            int32_t* topk_idx, moe_diag* diag, cudaStream_t s);
// Hash routing selection and the balancing-bias update.
cudaError_t launch_hash_select(const int32_t* token_ids, const int32_t* tid2eid, int32_t vocab, int64_t n, int32_t k,
                               int32_t E, int32_t* topk_idx, moe_diag* status, cudaStream_t s);
cudaError_t launch_bias_update(const int32_t* counts, int32_t E, float gamma, float* bias, cudaStream_t s);
// Gates of a given selection from the logits.
cudaError_t launch_gates(const RouteArgs& a, cudaStream_t s);

// Dispatch.
int64_t dispatch_blocks(int64_t n, int32_t k);
cudaError_t launch_dispatch(const int32_t* topk_idx, int64_t n, int32_t k, int32_t E, int32_t* blk_counts,
                            int32_t* counts, int32_t* offsets, int32_t* perm_token, int32_t* slot_dest,
                            bool scatter, moe_diag* diag, cudaStream_t s);
// The stable permutation alone, from the per-block bases and offsets a launch_dispatch over the
// same topk_idx left in blk_base and offsets.
cudaError_t launch_scatter(const int32_t* topk_idx, int64_t n, int32_t k, int32_t E, const int32_t* blk_base,
                           const int32_t* offsets, int32_t* perm_token, int32_t* slot_dest, cudaStream_t s);
// x_perm[slot_dest[t, j]] = x[t] for the kept slots (slot_dest >= 0), each token row read once.
cudaError_t launch_permute_rows(const void* x, const int32_t* slot_dest, int64_t n, int32_t k, int64_t row_bytes,
                                void* x_perm, cudaStream_t s);

// Combine.
cudaError_t launch_combine(const void* eo, const int32_t* slot_dest, const float* topk_w, const void* sh,
                           int64_t n, int32_t k, int32_t d, int dtype, void* y, cudaStream_t s);

// Expert parallelism: every rank's exchange buffers as seen from the calling device.
constexpr int kMaxEpRanks = MOE_EP_MAX_RANKS;
struct EpPeers {
  void* recv_x[kMaxEpRanks];
  void* recv_out[kMaxEpRanks];
  int32_t* counts[kMaxEpRanks];
  uint32_t* flags[kMaxEpRanks];
};
cudaError_t launch_ep_publish(const EpPeers& p, int32_t R, int32_t E, int32_t rank, const int32_t* counts,
                              cudaStream_t s);
cudaError_t launch_ep_dispatch(const EpPeers& p, int32_t R, int32_t E, int32_t rank, int64_t recv_rows,
                               const int32_t* table, const int32_t* offsets, const int32_t* perm_token,
                               const void* x, int64_t max_rows, int64_t row_bytes, int32_t* recv_offsets,
                               moe_diag* status, cudaStream_t s);
cudaError_t launch_ep_combine(const EpPeers& p, int32_t R, int32_t E, int32_t rank, int64_t recv_rows,
                              const int32_t* table, const int32_t* offsets, const int32_t* topk_idx,
                              const int32_t* slot_dest, const float* topk_w, const void* sh, int64_t n, int32_t k,
                              int32_t d, int dtype, void* y, cudaStream_t s);
cudaError_t launch_ep_barrier(const EpPeers& p, int32_t R, int32_t rank, uint64_t timeout_ns, moe_diag* status,
                              cudaStream_t s);

// Small utilities.
cudaError_t launch_fill_i32(int32_t* p, int64_t count, int32_t value, cudaStream_t s);
cudaError_t launch_set_offsets2(int32_t* p, int64_t n, cudaStream_t s);

}  // namespace moe
