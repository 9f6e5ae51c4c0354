// ep.cu -- expert parallelism over R ranks: rank q owns the routed experts
// [q E/R, (q+1) E/R) (page "15. DeepSeek: MLA, MoE and MTP", section "V3 MoE:
// how 8 of 256 experts are chosen": one expert group per node; page "MoE
// architecture revealed", section 4.2: experts spread evenly over the GPUs, the
// routing decision known to all of them).
//
// Exchange steps of one layer, each a kernel that takes every rank's buffer as
// a pointer (its own memory for the calling rank, a peer mapping otherwise):
//   publish   the rank's per-expert slot counts into row `rank` of every
//             rank's [R, E] count table;
//   dispatch  each kept slot's token row, pushed with 16-byte stores straight
//             into the owner's receive buffer (no local permuted copy);
//   combine   y[t] = sum_j w[t, j] * out_{owner}[row] + shared(x[t]), the
//             expert rows pulled from the owners' output buffers;
//   barrier   flag words with a bounded wait between the steps (one rank per
//             process); all ranks driven by one process on one device run the
//             steps in stream order instead.
// Receive layout at owner q: its experts in order; inside an expert, the
// source ranks in order; inside a source, that rank's stable slot order. With
// the ranks' tokens concatenated in rank order this is the single-device
// stable permutation restricted to q's experts, so every expert sees its rows
// in the same order as on one device.
#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

constexpr int kEpThreads = 256;

// For source rank s: base[e] = first receive row (at e's owner) of s's slots with expert e;
// total[q] = rows owner q receives from all ranks. T is the [R, E] count table.
__device__ void recv_bases(const int32_t* T, int R, int E, int s, int32_t* col, int32_t* base, int32_t* total) {
  const int Eq = E / R;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int c = 0;
    for (int r = 0; r < R; ++r) c += T[(int64_t)r * E + e];
    col[e] = c;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int q0 = (e / Eq) * Eq;
    int b = 0;
    for (int f = q0; f < e; ++f) b += col[f];
    for (int r = 0; r < s; ++r) b += T[(int64_t)r * E + e];
    base[e] = b;
  }
  for (int q = threadIdx.x; q < R; q += blockDim.x) {
    int t = 0;
    for (int f = q * Eq; f < (q + 1) * Eq; ++f) t += col[f];
    total[q] = t;
  }
  __syncthreads();
}

__global__ void ep_publish_kernel(EpPeers peers, int R, int E, int rank, const int32_t* counts) {
  for (int i = threadIdx.x; i < R * E; i += blockDim.x) {
    const int q = i / E, e = i % E;
    peers.counts[q][(int64_t)rank * E + e] = counts[e];
  }
  __threadfence_system();
}

// One warp per locally permuted row r: source token perm_token[r], expert e (from the local
// offsets), pushed to row base[e] + (r - offsets[e]) of the owner's receive buffer. Block 0 also
// writes this rank's own receive offsets (its experts' row ranges, clamped to recv_rows).
__global__ void __launch_bounds__(kEpThreads)
    ep_dispatch_kernel(EpPeers peers, int R, int E, int rank, int64_t recv_rows, const int32_t* T,
                       const int32_t* offsets, const int32_t* perm_token, const uint4* x, int64_t vec_per_row,
                       int32_t* recv_offsets, moe_diag* status) {
  __shared__ int32_t col[kMaxExperts], base[kMaxExperts], total[kMaxEpRanks], off[kMaxExperts + 1];
  for (int e = threadIdx.x; e <= E; e += blockDim.x) off[e] = offsets[e];
  recv_bases(T, R, E, rank, col, base, total);
  const int Eq = E / R;
  if (blockIdx.x == 0) {
    if (threadIdx.x == 0) {
      int acc = 0;
      for (int i = 0; i < Eq; ++i) {
        recv_offsets[i] = (int32_t)(acc < recv_rows ? acc : recv_rows);
        acc += col[rank * Eq + i];
      }
      recv_offsets[Eq] = (int32_t)(acc < recv_rows ? acc : recv_rows);
      for (int q = 0; q < R; ++q)
        if (total[q] > recv_rows) set_status(status, MOE_ERR_WORKSPACE);
    }
  }
  const int64_t rows = off[E];
  const int lane = threadIdx.x & 31;
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t r = warp; r < rows; r += nw) {
    int lo = 0, hi = E - 1;  // expert of row r: last e with off[e] <= r
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (off[mid] <= r) lo = mid; else hi = mid - 1;
    }
    const int e = lo;
    const int64_t dst = base[e] + (r - off[e]);
    if (dst >= recv_rows) continue;  // reported above; the owner's receive buffer is too small
    const uint4* src = x + (int64_t)perm_token[r] * vec_per_row;
    uint4* out = static_cast<uint4*>(peers.recv_x[e / Eq]) + dst * vec_per_row;
    for (int64_t v = lane; v < vec_per_row; v += 32) out[v] = __ldg(src + v);
  }
  __threadfence_system();
}

// y[t] = sum_j w[t, j] * out_owner(e_j)[row_j] (+ sh[t]) in binary32, slot order then shared:
// the same order as the single-device combine.
template <typename T>
__global__ void __launch_bounds__(kEpThreads)
    ep_combine_kernel(EpPeers peers, int R, int E, int rank, int64_t recv_rows, const int32_t* Tc,
                      const int32_t* offsets, const int32_t* topk_idx, const int32_t* slot_dest,
                      const float* topk_w, const T* sh, int64_t n, int k, int d, T* y) {
  __shared__ int32_t col[kMaxExperts], base[kMaxExperts], total[kMaxEpRanks], off[kMaxExperts + 1];
  for (int e = threadIdx.x; e <= E; e += blockDim.x) off[e] = offsets[e];
  recv_bases(Tc, R, E, rank, col, base, total);
  const int Eq = E / R;
  constexpr int V = 16 / sizeof(T);
  const int vpr = d / V;
  const int64_t work = n * vpr;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < work; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = i / vpr;
    const int c = (int)(i % vpr) * V;
    float acc[V];
#pragma unroll
    for (int q = 0; q < V; ++q) acc[q] = 0.0f;
    for (int j = 0; j < k; ++j) {
      const int pos = slot_dest[t * k + j];
      if (pos < 0) continue;
      const int e = topk_idx[t * k + j];
      const int64_t row = base[e] + (pos - off[e]);
      if (row >= recv_rows) continue;
      const float w = topk_w[t * k + j];
      const T* src = static_cast<const T*>(peers.recv_out[e / Eq]);
      const uint4 v = *reinterpret_cast<const uint4*>(src + row * d + c);
      const T* vs = reinterpret_cast<const T*>(&v);
#pragma unroll
      for (int q = 0; q < V; ++q) acc[q] = fmaf(w, to_f32(vs[q]), acc[q]);
    }
    if (sh) {
      const uint4 v = *reinterpret_cast<const uint4*>(sh + t * d + c);
      const T* vs = reinterpret_cast<const T*>(&v);
#pragma unroll
      for (int q = 0; q < V; ++q) acc[q] += to_f32(vs[q]);
    }
    uint4 out;
    T* os = reinterpret_cast<T*>(&out);
#pragma unroll
    for (int q = 0; q < V; ++q) os[q] = from_f32<T>(acc[q]);
    *reinterpret_cast<uint4*>(y + t * d + c) = out;
  }
}

__device__ __forceinline__ uint64_t ep_globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void st_release_sys(uint32_t* p, uint32_t v) {
  asm volatile("st.release.sys.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t ld_acquire_sys(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Barrier of one rank: flags[q][rank] = epoch for every q, then wait (bounded) until every
// flags[rank][q] has reached the epoch. flags[rank][R] is this rank's epoch counter (only it
// writes there). A rank whose status word already holds an error does not wait.
__global__ void ep_barrier_kernel(EpPeers peers, int R, int rank, uint64_t timeout_ns, moe_diag* status) {
  __shared__ uint32_t epoch;
  uint32_t* mine = peers.flags[rank];
  if (threadIdx.x == 0) {
    epoch = mine[R] + 1u;
    mine[R] = epoch;
  }
  __syncthreads();
  const uint32_t ep = epoch;
  const int q = threadIdx.x;
  if (q >= R) return;
  __threadfence_system();
  st_release_sys(peers.flags[q] + rank, ep);
  const bool failed = *reinterpret_cast<volatile int32_t*>(&status->status) != 0;
  if (failed) return;
  const uint64_t t0 = ep_globaltimer();
  for (uint32_t it = 0;; ++it) {
    if ((int32_t)(ld_acquire_sys(mine + q) - ep) >= 0) break;
    if ((it & 63u) == 63u && ep_globaltimer() - t0 > timeout_ns) {
      set_status(status, MOE_ERR_TIMEOUT);
      break;
    }
  }
  __threadfence_system();
}

unsigned ep_grid(int64_t work, int per_block) {
  const int64_t b = ceil_div(work, per_block);
  return (unsigned)(b < 148 * 16 ? (b > 0 ? b : 1) : 148 * 16);
}

}  // namespace

cudaError_t launch_ep_publish(const EpPeers& p, int32_t R, int32_t E, int32_t rank, const int32_t* counts,
                              cudaStream_t s) {
  ep_publish_kernel<<<1, kEpThreads, 0, s>>>(p, R, E, rank, counts);
  return cudaGetLastError();
}

cudaError_t launch_ep_dispatch(const EpPeers& p, int32_t R, int32_t E, int32_t rank, int64_t recv_rows,
                               const int32_t* table, const int32_t* offsets, const int32_t* perm_token,
                               const void* x, int64_t max_rows, int64_t row_bytes, int32_t* recv_offsets,
                               moe_diag* status, cudaStream_t s) {
  const unsigned grid = ep_grid(max_rows * 32, kEpThreads);
  ep_dispatch_kernel<<<grid, kEpThreads, 0, s>>>(p, R, E, rank, recv_rows, table, offsets, perm_token,
                                                 static_cast<const uint4*>(x), row_bytes / 16, recv_offsets, status);
  return cudaGetLastError();
}

cudaError_t launch_ep_combine(const EpPeers& p, int32_t R, int32_t E, int32_t rank, int64_t recv_rows,
                              const int32_t* table, const int32_t* offsets, const int32_t* topk_idx,
                              const int32_t* slot_dest, const float* topk_w, const void* sh, int64_t n, int32_t k,
                              int32_t d, int dtype, void* y, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  const int V = dtype == MOE_F32 ? 4 : 8;
  const unsigned grid = ep_grid(n * (d / V), kEpThreads);
  if (dtype == MOE_F32)
    ep_combine_kernel<float><<<grid, kEpThreads, 0, s>>>(p, R, E, rank, recv_rows, table, offsets, topk_idx,
                                                         slot_dest, topk_w, static_cast<const float*>(sh), n, k, d,
                                                         static_cast<float*>(y));
  else
    ep_combine_kernel<bf16><<<grid, kEpThreads, 0, s>>>(p, R, E, rank, recv_rows, table, offsets, topk_idx,
                                                        slot_dest, topk_w, static_cast<const bf16*>(sh), n, k, d,
                                                        static_cast<bf16*>(y));
  return cudaGetLastError();
}

cudaError_t launch_ep_barrier(const EpPeers& p, int32_t R, int32_t rank, uint64_t timeout_ns, moe_diag* status,
                              cudaStream_t s) {
  ep_barrier_kernel<<<1, 32, 0, s>>>(p, R, rank, timeout_ns, status);
  return cudaGetLastError();
}

}  // namespace moe
