// dispatch.cu -- per-expert histogram, exclusive scan, stable permutation and
// row gather; the gate-weighted combine; small utilities.
//
// Position of slot (t, j) with expert e = offsets[e] + number of earlier slots
// (t' < t) with expert e, i.e. a stable counting sort of the flattened slots
// a = t*k + j by expert (a token holds an expert at most once, so the order
// of slots inside one token never matters). No global atomics: each block
// counts a fixed range of slots, a single block scans the per-block counts,
// and each block then ranks its slots with warp match/ballot prefix counts.
#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

constexpr int kItems = 2048;   // slots per dispatch block
constexpr int kThreads = 256;  // 8 warps; a block walks its slots in rounds of 256

__global__ void __launch_bounds__(kThreads) count_kernel(const int32_t* idx, int64_t total, int E,
                                                       int32_t* blk_counts) {
  __shared__ int cnt[kMaxExperts];
  for (int e = threadIdx.x; e < E; e += kThreads) cnt[e] = 0;
  __syncthreads();
  const int64_t a0 = (int64_t)blockIdx.x * kItems;
  for (int i = threadIdx.x; i < kItems; i += kThreads) {
    const int64_t a = a0 + i;
    if (a < total) {
      const int e = idx[a];
      if (e >= 0) atomicAdd(&cnt[e], 1);
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += kThreads) blk_counts[(int64_t)blockIdx.x * E + e] = cnt[e];
}

// One block: per-expert exclusive scan over blocks (in place), then over experts. Thread e reads
// eight blocks' counts before it writes their bases, so the walk over blocks costs a few memory
// latencies; the scan over experts is a warp-shuffle scan.
__global__ void __launch_bounds__(kMaxExperts) scan_kernel(int32_t* blk_counts, int nblk, int E, int32_t* counts,
                                                         int32_t* offsets, moe_diag* diag) {
  constexpr int B = 8;
  __shared__ int warp_tot[kMaxExperts / 32], warp_max[kMaxExperts / 32];
  const int e = threadIdx.x, lane = e & 31, wid = e >> 5;
  int run = 0;
  if (e < E) {
    for (int b0 = 0; b0 < nblk; b0 += B) {
      int c[B];
#pragma unroll
      for (int q = 0; q < B; ++q) c[q] = b0 + q < nblk ? blk_counts[(int64_t)(b0 + q) * E + e] : 0;
#pragma unroll
      for (int q = 0; q < B; ++q)
        if (b0 + q < nblk) {
          blk_counts[(int64_t)(b0 + q) * E + e] = run;
          run += c[q];
        }
    }
    if (counts) counts[e] = run;
  }
  // exclusive scan of the per-expert totals in expert order, and their maximum
  int incl = run, mx = run;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int v = __shfl_up_sync(0xFFFFFFFFu, incl, off);
    if (lane >= off) incl += v;
    mx = max(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, off));
  }
  if (lane == 31) warp_tot[wid] = incl;
  if (lane == 0) warp_max[wid] = mx;
  __syncthreads();
  int base = 0, total = 0, gmax = 0;
  for (int w = 0; w < kMaxExperts / 32; ++w) {
    base += w < wid ? warp_tot[w] : 0;
    total += warp_tot[w];
    gmax = max(gmax, warp_max[w]);
  }
  if (e < E) offsets[e] = base + incl - run;
  if (e == 0) {
    offsets[E] = total;
    if (diag) diag->max_load = gmax;
  }
}

__global__ void __launch_bounds__(kThreads) scatter_kernel(const int32_t* idx, int64_t total, int k, int E,
                                                         const int32_t* blk_base, const int32_t* offsets,
                                                         int32_t* perm_token, int32_t* slot_dest) {
  __shared__ int run[kMaxExperts];
  __shared__ int wc[kThreads / 32][kMaxExperts];
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  for (int e = tid; e < E; e += kThreads) run[e] = offsets[e] + blk_base[(int64_t)blockIdx.x * E + e];
  const int64_t a0 = (int64_t)blockIdx.x * kItems;
  for (int r0 = 0; r0 < kItems; r0 += kThreads) {
    for (int i = tid; i < (kThreads / 32) * E; i += kThreads) (&wc[0][0])[(i / E) * kMaxExperts + i % E] = 0;
    __syncthreads();
    const int64_t a = a0 + r0 + tid;
    const int e = a < total ? idx[a] : -1;
    const unsigned peers = __match_any_sync(0xFFFFFFFFu, e);
    const int rank_in_warp = __popc(peers & ((1u << lane) - 1u));
    if (e >= 0 && rank_in_warp == 0) wc[wid][e] = __popc(peers);
    __syncthreads();
    if (a < total) {
      if (e >= 0) {
        int pos = run[e] + rank_in_warp;
        for (int w = 0; w < wid; ++w) pos += wc[w][e];
        perm_token[pos] = (int32_t)(a / k);
        slot_dest[a] = pos;
      } else {
        slot_dest[a] = -1;
      }
    }
    __syncthreads();
    for (int x = tid; x < E; x += kThreads) {
      int s = 0;
      for (int w = 0; w < kThreads / 32; ++w) s += wc[w][x];
      run[x] += s;
    }
    __syncthreads();
  }
}

// x_perm[slot_dest[t, j]] = x[t] for every kept slot (slot_dest >= 0), token-major: one warp per
// token reads its row once (16-byte vectors, four per lane in flight) and writes it to each of its
// k positions, so x crosses HBM once instead of once per slot.
__global__ void __launch_bounds__(256) permute_rows_kernel(const uint4* x, const int32_t* slot_dest, int64_t n,
                                                           int k, int64_t vec_per_row, uint4* x_perm) {
  constexpr int U = 4;
  const int lane = threadIdx.x & 31;
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t t = warp; t < n; t += nw) {
    const int mine = lane < k ? slot_dest[t * k + lane] : -1;
    const uint4* src = x + t * vec_per_row;
    for (int64_t v0 = lane; v0 < vec_per_row; v0 += 32 * U) {
      uint4 val[U];
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (v0 + 32 * u < vec_per_row) val[u] = __ldg(src + v0 + 32 * u);
      for (int j = 0; j < k; ++j) {
        const int p = __shfl_sync(0xffffffffu, mine, j);
        if (p < 0) continue;  // a slot the capacity rule dropped
        uint4* dst = x_perm + (int64_t)p * vec_per_row;
#pragma unroll
        for (int u = 0; u < U; ++u)
          if (v0 + 32 * u < vec_per_row) dst[v0 + 32 * u] = val[u];
      }
    }
  }
}

// y[t] = sum_j w[t, j] * eo[slot_dest[t, j]] (+ sh[t]), binary32, slot order then shared.
template <typename T>
__global__ void __launch_bounds__(256) combine_kernel(const T* eo, const int32_t* slot_dest, const float* topk_w,
                                                    const T* sh, int64_t n, int k, int d, T* y) {
  constexpr int V = 16 / sizeof(T);  // elements per 16-byte vector
  const int vpr = d / V;
  const int64_t total = n * vpr;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = i / vpr;
    const int c = (int)(i % vpr) * V;
    float acc[V];
#pragma unroll
    for (int q = 0; q < V; ++q) acc[q] = 0.0f;
    for (int j = 0; j < k; ++j) {
      const int pos = slot_dest[t * k + j];
      if (pos < 0) continue;
      const float w = topk_w[t * k + j];
      const uint4 v = *reinterpret_cast<const uint4*>(eo + (int64_t)pos * d + c);
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

__global__ void fill_i32_kernel(int32_t* p, int64_t count, int32_t v) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count; i += (int64_t)gridDim.x * blockDim.x)
    p[i] = v;
}

__global__ void set_offsets2_kernel(int32_t* p, int64_t n) {
  if (threadIdx.x == 0) {
    p[0] = 0;
    p[1] = (int32_t)n;
  }
}

unsigned grid_for(int64_t work, int per_block) {
  const int64_t b = ceil_div(work, per_block);
  return (unsigned)(b < 148 * 32 ? (b > 0 ? b : 1) : 148 * 32);
}

}  // namespace

int64_t dispatch_blocks(int64_t n, int32_t k) { return ceil_div(n * k, kItems); }

cudaError_t launch_scatter(const int32_t* topk_idx, int64_t n, int32_t k, int32_t E, const int32_t* blk_base,
                           const int32_t* offsets, int32_t* perm_token, int32_t* slot_dest, cudaStream_t s) {
  const int64_t nblk = dispatch_blocks(n, k);
  if (nblk > 0)
    scatter_kernel<<<(unsigned)nblk, kThreads, 0, s>>>(topk_idx, n * k, k, E, blk_base, offsets, perm_token, slot_dest);
  return cudaGetLastError();
}

cudaError_t launch_dispatch(const int32_t* topk_idx, int64_t n, int32_t k, int32_t E, int32_t* blk_counts,
                            int32_t* counts, int32_t* offsets, int32_t* perm_token, int32_t* slot_dest,
                            bool scatter, moe_diag* diag, cudaStream_t s) {
  const int64_t total = n * k;
  const int64_t nblk = dispatch_blocks(n, k);
  if (nblk > 0) count_kernel<<<(unsigned)nblk, kThreads, 0, s>>>(topk_idx, total, E, blk_counts);
  scan_kernel<<<1, kMaxExperts, 0, s>>>(blk_counts, (int)nblk, E, counts, offsets, diag);
  if (nblk > 0 && scatter)
    scatter_kernel<<<(unsigned)nblk, kThreads, 0, s>>>(topk_idx, total, k, E, blk_counts, offsets, perm_token,
                                                       slot_dest);
  return cudaGetLastError();
}

cudaError_t launch_permute_rows(const void* x, const int32_t* slot_dest, int64_t n, int32_t k, int64_t row_bytes,
                                void* x_perm, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  permute_rows_kernel<<<grid_for(n * 32, 256), 256, 0, s>>>(static_cast<const uint4*>(x), slot_dest, n, k,
                                                            row_bytes / 16, static_cast<uint4*>(x_perm));
  return cudaGetLastError();
}

cudaError_t launch_combine(const void* eo, const int32_t* slot_dest, const float* topk_w, const void* sh,
                           int64_t n, int32_t k, int32_t d, int dtype, void* y, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  const int V = dtype == MOE_F32 ? 4 : 8;
  const unsigned grid = grid_for(n * (d / V), 256);
  if (dtype == MOE_F32)
    combine_kernel<float><<<grid, 256, 0, s>>>(static_cast<const float*>(eo), slot_dest, topk_w,
                                                static_cast<const float*>(sh), n, k, d, static_cast<float*>(y));
  else
    combine_kernel<bf16><<<grid, 256, 0, s>>>(static_cast<const bf16*>(eo), slot_dest, topk_w,
                                               static_cast<const bf16*>(sh), n, k, d, static_cast<bf16*>(y));
  return cudaGetLastError();
}

cudaError_t launch_fill_i32(int32_t* p, int64_t count, int32_t value, cudaStream_t s) {
  if (count <= 0) return cudaSuccess;
  fill_i32_kernel<<<grid_for(count, 256), 256, 0, s>>>(p, count, value);
  return cudaGetLastError();
}

cudaError_t launch_set_offsets2(int32_t* p, int64_t n, cudaStream_t s) {
  set_offsets2_kernel<<<1, 32, 0, s>>>(p, n);
  return cudaGetLastError();
}

}  // namespace moe
