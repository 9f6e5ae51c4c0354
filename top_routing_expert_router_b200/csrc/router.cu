// router.cu -- scoring, group-limited top-k selection, gate weights and the
// expert-capacity rule. One warp per token: the E <= 256 logits of a token
// live in registers (EPL = E/32 per lane) and every selection step is a
// butterfly shuffle reduction.
//
// Definitions (page "15. DeepSeek: MLA, MoE and MTP", section "V3 MoE: how 8
// of 256 experts are chosen"; page "MoE architecture revealed", section 3.1;
// page "1.8T parameters / 2% per token", sections 2.2 and 4.1):
//   softmax: select on the logits l (softmax is increasing), gates
//            p_j = e^{l_j - m} / sum_E e^{l - m} (renormalised over the kept
//            slots when asked), times routed_scaling_factor;
//   sigmoid: s = sigmoid(l), c = s + bias (selection only); groups of E/G
//            experts scored by the sum of their two best c; the topk_group
//            best groups stay eligible; top-k of c among them; gates from s,
//            divided by their sum when asked, times routed_scaling_factor.
// Ties go to the lower expert (group) index; slots are in descending score.
//
// Exactness: logits arrive in binary32. A decision is certified when every
// gap it depends on exceeds twice the binary32 error bound delta (group cut:
// four times, a group score holds two values); otherwise the warp recomputes
// the token's logits in binary64 from x and W_r and decides again, so that the
// indices equal those of the binary64 definition.
#include <float.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

constexpr unsigned kFull = 0xFFFFFFFFu;
constexpr int kWarpsPerBlock = 8;

struct VE {
  double v;
  int e;
};

// Best of the warp: larger value, then lower index. Every lane gets the result.
__device__ __forceinline__ VE warp_best(VE x) {
#pragma unroll
  for (int off = 16; off; off >>= 1) {
    const double ov = __shfl_xor_sync(kFull, x.v, off);
    const int oe = __shfl_xor_sync(kFull, x.e, off);
    if (ov > x.v || (ov == x.v && oe < x.e)) {
      x.v = ov;
      x.e = oe;
    }
  }
  return x;
}

__device__ __forceinline__ double warp_max(double v) {
#pragma unroll
  for (int off = 16; off; off >>= 1) v = fmax(v, __shfl_xor_sync(kFull, v, off));
  return v;
}

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int off = 16; off; off >>= 1) v += __shfl_xor_sync(kFull, v, off);
  return v;
}

__device__ __forceinline__ double sigmoid_d(double z) { return 1.0 / (1.0 + exp(-z)); }

template <int EPL>
__device__ __forceinline__ double pick(const double (&r)[EPL], int j) {
  double out = 0.0;
#pragma unroll
  for (int i = 0; i < EPL; ++i)
    if (i == j) out = r[i];
  return out;
}

// Selection of one token. Writes the ranked experts to rank[0..R) (R = k, or
// every eligible expert when `full_ranking`). Returns false when `check` is set
// and some gap the decision depends on is within the binary32 error bound.
template <int EPL>
__device__ bool decide(const RouteArgs& a, const double (&l)[EPL], bool check, bool full_ranking,
                       int16_t* rank, int* n_ranked) {
  const int lane = threadIdx.x & 31;
  const int E = a.E;
  double v[EPL];
  bool valid[EPL];
  double amax = 0.0;
#pragma unroll
  for (int j = 0; j < EPL; ++j) {
    const int e = lane + 32 * j;
    valid[j] = e < E;
    if (valid[j]) {
      if (a.score_fn == MOE_SCORE_SIGMOID)
        v[j] = sigmoid_d(l[j]) + (a.bias ? (double)a.bias[e] : 0.0);
      else
        v[j] = l[j];
      amax = fmax(amax, fabs(l[j]));
    } else {
      v[j] = -INFINITY;
    }
  }
  double delta_v = 0.0;
  if (check) {
    amax = warp_max(amax);
    const double delta_l = ldexp(fmax(1.0, amax), -14);
    delta_v = a.score_fn == MOE_SCORE_SIGMOID ? 0.25 * delta_l : delta_l;
  }
  bool ok = true;

  // Group limit: keep the topk_group groups with the largest sum of two best scores.
  bool elig[EPL];
#pragma unroll
  for (int j = 0; j < EPL; ++j) elig[j] = valid[j];
  if (a.G > 1) {
    const int per = E / a.G;
    double gs[kMaxGroups];
    for (int g = 0; g < a.G; ++g) {
      double t1 = -INFINITY, t2 = -INFINITY;
#pragma unroll
      for (int j = 0; j < EPL; ++j) {
        const int e = lane + 32 * j;
        if (valid[j] && e / per == g) {
          if (v[j] > t1) {
            t2 = t1;
            t1 = v[j];
          } else if (v[j] > t2) {
            t2 = v[j];
          }
        }
      }
#pragma unroll
      for (int off = 16; off; off >>= 1) {
        const double o1 = __shfl_xor_sync(kFull, t1, off);
        const double o2 = __shfl_xor_sync(kFull, t2, off);
        const double hi = fmax(t1, o1);
        const double lo = fmax(fmin(t1, o1), fmax(t2, o2));
        t1 = hi;
        t2 = lo;
      }
      gs[g] = t1 + t2;
    }
    uint32_t keep = 0;
    double min_kept = INFINITY, max_drop = -INFINITY;
    for (int g = 0; g < a.G; ++g) {
      int better = 0;
      for (int h = 0; h < a.G; ++h) better += (gs[h] > gs[g]) || (gs[h] == gs[g] && h < g);
      if (better < a.topk_group) {
        keep |= 1u << g;
        min_kept = fmin(min_kept, gs[g]);
      } else {
        max_drop = fmax(max_drop, gs[g]);
      }
    }
    if (check && a.topk_group < a.G && !(min_kept - max_drop > 4.0 * delta_v)) ok = false;
#pragma unroll
    for (int j = 0; j < EPL; ++j) {
      const int e = lane + 32 * j;
      elig[j] = valid[j] && ((keep >> (e / per)) & 1u);
    }
  }

  // Ranked selection by repeated warp arg-max.
  int n_elig = 0;
#pragma unroll
  for (int j = 0; j < EPL; ++j) n_elig += elig[j];
#pragma unroll
  for (int off = 16; off; off >>= 1) n_elig += __shfl_xor_sync(kFull, n_elig, off);
  const int want = full_ranking ? n_elig : min(n_elig, check ? a.k + 1 : a.k);
  uint32_t taken = 0;
  double prev = 0.0;
  for (int r = 0; r < want; ++r) {
    VE best{-INFINITY, 0x7FFFFFFF};
#pragma unroll
    for (int j = 0; j < EPL; ++j) {
      const int e = lane + 32 * j;
      if (elig[j] && !((taken >> j) & 1u) && (v[j] > best.v || (v[j] == best.v && e < best.e))) {
        best.v = v[j];
        best.e = e;
      }
    }
    best = warp_best(best);
    if ((best.e & 31) == lane) taken |= 1u << (best.e >> 5);
    if (check && r > 0 && (full_ranking || r <= a.k) && !(prev - best.v > 2.0 * delta_v)) ok = false;
    prev = best.v;
    if (lane == 0 && (full_ranking || r < a.k)) rank[r] = (int16_t)best.e;
  }
  *n_ranked = full_ranking ? n_elig : min(n_elig, a.k);
  __syncwarp();
  return ok;
}

// Gate weights of the slots in idx[0..k) (entries < 0 are dropped slots).
// Lane j < k returns the weight of slot j.
template <int EPL>
__device__ float gates(const RouteArgs& a, const double (&l)[EPL], const int* idx_of_slot) {
  const int lane = threadIdx.x & 31;
  double m = -INFINITY;
  if (a.score_fn == MOE_SCORE_SOFTMAX) {
#pragma unroll
    for (int j = 0; j < EPL; ++j)
      if (lane + 32 * j < a.E) m = fmax(m, l[j]);
    m = warp_max(m);
  }
  double z = 0.0;
  if (a.score_fn == MOE_SCORE_SOFTMAX) {
#pragma unroll
    for (int j = 0; j < EPL; ++j)
      if (lane + 32 * j < a.E) z += exp(l[j] - m);
    z = warp_sum(z);
  }
  double mine = 0.0;
  for (int r = 0; r < a.k; ++r) {
    const int e = idx_of_slot[r];
    const int src = e >= 0 ? (e & 31) : 0;
    const double le = __shfl_sync(kFull, pick(l, e >= 0 ? (e >> 5) : 0), src);
    double p = 0.0;
    if (e >= 0) p = a.score_fn == MOE_SCORE_SOFTMAX ? exp(le - m) / z : sigmoid_d(le);
    if (lane == r) mine = p;
  }
  double denom = 1.0;
  if (a.renorm) denom = warp_sum(lane < a.k ? mine : 0.0);
  return (float)(mine / denom * (double)a.rsf);
}

template <int EPL>
__device__ void refine_logits(const RouteArgs& a, int64_t t, double (&l)[EPL]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int j = 0; j < EPL; ++j) {
    const int e = lane + 32 * j;
    double acc = 0.0;
    if (e < a.E) {
      if (a.dtype == MOE_BF16) {
        const uint4* xr = reinterpret_cast<const uint4*>(static_cast<const bf16*>(a.x) + t * a.d);
        const uint4* wr = reinterpret_cast<const uint4*>(static_cast<const bf16*>(a.w_r) + (int64_t)e * a.d);
        for (int i = 0; i < a.d / 8; ++i) {
          const uint4 xv = xr[i], wv = __ldg(wr + i);
          const bf16* xs = reinterpret_cast<const bf16*>(&xv);
          const bf16* ws = reinterpret_cast<const bf16*>(&wv);
#pragma unroll
          for (int q = 0; q < 8; ++q) acc = fma(to_f64(xs[q]), to_f64(ws[q]), acc);
        }
      } else {
        const float4* xr = reinterpret_cast<const float4*>(static_cast<const float*>(a.x) + t * a.d);
        const float4* wr = reinterpret_cast<const float4*>(static_cast<const float*>(a.w_r) + (int64_t)e * a.d);
        for (int i = 0; i < a.d / 4; ++i) {
          const float4 xv = xr[i], wv = __ldg(wr + i);
          acc = fma((double)xv.x, (double)wv.x, acc);
          acc = fma((double)xv.y, (double)wv.y, acc);
          acc = fma((double)xv.z, (double)wv.z, acc);
          acc = fma((double)xv.w, (double)wv.w, acc);
        }
      }
    }
    l[j] = acc;
  }
}

template <int EPL>
__global__ void __launch_bounds__(32 * kWarpsPerBlock) route_kernel(RouteArgs a) {
  __shared__ int16_t s_rank[kWarpsPerBlock][kMaxExperts];
  __shared__ int s_idx[kWarpsPerBlock][kMaxTopK];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const bool full_ranking = a.ranking != nullptr;
  for (int64_t t = warp; t < a.n; t += nwarps) {
    double l[EPL];
#pragma unroll
    for (int j = 0; j < EPL; ++j) {
      const int e = lane + 32 * j;
      l[j] = e < a.E ? (double)a.logits[t * a.E + e] : 0.0;
    }
    int nr = 0;
    bool ok = decide<EPL>(a, l, true, full_ranking, s_rank[wib], &nr);
    if (!ok) {
      refine_logits<EPL>(a, t, l);
      decide<EPL>(a, l, false, full_ranking, s_rank[wib], &nr);
      if (lane == 0 && a.diag) atomicAdd(&a.diag->refined_tokens, 1);
    }
    if (full_ranking) {
      for (int r = lane; r < a.E; r += 32) a.ranking[t * a.E + r] = r < nr ? (uint16_t)s_rank[wib][r] : (uint16_t)0xFFFF;
      continue;
    }
    if (lane < a.k) s_idx[wib][lane] = lane < nr ? (int)s_rank[wib][lane] : -1;
    __syncwarp();
    const float w = gates<EPL>(a, l, s_idx[wib]);
    if (lane < a.k) {
      a.topk_idx[t * a.k + lane] = s_idx[wib][lane];
      a.topk_w[t * a.k + lane] = w;
    }
    __syncwarp();
  }
}

// Gates of an existing selection (after the capacity rule), from binary32 logits.
template <int EPL>
__global__ void __launch_bounds__(32 * kWarpsPerBlock) gates_kernel(RouteArgs a) {
  __shared__ int s_idx[kWarpsPerBlock][kMaxTopK];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t t = warp; t < a.n; t += nwarps) {
    double l[EPL];
#pragma unroll
    for (int j = 0; j < EPL; ++j) {
      const int e = lane + 32 * j;
      l[j] = e < a.E ? (double)a.logits[t * a.E + e] : 0.0;
    }
    if (lane < a.k) s_idx[wib][lane] = a.topk_idx[t * a.k + lane];
    __syncwarp();
    const float w = gates<EPL>(a, l, s_idx[wib]);
    if (lane < a.k) a.topk_w[t * a.k + lane] = w;
    __syncwarp();
  }
}

// ---- capacity ------------------------------------------------------------------
// Token order, first come first served ("1.8T parameters / 2% per token",
// section 2.2). Between two fill events every token simply takes the first k
// non-full experts of its ranking, so the block evaluates a chunk of 1024
// tokens at once, finds the first token at which some expert reaches C,
// commits the chunk up to that token, marks the filled experts and continues
// after it. There are at most E fill events.
constexpr int kCapThreads = 1024;

__global__ void __launch_bounds__(kCapThreads) capacity_kernel(const uint16_t* ranking, int64_t n, int E, int k,
                                                            int64_t C, int policy, int32_t* topk_idx,
                                                            moe_diag* diag) {
  __shared__ int cnt[kMaxExperts];
  __shared__ int ccnt[kMaxExperts];
  __shared__ uint32_t full[kMaxExperts / 32];
  __shared__ uint32_t ballots[kCapThreads / 32];
  __shared__ int cand[kMaxExperts];
  __shared__ int n_cand;
  __shared__ int stop;
  __shared__ unsigned long long s_over, s_drop;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  for (int e = tid; e < kMaxExperts; e += kCapThreads) cnt[e] = 0;
  if (tid < kMaxExperts / 32) full[tid] = 0;
  if (tid == 0) s_over = s_drop = 0;
  __syncthreads();
  unsigned long long my_over = 0, my_drop = 0;
  int64_t base = 0;
  while (base < n) {
    const int64_t t = base + tid;
    const bool valid = t < n;
    int ch[kMaxTopK];
    int over = 0;
    for (int j = 0; j < k; ++j) ch[j] = -1;
    if (valid) {
      const uint16_t* rk = ranking + t * E;
      if (policy == MOE_CAP_OVERFLOW_NEXT) {
        int taken = 0;
        for (int r = 0; r < E && taken < k; ++r) {
          const int e = rk[r];
          if (e == 0xFFFF) break;
          if (!((full[e >> 5] >> (e & 31)) & 1u)) {
            ch[taken++] = e;
            over += r >= k;
          }
        }
      } else {
        for (int j = 0; j < k; ++j) {
          const int e = rk[j];
          ch[j] = (e != 0xFFFF && !((full[e >> 5] >> (e & 31)) & 1u)) ? e : -1;
        }
      }
    }
    for (int e = tid; e < E; e += kCapThreads) ccnt[e] = 0;
    if (tid == 0) {
      n_cand = 0;
      stop = kCapThreads;
    }
    __syncthreads();
    if (valid)
      for (int j = 0; j < k; ++j)
        if (ch[j] >= 0) atomicAdd(&ccnt[ch[j]], 1);
    __syncthreads();
    for (int e = tid; e < E; e += kCapThreads)
      if (cnt[e] < C && cnt[e] + ccnt[e] >= C) cand[atomicAdd(&n_cand, 1)] = e;
    __syncthreads();
    const int nc = n_cand;
    for (int c = 0; c < nc; ++c) {
      const int e = cand[c];
      bool mine = false;
      if (valid)
        for (int j = 0; j < k; ++j) mine |= ch[j] == e;
      const uint32_t b = __ballot_sync(kFull, mine);
      if (lane == 0) ballots[wid] = b;
      __syncthreads();
      if (tid == 0) {
        int need = (int)(C - cnt[e]);  // this expert's C-th slot is taken by the need-th chooser
        for (int w = 0; w < kCapThreads / 32; ++w) {
          const int pc = __popc(ballots[w]);
          if (need <= pc) {
            uint32_t bb = ballots[w];
            for (int q = 1; q < need; ++q) bb &= bb - 1;
            const int pos = w * 32 + __ffs(bb) - 1;
            if (pos < stop) stop = pos;
            break;
          }
          need -= pc;
        }
      }
      __syncthreads();
    }
    const int s = stop;  // relative index of the last committed token
    const bool commit = valid && tid <= s;
    if (commit) {
      for (int j = 0; j < k; ++j) topk_idx[t * k + j] = ch[j];
      my_over += over;
      for (int j = 0; j < k; ++j) my_drop += ch[j] < 0;
    }
    if (s < kCapThreads) {
      for (int e = tid; e < E; e += kCapThreads) ccnt[e] = 0;
      __syncthreads();
      if (commit)
        for (int j = 0; j < k; ++j)
          if (ch[j] >= 0) atomicAdd(&ccnt[ch[j]], 1);
      __syncthreads();
    }
    for (int e = tid; e < E; e += kCapThreads) {
      cnt[e] += ccnt[e];
      if (cnt[e] >= C) atomicOr(&full[e >> 5], 1u << (e & 31));
    }
    __syncthreads();
    base += s < kCapThreads ? (int64_t)s + 1 : (int64_t)kCapThreads;
  }
  atomicAdd(&s_over, my_over);
  atomicAdd(&s_drop, my_drop);
  __syncthreads();
  if (tid == 0 && diag) {
    diag->overflowed = (int32_t)s_over;
    diag->dropped = (int32_t)s_drop;
  }
}

int epl_for(int E) { return E <= 32 ? 1 : E <= 64 ? 2 : E <= 128 ? 4 : 8; }

unsigned route_grid(int64_t n) {
  const int64_t blocks = ceil_div(n, kWarpsPerBlock);
  return (unsigned)(blocks < 148 * 16 ? blocks : 148 * 16);
}

}  // namespace

cudaError_t launch_route(const RouteArgs& a, cudaStream_t s) {
  if (a.n <= 0) return cudaSuccess;
  const unsigned grid = route_grid(a.n);
  const unsigned block = 32 * kWarpsPerBlock;
  switch (epl_for(a.E)) {
    case 1: route_kernel<1><<<grid, block, 0, s>>>(a); break;
    case 2: route_kernel<2><<<grid, block, 0, s>>>(a); break;
    case 4: route_kernel<4><<<grid, block, 0, s>>>(a); break;
    default: route_kernel<8><<<grid, block, 0, s>>>(a); break;
  }
  return cudaGetLastError();
}

cudaError_t launch_gates(const RouteArgs& a, cudaStream_t s) {
  if (a.n <= 0) return cudaSuccess;
  const unsigned grid = route_grid(a.n);
  const unsigned block = 32 * kWarpsPerBlock;
  switch (epl_for(a.E)) {
    case 1: gates_kernel<1><<<grid, block, 0, s>>>(a); break;
    case 2: gates_kernel<2><<<grid, block, 0, s>>>(a); break;
    case 4: gates_kernel<4><<<grid, block, 0, s>>>(a); break;
    default: gates_kernel<8><<<grid, block, 0, s>>>(a); break;
  }
  return cudaGetLastError();
}

cudaError_t launch_capacity(const uint16_t* ranking, int64_t n, int32_t E, int32_t k, int64_t C, int policy,
                            int32_t* topk_idx, moe_diag* diag, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  capacity_kernel<<<1, kCapThreads, 0, s>>>(ranking, n, E, k, C, policy, topk_idx, diag);
  return cudaGetLastError();
}

}  // namespace moe
