// capacity.cu -- the expert-capacity rule on many SMs at once.
//
// Rule (page "1.8T parameters / 2% per token", section 2.2: an expert takes at
// most C tokens per batch and the excess is forced to the next-best expert;
// section 4.2: drop_tokens): tokens in order, first come first served.
//   OVERFLOW_NEXT: token t takes the first k experts of its ranking that are
//                  not full at its turn;
//   DROP:          token t keeps its top k, and a slot whose expert is full at
//                  its turn is dropped.
// Every kept slot adds one to its expert's count; an expert is full at C.
//
// Between two fill events every token's choice depends only on the set F of
// full experts. The tokens are cut into ranges of 1024, one per CTA, one token
// per thread; a CTA resolves its own range like the one-CTA kernel does a
// window: it counts its tokens' choices, finds the first token at which some
// expert reaches C (ballot prefixes in token order), commits up to it, marks
// the expert full, lets the later tokens walk on, and repeats. The counts and
// full set it starts from are its predecessor's final ones, handed over
// through a flag (release/acquire); while it waits, its tokens' rankings are
// already staged and their choices taken under no full expert, so only the
// tokens that held an expert filled upstream walk on afterwards. The grid is
// launched cooperatively (every CTA resident, so a wait always ends), and
// every wait is bounded.
#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace moe {
namespace {

using namespace ptx;

constexpr unsigned kFull = 0xFFFFFFFFu;
constexpr int kThreads = 1024;  // tokens per CTA
constexpr uint64_t kBarrierTimeoutNs = 2000000000ull;
constexpr int kPrefix = 64;  // ranking entries per token staged in shared memory
constexpr size_t kMaxDynSmem = 200 * 1024;  // dynamic shared memory of the largest grid

// 32-bit words per staged ranking prefix of P entries: enough for P and odd, so that lanes reading
// the same position of their rows hit 32 different banks.
__host__ __device__ constexpr int prefix_words(int P) { return ((P + 1) / 2) | 1; }

// State handed from CTA b to CTA b + 1: the counts and the full set after CTA b's tokens, and a
// flag (0: not yet, 1: ready, 2: the chain was abandoned upstream).
struct ChainState {
  int32_t flag;
  uint32_t full[kMaxExperts / 32];
  int32_t cnt[kMaxExperts];
};
__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Bounded wait (thread 0) for the predecessor's state; false if it never came or was abandoned.
__device__ bool wait_for(const ChainState* prev, moe_diag* status) {
  const uint64_t t0 = globaltimer();
  for (;;) {
    const uint32_t f = ld_acquire(reinterpret_cast<const uint32_t*>(&prev->flag));
    if (f == 1) return true;
    if (f == 2) return false;
    if (globaltimer() - t0 > kBarrierTimeoutNs) {
      set_status(status, MOE_ERR_TIMEOUT);
      return false;
    }
    __nanosleep(32);
  }
}

// counts[e] += 1 for every lane whose slot holds e (e < 0: nothing), one shared-memory atomic per
// distinct expert in the warp.
__device__ __forceinline__ void warp_count(int* counts, int e) {
  const unsigned peers = __match_any_sync(kFull, e);
  if (e >= 0 && (threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&counts[e], __popc(peers));
}

// A token's current choices and their ranking positions (registers for k known at compile time).
template <int KA, bool REG>
struct Slots {
  int v[KA];
  __device__ __forceinline__ int get(int i) const {
    if constexpr (REG) {
      int r = -1;
#pragma unroll
      for (int q = 0; q < KA; ++q)
        if (q == i) r = v[q];
      return r;
    } else {
      return v[i];
    }
  }
  __device__ __forceinline__ void set(int i, int x) {
    if constexpr (REG) {
#pragma unroll
      for (int q = 0; q < KA; ++q)
        if (q == i) v[q] = x;
    } else {
      v[i] = x;
    }
  }
};

template <int KT>
__global__ void __launch_bounds__(kThreads) capacity_grid_kernel(CapacityArgs a, ChainState* chain) {
  constexpr int KA = KT > 0 ? KT : kMaxTopK;
  const int k = KT > 0 ? KT : a.k;
  const int E = a.E;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  __shared__ int cnt_s[kMaxExperts];   // counts so far (the predecessor's, then this range's commits)
  __shared__ int hist[kMaxExperts];        // choices of the uncommitted tokens, per expert
  __shared__ int hist_taken[kMaxExperts];  // choices of the tokens a round commits
  __shared__ uint32_t full_s[kMaxExperts / 32];
  __shared__ int cand[kMaxExperts];
  __shared__ int8_t cidx[kMaxExperts];   // place of an expert in cand (-1: not a candidate)
  __shared__ int n_cand;
  __shared__ uint32_t bal[32][kThreads / 32];  // per candidate of a batch: which tokens of each warp hold it
  __shared__ int s_stop;
  __shared__ int s_ok;
  __shared__ unsigned long long s_over, s_drop;
  extern __shared__ uint32_t srows[];  // the tokens' ranking prefixes (kPrefix entries, odd word stride)
  const int64_t t = (int64_t)blockIdx.x * kThreads + tid;
  const bool valid = t < a.n;
  const int cnt_tok = (int)((a.n - (int64_t)blockIdx.x * kThreads) < kThreads ? (a.n - (int64_t)blockIdx.x * kThreads)
                                                                               : kThreads);
  const uint16_t* row = a.ranking + (valid ? t : 0) * E;
  // the first P entries of this token's ranking in shared memory: a token walking past full experts
  // reads them at shared-memory latency instead of one dependent global load per step
  const int P = E < kPrefix ? E : kPrefix;
  uint32_t* srow32 = srows + tid * prefix_words(P);
  const uint16_t* srow = reinterpret_cast<const uint16_t*>(srow32);
  if (valid) {
    if (E % 8 == 0) {
      const uint4* src = reinterpret_cast<const uint4*>(row);
      for (int v = 0; v < P / 8; ++v) {
        const uint4 q4 = src[v];
        srow32[4 * v] = q4.x;
        srow32[4 * v + 1] = q4.y;
        srow32[4 * v + 2] = q4.z;
        srow32[4 * v + 3] = q4.w;
      }
    } else {
      uint16_t* d16 = reinterpret_cast<uint16_t*>(srow32);
      for (int c = 0; c < P; ++c) d16[c] = row[c];
    }
  }
  Slots<KA, (KT > 0)> ch, pos;
  int taken = 0, cursor = 0;
  unsigned long long my_over = 0, my_drop = 0;
  if (tid == 0) s_over = s_drop = 0;
  for (int w = tid; w < kMaxExperts / 32; w += kThreads) full_s[w] = 0;
  for (int e = tid; e < kMaxExperts; e += kThreads) cidx[e] = -1;
  __syncthreads();
  auto is_full = [&](int e) { return (full_s[e >> 5] >> (e & 31)) & 1u; };
  // walk on from the cursor until k non-full experts are held
  auto refill = [&]() {
    while (taken < k && cursor < E) {
      const int e = cursor < P ? srow[cursor] : row[cursor];
      if (e == 0xFFFF) {
        cursor = E;
        break;
      }
      if (!is_full(e)) {
        ch.set(taken, e);
        pos.set(taken, cursor);
        ++taken;
      }
      ++cursor;
    }
  };
  auto slot = [&](int j) {
    if (a.policy == MOE_CAP_OVERFLOW_NEXT) return j < taken ? ch.get(j) : -1;
    return ch.get(j);
  };
  // drop the experts that are full now; under OVERFLOW_NEXT walk on to replace them
  auto drop_full = [&]() -> bool {
    bool changed = false;
    if (a.policy == MOE_CAP_OVERFLOW_NEXT) {
      int kept = 0;
      for (int j = 0; j < k; ++j)
        if (j < taken) {
          const int cj = ch.get(j);
          if (!is_full(cj)) {
            const int pj = pos.get(j);
            ch.set(kept, cj);
            pos.set(kept, pj);
            ++kept;
          }
        }
      if (kept < taken) {
        taken = kept;
        refill();
        changed = true;
      }
    } else {
      for (int j = 0; j < k; ++j)
        if (ch.get(j) >= 0 && is_full(ch.get(j))) {
          ch.set(j, -1);
          changed = true;
        }
    }
    return changed;
  };
  // this token's choices in or out of the histogram
  auto count_mine = [&](int sign) {
    for (int j = 0; j < k; ++j) {
      const int e = slot(j);
      if (e >= 0) atomicAdd(&hist[e], sign);
    }
  };
  auto commit = [&]() {
    for (int j = 0; j < k; ++j) {
      const int e = slot(j);
      a.topk_idx[t * k + j] = e;
      my_drop += e < 0;
      if (a.policy == MOE_CAP_OVERFLOW_NEXT && j < taken) my_over += pos.get(j) >= k;
    }
  };
  // choices under no full expert, while the predecessor resolves its range
  if (valid) {
    if (a.policy == MOE_CAP_OVERFLOW_NEXT) {
      refill();
    } else {
      for (int j = 0; j < k; ++j) {
        const int e = j < P ? srow[j] : row[j];
        ch.set(j, e != 0xFFFF ? e : -1);
      }
    }
  }
  ChainState* mine = chain + blockIdx.x;
  // Full sets only grow along the chain, so the experts full after CTA b - 2 are full at this CTA's
  // turn too: its tokens walk past them while CTA b - 1 still works, and the histogram of the
  // resulting choices is taken before the last wait.
  if (blockIdx.x >= 2) {
    if (tid == 0) s_ok = wait_for(chain + blockIdx.x - 2, a.status) ? 1 : 0;
    __syncthreads();
    if (!s_ok) {
      if (tid == 0) atomicExch(&mine->flag, 2);  // abandon the rest of the chain at once
      return;
    }
    for (int w = tid; w < kMaxExperts / 32; w += kThreads) full_s[w] = __ldcg(&chain[blockIdx.x - 2].full[w]);
    __syncthreads();
    if (valid) drop_full();
  }
  for (int e = tid; e < E; e += kThreads) hist[e] = 0;
  __syncthreads();
  for (int j = 0; j < k; ++j) warp_count(hist, valid ? slot(j) : -1);
  // the predecessor's counts and full set (other CTAs wrote them: read from L2, not L1)
  if (tid == 0) s_ok = blockIdx.x == 0 ? 1 : (wait_for(chain + blockIdx.x - 1, a.status) ? 1 : 0);
  __syncthreads();
  if (!s_ok) {
    if (tid == 0) atomicExch(&mine->flag, 2);
    return;
  }
  if (blockIdx.x == 0) {
    for (int e = tid; e < kMaxExperts; e += kThreads) cnt_s[e] = 0;
  } else {
    const ChainState* prev = chain + blockIdx.x - 1;
    for (int e = tid; e < kMaxExperts; e += kThreads) cnt_s[e] = __ldcg(&prev->cnt[e]);
    for (int w = tid; w < kMaxExperts / 32; w += kThreads) full_s[w] = __ldcg(&prev->full[w]);
  }
  __syncthreads();
  // tokens that held an expert CTA b - 1 filled walk on; the histogram follows them
  if (valid) {
    Slots<KA, (KT > 0)> ch0 = ch;
    const int taken0 = taken;
    if (blockIdx.x > 0 && drop_full()) {
      for (int j = 0; j < k; ++j) {
        const int e = a.policy == MOE_CAP_OVERFLOW_NEXT ? (j < taken0 ? ch0.get(j) : -1) : ch0.get(j);
        if (e >= 0) atomicSub(&hist[e], 1);
      }
      count_mine(1);
    }
  }
  // from here on hist holds the choices of every uncommitted token of the range
  int f = 0;  // first token of the range not committed yet (uniform across the CTA)
  for (;;) {
    const bool active = valid && tid >= f;
    if (tid == 0) {
      n_cand = 0;
      s_stop = kThreads;
    }
    __syncthreads();
    for (int e = tid; e < E; e += kThreads)
      if (!is_full(e) && cnt_s[e] + hist[e] >= a.C) {
        const int c = atomicAdd(&n_cand, 1);
        cand[c] = e;
        cidx[e] = (int8_t)(c < 127 ? c : 127);
      }
    __syncthreads();
    const int nc = n_cand;
    // The token at which each candidate expert reaches C: its (C - count)-th chooser in token
    // order. Candidates go 32 at a time: every warp ballots all of them, then warp q finds
    // candidate q's chooser with a prefix over the warps' counts.
    for (int c0 = 0; c0 < nc; c0 += 32) {
      const int nb = nc - c0 < 32 ? nc - c0 : 32;
      uint32_t held = 0;  // bit q: this token holds candidate c0 + q
      if (active)
        for (int j = 0; j < k; ++j) {
          const int e = slot(j);
          if (e >= 0) {
            const int q = nc <= 127 ? (int)cidx[e] - c0 : -1;
            if (q >= 0 && q < nb && cand[c0 + q] == e) {
              held |= 1u << q;
            } else if (nc > 127) {
              for (int qq = 0; qq < nb; ++qq) held |= cand[c0 + qq] == e ? 1u << qq : 0u;
            }
          }
        }
      for (int q = 0; q < nb; ++q) {
        const uint32_t b = __ballot_sync(kFull, (held >> q) & 1u);
        if (lane == 0) bal[q][wid] = b;
      }
      __syncthreads();
      if (wid < nb) {
        const int e = cand[c0 + wid];
        const int need = (int)(a.C - cnt_s[e]);
        const uint32_t bw = bal[wid][lane];
        const int pc = __popc(bw);
        int incl = pc;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const int v = __shfl_up_sync(kFull, incl, off);
          if (lane >= off) incl += v;
        }
        if (incl - pc < need && need <= incl) {
          uint32_t bb = bw;
          for (int q = 1; q < need - (incl - pc); ++q) bb &= bb - 1;
          atomicMin(&s_stop, lane * 32 + __ffs(bb) - 1);
        }
      }
      __syncthreads();
    }
    for (int c = tid; c < nc; c += kThreads) cidx[cand[c]] = -1;
    const int stop = s_stop;  // last token committed in this step (kThreads: the rest of the range)
    const bool take = active && tid <= stop;
    if (stop < kThreads) {
      // the committed tokens' counts; hist keeps those of the tokens after them
      for (int e = tid; e < E; e += kThreads) hist_taken[e] = 0;
      __syncthreads();
      for (int j = 0; j < k; ++j) warp_count(hist_taken, take ? slot(j) : -1);
      __syncthreads();
    }
    if (take) commit();
    for (int e = tid; e < E; e += kThreads) {
      if (stop < kThreads) {
        cnt_s[e] += hist_taken[e];
        hist[e] -= hist_taken[e];
      } else {
        cnt_s[e] += hist[e];
      }
      if (cnt_s[e] >= a.C) atomicOr(&full_s[e >> 5], 1u << (e & 31));
    }
    __syncthreads();
    if (stop >= cnt_tok - 1) break;
    f = stop + 1;
    // the later tokens holding the expert that just filled walk on; the histogram follows them,
    // so the next round needs no recount
    if (valid && tid >= f) {
      Slots<KA, (KT > 0)> ch0 = ch;
      const int taken0 = taken;
      if (drop_full()) {
        for (int j = 0; j < k; ++j) {
          const int e = a.policy == MOE_CAP_OVERFLOW_NEXT ? (j < taken0 ? ch0.get(j) : -1) : ch0.get(j);
          if (e >= 0) atomicSub(&hist[e], 1);
        }
        count_mine(1);
      }
    }
  }
  // hand the counts and full set on
  for (int e = tid; e < kMaxExperts; e += kThreads) mine->cnt[e] = cnt_s[e];
  for (int w = tid; w < kMaxExperts / 32; w += kThreads) mine->full[w] = full_s[w];
  __threadfence();
  __syncthreads();
  if (tid == 0) atomicExch(&mine->flag, 1);
  atomicAdd(&s_over, my_over);
  atomicAdd(&s_drop, my_drop);
  __syncthreads();
  if (tid == 0 && a.diag) {
    atomicAdd(&a.diag->overflowed, (int32_t)s_over);
    atomicAdd(&a.diag->dropped, (int32_t)s_drop);
  }
}

// Dynamic shared memory: the staged ranking prefixes of the CTA's tokens.
size_t dyn_smem(unsigned grid, int E) {
  (void)grid;
  const int P = E < kPrefix ? E : kPrefix;
  return (size_t)kThreads * prefix_words(P) * sizeof(uint32_t);
}

template <int KT>
cudaError_t launch_t(CapacityArgs a, ChainState* g, unsigned grid, cudaStream_t s) {
  static std::atomic<uint64_t> attr{0};
  const size_t smem = dyn_smem(grid, a.E);
  if (smem > 48 * 1024) {
    // the largest grid capacity_grid_fits accepts (static shared memory comes on top)
    const cudaError_t e = set_smem_limit(attr, (const void*)capacity_grid_kernel<KT>, kMaxDynSmem);
    if (e != cudaSuccess) return e;
  }
  void* args[] = {&a, &g};
  return cudaLaunchCooperativeKernel((const void*)capacity_grid_kernel<KT>, dim3(grid), dim3(kThreads), args, smem, s);
}

// CTAs of the kernel that fit on the current device at once (queried once per device).
// CTAs of the kernel that fit on the current device at once: one per SM (1024 threads at up to 64
// registers fill an SM's register file), so the SM count, read once per device.
int resident_blocks() {
  constexpr int kMaxDevices = 64;
  static std::atomic<int> cached[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 0;
  if (dev < kMaxDevices && cached[dev].load() > 0) return cached[dev].load();
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) return 0;
  if (dev < kMaxDevices) cached[dev].store(sms);
  return sms;
}

}  // namespace

int64_t capacity_grid_scratch_bytes(int64_t n, int32_t E) {
  (void)E;
  return ceil_div(n, kThreads) * (int64_t)sizeof(ChainState);
}

bool capacity_grid_fits(int64_t n, int32_t E) {
  const int64_t blocks = ceil_div(n, kThreads);
  // one CTA per SM, and every CTA's count row in shared memory next to the static arrays
  return blocks >= 1 && blocks <= resident_blocks() && dyn_smem((unsigned)blocks, E) <= kMaxDynSmem;
}

cudaError_t launch_capacity_grid(const CapacityArgs& a, void* scratch, cudaStream_t s) {
  if (a.n <= 0) return cudaSuccess;
  if (reinterpret_cast<uintptr_t>(scratch) % 16) return cudaErrorInvalidValue;
  ChainState* g = static_cast<ChainState*>(scratch);
  CapacityArgs b = a;
  const unsigned grid = (unsigned)ceil_div(a.n, kThreads);
  cudaError_t e = cudaMemsetAsync(g, 0, (size_t)grid * sizeof(ChainState), s);  // every flag 0
  if (e != cudaSuccess) return e;
  switch (a.k) {
    case 1: return launch_t<1>(b, g, grid, s);
    case 2: return launch_t<2>(b, g, grid, s);
    case 4: return launch_t<4>(b, g, grid, s);
    case 8: return launch_t<8>(b, g, grid, s);
    default: return launch_t<0>(b, g, grid, s);
  }
}

}  // namespace moe
