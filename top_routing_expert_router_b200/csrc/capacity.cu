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
// full experts, so the rule is a sequence of rounds. In a round each CTA (one
// token per thread, a contiguous token range per CTA) counts the choices of its
// uncommitted tokens under F; after a grid barrier every CTA scans those counts
// in token order and finds the first CTA b* in whose range some expert reaches
// C; CTA b* finds the exact token t* by ballots in token order, sets the new
// counts and F; after a second barrier every token up to t* commits its choice
// and the later tokens drop the experts that filled (and, under OVERFLOW_NEXT,
// walk on down their rankings). A round without any expert reaching C commits
// everything. There are at most E fill events. The grid is launched
// cooperatively (every CTA resident), and every barrier wait is bounded.
#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace moe {
namespace {

using namespace ptx;

constexpr unsigned kFull = 0xFFFFFFFFu;
constexpr int kThreads = 1024;  // tokens per CTA
constexpr uint64_t kBarrierTimeoutNs = 2000000000ull;
constexpr int kNone = 0x7FFFFFFF;
constexpr int kPrefix = 64;  // ranking entries per token staged in shared memory
constexpr size_t kMaxDynSmem = 200 * 1024;  // dynamic shared memory of the largest grid

// 32-bit words per staged ranking prefix of P entries: enough for P and odd, so that lanes reading
// the same position of their rows hit 32 different banks.
__host__ __device__ constexpr int prefix_words(int P) { return ((P + 1) / 2) | 1; }

// Global state of one round, double-buffered by round parity (CTAs still reading round r's
// copy while CTA b* writes round r + 1's).
struct RoundState {
  int32_t fill_tok;  // last committed token of the round (n - 1: all)
  uint32_t full[kMaxExperts / 32];
  int32_t cnt[kMaxExperts];
};

struct GridCtl {
  uint32_t count;  // barrier arrivals
  uint32_t gen;    // barrier generation
  int32_t abort;
  int32_t pad;
  RoundState st[2];
};

__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Bounded grid barrier; false (uniform over the CTA) after a timeout or another CTA's abort.
__device__ bool grid_sync(GridCtl* g, uint32_t nblocks, uint32_t& gen, moe_diag* status) {
  __shared__ int s_ok;
  __syncthreads();
  if (threadIdx.x == 0) {
    int ok = 1;
    const uint32_t my = gen;
    __threadfence();
    if (atomicAdd(&g->count, 1u) == nblocks - 1) {
      atomicExch(&g->count, 0u);
      __threadfence();
      atomicExch(&g->gen, my + 1);
    } else {
      const uint64_t t0 = globaltimer();
      while (ld_acquire(&g->gen) == my) {
        if (*reinterpret_cast<volatile int32_t*>(&g->abort)) {
          ok = 0;
          break;
        }
        if (globaltimer() - t0 > kBarrierTimeoutNs) {
          atomicExch(&g->abort, 1);
          set_status(status, MOE_ERR_TIMEOUT);
          ok = 0;
          break;
        }
        __nanosleep(64);
      }
    }
    __threadfence();
    gen = my + 1;
    s_ok = ok;
  }
  __syncthreads();
  return s_ok != 0;
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
__global__ void __launch_bounds__(kThreads) capacity_grid_kernel(CapacityArgs a, GridCtl* g) {
  constexpr int KA = KT > 0 ? KT : kMaxTopK;
  const int k = KT > 0 ? KT : a.k;
  const int E = a.E;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  __shared__ int hist[kMaxExperts];
  __shared__ uint32_t full_s[kMaxExperts / 32];
  __shared__ int cross[kMaxExperts];  // CTA where expert e reaches C this round (kNone: nowhere)
  __shared__ int need[kMaxExperts];   // choosers of e in that CTA up to and including the filling one
  __shared__ uint32_t ballots[kThreads / 32];
  __shared__ int cnt_s[kMaxExperts];        // committed counts at the start of the round
  __shared__ uint32_t nfull_s[kMaxExperts / 32];
  __shared__ int s_bstar, s_tloc;
  __shared__ unsigned long long s_over, s_drop;
  extern __shared__ int hist_all[];           // [gridDim.x][E]: every CTA's counts of this round, then
                                              // the tokens' ranking prefixes (kPrefix entries, odd word stride)
  const int64_t t = (int64_t)blockIdx.x * kThreads + tid;
  const bool valid = t < a.n;
  const uint16_t* row = a.ranking + (valid ? t : 0) * E;
  // the first P entries of this token's ranking in shared memory: a token walking past full experts
  // reads them at shared-memory latency instead of one dependent global load per step
  const int P = E < kPrefix ? E : kPrefix;
  uint32_t* srow32 = reinterpret_cast<uint32_t*>(hist_all + gridDim.x * E) + tid * prefix_words(P);
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
  uint32_t gen = 0;
  Slots<KA, (KT > 0)> ch, pos;
  int taken = 0, cursor = 0;
  bool committed = !valid;
  unsigned long long my_over = 0, my_drop = 0;
  if (tid == 0) s_over = s_drop = 0;
  for (int w = tid; w < kMaxExperts / 32; w += kThreads) full_s[w] = 0;
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
  const uint32_t nblocks = gridDim.x;
  for (int r = 0;; ++r) {
    const RoundState& cur = g->st[r & 1];
    RoundState& nxt = g->st[(r + 1) & 1];
    // 1. this CTA's per-expert counts of the uncommitted choices
    for (int e = tid; e < E; e += kThreads) hist[e] = 0;
    __syncthreads();
    for (int j = 0; j < k; ++j) warp_count(hist, committed ? -1 : slot(j));
    __syncthreads();
    for (int e = tid; e < E; e += kThreads) a.hist[(int64_t)blockIdx.x * E + e] = hist[e];
    if (!grid_sync(g, nblocks, gen, a.status)) return;
    // 2. in token order over the CTAs: where does each non-full expert reach C?
    // (every CTA's row, the counts and the full set are read once, in parallel, from L2: other
    // CTAs wrote them, so never through a possibly stale L1 line)
    if (tid == 0) s_bstar = kNone;
    for (int i = tid; i < (int)nblocks * E; i += kThreads) hist_all[i] = __ldcg(&a.hist[i]);
    for (int e = tid; e < E; e += kThreads) cnt_s[e] = __ldcg(&cur.cnt[e]);
    for (int w = tid; w < kMaxExperts / 32; w += kThreads) nfull_s[w] = __ldcg(&cur.full[w]);
    __syncthreads();
    if (tid < E) {
      const int e = tid;
      int run = cnt_s[e];
      int cb = kNone, nd = 0;
      if (!((nfull_s[e >> 5] >> (e & 31)) & 1u)) {
        for (uint32_t b = 0; b < nblocks; ++b) {
          const int h = hist_all[b * E + e];
          if (run + h >= a.C) {
            cb = (int)b;
            nd = (int)(a.C - run);
            break;
          }
          run += h;
        }
      }
      cross[e] = cb;
      need[e] = nd;
      if (cb != kNone) atomicMin(&s_bstar, cb);
    }
    __syncthreads();
    const int bstar = s_bstar;
    // 3. CTA b*: the token at which the first expert fills, the counts up to it and the new F
    if ((int)blockIdx.x == bstar) {
      if (tid == 0) s_tloc = kNone;
      __syncthreads();
      for (int e = 0; e < E; ++e) {
        if (cross[e] != bstar) continue;
        bool mine = false;
        if (!committed)
          for (int j = 0; j < k; ++j) mine |= slot(j) == e;
        const uint32_t b = __ballot_sync(kFull, mine);
        if (lane == 0) ballots[wid] = b;
        __syncthreads();
        if (tid == 0) {
          int nd = need[e];
          for (int w = 0; w < kThreads / 32; ++w) {
            const int pc = __popc(ballots[w]);
            if (nd <= pc) {
              uint32_t bb = ballots[w];
              for (int q = 1; q < nd; ++q) bb &= bb - 1;
              const int at = w * 32 + __ffs(bb) - 1;
              if (at < s_tloc) s_tloc = at;
              break;
            }
            nd -= pc;
          }
        }
        __syncthreads();
      }
      const int tloc = s_tloc;
      for (int e = tid; e < E; e += kThreads) hist[e] = 0;
      __syncthreads();
      for (int j = 0; j < k; ++j) warp_count(hist, (!committed && tid <= tloc) ? slot(j) : -1);
      __syncthreads();
      // counts up to and including the filling token: the committed ones, every earlier CTA's
      // row, and this CTA's tokens up to it; an expert is full from C on
      if (tid < E) {
        const int e = tid;
        int c = cnt_s[e] + hist[e];
        for (int b = 0; b < bstar; ++b) c += hist_all[b * E + e];
        nxt.cnt[e] = c;
        if (c >= a.C) atomicOr(&nfull_s[e >> 5], 1u << (e & 31));
      }
      __syncthreads();
      for (int w = tid; w < kMaxExperts / 32; w += kThreads) nxt.full[w] = nfull_s[w];
      if (tid == 0) nxt.fill_tok = (int)((int64_t)blockIdx.x * kThreads + tloc);
    }
    if (bstar == kNone) {
      // no expert fills among the remaining tokens: everything commits as it stands
      if (!committed) {
        for (int j = 0; j < k; ++j) {
          const int e = slot(j);
          a.topk_idx[t * k + j] = e;
          my_drop += e < 0;
          if (a.policy == MOE_CAP_OVERFLOW_NEXT && j < taken) my_over += pos.get(j) >= k;
        }
        committed = true;
      }
      break;
    }
    if (!grid_sync(g, nblocks, gen, a.status)) return;
    // 4. commit up to the filling token; later tokens drop the experts that filled
    // other CTAs' writes are read from L2 (__ldcg), never from a stale L1 line
    const int64_t last = __ldcg(&nxt.fill_tok);
    for (int w = tid; w < kMaxExperts / 32; w += kThreads) full_s[w] = __ldcg(&nxt.full[w]);
    __syncthreads();
    if (!committed) {
      if (t <= last) {
        for (int j = 0; j < k; ++j) {
          const int e = slot(j);
          a.topk_idx[t * k + j] = e;
          my_drop += e < 0;
          if (a.policy == MOE_CAP_OVERFLOW_NEXT && j < taken) my_over += pos.get(j) >= k;
        }
        committed = true;
      } else if (a.policy == MOE_CAP_OVERFLOW_NEXT) {
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
        }
      } else {
        for (int j = 0; j < k; ++j)
          if (ch.get(j) >= 0 && is_full(ch.get(j))) ch.set(j, -1);
      }
    }
  }
  atomicAdd(&s_over, my_over);
  atomicAdd(&s_drop, my_drop);
  __syncthreads();
  if (tid == 0 && a.diag) {
    atomicAdd(&a.diag->overflowed, (int32_t)s_over);
    atomicAdd(&a.diag->dropped, (int32_t)s_drop);
  }
}

// Dynamic shared memory of a grid of `grid` CTAs: every CTA's row of per-expert counts, and the
// staged ranking prefixes of the CTA's tokens.
size_t dyn_smem(unsigned grid, int E) {
  const int P = E < kPrefix ? E : kPrefix;
  return (size_t)grid * E * sizeof(int) + (size_t)kThreads * prefix_words(P) * sizeof(uint32_t);
}

template <int KT>
cudaError_t launch_t(CapacityArgs a, GridCtl* g, unsigned grid, cudaStream_t s) {
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
  return (int64_t)sizeof(GridCtl) + ceil_div(n, kThreads) * E * 4;
}

bool capacity_grid_fits(int64_t n, int32_t E) {
  const int64_t blocks = ceil_div(n, kThreads);
  // one CTA per SM, and every CTA's count row in shared memory next to the static arrays
  return blocks >= 1 && blocks <= resident_blocks() && dyn_smem((unsigned)blocks, E) <= kMaxDynSmem;
}

cudaError_t launch_capacity_grid(const CapacityArgs& a, void* scratch, cudaStream_t s) {
  if (a.n <= 0) return cudaSuccess;
  if (reinterpret_cast<uintptr_t>(scratch) % 16) return cudaErrorInvalidValue;
  GridCtl* g = static_cast<GridCtl*>(scratch);
  CapacityArgs b = a;
  b.hist = reinterpret_cast<int32_t*>(static_cast<char*>(scratch) + sizeof(GridCtl));
  cudaError_t e = cudaMemsetAsync(g, 0, sizeof(GridCtl), s);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)ceil_div(a.n, kThreads);
  switch (a.k) {
    case 1: return launch_t<1>(b, g, grid, s);
    case 2: return launch_t<2>(b, g, grid, s);
    case 4: return launch_t<4>(b, g, grid, s);
    case 8: return launch_t<8>(b, g, grid, s);
    default: return launch_t<0>(b, g, grid, s);
  }
}

}  // namespace moe
