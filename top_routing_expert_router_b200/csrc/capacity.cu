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
// per thread; a CTA resolves its range in rounds: from its tokens' current
// choices it finds the first token at which some expert reaches C (ballot
// prefixes in token order), marks that expert full, lets the later tokens that
// held it walk on, and repeats. The tokens before the filling token keep their
// choices for good. The counts it starts from are its predecessor's final ones
// (an expert is full once its count reaches C, and a full expert's count is
// exactly C), each handed over as its own self-validating word; while it
// waits, its tokens' rankings are already staged and their choices taken under
// the full set of the CTA two places up the chain, so only the tokens that
// held an expert filled just upstream walk on afterwards. The grid is launched
// cooperatively (every CTA resident, so a wait always ends), and every wait is
// bounded.
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
constexpr int kPosWords = 17;  // 32-bit words per token of the inverse ranking (64 bytes + 4: odd stride)

// 32-bit words per staged ranking prefix of P entries: enough for P and odd, so that lanes reading
// the same position of their rows hit 32 different banks.
__host__ __device__ constexpr int prefix_words(int P) { return ((P + 1) / 2) | 1; }
// Up to 64 experts (E a multiple of 8) every token's whole ranking is staged, and its inverse too.
__host__ __device__ constexpr bool mask_capable(int E) { return E <= 64 && E % 8 == 0; }

// State handed from CTA b to CTA b + 1: the expert counts after CTA b's tokens, word e holding
// count[e] + 1 (0: not written yet; kAbandoned: the chain was abandoned upstream). Each word is
// valid on its own, so a reader waits on exactly the words it needs and no fence or flag orders
// them; the full set is the experts whose count reached C.
struct ChainState {
  uint32_t cnt[kMaxExperts];
};
constexpr uint32_t kAbandoned = 0xFFFFFFFFu;

__device__ __forceinline__ uint32_t ld_relaxed(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_relaxed(uint32_t* p, uint32_t v) {
  asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Bounded wait for one word of a predecessor's state: count + 1, or 0 if it never came (timeout,
// status set) or the chain was abandoned.
__device__ uint32_t wait_word(const uint32_t* w, moe_diag* status) {
  uint32_t v = ld_relaxed(w);
  if (v != 0) return v == kAbandoned ? 0u : v;
  const uint64_t t0 = globaltimer();
  for (;;) {
    __nanosleep(32);
    v = ld_relaxed(w);
    if (v != 0) return v == kAbandoned ? 0u : v;
    if (globaltimer() - t0 > kBarrierTimeoutNs) {
      set_status(status, MOE_ERR_TIMEOUT);
      return 0;
    }
  }
}

// Every thread of the CTA: the counts (cnt != nullptr) and the full set of a predecessor's state,
// thread e waiting on word e; false (uniform) if any word never came.
__device__ bool take_state(const ChainState* src, int E, int64_t C, int* cnt, uint32_t* full, int* s_ok,
                           moe_diag* status) {
  const int tid = threadIdx.x;
  if (tid == 0) *s_ok = 1;
  __syncthreads();
  bool is_full = false;
  if (tid < E) {
    const uint32_t v = wait_word(&src->cnt[tid], status);
    if (v == 0) *s_ok = 0;
    const int c = (int)(v - 1u);
    if (cnt) cnt[tid] = v ? c : 0;
    is_full = v != 0 && c >= C;
  }
  const unsigned bits = __ballot_sync(0xFFFFFFFFu, is_full);
  if (tid < kMaxExperts && (tid & 31) == 0) full[tid >> 5] = bits;
  __syncthreads();
  return *s_ok != 0;
}

// Mark this CTA's state abandoned, so that the CTAs after it stop waiting.
__device__ void abandon(ChainState* mine, int E) {
  for (int e = threadIdx.x; e < E; e += blockDim.x) st_relaxed(&mine->cnt[e], kAbandoned);
}

// Position of the n-th (from 1) set bit of x, n <= popc(x): a binary search on popcounts.
__device__ __forceinline__ int nth_set_bit(uint32_t x, int n) {
  int pos = 0;
  int c = __popc(x & 0xFFFFu);
  if (n > c) { n -= c; pos += 16; x >>= 16; }
  c = __popc(x & 0xFFu);
  if (n > c) { n -= c; pos += 8; x >>= 8; }
  c = __popc(x & 0xFu);
  if (n > c) { n -= c; pos += 4; x >>= 4; }
  c = __popc(x & 0x3u);
  if (n > c) { n -= c; pos += 2; x >>= 2; }
  return pos + (n > (int)(x & 1u) ? 1 : 0);
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
  __shared__ int cnt0[kMaxExperts];     // counts before this range (the predecessor's)
  __shared__ int hist[kMaxExperts];     // the current choices of the range's tokens, per expert
                                        // (exact for experts that are not full)
  __shared__ uint32_t full_s[kMaxExperts / 32];
  __shared__ uint32_t applied_s[2];     // mask mode: the full set the tokens' masks already exclude
  __shared__ int cand[kMaxExperts];
  __shared__ int cstop[kMaxExperts];    // per candidate: the token at which it reaches C
  __shared__ uint32_t bal[32][kThreads / 32];  // per candidate of a batch: which tokens of each warp hold it
  __shared__ int s_stop;
  __shared__ int s_ok;
  __shared__ unsigned long long s_over, s_drop;
  extern __shared__ uint32_t srows[];  // the tokens' ranking prefixes (kPrefix entries, odd word stride)
  const int64_t t0 = (int64_t)blockIdx.x * kThreads;
  const int64_t t = t0 + tid;
  const bool valid = t < a.n;
  const int cnt_tok = (int)((a.n - t0) < kThreads ? (a.n - t0) : kThreads);
  const uint16_t* row = a.ranking + (valid ? t : 0) * E;
  // the first P entries of every token's ranking in shared memory: a token walking past full
  // experts reads them at shared-memory latency instead of one dependent global load per step
  const int P = E < kPrefix ? E : kPrefix;
  const int pw = prefix_words(P);
  uint32_t* srow32 = srows + tid * pw;
  const uint16_t* srow = reinterpret_cast<const uint16_t*>(srow32);
  // Mask mode (OVERFLOW_NEXT, at most 64 experts): a token's choices are the first k positions of
  // its ranking whose experts are not full, kept as a 64-bit mask of the available positions; the
  // inverse ranking turns an expert that fills into the one bit it clears, so a token whose expert
  // filled finds its next choice at once instead of stepping past every full expert. The first two
  // CTAs, whose staging is on the chain's critical path and which meet few full experts, walk.
  const bool mm = a.policy == MOE_CAP_OVERFLOW_NEXT && mask_capable(E) && blockIdx.x >= 2;
  uint8_t* pos_of = reinterpret_cast<uint8_t*>(srows + kThreads * pw);  // [kThreads][kPosWords words]
  if (mm)
    for (int w = 0; w < kPosWords; ++w) reinterpret_cast<uint32_t*>(pos_of)[tid * kPosWords + w] = 0xFFFFFFFFu;
  if (E % 8 == 0) {
    // the range's rows are contiguous: consecutive threads load consecutive 16-byte pieces, all of
    // a thread's loads in flight before the first store
    const int U = P / 8, R = E / 8;
    const int total = cnt_tok * U;
    const uint4* src = reinterpret_cast<const uint4*>(a.ranking + t0 * E);
    uint4 q4[kPrefix / 8];
#pragma unroll
    for (int v = 0; v < kPrefix / 8; ++v) {
      const int idx = tid + v * kThreads;
      if (idx < total) q4[v] = __ldg(&src[(int64_t)(idx / U) * R + idx % U]);
    }
#pragma unroll
    for (int v = 0; v < kPrefix / 8; ++v) {
      const int idx = tid + v * kThreads;
      if (idx < total) {
        uint32_t* d = srows + (idx / U) * pw + 4 * (idx % U);
        d[0] = q4[v].x;
        d[1] = q4[v].y;
        d[2] = q4[v].z;
        d[3] = q4[v].w;
      }
    }
    if (mm) {
      __syncthreads();  // every row's 0xFF (not ranked) fill is down
#pragma unroll
      for (int v = 0; v < kPrefix / 8; ++v) {
        const int idx = tid + v * kThreads;
        if (idx < total) {
          uint8_t* inv = pos_of + (idx / U) * (kPosWords * 4);
          const uint32_t w4[4] = {q4[v].x, q4[v].y, q4[v].z, q4[v].w};
#pragma unroll
          for (int h = 0; h < 8; ++h) {
            const uint32_t e = (w4[h >> 1] >> (16 * (h & 1))) & 0xFFFFu;
            if (e < 64u) inv[e] = (uint8_t)(8 * (idx % U) + h);
          }
        }
      }
    }
  } else if (valid) {
    uint16_t* d16 = reinterpret_cast<uint16_t*>(srow32);
    for (int c = 0; c < P; ++c) d16[c] = row[c];
  }
  Slots<KA, (KT > 0)> ch, pos;
  int taken = 0, cursor = 0;
  uint64_t avail = P == 64 ? ~0ull : (1ull << P) - 1, chosen = 0;  // mask mode: by ranking position
  if (tid == 0) s_over = s_drop = 0;
  if (tid < 2) applied_s[tid] = 0;
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
  // Drop the experts that are full now; under OVERFLOW_NEXT walk on to replace them. Returns the
  // first slot that holds a new choice (k: none). A dropped expert's count is not taken back: a
  // full expert's count is C, whatever its holders.
  auto drop_full = [&]() -> int {
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
      if (kept == taken) return k;
      taken = kept;
      refill();
      return kept;
    }
    for (int j = 0; j < k; ++j)
      if (ch.get(j) >= 0 && is_full(ch.get(j))) ch.set(j, -1);
    return k;
  };
  auto count_new = [&](int from) {
    for (int j = 0; j < k; ++j)
      if (j >= from && j < taken) atomicAdd(&hist[ch.get(j)], 1);
  };
  // mask mode: the choices are the first k available positions (0xFFFF ends the ranking)
  auto choose = [&]() {
    uint64_t m = avail;
    taken = 0;
    chosen = 0;
    for (int j = 0; j < k; ++j) {
      if (m == 0) break;
      const int p = __ffsll((long long)m) - 1;
      const int e = srow[p];
      if (e == 0xFFFF) break;
      ch.set(j, e);
      pos.set(j, p);
      chosen |= 1ull << p;
      ++taken;
      m &= m - 1;
    }
  };
  // mask mode: clear the positions of the experts filled since the masks were last brought up to
  // date; the hist of a new choice goes up (a left expert is full: its count is C anyway)
  auto apply_full = [&](bool counted) {
    uint64_t cleared = 0;
    const uint8_t* inv = pos_of + tid * (kPosWords * 4);
    for (int w = 0; w < 2; ++w) {
      uint32_t bits = full_s[w] & ~applied_s[w];
      while (bits) {
        const int p = inv[32 * w + __ffs(bits) - 1];
        bits &= bits - 1;
        if (p != 0xFF) cleared |= 1ull << p;
      }
    }
    avail &= ~cleared;
    if (!(chosen & cleared)) return;
    const uint64_t old = chosen;
    choose();
    if (counted)
      for (int j = 0; j < k; ++j)
        if (j < taken && !((old >> pos.get(j)) & 1ull)) atomicAdd(&hist[ch.get(j)], 1);
  };
  // choices under no full expert, while the predecessor resolves its range
  if (valid) {
    if (mm) {
      choose();
    } else if (a.policy == MOE_CAP_OVERFLOW_NEXT) {
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
    if (!take_state(chain + blockIdx.x - 2, E, a.C, nullptr, full_s, &s_ok, a.status)) {
      abandon(mine, E);  // abandon the rest of the chain at once
      return;
    }
    if (valid) {
      if (mm)
        apply_full(false);
      else
        drop_full();
    }
  }
  for (int e = tid; e < E; e += kThreads) hist[e] = 0;
  __syncthreads();
  if (tid < 2) applied_s[tid] = full_s[tid];  // before take_state below writes full_s
  for (int j = 0; j < k; ++j) warp_count(hist, valid ? slot(j) : -1);
  // the predecessor's counts and full set (other CTAs wrote them: read at L2, not L1)
  if (blockIdx.x == 0) {
    for (int e = tid; e < kMaxExperts; e += kThreads) cnt0[e] = 0;
    __syncthreads();
  } else if (!take_state(chain + blockIdx.x - 1, E, a.C, cnt0, full_s, &s_ok, a.status)) {
    abandon(mine, E);
    return;
  }
  // tokens that held an expert CTA b - 1 filled walk on; the histogram follows their new choices
  if (valid && blockIdx.x > 0) {
    if (mm)
      apply_full(true);
    else
      count_new(drop_full());
  }
  // Rounds. Committed tokens (those before f) never change their choices, so the token at which
  // expert e reaches C is its (C - cnt0[e])-th holder among all of the range's tokens, and an
  // expert is a candidate when cnt0[e] + hist[e] >= C. The first such token ends the round: the
  // experts that fill at it become full and the later tokens that held them walk on. Every warp
  // lists the candidates itself (the same list, in expert order) and ballots its tokens' holdings
  // of them, 32 candidates a batch; warp 0 finds each candidate's filling token from the warps'
  // counts and marks the experts that fill first. Three barriers a round, one when none fills.
  int f = 0;  // first token of the range not committed yet (uniform across the CTA)
  for (;;) {
    __syncthreads();  // choices and hist are up to date
    if (tid < 2) applied_s[tid] = full_s[tid];  // mask mode: every mask excludes these
    int nc = 0;
    int stop = kThreads;  // warp 0: the first filling token so far
    for (int bt = 0;; ++bt) {
      int idx = 0;
      for (int e0 = 0; e0 < E; e0 += 32) {
        const int e = e0 + lane;
        uint32_t m = __ballot_sync(kFull, e < E && !is_full(e) && cnt0[e] + hist[e] >= a.C);
        while (m) {
          const int ec = e0 + __ffs(m) - 1;
          m &= m - 1;
          if (idx >= 32 * bt && idx < 32 * bt + 32) {
            bool h = false;
            if (valid)
              for (int j = 0; j < k; ++j) h |= slot(j) == ec;
            const uint32_t b = __ballot_sync(kFull, h);
            if (lane == 0) bal[idx - 32 * bt][wid] = b;
          }
          if (bt == 0 && tid == 0) cand[idx] = ec;
          ++idx;
        }
      }
      nc = idx;
      if (nc == 0) break;
      __syncthreads();  // the batch's ballots are down
      if (wid == 0) {
        const int nb = nc - 32 * bt < 32 ? nc - 32 * bt : 32;
        for (int q = 0; q < nb; ++q) {
          const int e = cand[32 * bt + q];
          const int need = (int)(a.C - cnt0[e]);
          const uint32_t bw = bal[q][lane];  // lane w: the holders among warp w's tokens
          const int pc = __popc(bw);
          int incl = pc;
#pragma unroll
          for (int off = 1; off < 32; off <<= 1) {
            const int v = __shfl_up_sync(kFull, incl, off);
            if (lane >= off) incl += v;
          }
          int at = kThreads;  // fewer holders than needed: not while hist is exact
          if (incl - pc < need && need <= incl) at = lane * 32 + nth_set_bit(bw, need - (incl - pc));
          at = __reduce_min_sync(kFull, at);
          if (lane == 0) cstop[32 * bt + q] = at;
          stop = at < stop ? at : stop;
        }
      }
      if (32 * (bt + 1) >= nc) break;
      __syncthreads();  // warp 0 is done with bal before the next batch writes it
    }
    if (nc == 0) break;  // no expert fills in the rest of the range
    if (wid == 0) {
      __syncwarp();
      if (stop < kThreads)
        for (int c = lane; c < nc; c += 32)
          if (cstop[c] == stop) atomicOr(&full_s[cand[c] >> 5], 1u << (cand[c] & 31));
      if (lane == 0) s_stop = stop;
    }
    __syncthreads();  // the filling token and the new full set are out
    const int st = s_stop;
    if (st >= cnt_tok - 1) break;
    f = st + 1;
    // the later tokens holding an expert that just filled walk on; the histogram follows them
    if (valid && tid >= f) {
      if (mm)
        apply_full(true);
      else
        count_new(drop_full());
    }
  }
  // hand the counts on: C for a full expert, else the predecessor's count plus this range's
  for (int e = tid; e < E; e += kThreads)
    st_relaxed(&mine->cnt[e], (uint32_t)(is_full(e) ? (int)a.C : cnt0[e] + hist[e]) + 1u);
  // every token's final choices
  unsigned long long my_over = 0, my_drop = 0;
  if (valid)
    for (int j = 0; j < k; ++j) {
      const int e = slot(j);
      a.topk_idx[t * k + j] = e;
      my_drop += e < 0;
      if (a.policy == MOE_CAP_OVERFLOW_NEXT && j < taken) my_over += pos.get(j) >= k;
    }
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
  return (size_t)kThreads * (prefix_words(P) + (mask_capable(E) ? kPosWords : 0)) * sizeof(uint32_t);
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
  cudaError_t e = cudaMemsetAsync(g, 0, (size_t)grid * sizeof(ChainState), s);  // no word written yet
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
