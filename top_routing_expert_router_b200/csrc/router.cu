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

// Order-preserving key of a double: a larger value has a larger key. -0 is taken as +0 first, so
// that the two have one key as they compare equal.
__device__ __forceinline__ unsigned long long order_key(double v) {
  const unsigned long long b = (unsigned long long)__double_as_longlong(v + 0.0);
  return (b >> 63) ? ~b : (b | 0x8000000000000000ull);
}

// The value of an order key (-0 comes back as +0).
__device__ __forceinline__ double key_value(unsigned long long key) {
  return __longlong_as_double((long long)((key >> 63) ? (key & 0x7FFFFFFFFFFFFFFFull) : ~key));
}

// Lane holding the largest key of the warp (the lowest such lane on equal keys), by two warp
// reductions over the key's halves and a ballot.
__device__ __forceinline__ int warp_argmax_key(unsigned long long key) {
  const unsigned hi = (unsigned)(key >> 32), lo = (unsigned)key;
  const unsigned best_hi = __reduce_max_sync(kFull, hi);
  const unsigned best_lo = __reduce_max_sync(kFull, hi == best_hi ? lo : 0u);
  return __ffs(__ballot_sync(kFull, hi == best_hi && lo == best_lo)) - 1;
}

// Largest value of the warp (two warp reductions over its order key, then the value itself).
__device__ __forceinline__ double warp_max(double v) {
  const unsigned long long key = order_key(v);
  const unsigned hi = (unsigned)(key >> 32), lo = (unsigned)key;
  const unsigned best_hi = __reduce_max_sync(kFull, hi);
  const unsigned best_lo = __reduce_max_sync(kFull, hi == best_hi ? lo : 0u);
  const int src = __ffs(__ballot_sync(kFull, hi == best_hi && lo == best_lo)) - 1;
  return __shfl_sync(kFull, v, src);
}

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int off = 16; off; off >>= 1) v += __shfl_xor_sync(kFull, v, off);
  return v;
}

__device__ __forceinline__ double sigmoid_d(double z) { return 1.0 / (1.0 + exp(-z)); }

// sqrt(softplus(z)) ("sqrtsoftplus", page "15. DeepSeek: MLA, MoE and MTP", section V4).
__device__ __forceinline__ double sqrtsoftplus_d(double z) { return sqrt(fmax(z, 0.0) + log1p(exp(-fabs(z)))); }

// Raw score of the routers that add a selection bias.
__device__ __forceinline__ double raw_score(int score_fn, double z) {
  return score_fn == MOE_SCORE_SQRTSOFTPLUS ? sqrtsoftplus_d(z) : sigmoid_d(z);
}

template <int EPL>
__device__ __forceinline__ double pick(const double (&r)[EPL], int j) {
  double out = 0.0;
#pragma unroll
  for (int i = 0; i < EPL; ++i)
    if (i == j) out = r[i];
  return out;
}

// Selection values: softmax ranks the logits; sigmoid ranks s + bias.
template <int EPL>
__device__ __forceinline__ void selection_values(const RouteArgs& a, const double (&l)[EPL], double (&v)[EPL],
                                                 bool (&valid)[EPL]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int j = 0; j < EPL; ++j) {
    const int e = lane + 32 * j;
    valid[j] = e < a.E;
    if (valid[j])
      v[j] = a.score_fn != MOE_SCORE_SOFTMAX ? raw_score(a.score_fn, l[j]) + (a.bias ? (double)a.bias[e] : 0.0) : l[j];
    else
      v[j] = -INFINITY;
  }
}

// Group limit with per-expert uncertainty (bit j of `exact`: value is binary64;
// otherwise it may be off by delta_v). Sets *elig (bits over j) to the experts
// of the kept groups. Returns false when the group cut is not certain, with the
// inexact experts that could decide it in *mark. An expert can be in its group's
// true top two only if v >= (second largest v) - 2 delta_v; once all of those
// are exact the group score is exact.
template <int EPL>
__device__ bool decide_groups_32(const RouteArgs& a, const double (&v)[EPL], const bool (&valid)[EPL], uint32_t exact,
                                 double delta_v, uint32_t* elig, uint32_t* mark, unsigned long long* keys);

template <int EPL>
__device__ bool decide_groups(const RouteArgs& a, const double (&v)[EPL], const bool (&valid)[EPL], uint32_t exact,
                              double delta_v, uint32_t* elig, uint32_t* mark, unsigned long long* keys) {
  const int lane = threadIdx.x & 31;
  const int per = a.E / a.G;
  // groups of 32 experts, one per lane slot: every group's reduction at once (below)
  if (per == 32 && a.G == EPL) return decide_groups_32<EPL>(a, v, valid, exact, delta_v, elig, mark, keys);
  double gs[kMaxGroups], gu[kMaxGroups], t2s[kMaxGroups];
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
    bool inexact_cand = false;
#pragma unroll
    for (int j = 0; j < EPL; ++j) {
      const int e = lane + 32 * j;
      if (valid[j] && e / per == g && !((exact >> j) & 1u) && v[j] >= t2 - 2.0 * delta_v) inexact_cand = true;
    }
    gs[g] = t1 + t2;
    gu[g] = __any_sync(kFull, inexact_cand) ? 2.0 * delta_v : 0.0;
    t2s[g] = t2;
  }
  uint32_t keep = 0;
  double min_kept = INFINITY, max_drop = -INFINITY;
  for (int g = 0; g < a.G; ++g) {
    int better = 0;
    for (int h = 0; h < a.G; ++h) better += (gs[h] > gs[g]) || (gs[h] == gs[g] && h < g);
    if (better < a.topk_group) {
      keep |= 1u << g;
      min_kept = fmin(min_kept, gs[g] - gu[g]);
    } else {
      max_drop = fmax(max_drop, gs[g] + gu[g]);
    }
  }
  bool ok = true;
  uint32_t m = 0;
  if (a.topk_group < a.G && !(min_kept > max_drop)) {
    uint32_t involved = 0;
    for (int g = 0; g < a.G; ++g) {
      const bool kept = (keep >> g) & 1u;
      if (gu[g] > 0.0 && (kept ? gs[g] - gu[g] <= max_drop : gs[g] + gu[g] >= min_kept)) involved |= 1u << g;
    }
    if (involved) {
      ok = false;
#pragma unroll
      for (int j = 0; j < EPL; ++j) {
        const int e = lane + 32 * j;
        if (valid[j] && ((involved >> (e / per)) & 1u) && !((exact >> j) & 1u) && v[j] >= t2s[e / per] - 2.0 * delta_v)
          m |= 1u << j;
      }
    }
  }
  uint32_t el = 0;
#pragma unroll
  for (int j = 0; j < EPL; ++j) {
    const int e = lane + 32 * j;
    if (valid[j] && ((keep >> (e / per)) & 1u)) el |= 1u << j;
  }
  *elig = el;
  *mark = m;
  return ok;
}

// decide_groups for groups of exactly 32 experts with G = EPL: lane slot j of every lane holds
// expert lane + 32 j, which is in group j, so the two best values of all groups are reduced across
// the warp together (independent shuffle chains), with no per-expert group arithmetic.
template <int EPL>
__device__ bool decide_groups_32(const RouteArgs& a, const double (&v)[EPL], const bool (&valid)[EPL], uint32_t exact,
                                 double delta_v, uint32_t* elig, uint32_t* mark, unsigned long long* keys) {
  // The two best values of every group (the largest and the largest of the rest, equal to the
  // first on a tie) on integer order keys, which order like the values (binary64 comparisons and
  // min/max are slow next to integer ones when many warps decide at once). Group g is slot g of
  // every lane; through the warp's shared scratch each group goes to 32 / EPL lanes of EPL keys
  // each, which take their two best and merge them by shuffles, instead of one chain of warp
  // reductions per group and rank.
  const int lane = threadIdx.x & 31;
  constexpr int LPG = 32 / EPL;  // lanes per group
  __syncwarp();  // the scratch's previous readers are done
#pragma unroll
  for (int g = 0; g < EPL; ++g) keys[g * 32 + lane] = order_key(valid[g] ? v[g] : -INFINITY);
  __syncwarp();
  unsigned long long k1 = 0ull, k2 = 0ull;  // 0 is below the key of every value, -inf included
  const unsigned long long* mine = keys + (lane / LPG) * 32 + (lane % LPG) * EPL;
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    const unsigned long long kk = mine[(i + lane) % EPL];
    if (kk > k1) {
      k2 = k1;
      k1 = kk;
    } else if (kk > k2) {
      k2 = kk;
    }
  }
#pragma unroll
  for (int off = 1; off < LPG; off <<= 1) {
    const unsigned long long o1 = __shfl_xor_sync(kFull, k1, off);
    const unsigned long long o2 = __shfl_xor_sync(kFull, k2, off);
    const unsigned long long lo1 = k1 < o1 ? k1 : o1, hi2 = k2 > o2 ? k2 : o2;
    k1 = k1 > o1 ? k1 : o1;
    k2 = lo1 > hi2 ? lo1 : hi2;
  }
  double t1[EPL], t2[EPL];
#pragma unroll
  for (int g = 0; g < EPL; ++g) {
    t1[g] = key_value(__shfl_sync(kFull, k1, g * LPG));
    t2[g] = key_value(__shfl_sync(kFull, k2, g * LPG));
  }
  double gs[EPL], gu[EPL];
#pragma unroll
  for (int g = 0; g < EPL; ++g) {
    // an inexact expert could be among the group's true top two if v >= second best - 2 delta_v
    const bool cand = valid[g] && !((exact >> g) & 1u) && v[g] >= t2[g] - 2.0 * delta_v;
    gs[g] = t1[g] + t2[g];
    gu[g] = __any_sync(kFull, cand) ? 2.0 * delta_v : 0.0;
  }
  uint32_t keep = 0;
  double min_kept = INFINITY, max_drop = -INFINITY;
  unsigned long long gk[EPL];  // group scores as order keys: larger score, larger key
#pragma unroll
  for (int g = 0; g < EPL; ++g) gk[g] = order_key(gs[g]);
#pragma unroll
  for (int g = 0; g < EPL; ++g) {
    int better = 0;
#pragma unroll
    for (int h = 0; h < EPL; ++h) better += (gk[h] > gk[g]) || (gk[h] == gk[g] && h < g);
    if (better < a.topk_group) {
      keep |= 1u << g;
      min_kept = fmin(min_kept, gs[g] - gu[g]);
    } else {
      max_drop = fmax(max_drop, gs[g] + gu[g]);
    }
  }
  bool ok = true;
  uint32_t m = 0;
  if (a.topk_group < a.G && !(min_kept > max_drop)) {
    uint32_t involved = 0;
#pragma unroll
    for (int g = 0; g < EPL; ++g) {
      const bool kept = (keep >> g) & 1u;
      if (gu[g] > 0.0 && (kept ? gs[g] - gu[g] <= max_drop : gs[g] + gu[g] >= min_kept)) involved |= 1u << g;
    }
    if (involved) {
      ok = false;
#pragma unroll
      for (int g = 0; g < EPL; ++g)
        if (valid[g] && ((involved >> g) & 1u) && !((exact >> g) & 1u) && v[g] >= t2[g] - 2.0 * delta_v) m |= 1u << g;
    }
  }
  *elig = 0;
#pragma unroll
  for (int g = 0; g < EPL; ++g)
    if (valid[g] && ((keep >> g) & 1u)) *elig |= 1u << g;
  *mark = m;
  return ok;
}

// Top-k selection of one token with per-expert uncertainty. l[j] is the logit
// of expert lane + 32j; bit j of `exact` says it is the binary64 value,
// otherwise it is the binary32 GEMM result whose selection value may be off by
// up to delta_v. Writes the k kept experts to rank[0..k). Returns true when
// every comparison the decision depends on is certain: strictly separated
// intervals, or both sides exact (exact ties then follow the index rule).
// Otherwise sets, in *refine, the inexact experts an uncertain comparison involves.
template <int EPL>
__device__ bool decide(const RouteArgs& a, const double (&l)[EPL], uint32_t exact, double delta_v, int16_t* rank,
                       int* n_ranked, uint32_t* refine, unsigned long long* keys) {
  const int lane = threadIdx.x & 31;
  double v[EPL];
  bool valid[EPL];
  selection_values<EPL>(a, l, v, valid);
  auto unc = [&](int j) { return ((exact >> j) & 1u) ? 0.0 : delta_v; };
  bool ok = true;
  uint32_t mark = 0;
  uint32_t elig_mask = 0;
  if (a.G > 1) {
    if (!decide_groups<EPL>(a, v, valid, exact, delta_v, &elig_mask, &mark, keys)) ok = false;
  } else {
#pragma unroll
    for (int j = 0; j < EPL; ++j)
      if (valid[j]) elig_mask |= 1u << j;
  }
  int n_elig = __popc(elig_mask);
#pragma unroll
  for (int off = 16; off; off >>= 1) n_elig += __shfl_xor_sync(kFull, n_elig, off);
  const int want = min(n_elig, a.k);
  uint32_t taken = 0;
  double prev_lo = 0.0;
  int prev_e = -1;
  bool prev_exact = true;
  double top_lo = INFINITY;  // min over the kept experts of v - u
  unsigned long long vk[EPL];  // selection values as order keys
#pragma unroll
  for (int j = 0; j < EPL; ++j) vk[j] = order_key(v[j]);
  for (int r = 0; r < want; ++r) {
    // this lane's best untaken eligible expert (lower j first on equal keys), then the warp's
    unsigned long long bk = 0ull;
    int bj = -1;
#pragma unroll
    for (int j = 0; j < EPL; ++j)
      if (((elig_mask & ~taken) >> j) & 1u && (bj < 0 || vk[j] > bk)) {
        bk = vk[j];
        bj = j;
      }
    // the lowest expert index among the lanes holding the best key: lane + 32 j, so the lowest j,
    // then the lowest lane
    const unsigned bhi = __reduce_max_sync(kFull, bj >= 0 ? (unsigned)(bk >> 32) : 0u);
    const unsigned blo = __reduce_max_sync(kFull, bj >= 0 && (unsigned)(bk >> 32) == bhi ? (unsigned)bk : 0u);
    const bool top = bj >= 0 && (unsigned)(bk >> 32) == bhi && (unsigned)bk == blo;
    const unsigned be = __reduce_min_sync(kFull, top ? (unsigned)(lane + 32 * bj) : 0xFFFFFFFFu);
    VE best;
    best.e = (int)be;
    best.v = __shfl_sync(kFull, pick(v, bj < 0 ? 0 : bj), (int)(be & 31));
    const int owner = best.e & 31, jb = best.e >> 5;
    const bool b_exact = __shfl_sync(kFull, (int)((exact >> jb) & 1u), owner) != 0;
    const double bu = b_exact ? 0.0 : delta_v;
    if (lane == owner) taken |= 1u << jb;
    if (r > 0 && !(prev_exact && b_exact) && !(prev_lo > best.v + bu)) {
      // adjacent order not certain: refine whichever of the two is inexact
      ok = false;
      if (!prev_exact && (prev_e & 31) == lane) mark |= 1u << (prev_e >> 5);
      if (!b_exact && lane == owner) mark |= 1u << jb;
    }
    prev_lo = best.v - bu;
    prev_e = best.e;
    prev_exact = b_exact;
    top_lo = fmin(top_lo, best.v - bu);
    if (lane == 0) rank[r] = (int16_t)best.e;
  }
  if (want < n_elig) {
    // The cut between the k kept experts and every eligible expert below them.
    double below_hi = -INFINITY;
#pragma unroll
    for (int j = 0; j < EPL; ++j)
      if (((elig_mask & ~taken) >> j) & 1u) below_hi = fmax(below_hi, v[j] + unc(j));
    below_hi = warp_max(below_hi);
    if (!(top_lo > below_hi)) {
      bool any = false;
#pragma unroll
      for (int j = 0; j < EPL; ++j) {
        if (!((elig_mask >> j) & 1u) || ((exact >> j) & 1u)) continue;
        const bool mine = (taken >> j) & 1u;
        if (mine ? v[j] - delta_v <= below_hi : v[j] + delta_v >= top_lo) {
          mark |= 1u << j;
          any = true;
        }
      }
      if (__any_sync(kFull, any)) ok = false;
    }
  }
  *n_ranked = want;
  *refine = mark;
  __syncwarp();
  return ok;
}

// Full ranking of one token's eligible experts (the capacity rule needs it),
// by a bitonic sort across the warp: position p = lane * EPL + j. Each element
// carries its expert index and exactness. After the sort, adjacent pairs are
// certified like the top-k pairs; uncertain inexact experts are flagged in
// `flags` (per-warp shared, one byte per expert) and returned in *refine.
template <int EPL>
__device__ bool decide_full(const RouteArgs& a, const double (&l)[EPL], uint32_t exact, double delta_v,
                            int16_t* rank, uint8_t* flags, int* n_ranked, uint32_t* refine,
                            unsigned long long* keys) {
  const int lane = threadIdx.x & 31;
  const int E = a.E;
  double v0[EPL];
  bool valid[EPL];
  selection_values<EPL>(a, l, v0, valid);
  uint32_t elig_mask = 0;
  bool ok = true;
  uint32_t mark = 0;
  if (a.G > 1) {
    if (!decide_groups<EPL>(a, v0, valid, exact, delta_v, &elig_mask, &mark, keys)) ok = false;
  } else {
#pragma unroll
    for (int j = 0; j < EPL; ++j)
      if (valid[j]) elig_mask |= 1u << j;
  }
  // keys in sort layout: lane holds positions lane*EPL .. lane*EPL+EPL-1. The sort compares the
  // values' integer order keys (binary64 comparisons are slow next to integer ones when many
  // warps sort at once); the values come back from the keys afterwards.
  unsigned long long kk[EPL];
  int ke[EPL];  // expert | exact << 16, or -1 for empty
#pragma unroll
  for (int j = 0; j < EPL; ++j) {
    const int e = lane + 32 * j;
    const bool el = (elig_mask >> j) & 1u;
    kk[j] = order_key(el ? v0[j] : -INFINITY);
    ke[j] = el ? (e | (int)(((exact >> j) & 1u) << 16)) : (0x7FFF | (1 << 16));
  }
  auto key_better = [](unsigned long long ka, int ea, unsigned long long kb, int eb) {
    return ka > kb || (ka == kb && ea < eb);
  };
  constexpr int S = 32 * EPL;
#pragma unroll
  for (int k = 2; k <= S; k <<= 1) {
#pragma unroll
    for (int d = k >> 1; d > 0; d >>= 1) {
      if (d < EPL) {
#pragma unroll
        for (int j = 0; j < EPL; ++j) {
          const int jp = j ^ d;
          if (jp > j) {
            const int p = lane * EPL + j;
            const bool up = (p & k) == 0;  // block sorted best-first
            const bool swap = up ? key_better(kk[jp], ke[jp] & 0xFFFF, kk[j], ke[j] & 0xFFFF)
                                 : key_better(kk[j], ke[j] & 0xFFFF, kk[jp], ke[jp] & 0xFFFF);
            if (swap) {
              const unsigned long long tk = kk[j];
              kk[j] = kk[jp];
              kk[jp] = tk;
              const int te = ke[j];
              ke[j] = ke[jp];
              ke[jp] = te;
            }
          }
        }
      } else {
        const int ld = d / EPL;
#pragma unroll
        for (int j = 0; j < EPL; ++j) {
          const unsigned long long ok_ = __shfl_xor_sync(kFull, kk[j], ld);
          const int oe = __shfl_xor_sync(kFull, ke[j], ld);
          const int p = lane * EPL + j;
          const bool up = (p & k) == 0;
          const bool lower = (lane & ld) == 0;  // this element sits at the smaller position
          const bool other_better = key_better(ok_, oe & 0xFFFF, kk[j], ke[j] & 0xFFFF);
          // the smaller position keeps the better key in an ascending block
          const bool take = (lower == up) ? other_better : !other_better;
          if (take) {
            kk[j] = ok_;
            ke[j] = oe;
          }
        }
      }
    }
  }
  double kv[EPL];
#pragma unroll
  for (int j = 0; j < EPL; ++j) kv[j] = key_value(kk[j]);
  int n_elig = __popc(elig_mask);
#pragma unroll
  for (int off = 16; off; off >>= 1) n_elig += __shfl_xor_sync(kFull, n_elig, off);
  // certify adjacent pairs (p, p+1) inside the eligible prefix
  const double nxt_v = __shfl_down_sync(kFull, kv[0], 1);
  const int nxt_e = __shfl_down_sync(kFull, ke[0], 1);
  bool any_flag = false;
#pragma unroll
  for (int j = 0; j < EPL; ++j) {
    const int p = lane * EPL + j;
    if (p + 1 >= n_elig) continue;
    const double vb = (j + 1 < EPL) ? kv[(j + 1) % EPL] : nxt_v;
    const int eb = (j + 1 < EPL) ? ke[(j + 1) % EPL] : nxt_e;
    const bool ea_exact = (ke[j] >> 16) & 1, eb_exact = (eb >> 16) & 1;
    const double ua = ea_exact ? 0.0 : delta_v, ub = eb_exact ? 0.0 : delta_v;
    if (!(ea_exact && eb_exact) && !(kv[j] - ua > vb + ub)) {
      if (!ea_exact) flags[ke[j] & 0xFFFF] = 1;
      if (!eb_exact) flags[eb & 0xFFFF] = 1;
      any_flag = true;
    }
  }
#pragma unroll
  for (int j = 0; j < EPL; ++j) {
    const int p = lane * EPL + j;
    if (p < n_elig) rank[p] = (int16_t)(ke[j] & 0xFFFF);
  }
  if (__any_sync(kFull, any_flag)) {
    ok = false;
    __syncwarp();
#pragma unroll
    for (int j = 0; j < EPL; ++j) {
      const int e = lane + 32 * j;
      if (e < E && flags[e]) {
        mark |= 1u << j;
        flags[e] = 0;
      }
    }
  }
  __syncwarp();
  *n_ranked = n_elig;
  *refine = mark;
  return ok;
}

// Gate weights of the slots in idx[0..k) (entries < 0 are dropped slots).
// Lane j < k returns the weight of slot j.
// s_val: this warp's kMaxTopK doubles of shared memory.
template <int EPL>
__device__ float gates(const RouteArgs& a, const double (&l)[EPL], const int* idx_of_slot, double* s_val) {
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
  // the logit of each kept expert to its slot's lane (the lane owning the expert writes it), then
  // every slot's score at once
  for (int r = 0; r < a.k; ++r) {
    const int e = idx_of_slot[r];
    if (e >= 0 && (e & 31) == lane) s_val[r] = pick(l, e >> 5);
  }
  __syncwarp();
  double mine = 0.0;
  const int e_mine = lane < a.k ? idx_of_slot[lane] : -1;
  if (e_mine >= 0) {
    const double le = s_val[lane];
    mine = a.score_fn == MOE_SCORE_SOFTMAX ? exp(le - m) / z : raw_score(a.score_fn, le);
  }
  __syncwarp();  // s_val is the next token's
  double denom = 1.0;
  if (a.renorm) denom = warp_sum(lane < a.k ? mine : 0.0);
  // a dropped slot weighs 0, also when every slot of the token was dropped
  const bool kept = lane < a.k && idx_of_slot[lane] >= 0;
  return kept ? (float)(mine / denom * (double)a.rsf) : 0.0f;
}

// Binary64 dot products of x[t] with four rows of W_r at once (independent
// accumulators, the token's row read once per chunk); e < 0 entries are skipped
// and return 0.
__device__ void dot64x4(const RouteArgs& a, int64_t t, const int (&e)[4], double (&out)[4]) {
  const int lane = threadIdx.x & 31;
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
  if (a.dtype == MOE_BF16) {
    const uint4* xr = reinterpret_cast<const uint4*>(static_cast<const bf16*>(a.x) + t * a.d);
    const uint4* wr[4];
#pragma unroll
    for (int q = 0; q < 4; ++q)
      wr[q] = reinterpret_cast<const uint4*>(static_cast<const bf16*>(a.w_r) + (int64_t)(e[q] < 0 ? 0 : e[q]) * a.d);
#pragma unroll 2
    for (int i = lane; i < a.d / 8; i += 32) {
      const uint4 xv = __ldg(xr + i);
      const bf16* xs = reinterpret_cast<const bf16*>(&xv);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (e[q] < 0) continue;
        const uint4 wv = __ldg(wr[q] + i);
        const bf16* ws = reinterpret_cast<const bf16*>(&wv);
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[q] = fma(to_f64(xs[c]), to_f64(ws[c]), acc[q]);
      }
    }
  } else {
    const float4* xr = reinterpret_cast<const float4*>(static_cast<const float*>(a.x) + t * a.d);
    for (int i = lane; i < a.d / 4; i += 32) {
      const float4 xv = __ldg(xr + i);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (e[q] < 0) continue;
        const float4 wv = __ldg(reinterpret_cast<const float4*>(static_cast<const float*>(a.w_r) + (int64_t)e[q] * a.d) + i);
        acc[q] = fma((double)xv.x, (double)wv.x, acc[q]);
        acc[q] = fma((double)xv.y, (double)wv.y, acc[q]);
        acc[q] = fma((double)xv.z, (double)wv.z, acc[q]);
        acc[q] = fma((double)xv.w, (double)wv.w, acc[q]);
      }
    }
  }
#pragma unroll
  for (int q = 0; q < 4; ++q) out[q] = warp_sum(acc[q]);
}

// Replace the logits of the experts in `which` (bits over j, per lane) by
// binary64 values, four experts per pass over the token's row. Returns how many
// were recomputed.
template <int EPL>
__device__ int refine_logits(const RouteArgs& a, int64_t t, double (&l)[EPL], uint32_t which) {
  const int lane = threadIdx.x & 31;
  int total = 0;
  int e[4];
  int n = 0;
  auto flush = [&]() {
    double v[4];
    dot64x4(a, t, e, v);
#pragma unroll
    for (int q = 0; q < 4; ++q)
      if (e[q] >= 0 && (e[q] & 31) == lane) {
#pragma unroll
        for (int j = 0; j < EPL; ++j)
          if (j == (e[q] >> 5)) l[j] = v[q];
      }
    n = 0;
  };
#pragma unroll
  for (int j = 0; j < EPL; ++j) {
    uint32_t m = __ballot_sync(kFull, (which >> j) & 1u);
    total += __popc(m);
    while (m) {
      const int src = __ffs(m) - 1;
      m &= m - 1;
      e[n++] = src + 32 * j;
      if (n == 4) flush();
    }
  }
  if (n > 0) {
    for (int q = n; q < 4; ++q) e[q] = -1;
    flush();
  }
  return total;
}

// logits[t][e] (split 0's slot) = the sum of the split-K partials of (t, e) in split order: binary64
// sum, rounded once to binary32. One thread per logit with four splits' loads in flight, so the
// route kernel's warps read one row per token instead of a serial chain through every split.
__global__ void __launch_bounds__(256) sum_splits_kernel(float* logits, int splits, int64_t split_stride, int64_t n,
                                                       int64_t ld, int E) {
  const int64_t total = n * E;
  for (int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x; i < total; i += (int64_t)gridDim.x * 256) {
    const int64_t t = i / E;
    float* p0 = logits + t * ld + (i - t * E);
    double s = 0.0;
    int p = 0;
    for (; p + 4 <= splits; p += 4) {
      const float a0 = p0[(int64_t)p * split_stride], a1 = p0[(int64_t)(p + 1) * split_stride];
      const float a2 = p0[(int64_t)(p + 2) * split_stride], a3 = p0[(int64_t)(p + 3) * split_stride];
      s += (double)a0;
      s += (double)a1;
      s += (double)a2;
      s += (double)a3;
    }
    for (; p < splits; ++p) s += (double)p0[(int64_t)p * split_stride];
    *p0 = (float)s;
  }
}

// Load a token's logits, summing the split-K partial GEMM results in split order. The partials
// of four splits are loaded at once before they are added, so a many-way split costs a few
// memory latencies, not one per split.
template <int EPL>
__device__ __forceinline__ void load_logits(const RouteArgs& a, int64_t t, double (&l)[EPL]) {
  constexpr int P = 4;
  const int lane = threadIdx.x & 31;
  const float* row = a.logits + t * a.ldl + lane;
#pragma unroll
  for (int j = 0; j < EPL; ++j) l[j] = 0.0;
  for (int p0 = 0; p0 < a.splits; p0 += P) {
    float part[P][EPL];
#pragma unroll
    for (int q = 0; q < P; ++q)
#pragma unroll
      for (int j = 0; j < EPL; ++j)
        part[q][j] = (p0 + q < a.splits && lane + 32 * j < a.E)
                         ? __ldg(row + (int64_t)(p0 + q) * a.split_stride + 32 * j)
                         : 0.0f;
#pragma unroll
    for (int q = 0; q < P; ++q)
      if (p0 + q < a.splits)
#pragma unroll
        for (int j = 0; j < EPL; ++j) l[j] += (double)part[q][j];
  }
}

// Queue token t for the batched binary64 refinement: its index, the experts in `refine` (bits
// over j of expert lane + 32 j, ascending) as its candidate row (count -1 past kRouteCandMax), and
// one pair per candidate (a run padded to a multiple of four).
template <int EPL>
__device__ void defer_token(const RouteArgs& a, int64_t t, uint32_t refine) {
  const int lane = threadIdx.x & 31;
  int qpos = 0;
  if (lane == 0) {
    qpos = atomicAdd(a.defer_len, 1);
    a.defer_queue[qpos] = (int32_t)t;
  }
  qpos = __shfl_sync(kFull, qpos, 0);
  int32_t* cand = a.defer_cand + (int64_t)qpos * (kRouteCandMax + 1);
  double* cand_val = a.defer_cand_val + (int64_t)qpos * (kRouteCandMax + 1);
  const uint32_t below = (1u << lane) - 1u;
  int nc = 0;
#pragma unroll
  for (int j = 0; j < EPL; ++j) {
    const bool mine = (refine >> j) & 1u;
    const uint32_t m = __ballot_sync(kFull, mine);
    const int pos = nc + __popc(m & below);
    if (mine && pos < kRouteCandMax) {
      cand[1 + pos] = lane + 32 * j;
      cand_val[1 + pos] = 0.0;  // the refinement adds its two halves' sums here
    }
    nc += __popc(m);
  }
  if (nc <= kRouteCandMax) {
    // one run, padded with -1 to a multiple of four (the refinement takes four pairs of a token at once)
    const int padded = (nc + 3) & ~3;
    int base = 0;
    if (lane == 0) {
      cand[0] = nc;
      base = atomicAdd(a.defer_pair_count, padded);
    }
    base = __shfl_sync(kFull, base, 0);
    for (int c = lane; c < padded; c += 32)
      a.defer_pairs[base + c] = c < nc ? qpos * (kRouteCandMax + 1) + 1 + c : -1;
  } else if (lane == 0) {
    cand[0] = -1;  // too many: the second pass finds and refines them itself
  }
  __syncwarp();
}

template <int EPL, bool FULL>
__global__ void __launch_bounds__(32 * kWarpsPerBlock) route_kernel(RouteArgs a) {
  __shared__ int16_t s_rank[kWarpsPerBlock][kMaxExperts];
  __shared__ uint8_t s_flag[kWarpsPerBlock][kMaxExperts];
  __shared__ int s_idx[kWarpsPerBlock][kMaxTopK];
  __shared__ double s_val[kWarpsPerBlock][kMaxTopK];
  __shared__ unsigned long long s_keys[kWarpsPerBlock][kMaxExperts];  // the group cut's scratch
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  constexpr bool full_ranking = FULL;  // the capacity rule needs every eligible expert ranked
  for (int i = lane; i < kMaxExperts; i += 32) s_flag[wib][i] = 0;
  __syncwarp();
  uint32_t valid_mask = 0;
#pragma unroll
  for (int j = 0; j < EPL; ++j)
    if (lane + 32 * j < a.E) valid_mask |= 1u << j;
  // A warp's first token is fixed by its place in the grid; after that it takes the next one from a
  // shared cursor (past the first W = the grid's warps), so a token that needs binary64 refinement
  // holds up only its own warp, and a warp without a token leaves after one load, never touching
  // the cursor (the grid is sized before the queue's length is known).
  const int64_t count = a.queue ? (int64_t)*a.queue_len : a.n;
  const int64_t W = (int64_t)gridDim.x * kWarpsPerBlock;
  for (bool first = true;; first = false) {
    int64_t i = (int64_t)blockIdx.x * kWarpsPerBlock + wib;
    if (!first) {
      int tok = 0;
      if (lane == 0) tok = atomicAdd(a.cursor, 1);
      i = W + __shfl_sync(kFull, tok, 0);
    }
    if (i >= count) break;
    const int64_t t = a.queue ? (int64_t)a.queue[i] : i;
    double l[EPL];
    load_logits<EPL>(a, t, l);
    double amax = 0.0;
#pragma unroll
    for (int j = 0; j < EPL; ++j)
      if ((valid_mask >> j) & 1u) amax = fmax(amax, fabs(l[j]));
    amax = warp_max(amax);
    // binary32 error bound of the logits, mapped to selection values
    // (sigmoid' <= 1/4; sqrtsoftplus' = sigmoid / (2 sqrtsoftplus) < 1/2)
    const double delta_l = ldexp(fmax(1.0, amax), -13);
    const double delta_v = a.score_fn == MOE_SCORE_SIGMOID ? 0.25 * delta_l
                           : a.score_fn == MOE_SCORE_SQRTSOFTPLUS ? 0.5 * delta_l
                                                                  : delta_l;
    uint32_t exact = 0;
    int nr = 0;
    int n_refined = 0;
    if (a.cand) {
      // experts the one-pass router found near a decision boundary, already recomputed in binary64
      // lane q reads candidate q, then each value goes to the lane that owns its expert
      const int32_t* c = a.cand + i * (kRouteCandMax + 1);
      const double* cv = a.cand_val + i * (kRouteCandMax + 1);
      const int nc = c[0];
      const int my_e = lane < nc ? c[1 + lane] : -1;
      const double my_v = lane < nc ? cv[1 + lane] : 0.0;
      for (int q = 0; q < nc; ++q) {
        const int e = __shfl_sync(kFull, my_e, q);
        const double v = __shfl_sync(kFull, my_v, q);
        if ((e & 31) == lane) {
#pragma unroll
          for (int j = 0; j < EPL; ++j)
            if (j == (e >> 5)) {
              l[j] = v;
              exact |= 1u << j;
            }
        }
      }
      n_refined += nc > 0 ? nc : 0;
    }
    bool deferred = false;
    for (int it = 0;; ++it) {
      uint32_t refine = 0;
      bool ok;
      if constexpr (FULL)
        ok = decide_full<EPL>(a, l, exact, delta_v, s_rank[wib], s_flag[wib], &nr, &refine, s_keys[wib]);
      else
        ok = decide<EPL>(a, l, exact, delta_v, s_rank[wib], &nr, &refine, s_keys[wib]);
      if (ok) break;
      refine &= ~exact;
      if (it == 0 && a.defer_queue && __any_sync(kFull, refine != 0)) {
        // the marked experts of every such token are refined together (launch_refine), and the
        // token decided again by the second pass over the queue
        defer_token<EPL>(a, t, refine);
        deferred = true;
        break;
      }
      if (it >= 3 || !__any_sync(kFull, refine != 0)) {
        // not settled by the marked experts: first the experts near any boundary under four times
        // the margin (a superset), and only if that marks nothing new, every remaining logit
        uint32_t wide = 0;
        if (it < 6) {
          int nr_w = 0;
          if constexpr (FULL)
            decide_full<EPL>(a, l, exact, 4.0 * delta_v, s_rank[wib], s_flag[wib], &nr_w, &wide, s_keys[wib]);
          else
            decide<EPL>(a, l, exact, 4.0 * delta_v, s_rank[wib], &nr_w, &wide, s_keys[wib]);
          wide &= ~exact;
        }
        refine = __any_sync(kFull, wide != 0) ? wide : (valid_mask & ~exact);
      }
      n_refined += refine_logits<EPL>(a, t, l, refine);
      exact |= refine;
    }
    if (deferred) continue;
    if (n_refined && lane == 0 && a.diag) {
      atomicAdd(&a.diag->refined_tokens, 1);
      atomicAdd(&a.diag->refined_logits, n_refined);
    }
    if (full_ranking) {
      for (int r = lane; r < a.E; r += 32) a.ranking[t * a.E + r] = r < nr ? (uint16_t)s_rank[wib][r] : (uint16_t)0xFFFF;
      __syncwarp();
      continue;
    }
    if (lane < a.k) s_idx[wib][lane] = lane < nr ? (int)s_rank[wib][lane] : -1;
    __syncwarp();
    const float w = gates<EPL>(a, l, s_idx[wib], s_val[wib]);
    if (lane < a.k) {
      a.topk_idx[t * a.k + lane] = s_idx[wib][lane];
      a.topk_w[t * a.k + lane] = w;
    }
    __syncwarp();
  }
}

// Gates of an existing selection (after the capacity rule), from the binary32 logits.
template <int EPL>
__global__ void __launch_bounds__(32 * kWarpsPerBlock) gates_kernel(RouteArgs a) {
  __shared__ int s_idx[kWarpsPerBlock][kMaxTopK];
  __shared__ double s_val[kWarpsPerBlock][kMaxTopK];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t t = warp; t < a.n; t += nwarps) {
    double l[EPL];
    load_logits<EPL>(a, t, l);
    if (lane < a.k) s_idx[wib][lane] = a.topk_idx[t * a.k + lane];
    __syncwarp();
    const float w = gates<EPL>(a, l, s_idx[wib], s_val[wib]);
    if (lane < a.k) a.topk_w[t * a.k + lane] = w;
    __syncwarp();
  }
}

// ---- hash routing and the balancing-bias update ------------------------------------
// Hash routing (page "15. DeepSeek: MLA, MoE and MTP", section V4): the experts
// of token t are row token_ids[t] of the fixed table tid2eid [vocab, k]; the
// router only weights them (gates_kernel). Out-of-range ids or table entries
// leave the slot empty (-1) and report MOE_ERR_INVALID_ARG in the status word.
__global__ void hash_select_kernel(const int32_t* token_ids, const int32_t* tid2eid, int32_t vocab, int64_t n,
                                   int32_t k, int32_t E, int32_t* topk_idx, moe_diag* status) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n * k; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = i / k;
    const int32_t tok = token_ids[t];
    int32_t e = -1;
    if (tok >= 0 && tok < vocab) e = tid2eid[(int64_t)tok * k + i % k];
    if (e < 0 || e >= E) {
      e = -1;
      set_status(status, MOE_ERR_INVALID_ARG);
    }
    topk_idx[i] = e;
  }
}

// Auxiliary-loss-free balancing (same page, section V3): an expert that received
// more slots than the mean has its selection bias lowered by gamma, one below
// the mean raised by gamma; the mean is sum(counts) / E.
__global__ void bias_update_kernel(const int32_t* counts, int32_t E, float gamma, float* bias) {
  __shared__ double total;
  if (threadIdx.x == 0) {
    double s = 0.0;
    for (int e = 0; e < E; ++e) s += counts[e];
    total = s;
  }
  __syncthreads();
  const double mean = total / E;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const double c = counts[e];
    double b = (double)bias[e];
    if (c > mean) b -= (double)gamma;
    else if (c < mean) b += (double)gamma;
    bias[e] = (float)b;
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
constexpr int kCapPrefix = 64;  // ranking entries per token staged in shared memory

// 32-bit words per staged row: enough for P entries and odd, so that the lanes
// of a warp reading the same ranking position hit 32 different banks.
__host__ __device__ constexpr int cap_row_words(int P) { return ((P + 1) / 2) | 1; }

// counts[e] += 1 for every lane whose slot holds e (e < 0: nothing), one
// shared-memory atomic per distinct expert in the warp: popular experts would
// otherwise serialise hundreds of atomics on one address.
__device__ __forceinline__ void warp_count(int* counts, int e) {
  const unsigned peers = __match_any_sync(kFull, e);
  if (e >= 0 && (threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&counts[e], __popc(peers));
}

// The block holds a window of 1024 tokens, one per thread. Each token keeps
// its current choices and a cursor into its ranking; after a fill event only
// the tokens that lost a choice walk on from their cursor, so every ranking
// entry of a window is read at most once.
// A token's current choices and their ranking positions. For k known at
// compile time (REG) the slots live in registers (indexed through unrolled
// selects); otherwise in a local array of kMaxTopK.
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

template <int KT>  // KT = top_k when it is 1, 2, 4 or 8; 0 = any top_k up to kMaxTopK
__global__ void __launch_bounds__(kCapThreads) capacity_kernel(const uint16_t* ranking, int64_t n, int E, int k_arg,
                                                            int64_t C, int policy, int32_t* topk_idx,
                                                            moe_diag* diag) {
  constexpr int KA = KT > 0 ? KT : kMaxTopK;
  const int k = KT > 0 ? KT : k_arg;
  extern __shared__ __align__(16) uint16_t st[];  // [kCapThreads][2 * row words] staged ranking prefixes
  __shared__ int cnt[kMaxExperts];
  __shared__ int ccnt[kMaxExperts];
  __shared__ uint32_t full[kMaxExperts / 32];
  __shared__ uint32_t ballots[kCapThreads / 32];
  __shared__ int cand[kMaxExperts];
  __shared__ int n_cand;
  __shared__ int stop;
  __shared__ unsigned long long s_over, s_drop;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int P = E < kCapPrefix ? E : kCapPrefix;
  const int RW = cap_row_words(P);  // 32-bit words per staged row
  for (int e = tid; e < kMaxExperts; e += kCapThreads) cnt[e] = 0;
  if (tid < kMaxExperts / 32) full[tid] = 0;
  if (tid == 0) s_over = s_drop = 0;
  __syncthreads();
  auto is_full = [&](int e) { return (full[e >> 5] >> (e & 31)) & 1u; };
  unsigned long long my_over = 0, my_drop = 0;
  for (int64_t w0 = 0; w0 < n; w0 += kCapThreads) {
    const int cnt_tok = (int)((n - w0) < kCapThreads ? (n - w0) : kCapThreads);
    if (E % 8 == 0) {
      const int vpr = P / 8;  // 16-byte vectors per staged row, stored as four words each
      uint32_t* st32 = reinterpret_cast<uint32_t*>(st);
      for (int i = tid; i < cnt_tok * vpr; i += kCapThreads) {
        const int row = i / vpr, v = i % vpr;
        const uint4 q = reinterpret_cast<const uint4*>(ranking + (w0 + row) * E)[v];
        uint32_t* dst = st32 + row * RW + 4 * v;
        dst[0] = q.x;
        dst[1] = q.y;
        dst[2] = q.z;
        dst[3] = q.w;
      }
    } else {
      for (int i = tid; i < cnt_tok * P; i += kCapThreads) st[(i / P) * 2 * RW + i % P] = ranking[(w0 + i / P) * E + i % P];
    }
    __syncthreads();
    const int64_t t = w0 + tid;
    const bool valid = tid < cnt_tok;
    const uint16_t* srow = st + tid * 2 * RW;
    const uint16_t* grow = ranking + t * E;
    Slots<KA, (KT > 0)> ch;   // current choices (in ranking order); -1 = empty slot
    Slots<KA, (KT > 0)> pos;  // their ranking positions
    int taken = 0, cursor = 0;
    // walk on from the cursor until k non-full experts are held (overflow policy)
    auto refill = [&]() {
      while (taken < k && cursor < E) {
        const int e = cursor < P ? srow[cursor] : grow[cursor];
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
    if (valid) {
      if (policy == MOE_CAP_OVERFLOW_NEXT) {
        refill();
      } else {
        for (int j = 0; j < k; ++j) {
          const int e = srow[j];
          ch.set(j, (e != 0xFFFF && !is_full(e)) ? e : -1);
        }
      }
    }
    int f = 0;  // first window position not committed yet (uniform across the block)
    while (true) {
      const bool active = valid && tid >= f;
      auto slot = [&](int j) {
        if (policy == MOE_CAP_OVERFLOW_NEXT) return j < taken ? ch.get(j) : -1;
        return ch.get(j);
      };
      for (int e = tid; e < E; e += kCapThreads) ccnt[e] = 0;
      if (tid == 0) {
        n_cand = 0;
        stop = kCapThreads;
      }
      __syncthreads();
      for (int j = 0; j < k; ++j) warp_count(ccnt, active ? slot(j) : -1);
      __syncthreads();
      for (int e = tid; e < E; e += kCapThreads)
        if (cnt[e] < C && cnt[e] + ccnt[e] >= C) cand[atomicAdd(&n_cand, 1)] = e;
      __syncthreads();
      const int nc = n_cand;
      for (int c = 0; c < nc; ++c) {
        const int e = cand[c];
        bool mine = false;
        if (active)
          for (int j = 0; j < k; ++j) mine |= slot(j) == e;
        const uint32_t b = __ballot_sync(kFull, mine);
        if (lane == 0) ballots[wid] = b;
        __syncthreads();
        if (tid == 0) {
          int need = (int)(C - cnt[e]);  // this expert's C-th slot goes to its need-th chooser
          for (int w = 0; w < kCapThreads / 32; ++w) {
            const int pc = __popc(ballots[w]);
            if (need <= pc) {
              uint32_t bb = ballots[w];
              for (int q = 1; q < need; ++q) bb &= bb - 1;
              const int at = w * 32 + __ffs(bb) - 1;
              if (at < stop) stop = at;
              break;
            }
            need -= pc;
          }
        }
        __syncthreads();
      }
      const int s = stop;  // last committed window position (kCapThreads: all of them)
      const bool commit = active && tid <= s;
      if (commit) {
        for (int j = 0; j < k; ++j) {
          const int e = slot(j);
          topk_idx[t * k + j] = e;
          my_drop += e < 0;
          if (policy == MOE_CAP_OVERFLOW_NEXT && j < taken) my_over += pos.get(j) >= k;
        }
      }
      if (s < kCapThreads) {
        for (int e = tid; e < E; e += kCapThreads) ccnt[e] = 0;
        __syncthreads();
        for (int j = 0; j < k; ++j) warp_count(ccnt, commit ? slot(j) : -1);
        __syncthreads();
      }
      for (int e = tid; e < E; e += kCapThreads) {
        cnt[e] += ccnt[e];
        if (cnt[e] >= C) atomicOr(&full[e >> 5], 1u << (e & 31));
      }
      __syncthreads();
      if (s >= cnt_tok - 1) break;  // the whole window is committed
      f = s + 1;
      // tokens still to come drop the experts that just filled
      if (valid && tid >= f) {
        if (policy == MOE_CAP_OVERFLOW_NEXT) {
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
    __syncthreads();
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

// Persistent grid: as many blocks as fit on the device at once (tokens come
// from the cursor), never more than the tokens need.
template <int EPL, bool FULL>
cudaError_t launch_route_t(const RouteArgs& a, cudaStream_t s) {
  static int resident = 0;
  if (!resident) {
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, route_kernel<EPL, FULL>, 32 * kWarpsPerBlock, 0) !=
            cudaSuccess ||
        per_sm <= 0)
      per_sm = 1;
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    resident = per_sm * (sms > 0 ? sms : 148);
  }
  const int64_t need = ceil_div(a.n, kWarpsPerBlock);
  const unsigned grid = (unsigned)(need < resident ? need : resident);
  route_kernel<EPL, FULL><<<grid, 32 * kWarpsPerBlock, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_route(const RouteArgs& a, cudaStream_t s) {
  if (a.n <= 0) return cudaSuccess;
  if (!a.cursor) return cudaErrorInvalidValue;
  const bool full = a.ranking != nullptr;
  switch (epl_for(a.E)) {
    case 1: return full ? launch_route_t<1, true>(a, s) : launch_route_t<1, false>(a, s);
    case 2: return full ? launch_route_t<2, true>(a, s) : launch_route_t<2, false>(a, s);
    case 4: return full ? launch_route_t<4, true>(a, s) : launch_route_t<4, false>(a, s);
    default: return full ? launch_route_t<8, true>(a, s) : launch_route_t<8, false>(a, s);
  }
}

cudaError_t launch_sum_splits(float* logits, int32_t splits, int64_t split_stride, int64_t n, int64_t ld, int32_t E,
                              cudaStream_t s) {
  if (n <= 0 || splits <= 1) return cudaSuccess;
  const int64_t blocks = ceil_div(n * E, 256);
  sum_splits_kernel<<<(unsigned)(blocks < 148 * 16 ? blocks : 148 * 16), 256, 0, s>>>(logits, splits, split_stride, n,
                                                                                     ld, E);
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

cudaError_t launch_hash_select(const int32_t* token_ids, const int32_t* tid2eid, int32_t vocab, int64_t n, int32_t k,
                               int32_t E, int32_t* topk_idx, moe_diag* status, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  const int64_t blocks = ceil_div(n * k, 256);
  hash_select_kernel<<<(unsigned)(blocks < 148 * 8 ? blocks : 148 * 8), 256, 0, s>>>(token_ids, tid2eid, vocab, n, k, E,
                                                                                  topk_idx, status);
  return cudaGetLastError();
}

cudaError_t launch_bias_update(const int32_t* counts, int32_t E, float gamma, float* bias, cudaStream_t s) {
  bias_update_kernel<<<1, 256, 0, s>>>(counts, E, gamma, bias);
  return cudaGetLastError();
}

cudaError_t launch_capacity(const uint16_t* ranking, int64_t n, int32_t E, int32_t k, int64_t C, int policy,
                            int32_t* topk_idx, moe_diag* diag, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  const int P = E < kCapPrefix ? E : kCapPrefix;
  const size_t smem = (size_t)kCapThreads * cap_row_words(P) * sizeof(uint32_t);
  static std::atomic<uint64_t> attr[5];
  {
    const size_t bytes = (size_t)kCapThreads * cap_row_words(kCapPrefix) * sizeof(uint32_t);
    const void* fs[5] = {(const void*)capacity_kernel<1>, (const void*)capacity_kernel<2>,
                         (const void*)capacity_kernel<4>, (const void*)capacity_kernel<8>,
                         (const void*)capacity_kernel<0>};
    for (int i = 0; i < 5; ++i) {
      const cudaError_t e = set_smem_limit(attr[i], fs[i], bytes);
      if (e != cudaSuccess) return e;
    }
  }
  switch (k) {
    case 1: capacity_kernel<1><<<1, kCapThreads, smem, s>>>(ranking, n, E, k, C, policy, topk_idx, diag); break;
    case 2: capacity_kernel<2><<<1, kCapThreads, smem, s>>>(ranking, n, E, k, C, policy, topk_idx, diag); break;
    case 4: capacity_kernel<4><<<1, kCapThreads, smem, s>>>(ranking, n, E, k, C, policy, topk_idx, diag); break;
    case 8: capacity_kernel<8><<<1, kCapThreads, smem, s>>>(ranking, n, E, k, C, policy, topk_idx, diag); break;
    default: capacity_kernel<0><<<1, kCapThreads, smem, s>>>(ranking, n, E, k, C, policy, topk_idx, diag); break;
  }
  return cudaGetLastError();
}

}  // namespace moe
