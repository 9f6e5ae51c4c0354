// route_tc.cu -- the router in one pass: logits x W_r^T on the tensor cores, and
// the whole routing decision of every token in the epilogue that drains them.
//
// Definitions (page "15. DeepSeek: MLA, MoE and MTP", section "V3 MoE: how 8 of
// 256 experts are chosen"; page "MoE architecture revealed", section 3.1; page
// "1.8T parameters / 2% per token", section 4.1):
//   softmax : select on the logits l; gates e^{l_j - m} / sum_E e^{l - m}
//             (renormalised over the kept slots when asked) times rsf;
//   sigmoid : s = sigmoid(l), selection value c = s + bias; groups of E/G
//             experts scored by the sum of their two best c, the topk_group
//             best groups eligible, top-k of c among them; gates s_j / sum s
//             (when asked) times rsf; sqrtsoftplus likewise with
//             s = sqrt(softplus(l)) (section "V4").
// Ties go to the lower expert (group) index; slots are in descending score.
//
// Design (one CTA per SM, persistent over 128-token tiles, 192 threads):
//   warp 0      TMA producer: 128 x 64 tile of x and E x 64 tile of W_r per
//               stage, 4-stage ring of 128-byte-swizzled shared memory;
//   warp 1      TMEM owner (two 128 x 256 fp32 accumulators) and MMA issuer,
//               tcgen05.mma kind::f16, M = 128, N = E rounded up to 16;
//   warps 2..9  routing epilogue: two warps per TMEM lane quarter q, thread i
//               of each owning token row 32q + i, each half of its experts; they
//               read the logits from TMEM 32 columns at a time and decide in
//               binary32: group scores, group cut, the k best eligible experts
//               kept sorted by insertion, gates (partials exchanged through
//               shared memory, half 0 finishing).
// Exactness: the logits are binary32 sums, so a decision is kept only when
// every gap it depends on (group cut, adjacent kept experts, the k-th / (k+1)-th
// cut) exceeds twice the error bound of the selection values; any other token
// has its logits row written out and its index appended to a queue, and the
// warp-per-token router (router.cu) re-decides it, recomputing in binary64 the
// logits near a boundary. Indices therefore equal the binary64 definition.
#include <cuda.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace moe {
namespace {

using namespace ptx;

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_MAX_BYTES = 256 * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_MAX_BYTES;
constexpr int kThreads = 320;  // producer, MMA issuer, 8 epilogue warps
constexpr uint32_t TMEM_COLS = 512;
constexpr int kMaxK = 8;  // experts per token the epilogue keeps sorted in registers
constexpr int kCandMax = kRouteCandMax;  // experts listed for the binary64 refinement of a queued token
constexpr uint64_t kTimeoutNs = 2000000000ull;
constexpr int kXg = 2 + 16;                 // per token and half: |l| max, logit max, 16 group scores
constexpr int kXl = 3 * (kMaxK + 1) + 2;     // per token: half 1's list (values, logits, experts), count, softmax sum
constexpr int XCHG_BYTES = (2 * BM * kXg + BM * kXl + 256) * 4;  // and the selection bias

struct __align__(8) Ctl {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tmem_full[2];
  uint64_t tmem_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int32_t abort;
};

__device__ __noinline__ bool wait_bar(uint64_t* bar, uint32_t parity, Ctl* ctl, moe_diag* st) {
  const uint32_t b = smem_u32(bar);
  if (mbar_try(b, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try(b, parity)) return true;
    if ((it & 255u) == 0) {
      if (*reinterpret_cast<volatile int32_t*>(&ctl->abort)) return false;
      if (globaltimer() - t0 > kTimeoutNs) {
        atomicExch(&ctl->abort, 1);
        set_status(st, MOE_ERR_TIMEOUT);
        return false;
      }
    }
  }
}

// 32 lanes x 32 columns of fp32 from TMEM.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ uint32_t idesc_bf16(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}

// Selection score of the biased routers in the epilogue's fast form: sigmoid from ex2.approx and a
// correctly rounded reciprocal (absolute error below 2^-18 for any logit, which the certification
// margin adds); sqrtsoftplus in the accurate form.
__device__ __forceinline__ float sel_score(int score_fn, float l) {
  if (score_fn == MOE_SCORE_SIGMOID) return __frcp_rn(1.0f + __expf(-l));
  return sqrtf(fmaxf(l, 0.0f) + log1pf(expf(-fabsf(l))));
}

// Insert (v, l, e) into the list sorted by v descending (l: what the gate needs, the logit for
// softmax and the unbiased score otherwise); an equal v stays below the entries
// already there, which hold lower expert indices (experts arrive in ascending order).
__device__ __forceinline__ void insert(float (&lv)[kMaxK + 1], float (&ll)[kMaxK + 1], int (&le)[kMaxK + 1], float v,
                                       float l, int e) {
  if (!(v > lv[kMaxK])) return;
#pragma unroll
  for (int j = 0; j <= kMaxK; ++j) {
    if (v > lv[j]) {
      const float tv = lv[j], tl = ll[j];
      const int te = le[j];
      lv[j] = v;
      ll[j] = l;
      le[j] = e;
      v = tv;
      l = tl;
      e = te;
    }
  }
}

// SF: the score function (compile time, so each instance holds one); FAST: whole 32-expert chunks
// per half and groups of whole chunks, so the loops need no per-expert checks.
template <int SF, bool FAST>
__global__ void __launch_bounds__(kThreads, 1)
    route_tc_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_w,
                    RouteTcArgs p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Ctl* ctl = reinterpret_cast<Ctl*>(smem + STAGES * STAGE_BYTES);
  float* xg = reinterpret_cast<float*>(smem + STAGES * STAGE_BYTES + 256);  // partials of the two halves
  float* xl = xg + 2 * BM * kXg;                                            // half 1's candidate lists
  volatile int32_t* vote = reinterpret_cast<volatile int32_t*>(smem + STAGES * STAGE_BYTES + 128);
  float* sbias = xl + BM * kXl;                                             // selection bias (0 without)
  for (int e = threadIdx.x; e < 256; e += kThreads) sbias[e] = (p.bias && e < p.E) ? p.bias[e] : 0.0f;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles = (int)((p.n + BM - 1) / BM);
  const int num_kb = (p.d + BK - 1) / BK;
  const int n_mma = (p.E + 15) & ~15;

  if (threadIdx.x == 0) {
    ctl->abort = 0;
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&ctl->full[s], 1);
      mbar_init(&ctl->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&ctl->tmem_full[b], 1);
      mbar_init(&ctl->tmem_empty[b], 8);
    }
    mbar_init(&ctl->drain, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&ctl->tmem_base)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem_base = ctl->tmem_base;

  if (warp == 0) {
    // ================= TMA producer =================
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed[STAGES] = {0, 0, 0, 0};
      const uint32_t tx = A_BYTES + (uint32_t)n_mma * BK * 2;
      bool ok = true;
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_try(smem_u32(&ctl->empty[stage]), phase ^ 1u) &&
              !wait_bar(&ctl->empty[stage], phase ^ 1u, ctl, p.status)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + stage * STAGE_BYTES;
          mbar_expect_tx(&ctl->full[stage], tx);
          ++armed[stage];
          tma_load_2d(sa, &map_x, &ctl->full[stage], kb * BK, t * BM);
          tma_load_2d(sa + A_BYTES, &map_w, &ctl->full[stage], kb * BK, 0);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok)
        for (int s = 0; s < STAGES; ++s)
          if (armed[s]) mbar_drain(&ctl->full[s], (armed[s] - 1) & 1u);
    }
  } else if (warp == 1) {
    // ================= MMA issuer =================
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      const uint32_t idesc = idesc_bf16(n_mma);
      bool ok = true, issued = false;
      int i = 0;
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, ++i) {
        const int buf = i & 1;
        const uint32_t acc_phase = (uint32_t)(i >> 1) & 1u;
        if (!wait_bar(&ctl->tmem_empty[buf], acc_phase ^ 1u, ctl, p.status)) {
          ok = false;
          break;
        }
        fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(buf * 256);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_try(smem_u32(&ctl->full[stage]), phase) && !wait_bar(&ctl->full[stage], phase, ctl, p.status)) {
            ok = false;
            break;
          }
          const uint32_t sa = smem_u32(smem + stage * STAGE_BYTES);
          const uint64_t adesc = sw128_desc(sa);
          const uint64_t bdesc = sw128_desc(sa + A_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            asm volatile(
                "{\n\t.reg .pred p;\n\t"
                "setp.ne.b32 p, %4, 0;\n\t"
                "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
                "l"(adesc + (uint64_t)(2 * k)), "l"(bdesc + (uint64_t)(2 * k)), "r"(idesc), "r"((kb | k) != 0 ? 1 : 0)
                : "memory");
          }
          issued = true;
          asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                           smem_u32(&ctl->empty[stage]))
                       : "memory");
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                         smem_u32(&ctl->tmem_full[buf]))
                     : "memory");
      }
      if (!ok && issued) {
        asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                         smem_u32(&ctl->drain))
                     : "memory");
        mbar_drain(&ctl->drain, 0);
      }
    }
  } else {
    // ================= routing epilogue (warps 2..9) =================
    // Two warps per TMEM lane quarter q (the lanes a warp may read): both own the token rows
    // 32q .. 32q + 31, half 0 the experts [0, e_split), half 1 the rest (a whole number of groups
    // each). They exchange their partial group scores and softmax sums, decide the group cut
    // redundantly, each keep their k + 1 best eligible experts, and half 0 merges the two lists,
    // certifies and writes the token's routing.
    const int q = warp & 3;
    const int h = (warp - 2) >> 2;
    const int E = p.E, G = p.G, per = p.E / p.G, k = p.k;
    constexpr bool soft = SF == MOE_SCORE_SOFTMAX;
    const int Gh = G > 1 ? (G + 1) / 2 : 1;  // groups of half 0
    const int e_split = G > 1 ? Gh * per : min(E, ((E / 2 + 31) / 32) * 32);
    const int e_lo = h ? e_split : 0, e_hi = h ? E : e_split;
    const int g_lo = h ? Gh : 0;
    // derivative bound of the selection value in the logit (sigmoid' <= 1/4, sqrtsoftplus' < 1/2)
    constexpr float lip = SF == MOE_SCORE_SIGMOID ? 0.25f : SF == MOE_SCORE_SQRTSOFTPLUS ? 0.5f : 1.0f;
    // binary32 evaluation error of a non-softmax selection value (a few ulp of a value near 1)
    constexpr float eval_err = soft ? 0.0f : 0x1p-18f;
    // whole 32-expert chunks per half and groups of whole chunks: the loops need no per-expert checks
    constexpr bool fast = FAST;
    const int row = q * 32 + lane;
    float* xg_mine = xg + ((size_t)h * BM + row) * kXg;
    const float* xg_other = xg + ((size_t)(h ^ 1) * BM + row) * kXg;
    float* xl_row = xl + (size_t)row * kXl;
    auto pair_sync = [&]() { asm volatile("bar.sync %0, %1;" ::"r"(1 + q), "r"(64) : "memory"); };
    int i = 0;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++i) {
      const int buf = i & 1;
      const uint32_t acc_phase = (uint32_t)(i >> 1) & 1u;
      // both warps of the pair go on or stop together (a named barrier waits for both)
      const bool got = wait_bar(&ctl->tmem_full[buf], acc_phase, ctl, p.status);
      __syncwarp();
      if (lane == 0) vote[h * 4 + q] = got ? 1 : 0;
      pair_sync();
      if (!(vote[q] && vote[4 + q])) break;
      fence_after();
      const int64_t tok = (int64_t)t * BM + row;
      const bool valid = tok < p.n;
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * 256);
      // pass 1 over this half's experts: |l| max, softmax max, group scores (top-2 sums of c)
      float amax = 0.0f, m = -INFINITY;
      if constexpr (fast) {
        // whole 32-expert chunks, groups of whole chunks: no per-expert range or group checks
        float g1 = -INFINITY, g2 = -INFINITY;
        for (int c0 = e_lo; c0 < e_hi; c0 += 32) {
          float l[32];
          tmem_ld32(taddr + (uint32_t)c0, l);
          if (soft || G == 1) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              amax = fmaxf(amax, fabsf(l[j]));
              m = fmaxf(m, l[j]);
            }
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              amax = fmaxf(amax, fabsf(l[j]));
              const float v = sel_score(SF, l[j]) + sbias[c0 + j];
              g2 = fmaxf(g2, fminf(g1, v));
              g1 = fmaxf(g1, v);
            }
            if ((c0 + 32) % per == 0) {
              xg_mine[2 + (c0 / per) - g_lo] = g1 + g2;
              g1 = g2 = -INFINITY;
            }
          }
        }
      } else {
        float g1 = -INFINITY, g2 = -INFINITY;
        int gpos = 0, gidx = 0;  // place inside the current group, and the group (experts arrive in order)
        for (int c0 = e_lo & ~31; c0 < e_hi; c0 += 32) {
          float l[32];
          tmem_ld32(taddr + (uint32_t)c0, l);
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int e = c0 + j;
            if (e >= e_lo && e < e_hi) {
              amax = fmaxf(amax, fabsf(l[j]));
              m = fmaxf(m, l[j]);
              if (!soft && G > 1) {
                const float v = sel_score(SF, l[j]) + sbias[e];
                g2 = fmaxf(g2, fminf(g1, v));
                g1 = fmaxf(g1, v);
                if (++gpos == per) {
                  xg_mine[2 + gidx++] = g1 + g2;
                  g1 = g2 = -INFINITY;
                  gpos = 0;
                }
              }
            }
          }
        }
      }
      xg_mine[0] = amax;
      xg_mine[1] = m;
      pair_sync();
      amax = fmaxf(amax, xg_other[0]);
      m = fmaxf(m, xg_other[1]);
      const float dl = 0x1p-13f * fmaxf(1.0f, amax);  // binary32 error bound of a logit
      const float dv = lip * dl + eval_err;              // ... of a selection value
      // group cut: the topk_group best group scores, ties to the lower group index
      bool ok = true;
      uint32_t kept = 0xFFFFFFFFu;
      if (!soft && G > 1) {
        auto gs = [&](int g) { return g < Gh ? (h ? xg_other : xg_mine)[2 + g] : (h ? xg_mine : xg_other)[2 + g - Gh]; };
        kept = 0;
        float min_kept = INFINITY, max_drop = -INFINITY;
        for (int g = 0; g < G; ++g) {
          const float sg = gs(g);
          int better = 0;
          for (int hh = 0; hh < G; ++hh) {
            const float so = gs(hh);
            better += (so > sg) || (so == sg && hh < g);
          }
          if (better < p.topk_group) {
            kept |= 1u << g;
            min_kept = fminf(min_kept, sg);
          } else {
            max_drop = fmaxf(max_drop, sg);
          }
        }
        if (p.topk_group < G && !(min_kept - max_drop > 4.0f * dv + 0x1p-19f)) ok = false;
      }
      // pass 2: this half's k + 1 best eligible experts, sorted (and the softmax normaliser)
      float lv[kMaxK + 1], ll[kMaxK + 1];
      int le[kMaxK + 1];
#pragma unroll
      for (int j = 0; j <= kMaxK; ++j) {
        lv[j] = -INFINITY;
        ll[j] = 0.0f;
        le[j] = -1;
      }
      int n_elig = 0;
      float z = 0.0f;
      for (int c0 = e_lo & ~31; c0 < e_hi; c0 += 32) {
        int g = c0 / per, r = c0 - g * per;  // group of expert c0 and its place in the group
        // skip a chunk that lies in a dropped group of every token of the warp (TMEM loads are warp-wide)
        if (!soft && per >= 32 && r + 32 <= per && !__any_sync(0xFFFFFFFFu, (kept >> g) & 1u)) continue;
        float l[32];
        tmem_ld32(taddr + (uint32_t)c0, l);
        if constexpr (fast) {
          const bool keptg = (kept >> g) & 1u;  // the whole chunk is in group g
          n_elig += keptg ? 32 : 0;
          // selection values of the chunk, and which of them beat the list's current floor; the
          // few that do are inserted one by one (a small loop, not 32 inlined insertions)
          const float floor0 = lv[kMaxK];
          uint32_t hit = 0;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            float v;
            if (soft) {
              v = l[j];
              z += __expf(l[j] - m);
            } else {
              v = sel_score(SF, l[j]) + sbias[c0 + j];
            }
            l[j] = v;  // the logit itself is needed only for the few inserted experts (read back below)
            hit |= (keptg && v > floor0) ? 1u << j : 0u;
          }
          while (hit) {
            const int j = __ffs(hit) - 1;
            hit &= hit - 1;
            float v = 0.0f;
#pragma unroll
            for (int u = 0; u < 32; ++u) v = u == j ? l[u] : v;
            // the gate needs the logit (softmax) or the unbiased score (the others)
            if (v > lv[kMaxK]) insert(lv, ll, le, v, soft ? v : v - sbias[c0 + j], c0 + j);
          }
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int e = c0 + j;
            if (e >= e_lo && e < e_hi) {
              if (soft) z += __expf(l[j] - m);
              if ((kept >> g) & 1u) {
                ++n_elig;
                const float sc = soft ? l[j] : sel_score(SF, l[j]);
                const float v = soft ? sc : sc + sbias[e];
                insert(lv, ll, le, v, sc, e);
              }
            }
            if (++r == per) {
              r = 0;
              ++g;
            }
          }
        }
      }
      (void)g_lo;
      if (h == 1) {
        // hand the list to half 0; this warp is done with the accumulator
#pragma unroll
        for (int j = 0; j <= kMaxK; ++j) {
          xl_row[j] = lv[j];
          xl_row[kMaxK + 1 + j] = ll[j];
          xl_row[2 * (kMaxK + 1) + j] = __int_as_float(le[j]);
        }
        xl_row[3 * (kMaxK + 1)] = __int_as_float(n_elig);
        xl_row[3 * (kMaxK + 1) + 1] = z;
        fence_before();
        pair_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->tmem_empty[buf]);
        continue;
      }
      pair_sync();
      {
        // merge the other half's list (higher expert indices: on equal values this half's come first)
        float ov[kMaxK + 1], ol[kMaxK + 1];
        int oe[kMaxK + 1];
#pragma unroll
        for (int j = 0; j <= kMaxK; ++j) {
          ov[j] = xl_row[j];
          ol[j] = xl_row[kMaxK + 1 + j];
          oe[j] = __float_as_int(xl_row[2 * (kMaxK + 1) + j]);
        }
        n_elig += __float_as_int(xl_row[3 * (kMaxK + 1)]);
        z += xl_row[3 * (kMaxK + 1) + 1];
#pragma unroll
        for (int j = 0; j <= kMaxK; ++j) insert(lv, ll, le, ov[j], ol[j], oe[j] < 0 ? 0x7FFFFFFF : oe[j]);
      }
      // every order the result depends on must be certain: adjacent kept experts and the k-th / (k+1)-th cut
#pragma unroll
      for (int j = 0; j < kMaxK; ++j)
        if (j < k && j + 1 < n_elig && !(lv[j] - lv[j + 1] > 2.0f * dv)) ok = false;
      const bool spill = valid && !ok;
      if (valid && ok) {
        // gates of the k kept experts
        float w[kMaxK];
        float denom = 1.0f;
        if (soft) {
#pragma unroll
          for (int j = 0; j < kMaxK; ++j) w[j] = j < k ? expf(ll[j] - m) / z : 0.0f;
        } else {
#pragma unroll
          for (int j = 0; j < kMaxK; ++j) w[j] = j < k ? ll[j] : 0.0f;  // the unbiased scores
        }
        if (p.renorm) {
          float s = 0.0f;
#pragma unroll
          for (int j = 0; j < kMaxK; ++j) s += j < k ? w[j] : 0.0f;
          denom = s;
        }
#pragma unroll
        for (int j = 0; j < kMaxK; ++j)
          if (j < k) {
            p.topk_idx[tok * k + j] = le[j];
            p.topk_w[tok * k + j] = w[j] / denom * p.rsf;
          }
      }
      // not certain: hand the token to the binary64 router with its logits row (the TMEM loads are
      // warp-wide, so the whole warp reads when any lane spills). That router decides it from the
      // row in binary64, queues the experts an uncertain comparison involves for refine_kernel, and
      // decides it again with their binary64 logits.
      if (__any_sync(0xFFFFFFFFu, spill)) {
        float* lrow = p.logits + tok * p.ldl;
        for (int c0 = 0; c0 < E; c0 += 32) {
          float l[32];
          tmem_ld32(taddr + (uint32_t)c0, l);
          if (spill) {
#pragma unroll
            for (int j = 0; j < 32; j += 4)
              if (c0 + j + 4 <= E) {
                *reinterpret_cast<float4*>(lrow + c0 + j) = make_float4(l[j], l[j + 1], l[j + 2], l[j + 3]);
              } else {
#pragma unroll
                for (int u = 0; u < 4; ++u)
                  if (c0 + j + u < E) lrow[c0 + j + u] = l[j + u];
              }
          }
        }
        if (spill) p.queue[atomicAdd(p.queue_len, 1)] = (int32_t)tok;
      }
      fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->tmem_empty[buf]);
    }
  }

  fence_before();
  __syncthreads();
  fence_after();
  if (warp == 1) {
    __syncwarp();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS) : "memory");
  }
}

// One item of refine_kernel: the binary64 dot products of x[t] with the NQ listed rows of W_r over
// chunks [c_lo, c_hi) of 8 elements. NQ is the number of live pairs in the item's group of four (the
// padding of a token's run is at its end), so no conversion or DFMA is spent on padding.
template <int NQ>
__device__ __forceinline__ void refine_rows(const uint4* xr, const uint4* const (&wr)[4], int c_lo, int c_hi, int lane,
                                            double (&acc)[4]) {
  constexpr int U = 4;
  for (int c = c_lo + lane; c < c_hi; c += 32 * U) {
    uint4 xv[U], wv[NQ][U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int cc = c + 32 * u;
      xv[u] = cc < c_hi ? __ldg(xr + cc) : make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int q = 0; q < NQ; ++q) wv[q][u] = cc < c_hi ? __ldg(wr[q] + cc) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const bf16* xs = reinterpret_cast<const bf16*>(&xv[u]);
#pragma unroll
      for (int h = 0; h < 8; ++h) {
        const double xd = (double)__bfloat162float(xs[h]);
#pragma unroll
        for (int q = 0; q < NQ; ++q)
          acc[q] = fma(xd, (double)__bfloat162float(reinterpret_cast<const bf16*>(&wv[q][u])[h]), acc[q]);
      }
    }
  }
}

// Binary64 logits x[t] . W_r[e] of the listed (queued token, candidate expert) pairs. Each token's
// pairs are listed as one run padded with -1 to a multiple of four, so a warp takes four pairs of
// one token and one half of the rows: the token's row is read and widened once for the four
// experts, and only the live pairs of the four are computed. Products of two bf16 values are exact
// in binary64; the sums are DFMA, the lanes taking 16-byte chunks in turn with four chunks of every
// row in flight. The two halves' sums are added into the zeroed candidate values (two terms: the
// same result in either order). A warp's first item is fixed by its place in the grid (W warps);
// only a warp that finished one takes the next from the shared cursor, past the first W. A grid
// sized for the largest possible list then costs the warps without work one load each, and long
// lists still balance across the warps.
__global__ void __launch_bounds__(256) refine_kernel(RouteTcArgs p, int32_t* cursor) {
  const int lane = threadIdx.x & 31;
  const int quads = *p.pair_count / 4;
  const int nchunk = p.d / 8;
  const int W = (int)(gridDim.x * (blockDim.x / 32));
  for (int item = (int)(blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5)); item < 2 * quads;) {
    const int i = item >> 1, half = item & 1;
    const int c_lo = half ? nchunk / 2 : 0, c_hi = half ? nchunk : nchunk / 2;
    int slot[4], e[4];
    int live = 0;
    unsigned live_mask = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      slot[q] = p.pairs[4 * i + q];
      e[q] = slot[q] >= 0 ? p.cand[slot[q]] : -1;
      live += e[q] >= 0;
      live_mask |= (e[q] >= 0 ? 1u : 0u) << q;
    }
    const int64_t t = p.queue[slot[0] / (kCandMax + 1)];  // a run starts every group of four
    const uint4* xr = reinterpret_cast<const uint4*>(static_cast<const bf16*>(p.x) + t * p.d);
    const uint4* wr[4];
#pragma unroll
    for (int q = 0; q < 4; ++q)
      wr[q] = reinterpret_cast<const uint4*>(static_cast<const bf16*>(p.w_r) + (int64_t)(e[q] < 0 ? 0 : e[q]) * p.d);
    double acc[4] = {0.0, 0.0, 0.0, 0.0};
    // The live pairs lead the group (padding ends a run); every lane reads the same four pairs. Any
    // other pattern computes all four rows, a dead one from row 0, and keeps only the live sums.
    if (live == 4 || live_mask != (1u << live) - 1u) {
      refine_rows<4>(xr, wr, c_lo, c_hi, lane, acc);
    } else if (live == 3) {
      refine_rows<3>(xr, wr, c_lo, c_hi, lane, acc);
    } else if (live == 2) {
      refine_rows<2>(xr, wr, c_lo, c_hi, lane, acc);
    } else if (live == 1) {
      refine_rows<1>(xr, wr, c_lo, c_hi, lane, acc);
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      double v = acc[q];
#pragma unroll
      for (int off = 16; off; off >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, off);
      if (lane == 0 && slot[q] >= 0 && e[q] >= 0) atomicAdd(&p.cand_val[slot[q]], v);
    }
    int next = 0;
    if (lane == 0) next = atomicAdd(cursor, 1);
    item = W + __shfl_sync(0xFFFFFFFFu, next, 0);
  }
}

bool make_map(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)(cols * 2)};
  const cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static_assert(sizeof(Ctl) <= 128, "control block");
constexpr size_t kSmemBytes = 1024 + STAGES * STAGE_BYTES + 256 + XCHG_BYTES;
static_assert(kSmemBytes <= 232448, "dynamic shared memory above 227 KB");

}  // namespace

bool route_tc_supported(const RouteTcArgs& a) {
  const char* inj = getenv("MOE_TEST_NO_TENSOR_MAPS");
  if (inj && inj[0] == '1') return false;
  if (a.E < 1 || a.E > 256 || a.k < 1 || a.k > kMaxK || a.G < 1 || a.G > kMaxGroups || a.E % a.G != 0) return false;
  if ((a.G + 1) / 2 > 16) return false;  // group scores of a half in the exchange block
  if (a.d % 8 != 0 || a.ldl % 4 != 0 || a.ldl < a.E) return false;
  if (reinterpret_cast<uintptr_t>(a.x) % 16 || reinterpret_cast<uintptr_t>(a.w_r) % 16 ||
      reinterpret_cast<uintptr_t>(a.logits) % 16)
    return false;
  return encode_fn() != nullptr;
}

cudaError_t launch_route_tc(const RouteTcArgs& a, cudaStream_t s) {
  if (!route_tc_supported(a)) return cudaErrorNotSupported;
  if (a.n <= 0) return cudaSuccess;
  CUtensorMap mx, mw;
  if (!make_map(&mx, a.x, a.n, a.d, BM)) return cudaErrorInvalidValue;
  if (!make_map(&mw, a.w_r, a.E, a.d, (a.E + 15) & ~15)) return cudaErrorInvalidValue;
  // the instance: score function, and whether every half and group is a whole number of 32-expert chunks
  const int G = a.G, per = a.E / a.G;
  const int Gh = G > 1 ? (G + 1) / 2 : 1;
  const int e_split = G > 1 ? Gh * per : (a.E / 2 + 31) / 32 * 32 < a.E ? (a.E / 2 + 31) / 32 * 32 : a.E;
  const bool fast = a.E % 32 == 0 && e_split % 32 == 0 && (G == 1 || per % 32 == 0);
  using Kern = void (*)(const CUtensorMap, const CUtensorMap, RouteTcArgs);
  Kern kern;
  static std::atomic<uint64_t> attr[6];
  int which = 0;
  if (a.score_fn == MOE_SCORE_SOFTMAX) {
    kern = fast ? route_tc_kernel<MOE_SCORE_SOFTMAX, true> : route_tc_kernel<MOE_SCORE_SOFTMAX, false>;
    which = fast ? 0 : 1;
  } else if (a.score_fn == MOE_SCORE_SIGMOID) {
    kern = fast ? route_tc_kernel<MOE_SCORE_SIGMOID, true> : route_tc_kernel<MOE_SCORE_SIGMOID, false>;
    which = fast ? 2 : 3;
  } else {
    kern = fast ? route_tc_kernel<MOE_SCORE_SQRTSOFTPLUS, true> : route_tc_kernel<MOE_SCORE_SQRTSOFTPLUS, false>;
    which = fast ? 4 : 5;
  }
  {
    const cudaError_t e = set_smem_limit(attr[which], (const void*)kern, kSmemBytes);
    if (e != cudaSuccess) return e;
  }
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (sms <= 0) sms = 148;
  const int64_t tiles = ceil_div(a.n, BM);
  const unsigned grid = (unsigned)(tiles < sms ? tiles : sms);
  kern<<<grid, kThreads, kSmemBytes, s>>>(mx, mw, a);
  return cudaGetLastError();
}

cudaError_t launch_refine(const RouteTcArgs& a, cudaStream_t s) {
  if (a.n <= 0) return cudaSuccess;
  if (a.d % 8 != 0 || reinterpret_cast<uintptr_t>(a.x) % 16 || reinterpret_cast<uintptr_t>(a.w_r) % 16)
    return cudaErrorInvalidValue;
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (sms <= 0) sms = 148;
  // at most two warps per four listed pairs, and n * kRouteCandMax pairs can be listed
  const int64_t need = ceil_div(a.n * kCandMax / 2, 8);
  const unsigned grid = (unsigned)(need < sms * 8 ? need : sms * 8);
  refine_kernel<<<grid, 256, 0, s>>>(a, a.pair_count + 1);
  return cudaGetLastError();
}

}  // namespace moe
