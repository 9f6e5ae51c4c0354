// gemm_tc.cu -- grouped GEMM on the 5th-generation tensor cores (tcgen05).
//
// For every group g (an expert, or the single shared-expert / router problem)
// and every row r of that group:
//   plain : C[r, n]  = sum_k A[r, k] * B_g[n, k]
//   SwiGLU: C[r, i]  = silu(sum_k A[r, k] Bg_g[i, k]) * (sum_k A[r, k] Bu_g[i, k])
// (page "15. DeepSeek: MLA, MoE and MTP", section "671B and 37B": gate, up,
// down matrices; page "MoE" tag feed, activation functions: SwiGLU).
//
// Design (one CTA per SM, persistent, warp-specialised, 192 threads):
//   warp 0      TMA producer: 128x64 A tile + 256x64 B tile per stage into a
//               4-stage ring of 128B-swizzled shared memory (48 KB per stage);
//               for SwiGLU the B tile is 128 gate rows over 128 up rows of the
//               same output columns, so one MMA produces both.
//   warp 1      TMEM owner (512 columns = two 128x256 fp32 accumulators) and
//               MMA issuer: tcgen05.mma kind::f16 (bf16 x bf16 -> fp32),
//               M=128, N=256, K=16, four per stage; tcgen05.commit frees the
//               stage and, after the last stage, hands the accumulator over.
//   warps 2..5  epilogue: tcgen05.ld 32 lanes x 16 columns, SwiGLU in fp32,
//               bf16 (or fp32) stores of the rows inside the group; it drains
//               one accumulator while the MMA fills the other.
// Tiles are ordered (group, n-tile, m-tile) so that the CTAs running at the
// same time share B tiles through L2. Every mbarrier wait is bounded: past the
// limit the kernel records MOE_ERR_TIMEOUT in the status word, stops issuing,
// waits (bounded) for its copies and MMAs in flight, frees TMEM and returns.
#include <cuda.h>
#include <stdlib.h>
#include <string.h>

#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace moe {
namespace {

using namespace ptx;

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int BN_MAX = 256;
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BN_MAX * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int kThreads = 192;
constexpr uint32_t TMEM_COLS = 512;
constexpr int kMaxGroupsTc = 256;
constexpr uint64_t kTimeoutNs = 2000000000ull;      // 2 s for any single wait
constexpr uint64_t kTestTimeoutNs = 50000000ull;    // 50 ms under injected stalls

struct TcParams {
  int32_t G;
  const int32_t* offsets;  // [G + 1] row offsets, or nullptr: one group of M rows
  int32_t M;
  int32_t N;       // valid output columns per group
  int32_t K;
  int32_t n_mma;   // MMA N (multiple of 16, <= 256)
  int32_t n_out;   // output columns per tile (SwiGLU: n_mma / 2)
  int32_t b_rows;  // rows per group in the B tensor maps
  int32_t swiglu;
  int32_t out_f32;
  int32_t k_splits;   // split-K factor (partials to C + split * c_split_stride)
  int32_t kb_per;     // k-blocks per split
  void* C;
  int64_t ldc;
  int64_t c_split_stride;
  moe_diag* status;
  uint64_t timeout_ns;  // limit of any single barrier wait
  int32_t test_stall;   // fault injection: withhold the first copy of each CTA
  int32_t* tile_counter;  // SM-pair kernel: next tile to hand out (zeroed before the launch)
};

struct __align__(8) SmemCtl {
  uint64_t timeout_ns;
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tmem_full[2];
  uint64_t tmem_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int32_t abort;
  int32_t total_tiles;
  int32_t n_tiles;
  int32_t row_off[kMaxGroupsTc + 1];
  int32_t tile_off[kMaxGroupsTc + 1];
};

// Bounded wait for the phase of `parity` to complete. False on timeout or abort.
__device__ __noinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, SmemCtl* ctl, moe_diag* st) {
  const uint32_t b = smem_u32(bar);
  if (mbar_try(b, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try(b, parity)) return true;
    if ((it & 255u) == 0) {
      if (*reinterpret_cast<volatile int32_t*>(&ctl->abort)) return false;
      if (globaltimer() - t0 > ctl->timeout_ns) {
        atomicExch(&ctl->abort, 1);
        set_status(st, MOE_ERR_TIMEOUT);
        return false;
      }
    }
  }
}

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// kind::f16 instruction descriptor: bf16 A and B, fp32 D, both K-major, M = 128.
__device__ __forceinline__ uint32_t idesc_bf16(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// ---- tile mapping ----------------------------------------------------------------
struct Tile {
  int g, m, nt, split;
  int half;    // SM-pair kernel: half-height (M = 128) last tile of its group
  int lo, hi;  // SM-pair kernel: the group's rows
};

// Tiles of group g are tile_off[g] .. tile_off[g+1]-1, ordered split major,
// then n-tile, then m-tile.
__device__ __forceinline__ Tile decode(const SmemCtl* ctl, int G, int t, int& g_hint) {
  int g = g_hint;
  while (g + 1 <= G && ctl->tile_off[g + 1] <= t) ++g;
  g_hint = g;
  const int local = t - ctl->tile_off[g];
  const int mt = (ctl->row_off[g + 1] - ctl->row_off[g] + BM - 1) / BM;
  const int per_split = mt * ctl->n_tiles;
  const int rem = local % per_split;
  return Tile{g, rem % mt, rem / mt, local / per_split, 0, 0, 0};
}

__device__ __forceinline__ void store16(void* C, int64_t ldc, int64_t row, int col, int N, const float (&v)[16],
                                        bool f32) {
  if (f32) {
    float* p = static_cast<float*>(C) + row * ldc + col;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if (col + 4 * q + 4 <= N) {
        *reinterpret_cast<float4*>(p + 4 * q) = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e)  // last columns of a row whose width is not a multiple of 4
          if (col + 4 * q + e < N) p[4 * q + e] = v[4 * q + e];
      }
    }
  } else {
    bf16* p = static_cast<bf16*>(C) + row * ldc + col;
    uint4 lo, hi;
    __nv_bfloat162* l2 = reinterpret_cast<__nv_bfloat162*>(&lo);
    __nv_bfloat162* h2 = reinterpret_cast<__nv_bfloat162*>(&hi);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      l2[q] = __floats2bfloat162_rn(v[2 * q], v[2 * q + 1]);
      h2[q] = __floats2bfloat162_rn(v[8 + 2 * q], v[8 + 2 * q + 1]);
    }
    if (col + 8 <= N) *reinterpret_cast<uint4*>(p) = lo;
    if (col + 16 <= N) *reinterpret_cast<uint4*>(p + 8) = hi;
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                   const __grid_constant__ CUtensorMap map_b2, TcParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  SmemCtl* ctl = reinterpret_cast<SmemCtl*>(smem + STAGES * STAGE_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- set-up: group row offsets, tile offsets, barriers, TMEM ----
  if (threadIdx.x == 0) {
    int acc = 0;
    const int n_tiles = (p.N + p.n_out - 1) / p.n_out;
    for (int g = 0; g < p.G; ++g) {
      const int lo = p.offsets ? p.offsets[g] : 0;
      const int hi = p.offsets ? p.offsets[g + 1] : p.M;
      ctl->row_off[g] = lo;
      ctl->row_off[g + 1] = hi;
      ctl->tile_off[g] = acc;
      acc += ((hi - lo + BM - 1) / BM) * n_tiles * p.k_splits;
    }
    ctl->tile_off[p.G] = acc;
    ctl->total_tiles = acc;
    ctl->n_tiles = n_tiles;
    ctl->abort = 0;
    ctl->timeout_ns = p.timeout_ns;
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&ctl->full[s], 1);
      mbar_init(&ctl->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&ctl->tmem_full[b], 1);
      mbar_init(&ctl->tmem_empty[b], 4);
    }
    mbar_init(&ctl->drain, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&map_a);
    tma_prefetch_desc(&map_b);
    if (p.swiglu) tma_prefetch_desc(&map_b2);
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
  const int total = ctl->total_tiles;
  const int num_kb_all = (p.K + BK - 1) / BK;

  if (warp == 0) {
    // ================= TMA producer =================
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int g_hint = 0;
      uint32_t armed[STAGES] = {0, 0, 0, 0};
      const uint32_t tx = A_BYTES + (uint32_t)p.n_mma * BK * 2;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const Tile tl = decode(ctl, p.G, t, g_hint);
        const int row0 = ctl->row_off[tl.g] + tl.m * BM;
        const int brow = tl.g * p.b_rows + tl.nt * p.n_out;
        const int kb0 = tl.split * p.kb_per, kb1 = min(num_kb_all, kb0 + p.kb_per);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_try(smem_u32(&ctl->empty[stage]), phase ^ 1u) &&
              !mbar_wait(&ctl->empty[stage], phase ^ 1u, ctl, p.status)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + stage * STAGE_BYTES;
          uint8_t* sb = sa + A_BYTES;
          if (p.test_stall && t == (int)blockIdx.x && kb == kb0) {
            // injected fault: this stage is never filled, so the MMA's wait on it runs out
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
            continue;
          }
          mbar_expect_tx(&ctl->full[stage], tx);
          ++armed[stage];
          tma_load_2d(sa, &map_a, &ctl->full[stage], kb * BK, row0);
          if (p.swiglu) {
            tma_load_2d(sb, &map_b, &ctl->full[stage], kb * BK, brow);
            tma_load_2d(sb + (p.n_mma / 2) * BK * 2, &map_b2, &ctl->full[stage], kb * BK, brow);
          } else {
            tma_load_2d(sb, &map_b, &ctl->full[stage], kb * BK, brow);
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        // Let the copies already issued land before the block exits.
        for (int s = 0; s < STAGES; ++s)
          if (armed[s]) mbar_drain(&ctl->full[s], (armed[s] - 1) & 1u);
      }
    }
  } else if (warp == 1) {
    // ================= MMA issuer =================
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      const uint32_t idesc = idesc_bf16(p.n_mma);
      bool ok = true;
      bool issued = false;
      int i = 0;
      int g_hint = 0;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++i) {
        const Tile tl = decode(ctl, p.G, t, g_hint);
        const int nkb = min(num_kb_all, (tl.split + 1) * p.kb_per) - tl.split * p.kb_per;
        const int buf = i & 1;
        const uint32_t acc_phase = (uint32_t)(i >> 1) & 1u;
        if (!mbar_wait(&ctl->tmem_empty[buf], acc_phase ^ 1u, ctl, p.status)) {
          ok = false;
          break;
        }
        fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(buf * BN_MAX);
        for (int kb = 0; kb < nkb; ++kb) {
          // The copies completed on this barrier; the MMAs read them through the
          // async proxy as well, so no tcgen05 fence is needed here.
          if (!mbar_try(smem_u32(&ctl->full[stage]), phase) && !mbar_wait(&ctl->full[stage], phase, ctl, p.status)) {
            ok = false;
            break;
          }
          const uint32_t sa = smem_u32(smem + stage * STAGE_BYTES);
          const uint64_t adesc = sw128_desc(sa);
          const uint64_t bdesc = sw128_desc(sa + A_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)  // advance 16 elements = 32 bytes inside the swizzle atom
            mma_bf16(d_tmem, adesc + (uint64_t)(2 * k), bdesc + (uint64_t)(2 * k), idesc, (kb | k) != 0);
          issued = true;
          mma_commit(&ctl->empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit(&ctl->tmem_full[buf]);
      }
      if (!ok && issued) {
        // Wait for the MMAs already issued before TMEM is released.
        mma_commit(&ctl->drain);
        mbar_drain(&ctl->drain, 0);
      }
    }
  } else {
    // ================= epilogue (warps 2..5) =================
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int row_in_tile = q * 32 + lane;
    int g_hint = 0;
    int i = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++i) {
      const int buf = i & 1;
      const uint32_t acc_phase = (uint32_t)(i >> 1) & 1u;
      const Tile tl = decode(ctl, p.G, t, g_hint);
      const bool got = mbar_wait(&ctl->tmem_full[buf], acc_phase, ctl, p.status);
      __syncwarp();  // tcgen05.ld below is warp-aligned
      if (!got) break;
      fence_after();
      const int64_t row = (int64_t)ctl->row_off[tl.g] + tl.m * BM + row_in_tile;
      const bool valid = row < ctl->row_off[tl.g + 1];
      const int col0 = tl.nt * p.n_out;
      void* C = p.out_f32 ? (void*)(static_cast<float*>(p.C) + (int64_t)tl.split * p.c_split_stride)
                          : (void*)(static_cast<bf16*>(p.C) + (int64_t)tl.split * p.c_split_stride);
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * BN_MAX);
      if (p.swiglu) {
        for (int c = 0; c < p.n_out; c += 16) {
          float gv[16], uv[16];
          tmem_ld16(taddr + (uint32_t)c, gv);
          tmem_ld16(taddr + (uint32_t)(p.n_out + c), uv);
#pragma unroll
          for (int e = 0; e < 16; ++e) gv[e] = silu(gv[e]) * uv[e];
          if (valid && col0 + c < p.N) store16(C, p.ldc, row, col0 + c, p.N, gv, false);
        }
      } else {
        for (int c = 0; c < p.n_out; c += 16) {
          float v[16];
          tmem_ld16(taddr + (uint32_t)c, v);
          if (valid && col0 + c < p.N) store16(C, p.ldc, row, col0 + c, p.N, v, p.out_f32 != 0);
        }
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
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS)
                 : "memory");
  }
}

// ---- 2-SM variant (cta_group::2) -----------------------------------------------------
// A CTA pair (cluster of 2) computes a 256 x 256 tile: CTA r holds A rows
// [128r, 128r+128) of the tile and B rows [128r, 128r+128). The leader CTA
// (rank 0) issues tcgen05.mma.cta_group::2 with M = 256, which reads the peer's
// operand halves through the pair's shared memory, so each SM stages 32 KB per
// 64-k step instead of 48 KB. The last m-tile of a group whose remainder is at
// most 128 rows is a half-height tile: M = 128, 64 A rows per CTA, so groups
// are padded to 128 rows, not 256. For SwiGLU, CTA r stages gate rows
// [64r, 64r+64) of the tile's 128 output columns over the up rows of the same
// columns, so each output column finds its gate and up accumulators in one TMEM
// lane in both tile heights. Both CTAs' copies signal the leader's `full`
// barrier; the leader's commits are multicast to both CTAs; both epilogues
// report to the leader's `tmem_empty` barrier. No TMA multicast is used.
constexpr int BM2 = 256;        // rows per pair tile
constexpr int STAGES2 = 7;      // 7 x 32 KB ring; the group row offsets stay in global memory to make room
constexpr int A2_BYTES = 128 * BK * 2;
constexpr int A2_HALF_BYTES = 64 * BK * 2;  // half-height tile: 64 A rows per CTA
constexpr int B2_BYTES = 128 * BK * 2;
constexpr int STAGE2_BYTES = A2_BYTES + B2_BYTES;

constexpr int kTileSlots = 4;    // tile indices published ahead of the slowest reader
constexpr int kTileReaders = 10;  // leader MMA + 4 leader epilogue warps + peer producer + 4 peer epilogue warps

struct __align__(8) SmemCtl2 {
  uint64_t timeout_ns;
  uint64_t full[STAGES2];
  uint64_t empty[STAGES2];
  uint64_t tmem_full[2];
  uint64_t tmem_empty[2];
  uint64_t tile_full[kTileSlots];   // both CTAs: tile_ring[slot] holds the next tile
  uint64_t tile_empty[kTileSlots];  // leader CTA: every reader of both CTAs took the slot's tile
  int32_t tile_ring[kTileSlots];
  uint64_t drain;
  uint32_t tmem_base;
  int32_t abort;
  int32_t total_tiles;
  int32_t n_tiles;
  int32_t tile_off[kMaxGroupsTc + 1];
};

__device__ __forceinline__ void mma_bf16_pair(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

// Arrive on the barrier at this offset in both CTAs of the pair once the MMAs complete.
__device__ __forceinline__ void mma_commit_pair(uint64_t* bar) {
  const uint16_t mask = 0x3;
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(mask)
      : "memory");
}

__device__ __forceinline__ uint32_t idesc_bf16_pair(int m, int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

__device__ __forceinline__ int group_row(const TcParams& p, int g) {
  return p.offsets ? __ldg(p.offsets + g) : (g == 0 ? 0 : p.M);
}

__device__ __forceinline__ Tile decode2(const SmemCtl2* ctl, const TcParams& p, int t, int& g_hint) {
  int g = g_hint;
  while (g + 1 <= p.G && ctl->tile_off[g + 1] <= t) ++g;
  g_hint = g;
  const int local = t - ctl->tile_off[g];
  const int lo = group_row(p, g);
  const int rows = group_row(p, g + 1) - lo;
  const int mt = (rows + BM2 - 1) / BM2;
  const int m = local % mt;
  // the last m-tile is half height when at most 128 rows remain
  const int half = (m == mt - 1 && rows - m * BM2 <= BM2 / 2) ? 1 : 0;
  return Tile{g, m, local / mt, 0, half, lo, lo + rows};
}

__device__ __noinline__ bool mbar_wait2(uint64_t* bar, uint32_t parity, SmemCtl2* ctl, moe_diag* st) {
  const uint32_t b = smem_u32(bar);
  if (mbar_try(b, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try(b, parity)) return true;
    if ((it & 255u) == 0) {
      if (*reinterpret_cast<volatile int32_t*>(&ctl->abort)) return false;
      if (globaltimer() - t0 > ctl->timeout_ns) {
        atomicExch(&ctl->abort, 1);
        set_status(st, MOE_ERR_TIMEOUT);
        return false;
      }
    }
  }
}

__device__ __noinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, SmemCtl2* ctl, moe_diag* st) {
  const uint32_t b = smem_u32(bar);
  if (mbar_try_cluster(b, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_cluster(b, parity)) return true;
    if ((it & 255u) == 0) {
      if (*reinterpret_cast<volatile int32_t*>(&ctl->abort)) return false;
      if (globaltimer() - t0 > ctl->timeout_ns) {
        atomicExch(&ctl->abort, 1);
        set_status(st, MOE_ERR_TIMEOUT);
        return false;
      }
    }
  }
}

// Dynamic tile schedule of a CTA pair. The leader's producer takes the next
// tile index from the global counter and publishes it in slot i % kTileSlots of
// both CTAs; every other role reads it from there, so all roles of the pair
// walk the same tile sequence and the pairs stay within about one tile of each
// other in the global tile order (tiles that share B run at the same time).
__device__ int publish_tile(SmemCtl2* ctl, int i, const TcParams& p) {
  const int slot = i % kTileSlots;
  const uint32_t par = (uint32_t)(i / kTileSlots) & 1u;
  if (!mbar_wait_cluster(&ctl->tile_empty[slot], par ^ 1u, ctl, p.status)) return -1;
  const int t = atomicAdd(p.tile_counter, 1);
  ctl->tile_ring[slot] = t;
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(map_to_rank(&ctl->tile_ring[slot], 1)), "r"(t) : "memory");
  mbar_arrive(&ctl->tile_full[slot]);
  mbar_arrive_cluster(map_to_rank(&ctl->tile_full[slot], 1));
  return t;
}

// A reader's next tile (one thread per role); -1 after a timeout or an abort.
__device__ int take_tile(SmemCtl2* ctl, int i, uint32_t rank, const TcParams& p) {
  const int slot = i % kTileSlots;
  const uint32_t par = (uint32_t)(i / kTileSlots) & 1u;
  if (!mbar_wait_cluster(&ctl->tile_full[slot], par, ctl, p.status)) return -1;
  const int t = *reinterpret_cast<volatile int32_t*>(&ctl->tile_ring[slot]);
  if (rank == 0)
    mbar_arrive(&ctl->tile_empty[slot]);
  else
    mbar_arrive_cluster(map_to_rank(&ctl->tile_empty[slot], 0));
  return t;
}

__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc2_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_a_half,
                    const __grid_constant__ CUtensorMap map_b, const __grid_constant__ CUtensorMap map_b2, TcParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw2[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw2) + 1023) & ~uintptr_t(1023));
  SmemCtl2* ctl = reinterpret_cast<SmemCtl2*>(smem + STAGES2 * STAGE2_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();

  if (threadIdx.x == 0) {
    int acc = 0;
    const int n_tiles = (p.N + p.n_out - 1) / p.n_out;
    for (int g = 0; g < p.G; ++g) {
      const int lo = p.offsets ? p.offsets[g] : 0;
      const int hi = p.offsets ? p.offsets[g + 1] : p.M;
      ctl->tile_off[g] = acc;
      acc += ((hi - lo + BM2 - 1) / BM2) * n_tiles;
    }
    ctl->tile_off[p.G] = acc;
    ctl->total_tiles = acc;
    ctl->n_tiles = n_tiles;
    ctl->abort = 0;
    ctl->timeout_ns = p.timeout_ns;
    for (int s = 0; s < STAGES2; ++s) {
      mbar_init(&ctl->full[s], 1);
      mbar_init(&ctl->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&ctl->tmem_full[b], 1);
      mbar_init(&ctl->tmem_empty[b], 8);
    }
    for (int q = 0; q < kTileSlots; ++q) {
      mbar_init(&ctl->tile_full[q], 1);
      mbar_init(&ctl->tile_empty[q], kTileReaders);
    }
    mbar_init(&ctl->drain, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&map_a);
    tma_prefetch_desc(&map_a_half);
    tma_prefetch_desc(&map_b);
    if (p.swiglu) tma_prefetch_desc(&map_b2);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&ctl->tmem_base)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  fence_before();
  __syncthreads();
  cluster_sync();  // barriers of both CTAs initialised before any remote arrive or copy
  fence_after();
  const uint32_t tmem_base = ctl->tmem_base;
  const int total = ctl->total_tiles;
  const int num_kb = (p.K + BK - 1) / BK;
  bool aborted = false;

  if (warp == 0) {
    // ================= TMA producer (both CTAs) =================
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int g_hint = 0;
      for (int i = 0; !aborted; ++i) {
        const int t = rank == 0 ? publish_tile(ctl, i, p) : take_tile(ctl, i, rank, p);
        if (t < 0) {
          aborted = true;
          break;
        }
        if (t >= total) break;
        const Tile tl = decode2(ctl, p, t, g_hint);
        const bool half = tl.half != 0;
        const uint32_t tx = 2u * ((half ? A2_HALF_BYTES : A2_BYTES) + B2_BYTES);
        const CUtensorMap* amap = half ? &map_a_half : &map_a;
        const int row0 = tl.lo + tl.m * BM2 + (int)rank * (half ? 64 : 128);
        // SwiGLU: 64 gate rows over the 64 up rows of the same output columns; plain: 128 rows of B
        const int brow = p.swiglu ? tl.g * p.b_rows + tl.nt * p.n_out + (int)rank * 64
                                  : tl.g * p.b_rows + tl.nt * p.n_out + (int)rank * 128;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_try(smem_u32(&ctl->empty[stage]), phase ^ 1u) &&
              !mbar_wait2(&ctl->empty[stage], phase ^ 1u, ctl, p.status)) {
            aborted = true;
            break;
          }
          uint8_t* sa = smem + stage * STAGE2_BYTES;
          if (p.test_stall && i == 0 && kb == 0) {
            // injected fault: this stage is never filled, so the MMA's wait on it runs out
            if (++stage == STAGES2) {
              stage = 0;
              phase ^= 1u;
            }
            continue;
          }
          const uint32_t leader_full = map_to_rank(&ctl->full[stage], 0);
          if (rank == 0) mbar_expect_tx(&ctl->full[stage], tx);
          tma_load_2d_pair(sa, amap, leader_full, kb * BK, row0);
          if (p.swiglu) {
            tma_load_2d_pair(sa + A2_BYTES, &map_b, leader_full, kb * BK, brow);
            tma_load_2d_pair(sa + A2_BYTES + 64 * BK * 2, &map_b2, leader_full, kb * BK, brow);
          } else {
            tma_load_2d_pair(sa + A2_BYTES, &map_b, leader_full, kb * BK, brow);
          }
          if (++stage == STAGES2) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else if (warp == 1) {
    // ================= MMA issuer (leader CTA) =================
    if (lane == 0 && rank == 0) {
      int stage = 0;
      uint32_t phase = 0;
      const uint32_t idesc_full = idesc_bf16_pair(BM2, BN_MAX);
      const uint32_t idesc_half = idesc_bf16_pair(BM2 / 2, BN_MAX);
      bool issued = false;
      int g_hint = 0;
      for (int i = 0; !aborted; ++i) {
        const int t = take_tile(ctl, i, 0, p);
        if (t < 0) {
          aborted = true;
          break;
        }
        if (t >= total) break;
        const uint32_t idesc = decode2(ctl, p, t, g_hint).half ? idesc_half : idesc_full;
        const int buf = i & 1;
        const uint32_t acc_phase = (uint32_t)(i >> 1) & 1u;
        if (!mbar_wait2(&ctl->tmem_empty[buf], acc_phase ^ 1u, ctl, p.status)) {
          aborted = true;
          break;
        }
        fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(buf * BN_MAX);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_try(smem_u32(&ctl->full[stage]), phase) && !mbar_wait2(&ctl->full[stage], phase, ctl, p.status)) {
            aborted = true;
            break;
          }
          const uint32_t sa = smem_u32(smem + stage * STAGE2_BYTES);
          const uint64_t adesc = sw128_desc(sa);
          const uint64_t bdesc = sw128_desc(sa + A2_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            mma_bf16_pair(d_tmem, adesc + (uint64_t)(2 * k), bdesc + (uint64_t)(2 * k), idesc, (kb | k) != 0);
          issued = true;
          mma_commit_pair(&ctl->empty[stage]);
          if (++stage == STAGES2) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (aborted) break;
        mma_commit_pair(&ctl->tmem_full[buf]);
      }
      if (aborted && issued) {
        asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                         smem_u32(&ctl->drain))
                     : "memory");
        mbar_drain(&ctl->drain, 0);
      }
    }
  } else {
    // ================= epilogue (warps 2..5, both CTAs) =================
    // TMEM lane quarter q of CTA r. Full tile: lane = row 128r + 32q + lane,
    // column = MMA column n. Half tile (M = 128, 64 rows per CTA): MMA columns
    // [0, 128) sit in lanes 0..63 and columns [128, 256) in lanes 64..127, both
    // at TMEM columns [0, 128), so quarters 0-1 hold the first half of the
    // columns and quarters 2-3 the second half, each for rows 64r + 32(q & 1) + lane.
    const int q = warp & 3;
    const uint32_t leader_tmem_empty[2] = {map_to_rank(&ctl->tmem_empty[0], 0), map_to_rank(&ctl->tmem_empty[1], 0)};
    int g_hint = 0;
    for (int i = 0;; ++i) {
      int t = 0;
      if (lane == 0) t = take_tile(ctl, i, rank, p);
      t = __shfl_sync(0xffffffffu, t, 0);
      if (t < 0) {
        aborted = true;
        break;
      }
      if (t >= total) break;
      const int buf = i & 1;
      const uint32_t acc_phase = (uint32_t)(i >> 1) & 1u;
      const Tile tl = decode2(ctl, p, t, g_hint);
      const bool half = tl.half != 0;
      const bool got = mbar_wait2(&ctl->tmem_full[buf], acc_phase, ctl, p.status);
      __syncwarp();  // tcgen05.ld below is warp-aligned
      if (!got) {
        aborted = true;
        break;
      }
      fence_after();
      const int row_in_tile = half ? (int)rank * 64 + (q & 1) * 32 + lane : (int)rank * 128 + q * 32 + lane;
      const int64_t row = (int64_t)tl.lo + tl.m * BM2 + row_in_tile;
      const bool valid = row < tl.hi;
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * BN_MAX);
      if (p.swiglu) {
        // Output column j of the tile: gate at MMA column 128(j/64) + j%64, up 64 further.
        const int j0 = half ? (q >> 1) * 64 : 0;
        const int nj = half ? 64 : 128;
        const int col0 = tl.nt * p.n_out + j0;
        for (int c = 0; c < nj; c += 16) {
          const uint32_t gcol = half ? (uint32_t)c : (uint32_t)(128 * (c >> 6) + (c & 63));
          float gv[16], uv[16];
          tmem_ld16(taddr + gcol, gv);
          tmem_ld16(taddr + gcol + 64u, uv);
#pragma unroll
          for (int e = 0; e < 16; ++e) gv[e] = silu(gv[e]) * uv[e];
          if (valid && col0 + c < p.N) store16(p.C, p.ldc, row, col0 + c, p.N, gv, false);
        }
      } else {
        const int j0 = half ? (q >> 1) * 128 : 0;
        const int nj = half ? 128 : p.n_out;
        const int col0 = tl.nt * p.n_out + j0;
        for (int c = 0; c < nj; c += 16) {
          float v[16];
          tmem_ld16(taddr + (uint32_t)c, v);
          if (valid && col0 + c < p.N) store16(p.C, p.ldc, row, col0 + c, p.N, v, p.out_f32 != 0);
        }
      }
      fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(leader_tmem_empty[buf]);
    }
  }

  if (*reinterpret_cast<volatile int32_t*>(&ctl->abort)) spin_ns(1000000);  // let copies in flight land
  fence_before();
  __syncthreads();
  __syncwarp();
  cluster_sync();
  fence_after();
  if (warp == 1) {
    __syncwarp();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS)
                 : "memory");
  }
}

// ---- wide SM-pair variant: 256 x 512 tiles ------------------------------------------
// The pair computes a 256-row (or half-height 128-row) by 512-column tile with two
// tcgen05.mma.cta_group::2 of N = 256 per 16-wide k step, into one 512-column TMEM
// accumulator per CTA. Per 64-k stage each CTA stages its A rows (16 KB, 8 KB half) and two
// 128-row B blocks (32 KB): 48 KB for twice the MMA work of a 256 x 256 tile's 32 KB, so a
// stage of shared memory carries 25 % fewer bytes per FLOP. SwiGLU: block 0 holds gate rows
// [j0 + 128r, +128) and block 1 the up rows of the same columns (MMA 0 -> TMEM columns
// [0, 256) = gate, MMA 1 -> [256, 512) = up), 256 outputs per tile; plain: block 0 rows
// j0 + 128r, block 1 rows j0 + 256 + 128r, 512 outputs. With one accumulator the epilogue
// of a tile does not overlap the next tile's main loop, so eight epilogue warps (two per TMEM
// lane quarter, each half of the columns) drain it.
constexpr int STAGESW = 4;
constexpr int BW_BLOCK_BYTES = 128 * BK * 2;
constexpr int STAGEW_BYTES = A2_BYTES + 2 * BW_BLOCK_BYTES;
constexpr int kThreadsW = 320;  // producer, MMA issuer, 8 epilogue warps
constexpr int kTileReadersW = 18;  // leader MMA + 8 leader epilogue warps + peer producer + 8 peer epilogue warps
static_assert(STAGESW <= STAGES2, "the control block's barrier arrays hold STAGES2 stages");

__global__ void __launch_bounds__(kThreadsW, 1)
    gemm_tc2w_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_a_half,
                     const __grid_constant__ CUtensorMap map_b, const __grid_constant__ CUtensorMap map_b2,
                     TcParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw_w[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw_w) + 1023) & ~uintptr_t(1023));
  SmemCtl2* ctl = reinterpret_cast<SmemCtl2*>(smem + STAGESW * STAGEW_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();

  if (threadIdx.x == 0) {
    int acc = 0;
    const int n_tiles = (p.N + p.n_out - 1) / p.n_out;
    for (int g = 0; g < p.G; ++g) {
      const int lo = p.offsets ? p.offsets[g] : 0;
      const int hi = p.offsets ? p.offsets[g + 1] : p.M;
      ctl->tile_off[g] = acc;
      acc += ((hi - lo + BM2 - 1) / BM2) * n_tiles;
    }
    ctl->tile_off[p.G] = acc;
    ctl->total_tiles = acc;
    ctl->n_tiles = n_tiles;
    ctl->abort = 0;
    ctl->timeout_ns = p.timeout_ns;
    for (int s = 0; s < STAGESW; ++s) {
      mbar_init(&ctl->full[s], 1);
      mbar_init(&ctl->empty[s], 1);
    }
    mbar_init(&ctl->tmem_full[0], 1);
    mbar_init(&ctl->tmem_empty[0], 16);
    for (int q = 0; q < kTileSlots; ++q) {
      mbar_init(&ctl->tile_full[q], 1);
      mbar_init(&ctl->tile_empty[q], kTileReadersW);
    }
    mbar_init(&ctl->drain, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&map_a);
    tma_prefetch_desc(&map_a_half);
    tma_prefetch_desc(&map_b);
    if (p.swiglu) tma_prefetch_desc(&map_b2);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&ctl->tmem_base)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  fence_before();
  __syncthreads();
  cluster_sync();
  fence_after();
  const uint32_t tmem_base = ctl->tmem_base;
  const int total = ctl->total_tiles;
  const int num_kb = (p.K + BK - 1) / BK;
  bool aborted = false;

  if (warp == 0) {
    // ================= TMA producer (both CTAs) =================
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int g_hint = 0;
      for (int i = 0; !aborted; ++i) {
        const int t = rank == 0 ? publish_tile(ctl, i, p) : take_tile(ctl, i, rank, p);
        if (t < 0) {
          aborted = true;
          break;
        }
        if (t >= total) break;
        const Tile tl = decode2(ctl, p, t, g_hint);
        const bool half = tl.half != 0;
        const uint32_t tx = 2u * ((half ? A2_HALF_BYTES : A2_BYTES) + 2 * BW_BLOCK_BYTES);
        const CUtensorMap* amap = half ? &map_a_half : &map_a;
        const int row0 = tl.lo + tl.m * BM2 + (int)rank * (half ? 64 : 128);
        const int brow0 = tl.g * p.b_rows + tl.nt * p.n_out + (int)rank * 128;
        const int brow1 = p.swiglu ? brow0 : brow0 + 256;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_try(smem_u32(&ctl->empty[stage]), phase ^ 1u) &&
              !mbar_wait2(&ctl->empty[stage], phase ^ 1u, ctl, p.status)) {
            aborted = true;
            break;
          }
          uint8_t* sa = smem + stage * STAGEW_BYTES;
          const uint32_t leader_full = map_to_rank(&ctl->full[stage], 0);
          if (rank == 0) mbar_expect_tx(&ctl->full[stage], tx);
          tma_load_2d_pair(sa, amap, leader_full, kb * BK, row0);
          tma_load_2d_pair(sa + A2_BYTES, &map_b, leader_full, kb * BK, brow0);
          tma_load_2d_pair(sa + A2_BYTES + BW_BLOCK_BYTES, p.swiglu ? &map_b2 : &map_b, leader_full, kb * BK, brow1);
          if (++stage == STAGESW) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else if (warp == 1) {
    // ================= MMA issuer (leader CTA) =================
    if (lane == 0 && rank == 0) {
      int stage = 0;
      uint32_t phase = 0;
      const uint32_t idesc_full = idesc_bf16_pair(BM2, BN_MAX);
      const uint32_t idesc_half = idesc_bf16_pair(BM2 / 2, BN_MAX);
      bool issued = false;
      int g_hint = 0;
      for (int i = 0; !aborted; ++i) {
        const int t = take_tile(ctl, i, 0, p);
        if (t < 0) {
          aborted = true;
          break;
        }
        if (t >= total) break;
        const uint32_t idesc = decode2(ctl, p, t, g_hint).half ? idesc_half : idesc_full;
        if (!mbar_wait2(&ctl->tmem_empty[0], (uint32_t)(i & 1) ^ 1u, ctl, p.status)) {
          aborted = true;
          break;
        }
        fence_after();
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_try(smem_u32(&ctl->full[stage]), phase) && !mbar_wait2(&ctl->full[stage], phase, ctl, p.status)) {
            aborted = true;
            break;
          }
          const uint32_t sa = smem_u32(smem + stage * STAGEW_BYTES);
          const uint64_t adesc = sw128_desc(sa);
          const uint64_t bdesc0 = sw128_desc(sa + A2_BYTES);
          const uint64_t bdesc1 = sw128_desc(sa + A2_BYTES + BW_BLOCK_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint32_t acc = (kb | k) != 0;
            mma_bf16_pair(tmem_base, adesc + (uint64_t)(2 * k), bdesc0 + (uint64_t)(2 * k), idesc, acc);
            mma_bf16_pair(tmem_base + 256u, adesc + (uint64_t)(2 * k), bdesc1 + (uint64_t)(2 * k), idesc, acc);
          }
          issued = true;
          mma_commit_pair(&ctl->empty[stage]);
          if (++stage == STAGESW) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (aborted) break;
        mma_commit_pair(&ctl->tmem_full[0]);
      }
      if (aborted && issued) {
        asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                         smem_u32(&ctl->drain))
                     : "memory");
        mbar_drain(&ctl->drain, 0);
      }
    }
  } else {
    // ================= epilogue (warps 2..9, both CTAs) =================
    // Lane quarter q = warp % 4 (the TMEM lanes this warp may read), column half hh.
    // Full tile: lane = row 128r + 32q + lane. Half tile: quarters 0-1 hold MMA columns
    // [0, 128) and quarters 2-3 columns [128, 256) of each MMA, for rows 64r + 32(q & 1) + lane,
    // at TMEM columns [0, 128) (MMA 0) and [256, 384) (MMA 1).
    const int q = warp & 3;
    const int hh = (warp - 2) >> 2;
    const uint32_t leader_tmem_empty = map_to_rank(&ctl->tmem_empty[0], 0);
    int g_hint = 0;
    for (int i = 0;; ++i) {
      int t = 0;
      if (lane == 0) t = take_tile(ctl, i, rank, p);
      t = __shfl_sync(0xffffffffu, t, 0);
      if (t < 0) {
        aborted = true;
        break;
      }
      if (t >= total) break;
      const Tile tl = decode2(ctl, p, t, g_hint);
      const bool half = tl.half != 0;
      const bool got = mbar_wait2(&ctl->tmem_full[0], (uint32_t)(i & 1), ctl, p.status);
      __syncwarp();
      if (!got) {
        aborted = true;
        break;
      }
      fence_after();
      const int row_in_tile = half ? (int)rank * 64 + (q & 1) * 32 + lane : (int)rank * 128 + q * 32 + lane;
      const int64_t row = (int64_t)tl.lo + tl.m * BM2 + row_in_tile;
      const bool valid = row < tl.hi;
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16);
      const int tile_col = tl.nt * p.n_out;
      if (p.swiglu) {
        // output column j of the tile: gate at MMA-0 column j, up at MMA-1 column j
        const int j0 = half ? (q >> 1) * 128 + hh * 64 : hh * 128;
        const int nj = half ? 64 : 128;
        const uint32_t tcol = half ? (uint32_t)(hh * 64) : (uint32_t)(hh * 128);
        for (int c = 0; c < nj; c += 16) {
          float gv[16], uv[16];
          tmem_ld16(taddr + tcol + (uint32_t)c, gv);
          tmem_ld16(taddr + 256u + tcol + (uint32_t)c, uv);
#pragma unroll
          for (int e = 0; e < 16; ++e) gv[e] = silu(gv[e]) * uv[e];
          if (valid && tile_col + j0 + c < p.N) store16(p.C, p.ldc, row, tile_col + j0 + c, p.N, gv, false);
        }
      } else {
        // output column j < 256 at MMA-0 column j, j >= 256 at MMA-1 column j - 256
        const int j0 = half ? hh * 256 + (q >> 1) * 128 : hh * 256;
        const int nj = half ? 128 : 256;
        const uint32_t tcol = (uint32_t)(hh * 256);
        for (int c = 0; c < nj; c += 16) {
          float v[16];
          tmem_ld16(taddr + tcol + (uint32_t)c, v);
          if (valid && tile_col + j0 + c < p.N) store16(p.C, p.ldc, row, tile_col + j0 + c, p.N, v, p.out_f32 != 0);
        }
      }
      fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(leader_tmem_empty);
    }
  }

  if (*reinterpret_cast<volatile int32_t*>(&ctl->abort)) spin_ns(1000000);  // let copies in flight land
  fence_before();
  __syncthreads();
  __syncwarp();
  cluster_sync();
  fence_after();
  if (warp == 1) {
    __syncwarp();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS)
                 : "memory");
  }
}

// ---- host side -----------------------------------------------------------------
// 2-D bf16 tensor [rows, cols] (cols contiguous), box [box_rows, 64], 128-byte swizzle.
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

int num_sms() {
  static int sms = 0;
  if (!sms) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (sms <= 0) sms = 148;
  }
  return sms;
}

// Clusters of two CTAs of a pair kernel (gemm_tc2_kernel, or the wide gemm_tc2w_kernel) that fit
// on the device at once, per device.
int max_resident_pairs(const cudaLaunchConfig_t& cfg, bool wide) {
  static int cached[2][64] = {{0}};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return 0;
  if (!cached[wide][dev]) {
    cudaLaunchConfig_t q = cfg;
    q.gridDim = dim3((unsigned)num_sms(), 1, 1);
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, wide ? (void*)gemm_tc2w_kernel : (void*)gemm_tc2_kernel, &q) !=
            cudaSuccess ||
        clusters <= 0)
      return 0;
    cached[wide][dev] = clusters;
  }
  return cached[wide][dev];
}

constexpr size_t kSmemBytes = 1024 + STAGES * STAGE_BYTES + sizeof(SmemCtl);
constexpr size_t kSmemBytes2 = 1024 + STAGES2 * STAGE2_BYTES + sizeof(SmemCtl2);
constexpr size_t kSmemBytesW = 1024 + STAGESW * STAGEW_BYTES + sizeof(SmemCtl2);
static_assert(kSmemBytes <= 232448 && kSmemBytes2 <= 232448 && kSmemBytesW <= 232448,
              "dynamic shared memory above 227 KB");

// Wide pair tiles (256 x 512): half as many n-tiles re-read each group's rows. Taken by the gate/up
// (SwiGLU) GEMM of many small groups (at most 768 rows per group on average, the DeepSeek shapes)
// and by both GEMMs of one dense group (the shared experts). Measured ~2 % faster on the routed
// DeepSeek gate/up GEMM and 4-7 % on the V3 shared expert's, and 3-4 % more on the shared down
// GEMM, at full clock and under the power cap. The grouped down GEMM (K = 2048 or less) and groups
// of ~1024 rows are slower with them: a wide tile's epilogue cannot overlap the next tile.
// MOE_TC_WIDE=1 selects them for every SM-pair GEMM, =gate for the gate/up GEMM only, =0 for none.
bool use_wide_tiles(bool swiglu, int64_t rows, int32_t groups) {
  const char* w = getenv("MOE_TC_WIDE");
  if (!w) return groups == 1 || (swiglu && rows <= 768 * (int64_t)groups);
  if (w[0] == '1') return true;
  return swiglu && strcmp(w, "gate") == 0;
}

// SM-pair tiles stage fewer bytes per FLOP and, with half-height last tiles,
// pad groups to 128 rows like the single-SM tiles; they are used once groups
// average at least 128 rows. Below that (decode) every tile is mostly padding
// and the single-SM kernel keeps twice as many independent weight streams in
// flight. MOE_TC_MODE=1sm|2sm overrides the choice (tuning and tests).
bool use_pair_tiles(const GemmArgs& a, bool swiglu, bool out_f32) {
  if (a.k_splits > 1 || out_f32) return false;
  if (!swiglu && a.N < BN_MAX) return false;
  const char* mode = getenv("MOE_TC_MODE");
  if (mode && strcmp(mode, "1sm") == 0) return false;
  if (mode && strcmp(mode, "2sm") == 0) return true;
  return a.M / (a.offsets ? a.G : 1) >= 128;
}

}  // namespace

bool gemm_tc_supported(const GemmArgs& a, bool swiglu, bool out_f32) {
  // MOE_TEST_NO_TENSOR_MAPS=1 makes every shape unsupported (test of the error path).
  const char* inj = getenv("MOE_TEST_NO_TENSOR_MAPS");
  if (inj && inj[0] == '1') return false;
  // binary32 outputs store a row's last columns one by one; bf16 outputs need whole 8-column chunks
  if (a.K % 8 != 0 || (!out_f32 && a.N % 8 != 0) || a.N <= 0 || a.K <= 0) return false;
  if (a.G > kMaxGroupsTc || a.M >= ((int64_t)1 << 31)) return false;
  if (a.lda != a.K) return false;
  if (swiglu && out_f32) return false;
  if (a.k_splits > 1 && (swiglu || !out_f32)) return false;
  if (out_f32 && a.ldc % 4 != 0) return false;
  if (!out_f32 && a.ldc % 8 != 0) return false;
  if (reinterpret_cast<uintptr_t>(a.A) % 16 || reinterpret_cast<uintptr_t>(a.B) % 16 ||
      reinterpret_cast<uintptr_t>(a.C) % 16 || (swiglu && reinterpret_cast<uintptr_t>(a.B2) % 16))
    return false;
  return encode_fn() != nullptr;
}

cudaError_t launch_gemm_tc(const GemmArgs& a, bool swiglu, bool out_f32, moe_diag* status, cudaStream_t s) {
  if (!gemm_tc_supported(a, swiglu, out_f32)) return cudaErrorNotSupported;
  if (a.M <= 0) return cudaSuccess;
  TcParams p{};
  p.G = a.G;
  p.offsets = a.offsets;
  p.M = (int32_t)a.M;
  p.N = a.N;
  p.K = a.K;
  if (swiglu) {
    p.n_mma = BN_MAX;
    p.n_out = BN_MAX / 2;
  } else {
    p.n_mma = a.N >= BN_MAX ? BN_MAX : (int32_t)align_up(a.N, 16);
    p.n_out = p.n_mma;
  }
  p.b_rows = a.N;
  p.swiglu = swiglu;
  p.out_f32 = out_f32;
  {
    // Split-K: every split owns at least one k-block.
    const int num_kb = (int)ceil_div(a.K, BK);
    const int want = a.k_splits < 1 ? 1 : (a.k_splits > num_kb ? num_kb : a.k_splits);
    p.kb_per = (int)ceil_div(num_kb, want);
    p.k_splits = (int)ceil_div(num_kb, p.kb_per);
    if (p.k_splits != a.k_splits) return cudaErrorInvalidValue;  // caller sized its partials for a.k_splits
  }
  p.C = a.C;
  p.ldc = a.ldc;
  p.c_split_stride = a.c_split_stride;
  p.status = status;
  // MOE_TEST_STALL=1 injects a stalled pipeline stage to exercise the bounded
  // waits and the MOE_ERR_TIMEOUT status path (fault injection for tests).
  const char* stall = getenv("MOE_TEST_STALL");
  p.test_stall = stall && stall[0] == '1';
  p.timeout_ns = p.test_stall ? kTestTimeoutNs : kTimeoutNs;
  p.tile_counter = a.tile_counter;
  CUtensorMap ma, mb, mb2;
  const int64_t b_total_rows = (int64_t)a.G * a.N;
  const bool pair = use_pair_tiles(a, swiglu, out_f32);
  // Rows of B one CTA stages per copy. One SM: SwiGLU gate and up halves of 128
  // rows, or the whole plain tile. SM pair: each CTA holds 128 of the tile's 256
  // B rows, as 64 gate over 64 up rows for SwiGLU.
  const int b_box = pair ? (swiglu ? p.n_mma / 4 : p.n_mma / 2) : (swiglu ? p.n_mma / 2 : p.n_mma);
  // Every copy must fit the shared-memory slot it lands in.
  const int b_slot_rows = pair ? (swiglu ? B2_BYTES / (BK * 2) / 2 : B2_BYTES / (BK * 2)) : (swiglu ? BN_MAX / 2 : BN_MAX);
  if (b_box > b_slot_rows || (pair && (p.n_mma != BN_MAX || A2_BYTES != BM * BK * 2 || 2 * A2_HALF_BYTES != A2_BYTES)))
    return cudaErrorInvalidValue;
  if (!make_map(&ma, a.A, a.M, a.K, BM)) return cudaErrorInvalidValue;
  CUtensorMap ma_half;
  if (pair && !make_map(&ma_half, a.A, a.M, a.K, BM / 2)) return cudaErrorInvalidValue;
  const bool wide = pair && use_wide_tiles(swiglu, a.M, a.G);
  const int b_box_used = wide ? 128 : b_box;
  if (!make_map(&mb, a.B, b_total_rows, a.K, b_box_used)) return cudaErrorInvalidValue;
  if (swiglu) {
    if (!make_map(&mb2, a.B2, b_total_rows, a.K, b_box_used)) return cudaErrorInvalidValue;
  } else {
    mb2 = mb;
  }
  if (wide) {
    // 256 outputs per tile for SwiGLU (gate and up of 256 columns), 512 for plain tiles
    p.n_out = swiglu ? 256 : 512;
    static std::atomic<uint64_t> attrw{0};
    {
      const cudaError_t e = set_smem_limit(attrw, (const void*)gemm_tc2w_kernel, kSmemBytesW);
      if (e != cudaSuccess) return e;
    }
    const int64_t max_tiles_w = (ceil_div(a.M, BM2) + (a.offsets ? a.G : 0)) * ceil_div(a.N, p.n_out);
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kThreadsW, 1, 1);
    cfg.dynamicSmemBytes = kSmemBytesW;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (!a.tile_counter) return cudaErrorInvalidValue;
    {
      const cudaError_t e = cudaMemsetAsync(a.tile_counter, 0, sizeof(int32_t), s);
      if (e != cudaSuccess) return e;
    }
    const int pairs_resident = max_resident_pairs(cfg, true);
    if (pairs_resident <= 0) return cudaErrorInvalidConfiguration;
    const int64_t pairs = max_tiles_w < pairs_resident ? max_tiles_w : pairs_resident;
    cfg.gridDim = dim3((unsigned)(2 * pairs), 1, 1);
    return cudaLaunchKernelEx(&cfg, gemm_tc2w_kernel, ma, ma_half, mb, mb2, p);
  }
  const int64_t n_tiles_all = ceil_div(a.N, p.n_out);
  if (pair) {
    static std::atomic<uint64_t> attr2{0};
    {
      const cudaError_t e = set_smem_limit(attr2, (const void*)gemm_tc2_kernel, kSmemBytes2);
      if (e != cudaSuccess) return e;
    }
    const int64_t max_pair_tiles = (ceil_div(a.M, BM2) + (a.offsets ? a.G : 0)) * n_tiles_all;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = kSmemBytes2;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // Tiles are dealt round-robin to a persistent grid, so every pair must be
    // resident at once: a pair that only starts when another one exits would
    // run its whole share after the others. On parts whose GPCs hold odd SM
    // counts fewer than SMs/2 pairs fit, hence the occupancy query.
    if (!a.tile_counter) return cudaErrorInvalidValue;
    {
      const cudaError_t e = cudaMemsetAsync(a.tile_counter, 0, sizeof(int32_t), s);
      if (e != cudaSuccess) return e;
    }
    const int pairs_resident = max_resident_pairs(cfg, false);
    if (pairs_resident <= 0) return cudaErrorInvalidConfiguration;
    const int64_t pairs = max_pair_tiles < pairs_resident ? max_pair_tiles : pairs_resident;
    cfg.gridDim = dim3((unsigned)(2 * pairs), 1, 1);
    return cudaLaunchKernelEx(&cfg, gemm_tc2_kernel, ma, ma_half, mb, mb2, p);
  }
  static std::atomic<uint64_t> attr1{0};
  {
    const cudaError_t e = set_smem_limit(attr1, (const void*)gemm_tc_kernel, kSmemBytes);
    if (e != cudaSuccess) return e;
  }
  // Upper bound on the tiles: every group may add one partial m-tile.
  const int64_t n_tiles = ceil_div(a.N, p.n_out);
  const int64_t max_tiles = (ceil_div(a.M, BM) + (a.offsets ? a.G : 0)) * n_tiles * p.k_splits;
  const int grid = (int)(max_tiles < num_sms() ? max_tiles : num_sms());
  gemm_tc_kernel<<<grid, kThreads, kSmemBytes, s>>>(ma, mb, mb2, p);
  return cudaGetLastError();
}

}  // namespace moe
