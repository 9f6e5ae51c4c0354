// gemm_fp8_pair.cu -- grouped GEMM of the FP8 experts on CTA pairs (cta_group::2).
//
// Same operation as gemm_fp8.cu (page "15. DeepSeek: MLA, MoE and MTP", FP8
// section: E4M3 inputs, one UE8M0 scale per 1 x 128 activation tile and per
// 128 x 128 weight block), for groups of at least 128 rows on average.
//
// A CTA pair (cluster of 2) computes a 256 x 256 tile with
// tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale (M = 256, N = 256, K = 32):
// CTA r holds A rows [128r, 128r+128) of the tile and B rows [128r, 128r+128)
// (SwiGLU: gate rows [64r, 64r+64) of the tile's 128 output columns over the up
// rows of the same columns), so each SM copies 32 KB per 128-k stage instead of
// the 48 KB of a one-SM 128 x 256 tile. Scale factors: each CTA stages the scale
// block of its own 128 A rows and the two blocks of all 256 B rows at the same
// shared-memory offsets, and the leader's tcgen05.cp.cta_group::2 copies each
// CTA's blocks into that CTA's TMEM. A scale word carries four k blocks (byte j:
// block 4q + j), so the scale factors move once per four stages. Both come from
// memory by TMA like the operands: A's from the quantiser, B's from blocks that
// sfb_blocks_kernel lays out before the GEMM (1 KB per tile and four k blocks),
// so no thread writes shared memory and the peer CTA never has to signal the
// leader (a cluster-scope release per stage held its copies back). The
// accumulator takes 256 TMEM columns and the scale factors the next 24, so there
// is one accumulator: the epilogue of a tile does not overlap the next tile.
//
// Roles (192 threads per CTA):
//   warp 0      producer in both CTAs (one thread): TMA copies of its A and B
//               halves and, every fourth stage, of its A scale block and the
//               tile's B scale blocks, all completing on the leader's `full`
//               barrier. The leader's producer takes tiles from a global counter
//               and publishes them to both CTAs (dynamic schedule).
//   warp 1      leader only: TMEM owner of the pair and MMA issuer; its commits
//               arrive on the barriers of both CTAs.
//   warps 2..5  epilogue in both CTAs: tcgen05.ld, SwiGLU in fp32, bf16 stores.
// Every wait is bounded; past the limit the kernel records MOE_ERR_TIMEOUT, stops
// issuing and drains. No TMA multicast is used.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace moe {
namespace {

using namespace ptx;

constexpr int BK = 128;              // k per stage, in E4M3 elements (128 bytes per row)
constexpr int SF_BYTES = 512;        // one 128-row scale-factor block
constexpr int STAGES = 6;
constexpr int A_BYTES = 128 * BK;    // this CTA's 128 A rows
constexpr int B_BYTES = 128 * BK;    // this CTA's 128 B rows
constexpr int STAGE_BYTES = (A_BYTES + B_BYTES + 3 * SF_BYTES + 1023) / 1024 * 1024;  // + SFA + two SFB blocks
constexpr int SFB_WORDS = 256;       // B scale words of one tile and four k blocks (two 512-byte blocks)
constexpr int kThreads = 192;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t SF_COL0 = 256;    // after the accumulator
constexpr uint32_t SF_COLS = 12;     // per slot: A (4 columns) and B (two blocks of 4)
constexpr int kMaxPairGroups = 256;
constexpr int kTileSlots = 4;
constexpr int kTileReaders = 10;     // leader MMA + 4 leader epilogue warps + peer producer + 4 peer epilogue warps
constexpr uint64_t kTimeoutNs = 2000000000ull;
static_assert(SF_COL0 + 2 * SF_COLS <= TMEM_COLS, "TMEM budget");

struct PairParams {
  int32_t G;
  const int32_t* offsets;
  int32_t M;
  int32_t N;       // valid output columns per group
  int32_t K;
  int32_t n_out;   // output columns per tile (SwiGLU 128, plain 256)
  int32_t b_rows;  // rows per group in B
  int32_t swiglu;
  const uint8_t* sb;   // B scale bytes [G][ceil(b_rows/128)][K/128]
  const uint8_t* sb2;  // up-matrix scale bytes (SwiGLU)
  void* C;
  int64_t ldc;
  moe_diag* status;
  int32_t* tile_counter;  // zeroed before the launch
};

struct __align__(8) Ctl {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tmem_full;
  uint64_t tmem_empty;
  uint64_t tile_full[kTileSlots];
  uint64_t tile_empty[kTileSlots];
  int32_t tile_ring[kTileSlots];
  uint64_t drain;
  uint32_t tmem_base;
  int32_t abort;
  int32_t total_tiles;
  int32_t row_off[kMaxPairGroups + 1];
  int32_t tile_off[kMaxPairGroups + 1];  // first pair tile of each group
  int32_t sf_off[kMaxPairGroups + 1];    // first 128-row scale tile of each group
};

// Bounded wait for the phase of `parity`. False on timeout or abort.
template <bool CLUSTER>
__device__ __noinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, Ctl* ctl, moe_diag* st) {
  const uint32_t b = smem_u32(bar);
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 0;; ++it) {
    if (CLUSTER ? mbar_try_cluster(b, parity) : mbar_try(b, parity)) return true;
    if ((it & 255u) == 255u) {
      if (*reinterpret_cast<volatile int32_t*>(&ctl->abort)) return false;
      if (globaltimer() - t0 > kTimeoutNs) {
        atomicExch(&ctl->abort, 1);
        set_status(st, MOE_ERR_TIMEOUT);
        return false;
      }
    }
  }
}

// kind::mxf8f6f4: E4M3 A and B, K-major, UE8M0 scales, M = 256, N = 256; scale byte `id`.
__device__ __forceinline__ uint32_t idesc_pair(int id) {
  return ((uint32_t)id << 4) | ((uint32_t)(256 >> 3) << 17) | (1u << 23) | ((uint32_t)(256 >> 4) << 24) |
         ((uint32_t)id << 29);
}

__device__ __forceinline__ void mma_pair(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t sfa,
                                         uint32_t sfb, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb)
      : "memory");
}

// Each CTA's block at this shared-memory offset into the same TMEM address of that CTA.
__device__ __forceinline__ void sf_copy_pair(uint32_t taddr, uint64_t desc) {
  asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(desc) : "memory");
}

// Arrive on the barrier at this offset in both CTAs of the pair once the MMAs complete.
__device__ __forceinline__ void commit_pair(uint64_t* bar) {
  const uint16_t mask = 0x3;
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(mask)
      : "memory");
}

__device__ __forceinline__ void store16(bf16* C, int64_t ldc, int64_t row, int col, int N, const float (&v)[16]) {
  bf16* p = C + row * ldc + col;
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

struct Tile {
  int g, m, nt;
};

__device__ __forceinline__ Tile decode(const Ctl* ctl, int G, int t, int& g_hint) {
  int g = g_hint;
  while (g + 1 <= G && ctl->tile_off[g + 1] <= t) ++g;
  g_hint = g;
  const int local = t - ctl->tile_off[g];
  const int mt = (ctl->row_off[g + 1] - ctl->row_off[g] + 255) / 256;
  return Tile{g, local % mt, local / mt};
}

// Dynamic tile schedule (as in the bf16 pair kernel): the leader's producer takes the next tile
// from the global counter and publishes it in slot i % kTileSlots of both CTAs.
__device__ int publish_tile(Ctl* ctl, int i, const PairParams& p) {
  const int slot = i % kTileSlots;
  const uint32_t par = (uint32_t)(i / kTileSlots) & 1u;
  if (!mbar_wait<true>(&ctl->tile_empty[slot], par ^ 1u, ctl, p.status)) return -1;
  const int t = atomicAdd(p.tile_counter, 1);
  ctl->tile_ring[slot] = t;
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(map_to_rank(&ctl->tile_ring[slot], 1)), "r"(t) : "memory");
  mbar_arrive(&ctl->tile_full[slot]);
  mbar_arrive_cluster(map_to_rank(&ctl->tile_full[slot], 1));
  return t;
}

__device__ int take_tile(Ctl* ctl, int i, uint32_t rank, const PairParams& p) {
  const int slot = i % kTileSlots;
  const uint32_t par = (uint32_t)(i / kTileSlots) & 1u;
  if (!mbar_wait<true>(&ctl->tile_full[slot], par, ctl, p.status)) return -1;
  const int t = *reinterpret_cast<volatile int32_t*>(&ctl->tile_ring[slot]);
  if (rank == 0)
    mbar_arrive(&ctl->tile_empty[slot]);
  else
    mbar_arrive_cluster(map_to_rank(&ctl->tile_empty[slot], 0));
  return t;
}

// B scale words of every (group, tile, four k blocks) in the layout the GEMM stages: 256 words,
// two 128-row blocks (MMA rows 0..127 from CTA 0's B rows, 128..255 from CTA 1's), row p of a
// block at word 4 (p % 32) + p / 32, byte j of a word the UE8M0 byte of k block 4q + j. SwiGLU:
// in both blocks rows 0..63 are gate rows and 64..127 up rows of the tile's 128 output columns,
// which lie in one 128-row weight block; plain: the tile's two consecutive 128-row blocks.
__global__ void sfb_blocks_kernel(const uint8_t* sb, const uint8_t* sb2, int G, int n_tiles, int nkb, int nbr,
                                  int swiglu, uint32_t* out) {
  const int nq = (nkb + 3) / 4;
  const int64_t total = (int64_t)G * n_tiles * nq * SFB_WORDS;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const int w = (int)(i % SFB_WORDS);
    const int64_t blk = i / SFB_WORDS;
    const int qd = (int)(blk % nq);
    const int nt = (int)((blk / nq) % n_tiles);
    const int g = (int)(blk / ((int64_t)nq * n_tiles));
    const int half = w / 128, k = w % 128;
    const int prow = (k % 4) * 32 + k / 4;  // row of the 128-row block
    const uint8_t* src;
    if (swiglu) {
      src = (prow < 64 ? sb : sb2) + ((int64_t)g * nbr + nt) * nkb;
    } else {
      int br = 2 * nt + half;
      if (br > nbr - 1) br = nbr - 1;
      src = sb + ((int64_t)g * nbr + br) * nkb;
    }
    uint32_t word = 0;
    for (int j = 0; j < 4; ++j) {
      const int kb = 4 * qd + j;
      word |= (uint32_t)(kb < nkb ? src[kb] : 127u) << (8 * j);
    }
    out[i] = word;
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    gemm_fp8_pair_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                         const __grid_constant__ CUtensorMap map_b2, const __grid_constant__ CUtensorMap map_sfa,
                         const __grid_constant__ CUtensorMap map_sfb, PairParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Ctl* ctl = reinterpret_cast<Ctl*>(smem + STAGES * STAGE_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int n_tiles = (p.N + p.n_out - 1) / p.n_out;

  if (threadIdx.x == 0) {
    int acc = 0, sacc = 0;
    for (int g = 0; g < p.G; ++g) {
      const int lo = p.offsets ? p.offsets[g] : 0;
      const int hi = p.offsets ? p.offsets[g + 1] : p.M;
      ctl->row_off[g] = lo;
      ctl->row_off[g + 1] = hi;
      ctl->tile_off[g] = acc;
      ctl->sf_off[g] = sacc;
      acc += ((hi - lo + 255) / 256) * n_tiles;
      sacc += (hi - lo + 127) / 128;
    }
    ctl->tile_off[p.G] = acc;
    ctl->sf_off[p.G] = sacc;
    ctl->total_tiles = acc;
    ctl->abort = 0;
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&ctl->full[s], 1);  // the leader's expect_tx; both CTAs' copies complete bytes on it
      mbar_init(&ctl->empty[s], 1);
    }
    mbar_init(&ctl->tmem_full, 1);
    mbar_init(&ctl->tmem_empty, 8);
    for (int q = 0; q < kTileSlots; ++q) {
      mbar_init(&ctl->tile_full[q], 1);
      mbar_init(&ctl->tile_empty[q], kTileReaders);
    }
    mbar_init(&ctl->drain, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
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
  const int nkb = p.K / BK;
  const int nq = (nkb + 3) / 4;           // scale blocks per 128-row tile (four k blocks each)
  bool aborted = false;

  if (warp == 0) {
    // ================= producer (one thread, both CTAs) =================
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int g_hint = 0;
      const uint32_t leader_full0 = map_to_rank(&ctl->full[0], 0);
      for (int i = 0; !aborted; ++i) {
        const int t = rank == 0 ? publish_tile(ctl, i, p) : take_tile(ctl, i, rank, p);
        if (t < 0) {
          aborted = true;
          break;
        }
        if (t >= total) break;
        const Tile tl = decode(ctl, p.G, t, g_hint);
        const int row0 = ctl->row_off[tl.g] + tl.m * 256 + (int)rank * 128;
        // This CTA's A scale tile; a CTA whose rows all lie past the group reads the group's
        // last tile instead (its accumulator rows are never stored).
        const int sf_tiles_g = ctl->sf_off[tl.g + 1] - ctl->sf_off[tl.g];
        int sf_tile = 2 * tl.m + (int)rank;
        if (sf_tile > sf_tiles_g - 1) sf_tile = sf_tiles_g - 1;
        const int sf_row0 = (ctl->sf_off[tl.g] + sf_tile) * nq;
        const int sfb_row0 = (tl.g * n_tiles + tl.nt) * nq;
        const int brow = p.swiglu ? tl.g * p.b_rows + tl.nt * p.n_out + (int)rank * 64
                                  : tl.g * p.b_rows + tl.nt * p.n_out + (int)rank * 128;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_try(smem_u32(&ctl->empty[stage]), phase ^ 1u) &&
              !mbar_wait<false>(&ctl->empty[stage], phase ^ 1u, ctl, p.status)) {
            aborted = true;
            break;
          }
          uint8_t* sa = smem + stage * STAGE_BYTES;
          uint8_t* sbm = sa + A_BYTES;
          uint8_t* sfa_s = sbm + B_BYTES;
          uint8_t* sfb_s = sfa_s + SF_BYTES;
          const bool lead = (kb & 3) == 0;
          const uint32_t leader_full = leader_full0 + (uint32_t)(stage * sizeof(uint64_t));
          if (rank == 0)
            mbar_expect_tx(&ctl->full[stage], 2u * (A_BYTES + B_BYTES) + (lead ? 2u * 3u * SF_BYTES : 0u));
          tma_load_2d_pair(sa, &map_a, leader_full, kb * BK, row0);
          if (p.swiglu) {
            tma_load_2d_pair(sbm, &map_b, leader_full, kb * BK, brow);
            tma_load_2d_pair(sbm + 64 * BK, &map_b2, leader_full, kb * BK, brow);
          } else {
            tma_load_2d_pair(sbm, &map_b, leader_full, kb * BK, brow);
          }
          if (lead) {
            tma_load_2d_pair(sfa_s, &map_sfa, leader_full, 0, sf_row0 + (kb >> 2));
            tma_load_2d_pair(sfb_s, &map_sfb, leader_full, 0, sfb_row0 + (kb >> 2));
          }
          if (++stage == STAGES) {
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
      bool issued = false;
      for (int i = 0; !aborted; ++i) {
        const int t = take_tile(ctl, i, 0, p);
        if (t < 0) {
          aborted = true;
          break;
        }
        if (t >= total) break;
        if (!mbar_wait<true>(&ctl->tmem_empty, (uint32_t)(i & 1) ^ 1u, ctl, p.status)) {
          aborted = true;
          break;
        }
        fence_after();
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_try(smem_u32(&ctl->full[stage]), phase) &&
              !mbar_wait<false>(&ctl->full[stage], phase, ctl, p.status)) {
            aborted = true;
            break;
          }
          fence_after();
          const uint32_t sa = smem_u32(smem + stage * STAGE_BYTES);
          const uint32_t sfa_t = tmem_base + SF_COL0 + SF_COLS * (uint32_t)((kb >> 2) & 1);
          const uint32_t sfb_t = sfa_t + 4u;
          if ((kb & 3) == 0) {
            sf_copy_pair(sfa_t, sf_desc(sa + A_BYTES + B_BYTES));
            sf_copy_pair(sfb_t, sf_desc(sa + A_BYTES + B_BYTES + SF_BYTES));
            sf_copy_pair(sfb_t + 4u, sf_desc(sa + A_BYTES + B_BYTES + 2 * SF_BYTES));
          }
          const uint64_t adesc = sw128_desc(sa);
          const uint64_t bdesc = sw128_desc(sa + A_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 32; ++k)
            mma_pair(tmem_base, adesc + (uint64_t)(2 * k), bdesc + (uint64_t)(2 * k), idesc_pair(kb & 3), sfa_t, sfb_t,
                     (kb | k) != 0);
          issued = true;
          commit_pair(&ctl->empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (aborted) break;
        commit_pair(&ctl->tmem_full);
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
    // TMEM lane quarter q of CTA r holds tile rows 128r + 32q + lane; column n = MMA column n.
    const int q = warp & 3;
    const uint32_t leader_tmem_empty = map_to_rank(&ctl->tmem_empty, 0);
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
      const Tile tl = decode(ctl, p.G, t, g_hint);
      const bool got = mbar_wait<false>(&ctl->tmem_full, (uint32_t)(i & 1), ctl, p.status);
      __syncwarp();  // tcgen05.ld below is warp-aligned
      if (!got) {
        aborted = true;
        break;
      }
      fence_after();
      const int64_t row = (int64_t)ctl->row_off[tl.g] + tl.m * 256 + (int)rank * 128 + q * 32 + lane;
      const bool valid = row < ctl->row_off[tl.g + 1];
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16);
      bf16* C = static_cast<bf16*>(p.C);
      const int col0 = tl.nt * p.n_out;
      if (p.swiglu) {
        // Output column j of the tile: gate at MMA column 128 (j / 64) + j % 64, up 64 further.
        for (int c = 0; c < 128; c += 16) {
          const uint32_t gcol = (uint32_t)(128 * (c >> 6) + (c & 63));
          float gv[16], uv[16];
          tmem_ld16(taddr + gcol, gv);
          tmem_ld16(taddr + gcol + 64u, uv);
#pragma unroll
          for (int e = 0; e < 16; ++e) gv[e] = silu(gv[e]) * uv[e];
          if (valid && col0 + c < p.N) store16(C, p.ldc, row, col0 + c, p.N, gv);
        }
      } else {
        for (int c = 0; c < 256; c += 16) {
          float v[16];
          tmem_ld16(taddr + (uint32_t)c, v);
          if (valid && col0 + c < p.N) store16(C, p.ldc, row, col0 + c, p.N, v);
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
  cluster_sync();
  fence_after();
  if (warp == 1) {
    __syncwarp();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS)
                 : "memory");
  }
}

// ---- host side -----------------------------------------------------------------
// 2-D byte tensor [rows, cols], box [box_rows, 128], 128-byte swizzle.
bool make_map_u8(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols};
  const cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Scale-factor blocks as a 2-D tensor of 32-bit words [blocks, words], one block per box.
bool make_map_sf(CUtensorMap* m, const void* base, int64_t blocks, int words) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)words, (cuuint64_t)blocks};
  const cuuint64_t strides[1] = {(cuuint64_t)words * 4};
  const cuuint32_t box[2] = {(cuuint32_t)words, 1};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

constexpr size_t kSmemBytes = 1024 + STAGES * STAGE_BYTES + sizeof(Ctl);
static_assert(kSmemBytes <= 232448, "dynamic shared memory above 227 KB");

int num_sms() {
  int sms = 0, dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms > 0 ? sms : 148;
}

int max_resident_pairs(const cudaLaunchConfig_t& cfg) {
  static int cached[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return 0;
  if (!cached[dev]) {
    cudaLaunchConfig_t q = cfg;
    q.gridDim = dim3((unsigned)num_sms(), 1, 1);
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, (void*)gemm_fp8_pair_kernel, &q) != cudaSuccess || clusters <= 0)
      return 0;
    cached[dev] = clusters;
  }
  return cached[dev];
}

}  // namespace

int64_t fp8_pair_sfb_bytes(int32_t G, int32_t N, int32_t K, bool swiglu) {
  return (int64_t)G * ceil_div(N, swiglu ? 128 : 256) * ceil_div(K / BK, 4) * SFB_WORDS * 4;
}

cudaError_t launch_gemm_fp8_pair(const GemmFp8Args& a, bool swiglu, moe_diag* status, cudaStream_t s) {
  if (a.M <= 0) return cudaSuccess;
  if (a.tile_rows != 128 || !a.tile_counter || a.sf_blocks <= 0 || a.G > kMaxPairGroups || !a.sfb ||
      a.sfb_bytes < fp8_pair_sfb_bytes(a.G, a.N, a.K, swiglu))
    return cudaErrorInvalidValue;
  PairParams p{};
  p.G = a.G;
  p.offsets = a.offsets;
  p.M = (int32_t)a.M;
  p.N = a.N;
  p.K = a.K;
  p.n_out = swiglu ? 128 : 256;
  p.b_rows = a.N;
  p.swiglu = swiglu;
  p.sb = a.sb;
  p.sb2 = swiglu ? a.sb2 : a.sb;
  p.C = a.C;
  p.ldc = a.ldc;
  p.status = status;
  p.tile_counter = a.tile_counter;
  CUtensorMap ma, mb, mb2, msf;
  const int b_box = swiglu ? 64 : 128;
  if (!make_map_u8(&ma, a.A, a.M, a.K, 128)) return cudaErrorInvalidValue;
  if (!make_map_u8(&mb, a.B, (int64_t)a.G * a.N, a.K, b_box)) return cudaErrorInvalidValue;
  if (swiglu) {
    if (!make_map_u8(&mb2, a.B2, (int64_t)a.G * a.N, a.K, b_box)) return cudaErrorInvalidValue;
  } else {
    mb2 = mb;
  }
  const int n_tiles = (int)ceil_div(a.N, p.n_out);
  const int nkb = a.K / BK, nq = (nkb + 3) / 4;
  CUtensorMap msfb;
  if (!make_map_sf(&msf, a.sfa, a.sf_blocks, 128)) return cudaErrorInvalidValue;
  if (!make_map_sf(&msfb, a.sfb, (int64_t)a.G * n_tiles * nq, SFB_WORDS)) return cudaErrorInvalidValue;
  {
    const int64_t words = (int64_t)a.G * n_tiles * nq * SFB_WORDS;
    const int64_t blocks = ceil_div(words, 256);
    sfb_blocks_kernel<<<(unsigned)(blocks < 148 * 8 ? blocks : 148 * 8), 256, 0, s>>>(
        a.sb, swiglu ? a.sb2 : a.sb, a.G, n_tiles, nkb, (int)ceil_div(a.N, 128), swiglu ? 1 : 0, a.sfb);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  static std::atomic<uint64_t> attr{0};
  {
    const cudaError_t e = set_smem_limit(attr, (const void*)gemm_fp8_pair_kernel, kSmemBytes);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute la[1];
  la[0].id = cudaLaunchAttributeClusterDimension;
  la[0].val.clusterDim.x = 2;
  la[0].val.clusterDim.y = 1;
  la[0].val.clusterDim.z = 1;
  cfg.attrs = la;
  cfg.numAttrs = 1;
  {
    const cudaError_t e = cudaMemsetAsync(a.tile_counter, 0, sizeof(int32_t), s);
    if (e != cudaSuccess) return e;
  }
  // Every pair must be resident at once (the pairs take tiles from one counter).
  const int pairs_resident = max_resident_pairs(cfg);
  if (pairs_resident <= 0) return cudaErrorInvalidConfiguration;
  const int64_t max_tiles = (ceil_div(a.M, 256) + (a.offsets ? a.G : 0)) * n_tiles;
  const int64_t pairs = max_tiles < pairs_resident ? max_tiles : pairs_resident;
  cfg.gridDim = dim3((unsigned)(2 * pairs), 1, 1);
  return cudaLaunchKernelEx(&cfg, gemm_fp8_pair_kernel, ma, mb, mb2, msf, msfb, p);
}

}  // namespace moe
