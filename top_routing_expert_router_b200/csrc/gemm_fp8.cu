// gemm_fp8.cu -- grouped GEMM of the FP8 experts on the tcgen05 tensor cores.
//
// Page "15. DeepSeek: MLA, MoE and MTP", FP8 section: matrix inputs in E4M3,
// one UE8M0 scale per 1 x 128 tile of the activations A and per 128 x 128
// block of the weights B. For every group g and row r of that group:
//   plain : C[r, n] = sum_k (A[r, k] sa[r, k/128]) (B_g[n, k] sb_g[n/128, k/128])
//   SwiGLU: C[r, i] = silu(gate) * up, gate and up the plain sums with Bg_g, Bu_g
// computed by tcgen05.mma kind::mxf8f6f4.block_scale (E4M3 x E4M3 -> fp32 in
// TMEM, the scales applied by the tensor core per 32-wide k sub-block). C is bf16.
//
// Scale factors: a 32-bit scale word in TMEM holds four bytes and each MMA
// selects one of them. One scale covers a whole 128-wide k block, so the word
// of a row carries the scales of four consecutive k blocks (byte j: block
// 4q + j), and one copy into TMEM serves the MMAs of four stages.
//
// Design (one CTA per SM, persistent, warp-specialised, 192 threads):
//   warp 0      producer: per 128-k stage TMA copies of the 128 x 128 A tile and
//               the 128 x 128 B tile (SwiGLU: 64 gate over 64 up rows); every
//               fourth stage also a 512-byte bulk copy of A's scale-factor block
//               (laid out by the quantiser) and B's scale words, which the warp
//               writes from the block scale bytes (prefetched per tile).
//   warp 1      TMEM owner and MMA issuer: every fourth stage tcgen05.cp of both
//               scale-factor blocks into TMEM (32x128b.warpx4: rows p and p+32k
//               of the tile in lane p, column k), then per stage four MMAs of
//               K = 32 that select the scale byte of the stage's k block;
//               tcgen05.commit frees the stage.
//   warps 2..5  epilogue: tcgen05.ld, SwiGLU in fp32, bf16 stores.
// Every mbarrier wait is bounded like the bf16 kernels'.
// Short tiles (groups of a few rows, decode): an m-tile covers 32 rows and a
// stage holds only those 32 A rows next to the B tile, so 160 KB of weights
// stay in flight per SM (5 stages of 256-wide tiles, 10 of 128-wide). The MMA
// still reads a 128-row A operand; its rows 32..127 fall on the stage's B bytes
// and produce accumulator rows that are never stored.
#include <cuda.h>
#include <stdlib.h>
#include <string.h>

#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace moe {
namespace {

using namespace ptx;

constexpr int BM = 128, BK = 128;  // BK in E4M3 elements (128 bytes per row)
constexpr int A_BYTES = BM * BK, SF_BYTES = 512;  // SF_BYTES: one 128-row scale-factor block
constexpr int kThreads = 192;
constexpr uint32_t TMEM_COLS = 512;
constexpr int kMaxGroupsFp8 = 256;
constexpr uint64_t kTimeoutNs = 2000000000ull;

// Tile shapes: BN = 128 keeps two TMEM accumulators (the epilogue of one tile
// overlaps the next); BN = 256 halves the copies of A per MMA but leaves TMEM
// room for one accumulator next to the scale factors. BMR = rows of an m-tile
// (128, or 32 for short tiles).
template <int BN, int BMR>
struct Shape {
  static constexpr int ACC_BUFS = BN == 256 ? 1 : 2;
  static constexpr int A_STAGE = BMR * BK;  // A bytes copied per stage
  static constexpr int B_BYTES = BN * BK;
  static constexpr int SFB_BYTES = (BN / 128) * SF_BYTES;
  static constexpr int STAGE_BYTES = (A_STAGE + B_BYTES + SF_BYTES + SFB_BYTES + 1023) / 1024 * 1024;
  static constexpr int STAGES = BMR == 32 ? (BN == 256 ? 5 : 10) : (BN == 256 ? 4 : 6);
  static constexpr uint32_t SF_COL0 = ACC_BUFS * BN;   // scale factors after the accumulators
  static constexpr uint32_t SF_COLS = 4 + BN / 32;     // per slot: A (128 rows) and B (BN rows)
  static constexpr uint32_t SF_SLOTS = 2;              // four k blocks per slot, two slots in turn
  static_assert(SF_COL0 + SF_COLS * SF_SLOTS <= TMEM_COLS, "TMEM budget");
  static_assert(A_STAGE + B_BYTES >= A_BYTES, "the MMA's 128-row A operand stays inside its stage");
  static_assert(BMR == 128 || BMR == 32, "m-tile heights");
};

struct Fp8Params {
  int32_t G;
  const int32_t* offsets;
  int32_t M;
  int32_t N;      // valid output columns per group
  int32_t K;
  int32_t n_out;  // output columns per tile
  int32_t b_rows; // rows per group in B
  int32_t swiglu;
  const uint32_t* sfa;        // A scale-factor blocks from the quantiser
  const uint8_t* sb;          // B scale bytes [G][ceil(b_rows/128)][K/128]
  const uint8_t* sb2;         // up-matrix scale bytes (SwiGLU)
  void* C;
  int64_t ldc;
  moe_diag* status;
};

constexpr int kMaxStages = 10;

struct __align__(8) Ctl {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  uint64_t tmem_full[2];
  uint64_t tmem_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int32_t abort;
  int32_t total_tiles;
  int32_t n_tiles;
  int32_t row_off[kMaxGroupsFp8 + 1];
  int32_t tile_off[kMaxGroupsFp8 + 1];
  int32_t sf_off[kMaxGroupsFp8 + 1];  // first scale tile (one per m-tile) of each group
};

__device__ __noinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, Ctl* ctl, moe_diag* st) {
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

// Untiled bulk copy (16-byte aligned addresses, size a multiple of 16).
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// kind::mxf8f6f4 instruction descriptor: E4M3 A and B (format 0), K-major,
// UE8M0 scales, M = 128, N = BN; scale-factor byte `id` of A's and B's words.
__device__ __forceinline__ uint32_t idesc_fp8(int bn, int id) {
  return ((uint32_t)id << 4) | ((uint32_t)(bn >> 3) << 17) | (1u << 23) | ((uint32_t)(BM >> 4) << 24) |
         ((uint32_t)id << 29);
}

__device__ __forceinline__ void mma_fp8(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t sfa,
                                        uint32_t sfb, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb)
      : "memory");
}

__device__ __forceinline__ void sf_copy(uint32_t taddr, uint64_t desc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(desc) : "memory");
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

struct Tile {
  int g, m, nt;
};

// a[j] for a run-time j in 0..3. SELECT: by comparisons, which keeps the array in registers
// (measured 3 % faster on the FP8 prefill layer); otherwise by indexing, which puts it in local
// memory (measured 2 % faster on the FP8 decode layer with short tiles).
template <bool SELECT>
__device__ __forceinline__ uint32_t pick4(const uint32_t (&a)[4], int j) {
  if constexpr (SELECT) return j == 0 ? a[0] : (j == 1 ? a[1] : (j == 2 ? a[2] : a[3]));
  return a[j];
}

template <int BMR>
__device__ __forceinline__ Tile decode(const Ctl* ctl, int G, int t, int& g_hint) {
  int g = g_hint;
  while (g + 1 <= G && ctl->tile_off[g + 1] <= t) ++g;
  g_hint = g;
  const int local = t - ctl->tile_off[g];
  const int mt = (ctl->row_off[g + 1] - ctl->row_off[g] + BMR - 1) / BMR;
  return Tile{g, local % mt, local / mt};
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

template <int BN, int BMR>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_fp8_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                    const __grid_constant__ CUtensorMap map_b2, Fp8Params p) {
  using S = Shape<BN, BMR>;
  constexpr int STAGES = S::STAGES, STAGE_BYTES = S::STAGE_BYTES, B_BYTES = S::B_BYTES, A_STAGE = S::A_STAGE;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Ctl* ctl = reinterpret_cast<Ctl*>(smem + STAGES * STAGE_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    int acc = 0, sacc = 0;
    const int n_tiles = (p.N + p.n_out - 1) / p.n_out;
    for (int g = 0; g < p.G; ++g) {
      const int lo = p.offsets ? p.offsets[g] : 0;
      const int hi = p.offsets ? p.offsets[g + 1] : p.M;
      const int mt = (hi - lo + BMR - 1) / BMR;
      ctl->row_off[g] = lo;
      ctl->row_off[g + 1] = hi;
      ctl->tile_off[g] = acc;
      ctl->sf_off[g] = sacc;
      acc += mt * n_tiles;
      sacc += mt;
    }
    ctl->tile_off[p.G] = acc;
    ctl->sf_off[p.G] = sacc;
    ctl->total_tiles = acc;
    ctl->n_tiles = n_tiles;
    ctl->abort = 0;
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&ctl->full[s], 2);  // the producer's expect_tx arrival + its scale-word arrival
      mbar_init(&ctl->empty[s], 1);
    }
    for (int b = 0; b < S::ACC_BUFS; ++b) {
      mbar_init(&ctl->tmem_full[b], 1);
      mbar_init(&ctl->tmem_empty[b], 4);
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
  const int total = ctl->total_tiles;
  const int nkb = p.K / BK;
  const int nbr = (p.b_rows + 127) / 128;  // scale rows of B per group

  if (warp == 0) {
    // ================= producer (whole warp) =================
    int stage = 0;
    uint32_t phase = 0;
    int g_hint = 0;
    bool ok = true;
    uint32_t issued = 0;  // stages armed so far (stage s was armed (issued - 1 - s) / STAGES + 1 times)
    const uint32_t tx_tiles = A_STAGE + B_BYTES;  // TMA tiles; every fourth stage also A's scale block
    const int nq = (nkb + 3) / 4;                  // scale blocks per row tile (four k blocks each)
    // B scale bytes of a tile: lane l keeps k-blocks l, l + 32, l + 64, l + 96 of the gate (or
    // plain) block, the up block and, for plain 256-wide tiles, the next 128-row block. They are
    // loaded one tile ahead, so a tile's first stage does not wait for them.
    int pf_hint = 0;
    auto load_scales = [&](int tt, uint32_t (&g)[4], uint32_t (&u)[4], uint32_t (&nx)[4]) {
      if (tt >= total) return;
      const Tile tl = decode<BMR>(ctl, p.G, tt, pf_hint);
      const int brow_local = tl.nt * p.n_out;
      const uint8_t* sb_g = p.sb + ((int64_t)tl.g * nbr + brow_local / 128) * nkb;
      const uint8_t* sb2_g = p.swiglu ? p.sb2 + ((int64_t)tl.g * nbr + brow_local / 128) * nkb : sb_g;
      const uint8_t* sbn_g = sb_g + ((brow_local / 128 + 1 < nbr) ? nkb : 0);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int kb = lane + 32 * j;
        g[j] = kb < nkb ? sb_g[kb] : 127u;
        u[j] = kb < nkb ? sb2_g[kb] : 127u;
        nx[j] = kb < nkb ? sbn_g[kb] : 127u;
      }
    };
    uint32_t nsbg[4], nsbu[4], nsbn[4];
    load_scales(blockIdx.x, nsbg, nsbu, nsbn);
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
      const Tile tl = decode<BMR>(ctl, p.G, t, g_hint);
      const int row0 = ctl->row_off[tl.g] + tl.m * BMR;
      const int brow = tl.g * p.b_rows + tl.nt * p.n_out;
      const uint32_t* sfa_tile = p.sfa + (int64_t)(ctl->sf_off[tl.g] + tl.m) * nq * 128;
      uint32_t sbg[4], sbu[4], sbn[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        sbg[j] = nsbg[j];
        sbu[j] = nsbu[j];
        sbn[j] = nsbn[j];
      }
      load_scales(t + (int)gridDim.x, nsbg, nsbu, nsbn);
      for (int kb = 0; kb < nkb; ++kb) {
        int go = 1;
        if (lane == 0 && !mbar_try(smem_u32(&ctl->empty[stage]), phase ^ 1u) &&
            !mbar_wait(&ctl->empty[stage], phase ^ 1u, ctl, p.status))
          go = 0;
        go = __shfl_sync(0xffffffffu, go, 0);
        if (!go) {
          ok = false;
          break;
        }
        uint8_t* sa = smem + stage * STAGE_BYTES;
        uint8_t* sbm = sa + A_STAGE;
        uint8_t* sfa_s = sbm + B_BYTES;
        uint8_t* sfb_s = sfa_s + SF_BYTES;
        const bool lead = (kb & 3) == 0;  // first stage of four: carries the scale factors
        if (lane == 0) {
          mbar_expect_tx(&ctl->full[stage], tx_tiles + (lead ? SF_BYTES : 0u));
          tma_load_2d(sa, &map_a, &ctl->full[stage], kb * BK, row0);
          if (p.swiglu) {
            tma_load_2d(sbm, &map_b, &ctl->full[stage], kb * BK, brow);
            tma_load_2d(sbm + (BN / 2) * BK, &map_b2, &ctl->full[stage], kb * BK, brow);
          } else {
            tma_load_2d(sbm, &map_b, &ctl->full[stage], kb * BK, brow);
          }
          if (lead) bulk_load(sfa_s, sfa_tile + (int64_t)(kb >> 2) * 128, SF_BYTES, &ctl->full[stage]);
        }
        // B scale words, one 128-row block per 512 bytes: block row p at word 4 (p % 32) + p / 32,
        // byte j of the word the scale of k block kb + j. SwiGLU: the first BN/2 tile rows are gate
        // rows, the rest up rows (one scale block each, as BN/2 <= 128 rows never straddle a
        // 128-row block); plain: one block per 128 rows.
        if (lead) {
          auto quad = [&](const uint32_t(&a)[4]) {  // bytes of k blocks kb .. kb + 3 (kb + 3 <= 127)
            uint32_t w = 0;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int x = kb + i;
              w |= (__shfl_sync(0xffffffffu, pick4<BMR == 128>(a, x >> 5), x & 31) & 0xFFu) << (8 * i);
            }
            return w;
          };
          const uint32_t bg = quad(sbg);
          const uint32_t bu = quad(sbu);
          if (BN == 128) {
            const uint32_t w2 = p.swiglu ? bu : bg;
            *reinterpret_cast<uint4*>(sfb_s + 16 * lane) = make_uint4(bg, bg, w2, w2);
          } else {  // BN = 256: block 0 holds tile rows 0..127, block 1 rows 128..255
            const uint32_t w2 = p.swiglu ? bu : quad(sbn);
            *reinterpret_cast<uint4*>(sfb_s + 16 * lane) = make_uint4(bg, bg, bg, bg);
            *reinterpret_cast<uint4*>(sfb_s + SF_BYTES + 16 * lane) = make_uint4(w2, w2, w2, w2);
          }
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->full[stage]);
        ++issued;
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (!ok && lane == 0)
      for (uint32_t s = 0; s < (uint32_t)STAGES; ++s) {
        const uint32_t armed = issued > s ? (issued - 1 - s) / STAGES + 1 : 0;
        if (armed) mbar_drain(&ctl->full[s], (armed - 1) & 1u);
      }
  } else if (warp == 1) {
    // ================= MMA issuer =================
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true, issued = false;
      int i = 0;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++i) {
        const int buf = S::ACC_BUFS == 2 ? (i & 1) : 0;
        const uint32_t acc_phase = (uint32_t)(S::ACC_BUFS == 2 ? (i >> 1) : i) & 1u;
        if (!mbar_wait(&ctl->tmem_empty[buf], acc_phase ^ 1u, ctl, p.status)) {
          ok = false;
          break;
        }
        fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(buf * BN);
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_try(smem_u32(&ctl->full[stage]), phase) && !mbar_wait(&ctl->full[stage], phase, ctl, p.status)) {
            ok = false;
            break;
          }
          fence_after();
          const uint32_t sa = smem_u32(smem + stage * STAGE_BYTES);
          const uint32_t sfa_t = tmem_base + S::SF_COL0 + S::SF_COLS * (uint32_t)((kb >> 2) & 1);
          const uint32_t sfb_t = sfa_t + 4u;
          if ((kb & 3) == 0) {  // scale factors of k blocks kb .. kb + 3, copied once
            sf_copy(sfa_t, sf_desc(sa + A_STAGE + B_BYTES));
#pragma unroll
            for (int blk = 0; blk < BN / 128; ++blk)  // B rows 128 blk .. : TMEM columns 4 blk ..
              sf_copy(sfb_t + 4u * blk, sf_desc(sa + A_STAGE + B_BYTES + SF_BYTES + SF_BYTES * blk));
          }
          const uint64_t adesc = sw128_desc(sa);
          const uint64_t bdesc = sw128_desc(sa + A_STAGE);
#pragma unroll
          for (int k = 0; k < BK / 32; ++k)  // 32 E4M3 elements = 32 bytes per MMA
            mma_fp8(d_tmem, adesc + (uint64_t)(2 * k), bdesc + (uint64_t)(2 * k), idesc_fp8(BN, kb & 3), sfa_t,
                    sfb_t, (kb | k) != 0);
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
        mma_commit(&ctl->drain);
        mbar_drain(&ctl->drain, 0);
      }
    }
  } else {
    // ================= epilogue (warps 2..5) =================
    const int q = warp & 3;
    const int row_in_tile = q * 32 + lane;
    int g_hint = 0;
    int i = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++i) {
      const int buf = S::ACC_BUFS == 2 ? (i & 1) : 0;
      const uint32_t acc_phase = (uint32_t)(S::ACC_BUFS == 2 ? (i >> 1) : i) & 1u;
      const Tile tl = decode<BMR>(ctl, p.G, t, g_hint);
      const bool got = mbar_wait(&ctl->tmem_full[buf], acc_phase, ctl, p.status);
      __syncwarp();
      if (!got) break;
      fence_after();
      const int64_t row = (int64_t)ctl->row_off[tl.g] + tl.m * BMR + row_in_tile;
      const bool valid = row_in_tile < BMR && row < ctl->row_off[tl.g + 1];
      if (BMR < 128 && q * 32 >= BMR) {  // accumulator rows past a short tile: nothing to store
        fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->tmem_empty[buf]);
        continue;
      }
      const int col0 = tl.nt * p.n_out;
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * BN);
      bf16* C = static_cast<bf16*>(p.C);
      if (p.swiglu) {
        for (int c = 0; c < p.n_out; c += 16) {
          float gv[16], uv[16];
          tmem_ld16(taddr + (uint32_t)c, gv);
          tmem_ld16(taddr + (uint32_t)(p.n_out + c), uv);
#pragma unroll
          for (int e = 0; e < 16; ++e) gv[e] = silu(gv[e]) * uv[e];
          if (valid && col0 + c < p.N) store16(C, p.ldc, row, col0 + c, p.N, gv);
        }
      } else {
        for (int c = 0; c < p.n_out; c += 16) {
          float v[16];
          tmem_ld16(taddr + (uint32_t)c, v);
          if (valid && col0 + c < p.N) store16(C, p.ldc, row, col0 + c, p.N, v);
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
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS) : "memory");
  }
}

// ---- host side -----------------------------------------------------------------
// 2-D byte tensor [rows, cols] (cols contiguous), box [box_rows, 128], 128-byte swizzle.
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

template <int BN, int BMR>
constexpr size_t smem_bytes() {
  return 1024 + Shape<BN, BMR>::STAGES * Shape<BN, BMR>::STAGE_BYTES + sizeof(Ctl);
}
static_assert(smem_bytes<128, 128>() <= 232448 && smem_bytes<256, 128>() <= 232448 &&
                  smem_bytes<128, 32>() <= 232448 && smem_bytes<256, 32>() <= 232448,
              "dynamic shared memory above 227 KB");
static_assert(Shape<128, 128>::STAGES <= kMaxStages && Shape<256, 128>::STAGES <= kMaxStages &&
                  Shape<128, 32>::STAGES <= kMaxStages && Shape<256, 32>::STAGES <= kMaxStages,
              "barrier arrays");

template <int BN, int BMR>
cudaError_t launch_bn(const GemmFp8Args& a, bool swiglu, moe_diag* status, cudaStream_t s) {
  Fp8Params p{};
  p.G = a.G;
  p.offsets = a.offsets;
  p.M = (int32_t)a.M;
  p.N = a.N;
  p.K = a.K;
  p.n_out = swiglu ? BN / 2 : BN;
  p.b_rows = a.N;
  p.swiglu = swiglu;
  p.sfa = a.sfa;
  p.sb = a.sb;
  p.sb2 = swiglu ? a.sb2 : a.sb;
  p.C = a.C;
  p.ldc = a.ldc;
  p.status = status;
  CUtensorMap ma, mb, mb2;
  const int b_box = swiglu ? BN / 2 : BN;
  if (!make_map_u8(&ma, a.A, a.M, a.K, BMR)) return cudaErrorInvalidValue;
  if (!make_map_u8(&mb, a.B, (int64_t)a.G * a.N, a.K, b_box)) return cudaErrorInvalidValue;
  if (swiglu) {
    if (!make_map_u8(&mb2, a.B2, (int64_t)a.G * a.N, a.K, b_box)) return cudaErrorInvalidValue;
  } else {
    mb2 = mb;
  }
  static std::atomic<uint64_t> attr{0};
  {
    const cudaError_t e = set_smem_limit(attr, (const void*)gemm_fp8_kernel<BN, BMR>, smem_bytes<BN, BMR>());
    if (e != cudaSuccess) return e;
  }
  int sms = 0, dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (sms <= 0) sms = 148;
  const int64_t n_tiles = ceil_div(a.N, p.n_out);
  const int64_t max_tiles = (ceil_div(a.M, BMR) + (a.offsets ? a.G : 0)) * n_tiles;
  const int grid = (int)(max_tiles < sms ? max_tiles : sms);
  gemm_fp8_kernel<BN, BMR><<<grid, kThreads, smem_bytes<BN, BMR>(), s>>>(ma, mb, mb2, p);
  return cudaGetLastError();
}

}  // namespace

// Tile choice from the rows per group (M rows in G groups):
//  - >= 128 rows (prefill): 256 x 256 tiles on SM pairs (gemm_fp8_pair.cu). At the FP8 MMA rate
//    the L2 -> SM copies bound the kernel, and a pair copies 32 KB per SM and 128-k stage where a
//    one-SM 128 x 256 tile copies 48 KB.
//  - <= 16 rows (decode): short 32-row tiles, 128 wide with two accumulators and 10 stages:
//    weight streaming at HBM rate needs bytes in flight (160 KB of weights per SM), and a group of
//    a few rows needs none of a 128-row A tile. (256-wide short tiles, 5 stages, measured 13 %
//    slower on the DeepSeek-V3 decode layer.)
//  - otherwise 128 x 128 tiles with two accumulators.
// MOE_FP8_BN (tuning and tests): 128 | 256 force one-SM 128-row tiles of that width; pair forces
// the SM-pair tiles; s128 | s256 force the width of short tiles where the rule allows them. The workspace holds scale blocks for the
// short tiles whenever the rule could choose them.
bool fp8_short_rule(int64_t M, int32_t G) { return M <= 16 * (int64_t)G; }

int fp8_tile_rows(int64_t M, int32_t G) {
  const char* bn = getenv("MOE_FP8_BN");
  if (bn && bn[0] != 's') return 128;
  return fp8_short_rule(M, G) ? 32 : 128;
}

int64_t fp8_sf_tiles_bound(int64_t rows, int32_t G) { return ceil_div(rows, fp8_short_rule(rows, G) ? 32 : 128) + G; }

cudaError_t launch_gemm_fp8(const GemmFp8Args& a, bool swiglu, moe_diag* status, cudaStream_t s) {
  if (a.M <= 0) return cudaSuccess;
  if (a.K % BK != 0 || a.K / BK > 128 || a.N % 16 != 0 || a.N <= 0 || a.G < 1 || a.G > kMaxGroupsFp8)
    return cudaErrorInvalidValue;
  if (reinterpret_cast<uintptr_t>(a.A) % 16 || reinterpret_cast<uintptr_t>(a.B) % 16 ||
      reinterpret_cast<uintptr_t>(a.sfa) % 16 || reinterpret_cast<uintptr_t>(a.C) % 16 || a.ldc % 8 != 0 ||
      (swiglu && reinterpret_cast<uintptr_t>(a.B2) % 16))
    return cudaErrorInvalidValue;
  if (a.tile_rows != fp8_tile_rows(a.M, a.offsets ? a.G : 1)) return cudaErrorInvalidValue;
  const char* bn = getenv("MOE_FP8_BN");
  if (a.tile_rows == 32)
    return bn && strcmp(bn, "s256") == 0 ? launch_bn<256, 32>(a, swiglu, status, s)
                                         : launch_bn<128, 32>(a, swiglu, status, s);
  const bool big = a.M / (a.offsets ? a.G : 1) >= 128;
  const bool pair_ok = a.tile_counter && a.sfb && a.sfb_bytes >= fp8_pair_sfb_bytes(a.G, a.N, a.K, swiglu);
  if (bn ? strcmp(bn, "pair") == 0 : big && pair_ok) return launch_gemm_fp8_pair(a, swiglu, status, s);
  const bool wide = bn && bn[0] != 's' ? strcmp(bn, "256") == 0 : big;
  return wide ? launch_bn<256, 128>(a, swiglu, status, s) : launch_bn<128, 128>(a, swiglu, status, s);
}

}  // namespace moe
