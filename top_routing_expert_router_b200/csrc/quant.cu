// quant.cu -- FP8 (E4M3) quantisation of activation rows for the FP8 experts.
//
// Page "15. DeepSeek: MLA, MoE and MTP", FP8 section: matrix inputs in E4M3,
// one scale per 1 x 128 tile of activations, scales stored as UE8M0 (an 8-bit
// exponent, scale = 2^(byte - 127)). For every row and 128-column tile:
//   e      = the smallest integer with amax <= 448 * 2^e (0 when amax = 0),
//   code_c = E4M3 of v_c * 2^-e, round to nearest even (|v_c * 2^-e| <= 448).
// The scale of row r, tile t is written where the tensor-core GEMM reads it:
// 128-row GEMM tiles of each group (tile m of group g covers rows
// offsets[g] + 128m ...), one 512-byte block per (tile, 128-column tile) in the
// scale-factor layout of tcgen05.mma block scaling: the 32-bit word of tile
// row p sits at word 4 (p % 32) + p / 32 and holds the UE8M0 byte four times
// (one per 32-column sub-block, all equal for 1 x 128 tiles).
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

// UE8M0 exponent of a tile whose largest magnitude is amax (finite binary32).
__device__ __forceinline__ int ue8m0_exponent(float amax) {
  if (!(amax > 0.0f)) return 0;
  int x;
  const float f = frexpf(amax, &x);  // amax = f * 2^x, f in [0.5, 1)
  // amax <= 448 * 2^e  <=>  f * 2^(x - 8 - e) <= 1.75: e = x - 9 iff f <= 0.875, else x - 8
  int e = f <= 0.875f ? x - 9 : x - 8;
  return e < -127 ? -127 : (e > 127 ? 127 : e);
}

constexpr int kQuantWarps = 8;

// One warp per row; lane l holds columns 4l .. 4l+3 of each 128-column tile.
__global__ void __launch_bounds__(32 * kQuantWarps)
    quantize_rows_kernel(const bf16* src, const int32_t* src_row, const int32_t* offsets, int G, int64_t rows_single,
                         int cols, uint8_t* q, uint32_t* sf, uint8_t* sf_plain) {
  __shared__ int32_t tile_off[kMaxExperts + 1];  // first 128-row tile of each group
  __shared__ int32_t row_off[kMaxExperts + 1];
  if (threadIdx.x == 0) {
    int32_t acc = 0;
    for (int g = 0; g < G; ++g) {
      const int32_t lo = offsets ? offsets[g] : 0;
      const int32_t hi = offsets ? offsets[g + 1] : (int32_t)rows_single;
      row_off[g] = lo;
      row_off[g + 1] = hi;
      tile_off[g] = acc;
      acc += (hi - lo + 127) / 128;
    }
    tile_off[G] = acc;
  }
  __syncthreads();
  const int64_t rows = row_off[G];
  const int lane = threadIdx.x & 31;
  const int tiles = cols / 128;
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t r = warp; r < rows; r += nwarps) {
    // group of row r (offsets ascending), its 128-row GEMM tile and the row inside it
    int lo = 0, hi = G - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (row_off[mid] <= r) lo = mid; else hi = mid - 1;
    }
    const int g = lo;
    const int64_t local = r - row_off[g];
    const int64_t tile = tile_off[g] + local / 128;
    const int p = (int)(local % 128);
    const int64_t srow = src_row ? (int64_t)src_row[r] : r;
    const uint2* in = reinterpret_cast<const uint2*>(src + srow * cols);
    uint32_t* out = reinterpret_cast<uint32_t*>(q + r * cols);
    // eight tiles' loads in flight at a time, then their reductions and stores
    for (int t0 = 0; t0 < tiles; t0 += 8) {
      uint2 raws[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (t0 + u < tiles) raws[u] = __ldg(in + (t0 + u) * 32 + lane);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int t = t0 + u;
        if (t >= tiles) break;
        const uint2 raw = raws[u];
        const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&raw.x);
        const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&raw.y);
        const float v0 = __low2float(a), v1 = __high2float(a), v2 = __low2float(b), v3 = __high2float(b);
        float m = fmaxf(fmaxf(fabsf(v0), fabsf(v1)), fmaxf(fabsf(v2), fabsf(v3)));
#pragma unroll
        for (int off = 16; off; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
        const int e = ue8m0_exponent(m);
        // multiplying by 2^-e is exact for these magnitudes
        const __nv_fp8x2_storage_t c01 =
            __nv_cvt_float2_to_fp8x2(make_float2(ldexpf(v0, -e), ldexpf(v1, -e)), __NV_SATFINITE, __NV_E4M3);
        const __nv_fp8x2_storage_t c23 =
            __nv_cvt_float2_to_fp8x2(make_float2(ldexpf(v2, -e), ldexpf(v3, -e)), __NV_SATFINITE, __NV_E4M3);
        out[t * 32 + lane] = (uint32_t)c01 | ((uint32_t)c23 << 16);
        if (lane == 0) {
          const uint32_t byte = (uint32_t)(e + 127);
          if (sf_plain)
            sf_plain[r * tiles + t] = (uint8_t)byte;
          else
            sf[(tile * tiles + t) * 128 + 4 * (p % 32) + p / 32] = byte * 0x01010101u;
        }
      }
    }
  }
}

}  // namespace

int64_t fp8_sf_tiles_bound(int64_t rows, int32_t G) { return ceil_div(rows, 128) + G; }

cudaError_t launch_quantize_rows(const void* src, const int32_t* src_row, const int32_t* offsets, int32_t G,
                                 int64_t rows_bound, int32_t cols, uint8_t* q, uint32_t* sf, cudaStream_t s,
                                 uint8_t* sf_plain) {
  if (rows_bound <= 0) return cudaSuccess;
  if (cols % 128 != 0 || G < 1 || G > kMaxExperts) return cudaErrorInvalidValue;
  int64_t blocks = ceil_div(rows_bound, kQuantWarps);
  if (blocks > 148 * 16) blocks = 148 * 16;
  quantize_rows_kernel<<<(unsigned)blocks, 32 * kQuantWarps, 0, s>>>(static_cast<const bf16*>(src), src_row, offsets,
                                                                    G, rows_bound, cols, q, sf, sf_plain);
  return cudaGetLastError();
}

}  // namespace moe
