// quant.cu -- FP8 (E4M3) quantisation of activation rows for the FP8 experts.
//
// Page "15. DeepSeek: MLA, MoE and MTP", FP8 section: matrix inputs in E4M3,
// one scale per 1 x 128 tile of activations, scales stored as UE8M0 (an 8-bit
// exponent, scale = 2^(byte - 127)). For every row and 128-column tile:
//   e      = the smallest integer with amax <= 448 * 2^e (0 when amax = 0),
//   code_c = E4M3 of v_c * 2^-e, round to nearest even (|v_c * 2^-e| <= 448).
// The scale of row r, tile t is written where the tensor-core GEMM reads it:
// GEMM row tiles of TR = 128 (or 32) rows of each group (tile m of group g
// covers rows offsets[g] + TR m ...), one 512-byte block per (row tile, four
// consecutive 128-column tiles) in the scale-factor layout of tcgen05.mma block
// scaling: the 32-bit word of tile row p sits at word 4 (p % 32) + p / 32, and
// its byte j is the UE8M0 byte of column tile 4q + j (the GEMM's MMAs select the
// byte of their k block).
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

// UE8M0 exponent of a tile whose largest magnitude is amax (finite binary32):
// with amax = f * 2^x, f in [0.5, 1), amax <= 448 * 2^e  <=>  f * 2^(x - 8 - e) <= 1.75,
// so e = x - 9 when f <= 0.875 and x - 8 otherwise. For a normal amax = 1.m * 2^(E - 127)
// that is x = E - 126 and f <= 0.875 <=> m <= 0.75, read straight off the bits.
__device__ __forceinline__ int ue8m0_exponent(float amax) {
  if (!(amax > 0.0f)) return 0;
  const uint32_t u = __float_as_uint(amax);
  const int E = (int)(u >> 23);
  int e;
  if (E > 0) {
    e = (u & 0x7FFFFFu) <= 0x600000u ? E - 135 : E - 134;
  } else {  // binary32 subnormal
    int x;
    const float f = frexpf(amax, &x);
    e = f <= 0.875f ? x - 9 : x - 8;
  }
  return e < -127 ? -127 : (e > 127 ? 127 : e);
}

// 2^-e as a binary32 (normal for the exponents bf16 inputs produce, -127 <= e <= 119).
__device__ __forceinline__ float pow2_neg(int e) { return __uint_as_float((uint32_t)(127 - e) << 23); }

constexpr int kQuantWarps = 8;

// One warp per row, two 128-column tiles at a time (one per half-warp).
__global__ void __launch_bounds__(32 * kQuantWarps)
    quantize_rows_kernel(const bf16* src, const int32_t* src_row, const int32_t* offsets, int G, int64_t rows_single,
                         int cols, int TR, uint8_t* q, uint32_t* sf, uint8_t* sf_plain) {
  __shared__ int32_t tile_off[kMaxExperts + 1];  // first row tile of each group
  __shared__ int32_t row_off[kMaxExperts + 1];
  if (threadIdx.x == 0) {
    int32_t acc = 0;
    for (int g = 0; g < G; ++g) {
      const int32_t lo = offsets ? offsets[g] : 0;
      const int32_t hi = offsets ? offsets[g + 1] : (int32_t)rows_single;
      row_off[g] = lo;
      row_off[g + 1] = hi;
      tile_off[g] = acc;
      acc += (hi - lo + TR - 1) / TR;
    }
    tile_off[G] = acc;
  }
  __syncthreads();
  const int64_t rows = row_off[G];
  const int lane = threadIdx.x & 31;
  const int tiles = cols / 128;
  const int quads = (tiles + 3) / 4;  // scale blocks per row tile
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t r = warp; r < rows; r += nwarps) {
    // group of row r (offsets ascending), its GEMM row tile and the row inside it
    int lo = 0, hi = G - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (row_off[mid] <= r) lo = mid; else hi = mid - 1;
    }
    const int g = lo;
    const int64_t local = r - row_off[g];
    const int64_t tile = tile_off[g] + local / TR;
    const int p = (int)(local % TR);
    const int64_t srow = src_row ? (int64_t)src_row[r] : r;
    // Half-warp h of the warp owns tile 2c + h of chunk c (256 columns); lane l of a
    // half-warp holds columns 8 (l % 16) .. +7 of its tile: one 16-byte load and one
    // 8-byte store per lane, four chunks of loads in flight.
    const uint4* in = reinterpret_cast<const uint4*>(src + srow * cols);
    uint2* out = reinterpret_cast<uint2*>(q + r * cols);
    const int half = lane >> 4, hl = lane & 15;
    const unsigned hmask = half ? 0xffff0000u : 0x0000ffffu;
    const int chunks = (tiles + 1) / 2;
    for (int c0 = 0; c0 < chunks; c0 += 4) {
      uint4 raws[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int t = 2 * (c0 + u) + half;
        if (c0 + u < chunks && t < tiles) raws[u] = __ldg(in + t * 16 + hl);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int t = 2 * (c0 + u) + half;
        if (c0 + u >= chunks || t >= tiles) continue;  // uniform within each half-warp
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raws[u]);
        float v[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          v[2 * j] = __low2float(h2[j]);
          v[2 * j + 1] = __high2float(h2[j]);
        }
        float m = 0.0f;
#pragma unroll
        for (int j = 0; j < 8; ++j) m = fmaxf(m, fabsf(v[j]));
#pragma unroll
        for (int off = 8; off; off >>= 1) m = fmaxf(m, __shfl_xor_sync(hmask, m, off));
        const int e = ue8m0_exponent(m);
        const float sc = pow2_neg(e);  // multiplying by 2^-e is exact for these magnitudes
        uint32_t w[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const __nv_fp8x2_storage_t c01 = __nv_cvt_float2_to_fp8x2(
              make_float2(v[4 * j] * sc, v[4 * j + 1] * sc), __NV_SATFINITE, __NV_E4M3);
          const __nv_fp8x2_storage_t c23 = __nv_cvt_float2_to_fp8x2(
              make_float2(v[4 * j + 2] * sc, v[4 * j + 3] * sc), __NV_SATFINITE, __NV_E4M3);
          w[j] = (uint32_t)c01 | ((uint32_t)c23 << 16);
        }
        out[t * 16 + hl] = make_uint2(w[0], w[1]);
        if (hl == 0) {
          const uint32_t byte = (uint32_t)(e + 127);
          if (sf_plain)
            sf_plain[r * tiles + t] = (uint8_t)byte;
          else
            reinterpret_cast<uint8_t*>(sf)[(((tile * quads + (t >> 2)) * 128) + 4 * (p % 32) + p / 32) * 4 + (t & 3)] =
                (uint8_t)byte;
        }
      }
    }
  }
}

}  // namespace

cudaError_t launch_quantize_rows(const void* src, const int32_t* src_row, const int32_t* offsets, int32_t G,
                                 int64_t rows_bound, int32_t cols, int32_t tile_rows, uint8_t* q, uint32_t* sf,
                                 cudaStream_t s, uint8_t* sf_plain) {
  if (rows_bound <= 0) return cudaSuccess;
  if (cols % 128 != 0 || G < 1 || G > kMaxExperts || (tile_rows != 128 && tile_rows != 32))
    return cudaErrorInvalidValue;
  int64_t blocks = ceil_div(rows_bound, kQuantWarps);
  if (blocks > 148 * 16) blocks = 148 * 16;
  quantize_rows_kernel<<<(unsigned)blocks, 32 * kQuantWarps, 0, s>>>(static_cast<const bf16*>(src), src_row, offsets,
                                                                    G, rows_bound, cols, tile_rows, q, sf, sf_plain);
  return cudaGetLastError();
}

}  // namespace moe
