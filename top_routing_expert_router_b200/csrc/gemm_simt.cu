// gemm_simt.cu -- grouped GEMM on the CUDA cores (FFMA, binary32 accumulation).
//
// C[r, :] = A[r, :] B_g^T for the rows r of group g (plain), or
// C[r, :] = silu(A[r, :] Bg_g^T) * (A[r, :] Bu_g^T) (SwiGLU epilogue).
// Used for binary32 layers (whose 1e-4 tolerance rules out TF32 tensor cores)
// and for the router logits of small problems. Tiles: 64 rows x 64 output
// columns x 16 k, 256 threads, 4 x 4 outputs per thread (x2 for SwiGLU).
#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

constexpr int BM = 64, BN = 64, BK = 16;

template <typename T, typename TO, bool SWIGLU>
__global__ void __launch_bounds__(256) gemm_simt_kernel(GemmArgs a) {
  __shared__ float As[BK][BM + 4];
  __shared__ float Bs[BK][BN + 4];
  __shared__ float Us[SWIGLU ? BK : 1][BN + 4];

  // Map blockIdx.y to (group, m-tile) by walking the group row counts.
  int64_t row0 = 0, row_end = 0;
  int g = 0;
  {
    int64_t y = blockIdx.y;
    bool found = false;
    for (g = 0; g < a.G; ++g) {
      const int64_t lo = a.offsets ? a.offsets[g] : 0;
      const int64_t hi = a.offsets ? a.offsets[g + 1] : a.M;
      const int64_t tiles = ceil_div(hi - lo, BM);
      if (y < tiles) {
        row0 = lo + y * BM;
        row_end = hi;
        found = true;
        break;
      }
      y -= tiles;
    }
    if (!found) return;
  }
  const int col0 = blockIdx.x * BN;
  const T* A = static_cast<const T*>(a.A);
  const T* B = static_cast<const T*>(a.B) + (int64_t)g * a.b_group_stride;
  const T* U = SWIGLU ? static_cast<const T*>(a.B2) + (int64_t)g * a.b_group_stride : nullptr;

  const int tid = threadIdx.x;
  const int tr = tid / 16, tc = tid % 16;  // 16 x 16 threads, 4 x 4 outputs each
  float acc[4][4] = {};
  float accu[SWIGLU ? 4 : 1][SWIGLU ? 4 : 1] = {};

  for (int k0 = 0; k0 < a.K; k0 += BK) {
    // 64 x 16 tiles: each of the 256 threads loads 4 elements of A and of B (and U).
    for (int i = tid; i < BM * BK; i += 256) {
      const int r = i / BK, kk = i % BK;
      const int64_t row = row0 + r;
      const int k = k0 + kk;
      As[kk][r] = (row < row_end && k < a.K) ? to_f32(A[row * a.lda + k]) : 0.0f;
      const int col = col0 + r;
      Bs[kk][r] = (col < a.N && k < a.K) ? to_f32(B[(int64_t)col * a.K + k]) : 0.0f;
      if constexpr (SWIGLU) Us[kk][r] = (col < a.N && k < a.K) ? to_f32(U[(int64_t)col * a.K + k]) : 0.0f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float av[4], bv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) av[i] = As[kk][tr * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) bv[j] = Bs[kk][tc * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
      if constexpr (SWIGLU) {
        float uv[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) uv[j] = Us[kk][tc * 4 + j];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) accu[i][j] = fmaf(av[i], uv[j], accu[i][j]);
      }
    }
    __syncthreads();
  }
  TO* C = static_cast<TO*>(a.C);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t row = row0 + tr * 4 + i;
    if (row >= row_end) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int col = col0 + tc * 4 + j;
      if (col >= a.N) continue;
      float v = acc[i][j];
      if constexpr (SWIGLU) v = silu(v) * accu[i][j];
      C[row * a.ldc + col] = from_f32<TO>(v);
    }
  }
}

}  // namespace

int64_t gemm_simt_max_tiles_y(int64_t rows_total, int G) { return ceil_div(rows_total, BM) + G; }

cudaError_t launch_gemm_simt(const GemmArgs& a, int dtype, bool out_f32, bool swiglu, cudaStream_t s) {
  if (a.k_splits > 1) return cudaErrorInvalidValue;  // split-K is a tensor-core path feature
  const int64_t ty = gemm_simt_max_tiles_y(a.M, a.G);
  if (ty <= 0 || a.N <= 0) return cudaSuccess;
  dim3 grid((unsigned)ceil_div(a.N, BN), (unsigned)ty);
  if (dtype == MOE_F32) {
    if (swiglu)
      gemm_simt_kernel<float, float, true><<<grid, 256, 0, s>>>(a);
    else
      gemm_simt_kernel<float, float, false><<<grid, 256, 0, s>>>(a);
  } else if (out_f32) {
    gemm_simt_kernel<bf16, float, false><<<grid, 256, 0, s>>>(a);
  } else if (swiglu) {
    gemm_simt_kernel<bf16, bf16, true><<<grid, 256, 0, s>>>(a);
  } else {
    gemm_simt_kernel<bf16, bf16, false><<<grid, 256, 0, s>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace moe
