// Fused epilogues of the GLM-130B projections, shared by the GEMM kernels.
//
// GLM-130B paper card (wikillm.com): "Method" -- the feed-forward block is a GeGLU
// (FFN-up carries the two GLU branches, 2 x 32768 rows); "Paper vs code" -- biases
// stay FP16. paperlayer summary, section B.3: GeGLU feed-forward network.
//
//   bias:  Y[m,n] = fp16( s[n] acc[m,n] + b[n] ),  b fp16 in the natural row order.
//   GeGLU: with U = s acc + b over N = 2F rows, Y[m,j] = fp16( GELU(U[m,j]) U[m,F+j] ),
//          GELU(u) = u Phi(u) = 0.5 u (1 + erf(u / sqrt 2)), Y of shape [M, F].
// For the fused GeGLU the packed weights are stored in blocks of 16 rows (see
// glmq_quantize_geglu): packed row 16g + r holds natural row 8g + r for r < 8 and
// F + 8g + r - 8 for r >= 8, so each pair sits 8 rows apart in one block and reaches
// one thread (the decode MMA fragment's rows r and r + 8) or one warp (TMEM lanes).
#pragma once

#include <cuda_fp16.h>

namespace glmq {

__device__ __forceinline__ float gelu_exact(float u) { return 0.5f * u * (1.0f + erff(u * 0.70710678118654752f)); }

// Natural row of W held by packed row p of the GeGLU layout (F = N / 2).
__device__ __forceinline__ int geglu_natural_row(int p, int F) {
  const int g = p >> 4, r = p & 15;
  return r < 8 ? 8 * g + r : F + 8 * g + (r - 8);
}

// Output column of the pair whose first-half row is packed row p (p % 16 < 8).
__device__ __forceinline__ int geglu_column(int p) { return 8 * (p >> 4) + (p & 15); }

// Bias of packed row p (0 when there is no bias).
__device__ __forceinline__ float epilogue_bias(const __half* bias, int geglu, int p, int N) {
  if (bias == nullptr) return 0.0f;
  return __half2float(bias[geglu ? geglu_natural_row(p, N >> 1) : p]);
}

}  // namespace glmq
