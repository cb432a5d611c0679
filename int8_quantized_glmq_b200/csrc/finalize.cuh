// Finalize pass for GEMM calls whose tiles were split over K parts: the fp32 partial
// sums of all parts have been added into a scratch buffer ws [M, N]; this kernel
// applies the per-row scale, rounds to fp16 (the epilogue of the dequantizing linear
// layer, Y = fp16(s[n] * sum_k X q)) and returns ws to zero for the next call.
#pragma once

#include <cuda_fp16.h>
#include <cstdint>

#include "epilogue.cuh"
#include "glmq_ptx.cuh"

namespace glmq {

// Y[m, n] = fp16(s[n] * ws[m, n]) for split calls, columns n0 <= n < N (the split
// tiles' rows of W); returns those ws entries to zero.
// Grid: x covers the columns from n0 in groups of VEC per thread (one pass), y the
// token rows (rows m = blockIdx.y, blockIdx.y + gridDim.y, ...). VEC = 4 needs N % 4
// == 0 and n0 % 4 == 0, so every group is 16-byte aligned in ws and 8-byte aligned in
// Y and scale.
template <int VEC>
__global__ void __launch_bounds__(256) decode_finalize_kernel(float* __restrict__ ws, const __half* __restrict__ scale,
                                                              __half* __restrict__ Y, int M, int N, int n0) {
  // Let the next kernel in the stream launch now: its CTAs take their SM slots and run
  // their shared-memory prologue while this pass waits; every kernel launched with a
  // grid dependency here waits (griddep_wait) for this one before touching memory.
  griddep_launch_dependents();
  griddep_wait();   // the partial sums come from the kernel before this one
  const int n = n0 + (blockIdx.x * 256 + threadIdx.x) * VEC;
  if (n >= N) return;
  if constexpr (VEC == 4) {
    const uint2 sv = __ldg(reinterpret_cast<const uint2*>(scale + n));
    const float2 s01 = __half22float2(*reinterpret_cast<const __half2*>(&sv.x));
    const float2 s23 = __half22float2(*reinterpret_cast<const __half2*>(&sv.y));
    for (int m = blockIdx.y; m < M; m += gridDim.y) {
      const long long idx = static_cast<long long>(m) * N + n;
      const float4 v = __ldcg(reinterpret_cast<const float4*>(ws + idx));
      __stcg(reinterpret_cast<float4*>(ws + idx), make_float4(0.0f, 0.0f, 0.0f, 0.0f));
      const __half2 y01 = __floats2half2_rn(s01.x * v.x, s01.y * v.y);
      const __half2 y23 = __floats2half2_rn(s23.x * v.z, s23.y * v.w);
      uint2 o;
      o.x = *reinterpret_cast<const uint32_t*>(&y01);
      o.y = *reinterpret_cast<const uint32_t*>(&y23);
      *reinterpret_cast<uint2*>(Y + idx) = o;
    }
  } else {
    const float sn = __half2float(scale[n]);
    for (int m = blockIdx.y; m < M; m += gridDim.y) {
      const long long idx = static_cast<long long>(m) * N + n;
      const float v = __ldcg(ws + idx);
      __stcg(ws + idx, 0.0f);
      Y[idx] = __float2half_rn(sn * v);
    }
  }
}

// The same pass with a fused epilogue (a bias, and/or GeGLU over a GeGLU-layout
// weight): one thread per output column j >= j0 of a token row, Y of width N (bias
// only) or N / 2 (GeGLU). For GeGLU, output j reads packed rows pa = 16 (j / 8) + j % 8
// and pa + 8, and returns both scratch entries to zero; the packed rows from n0 on are
// the outputs from j0 = n0 / 2 on (n0 a multiple of 16).
__global__ void __launch_bounds__(256) finalize_epilogue_kernel(float* __restrict__ ws,
                                                                const __half* __restrict__ scale,
                                                                const __half* __restrict__ bias, int geglu,
                                                                __half* __restrict__ Y, int M, int N, int j0) {
  griddep_launch_dependents();   // as in decode_finalize_kernel
  griddep_wait();   // the partial sums come from the kernel before this one
  const int width = geglu ? (N >> 1) : N;
  const int j = j0 + blockIdx.x * 256 + threadIdx.x;
  if (j >= width) return;
  if (!geglu) {
    const float sj = __half2float(scale[j]);
    const float bj = bias ? __half2float(bias[j]) : 0.0f;
    for (int m = blockIdx.y; m < M; m += gridDim.y) {
      const long long idx = static_cast<long long>(m) * N + j;
      const float v = __ldcg(ws + idx);
      __stcg(ws + idx, 0.0f);
      Y[idx] = __float2half_rn(sj * v + bj);
    }
  } else {
    const int F = N >> 1;
    const int pa = 16 * (j >> 3) + (j & 7);
    const int pb = pa + 8;
    const float sa = __half2float(scale[pa]), sb = __half2float(scale[pb]);
    const float ba = bias ? __half2float(bias[j]) : 0.0f;
    const float bb = bias ? __half2float(bias[F + j]) : 0.0f;
    for (int m = blockIdx.y; m < M; m += gridDim.y) {
      const long long row = static_cast<long long>(m) * N;
      const float va = __ldcg(ws + row + pa), vb = __ldcg(ws + row + pb);
      __stcg(ws + row + pa, 0.0f);
      __stcg(ws + row + pb, 0.0f);
      const float ua = sa * va + ba, ub = sb * vb + bb;
      Y[static_cast<long long>(m) * F + j] = __float2half_rn(gelu_exact(ua) * ub);
    }
  }
}

}  // namespace glmq
