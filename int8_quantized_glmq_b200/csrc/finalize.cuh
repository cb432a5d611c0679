// Finalize pass for GEMM calls whose tiles were split over K parts: the fp32 partial
// sums of all parts have been added into a scratch buffer ws [M, N]; this kernel
// applies the per-row scale, rounds to fp16 (the epilogue of the dequantizing linear
// layer, Y = fp16(s[n] * sum_k X q)) and returns ws to zero for the next call.
//
// The pass sits on the critical path between two GEMM kernels, so it is built for
// latency: each thread loads up to kFinalizeRows token rows of its columns at once, and
// the per-column constants (scale, bias) are read before the grid-dependency wait. That
// is safe: they are not written by the GEMM kernel this pass follows, and that kernel
// had itself waited for every kernel before it (or, launched without a grid dependency,
// started only after them) before this pass could launch.
#pragma once

#include <cuda_fp16.h>
#include <cstdint>

#include "epilogue.cuh"
#include "glmq_ptx.cuh"

namespace glmq {

// Token rows a thread of decode_finalize_kernel<4> handles with its loads in flight together.
constexpr int kFinalizeRows = 16;

// Y[m, n] = fp16(s[n] * ws[m, n]) for split calls, columns n0 <= n < N (the split
// tiles' rows of W); returns those ws entries to zero.
// Grid: x covers the columns from n0 in groups of VEC per thread (one pass). VEC = 4:
// y covers the token rows in blocks of kFinalizeRows (rows m0 .. m0 + 15 with m0 =
// 16 blockIdx.y, 16 (blockIdx.y + gridDim.y), ...); it needs N % 4 == 0 and n0 % 4 ==
// 0, so every group is 16-byte aligned in ws and 8-byte aligned in Y and scale.
// VEC = 1: y covers single rows (m = blockIdx.y, blockIdx.y + gridDim.y, ...).
template <int VEC>
__global__ void __launch_bounds__(256) decode_finalize_kernel(float* __restrict__ ws, const __half* __restrict__ scale,
                                                              __half* __restrict__ Y, int M, int N, int n0) {
  // Let the next kernel in the stream launch now: its CTAs take their SM slots and run
  // their shared-memory prologue while this pass waits; every kernel launched with a
  // grid dependency here waits (griddep_wait) for this one before touching memory.
  griddep_launch_dependents();
  const int n = n0 + (blockIdx.x * 256 + threadIdx.x) * VEC;
  const bool live = n < N;
  uint2 sv = make_uint2(0, 0);
  float sn = 0.0f;
  if (live) {   // per-column constants before the wait (see the top of this file)
    if constexpr (VEC == 4) sv = __ldg(reinterpret_cast<const uint2*>(scale + n));
    else sn = __half2float(scale[n]);
  }
  griddep_wait();   // the partial sums come from the kernel before this one
  if (!live) return;
  if constexpr (VEC == 4) {
    const float2 s01 = __half22float2(*reinterpret_cast<const __half2*>(&sv.x));
    const float2 s23 = __half22float2(*reinterpret_cast<const __half2*>(&sv.y));
    constexpr int R = kFinalizeRows;
    for (int m0 = blockIdx.y * R; m0 < M; m0 += gridDim.y * R) {
      float4 v[R];
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const long long idx = static_cast<long long>(m0 + r) * N + n;
        v[r] = (m0 + r < M) ? __ldcg(reinterpret_cast<const float4*>(ws + idx)) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int r = 0; r < R; ++r) {
        if (m0 + r >= M) break;
        const long long idx = static_cast<long long>(m0 + r) * N + n;
        __stcg(reinterpret_cast<float4*>(ws + idx), make_float4(0.0f, 0.0f, 0.0f, 0.0f));
        const __half2 y01 = __floats2half2_rn(s01.x * v[r].x, s01.y * v[r].y);
        const __half2 y23 = __floats2half2_rn(s23.x * v[r].z, s23.y * v[r].w);
        uint2 o;
        o.x = *reinterpret_cast<const uint32_t*>(&y01);
        o.y = *reinterpret_cast<const uint32_t*>(&y23);
        *reinterpret_cast<uint2*>(Y + idx) = o;
      }
    }
  } else {
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
  const int width = geglu ? (N >> 1) : N;
  const int j = j0 + blockIdx.x * 256 + threadIdx.x;
  if (j >= width) {
    griddep_wait();
    return;
  }
  // per-column constants before the wait (see the top of this file)
  const int F = N >> 1;
  const int pa = geglu ? 16 * (j >> 3) + (j & 7) : j;
  const int pb = pa + 8;
  const float sa = __half2float(scale[pa]);
  const float sb = geglu ? __half2float(scale[pb]) : 0.0f;
  const float ba = bias ? __half2float(bias[j]) : 0.0f;
  const float bb = (bias && geglu) ? __half2float(bias[F + j]) : 0.0f;
  griddep_wait();   // the partial sums come from the kernel before this one
  if (!geglu) {
    const float sj = sa;
    const float bj = ba;
    for (int m = blockIdx.y; m < M; m += gridDim.y) {
      const long long idx = static_cast<long long>(m) * N + j;
      const float v = __ldcg(ws + idx);
      __stcg(ws + idx, 0.0f);
      Y[idx] = __float2half_rn(sj * v + bj);
    }
  } else {
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
