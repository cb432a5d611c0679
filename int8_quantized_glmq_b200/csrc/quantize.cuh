// One-shot weight quantization: fp16 W[N,K] -> packed INT4/INT8 codes + fp16 scale[N].
//
// GLM-130B paper card (wikillm.com), "Method": each output row of a linear
// layer gets one scale, absmax / 7, and the weights are rounded to integers in
// [-7, 7], two per byte. "Paper vs code": the divisor is 2^(b-1)-1, so INT8 uses
// absmax / 127, and the scale is computed per output row in FP16.
//
// Readings fixed by this library (the same ones the oracle states):
//   s = fp16_rn(fp32(a) / d),  q = clamp(rint(fp32(w) / fp32(s)), -d, d),
//   q = 0 on rows whose scale rounds to 0, round half to even,
//   INT4 byte j = (q[2j] & 0xF) | (q[2j+1] << 4)  (low nibble = even k).
//
// Kernel shape (HBM-bound): one CTA per row, 256 threads for rows up to 12288
// values and 512 or 1024 for longer rows (so a thread holds at most 8 chunks and
// enough CTAs stay resident to cover the memory latency). Each thread loads
// its 16-byte chunks of the row once with streaming 128-bit loads and keeps them
// in registers; the row absmax is a max over |w| (a warp reduce, then the warps
// through shared memory); the codes are formed from the
// registers and written with coalesced 4- or 8-byte stores. W is read exactly once.
//
// Exact rounding without a per-element IEEE divide: with r = 1/s rounded to
// nearest, t = fma(w, r, 1.5*2^23) leaves RNE(w*r) in the low mantissa bits of t.
// Let e = w*r - k (one fma). Because |w*r - w/s| <= (w/s)*2^-24 < 2^-16 for the
// quotients that occur (|w/s| < 192), |e| < 1/2 - 2^-15 proves k = RNE(w/s). The
// rare elements with |e| at or above that margin, and every element of a row
// whose scale is subnormal (where the clamp can fire), take an exact path that
// compares 2|w| with (2k +- 1)s; those products have at most 20 significant bits
// and are exact in fp32.
#pragma once

#include "epilogue.cuh"
#include "glmq_ptx.cuh"

namespace glmq {


// RNE(w / s) from a candidate kf within one of it, clamped to magnitude D, by exact
// comparisons of 2|w| with (2k +- 1) s.
template <int D>
__device__ __forceinline__ int exact_code_d(float w, float sf, float kf) {
  const float aw = fabsf(w);
  const int k0 = static_cast<int>(fabsf(kf));
  const float aw2 = aw + aw;                                   // exact
  const float hi = static_cast<float>(2 * k0 + 1) * sf;        // exact: <= 9 x 11 significant bits
  const float lo = static_cast<float>(2 * k0 - 1) * sf;        // exact
  int k = k0;
  if (aw2 > hi || (aw2 == hi && (k0 & 1))) {
    k = k0 + 1;
  } else if (aw2 < lo || (aw2 == lo && (k0 & 1))) {
    k = k0 - 1;
  }
  k = min(k, D);
  return (w < 0.0f) ? -k : k;
}

template <int BITS>
__device__ __forceinline__ int exact_code(float w, float sf, float kf) {
  return exact_code_d<(1 << (BITS - 1)) - 1>(w, sf, kf);
}

// Packed fp32 pairs (sm_100 f32x2 arithmetic): one instruction does two IEEE fp32
// operations, each rounded to nearest even exactly as the scalar instruction.
__device__ __forceinline__ float2 fma2_rn(float2 a, float2 b, float2 c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;"
      : "=l"(d)
      : "l"(*reinterpret_cast<unsigned long long*>(&a)), "l"(*reinterpret_cast<unsigned long long*>(&b)),
        "l"(*reinterpret_cast<unsigned long long*>(&c)));
  return *reinterpret_cast<float2*>(&d);
}

__device__ __forceinline__ float2 sub2_rn(float2 a, float2 b) {
  unsigned long long d;
  asm("sub.rn.f32x2 %0, %1, %2;"
      : "=l"(d)
      : "l"(*reinterpret_cast<unsigned long long*>(&a)), "l"(*reinterpret_cast<unsigned long long*>(&b)));
  return *reinterpret_cast<float2*>(&d);
}

// Codes for the 8 halves of one 16-byte chunk, as 32-bit words whose low bits hold
// the two's-complement code (the low byte is the int8 code; the low nibble the INT4
// code). Candidates and residuals are computed on fp32 pairs; a chunk whose largest
// residual reaches the margin (or every chunk of a row with a subnormal scale) takes
// the exact comparison path for all its elements.
template <int BITS>
__device__ __forceinline__ void chunk_codes(const uint4 v, float sf, float r, bool exact_all, uint32_t (&u)[8]) {
  constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
  constexpr float kMargin = 0.5f - 0x1p-15f;
  const uint32_t words[4] = {v.x, v.y, v.z, v.w};
  const float2 r2 = make_float2(r, r), nr2 = make_float2(-r, -r), m2 = make_float2(kMagic, kMagic);
  float2 w[4], k[4];
  float emax = 0.0f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    w[i] = __half22float2(*reinterpret_cast<const __half2*>(&words[i]));
    const float2 t = fma2_rn(w[i], r2, m2);          // RNE(w * r) in the low mantissa bits
    k[i] = sub2_rn(t, m2);                           // that integer, as a float
    const float2 e = fma2_rn(w[i], nr2, k[i]);       // k - w * r, exact
    emax = fmaxf(emax, fmaxf(fabsf(e.x), fabsf(e.y)));
    u[2 * i] = __float_as_uint(t.x);
    u[2 * i + 1] = __float_as_uint(t.y);
  }
  if (exact_all || emax >= kMargin) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      u[2 * i] = static_cast<uint32_t>(exact_code<BITS>(w[i].x, sf, k[i].x));
      u[2 * i + 1] = static_cast<uint32_t>(exact_code<BITS>(w[i].y, sf, k[i].y));
    }
  }
}

// Bytes [u0.b0, u1.b0, u2.b0, u3.b0]: the low bytes of four code words.
__device__ __forceinline__ uint32_t low_bytes4(uint32_t u0, uint32_t u1, uint32_t u2, uint32_t u3) {
  return prmt(prmt(u0, u1, 0x0040u), prmt(u2, u3, 0x0040u), 0x5410u);
}

// INT4: 8 code words -> one packed word, nibble j = code j & 0xF (low nibble = even k).
__device__ __forceinline__ uint32_t pack_int4_word(const uint32_t (&u)[8]) {
  const uint32_t b0 = low_bytes4(u[0], u[1], u[2], u[3]);       // code bytes k0..k3
  const uint32_t b1 = low_bytes4(u[4], u[5], u[6], u[7]);
  // byte 2i of y: (k_{2i} & 0xF) | (k_{2i+1} & 0xF) << 4  (odd bytes unused)
  const uint32_t y0 = lop3_sel(b0, b0 >> 4, 0x0F0F0F0Fu);
  const uint32_t y1 = lop3_sel(b1, b1 >> 4, 0x0F0F0F0Fu);
  return prmt(y0, y1, 0x6420u);
}

// One CTA of T threads per row; each thread holds CPT 16-byte chunks of the row.
// geglu_half = F > 0 writes the GeGLU row layout (output row 16g + r from input row
// 8g + r, r < 8, or F + 8g + r - 8); 0 keeps the natural order.
// At least 40 warps resident per SM (registers capped to fit): a row's loads are issued
// all at once and then waited for, so occupancy is what hides the memory latency.
constexpr int quantize_min_blocks(int T) { return T <= 256 ? 5 : (T <= 512 ? 2 : 1); }

template <int BITS, int CPT, int T>
__global__ void __launch_bounds__(T, quantize_min_blocks(T)) quantize_kernel(const __half* __restrict__ W, int K,
                                                     uint8_t* __restrict__ packed, __half* __restrict__ scale,
                                                     int geglu_half) {
  constexpr int D = (1 << (BITS - 1)) - 1;
  const long long row = blockIdx.x;
  const long long src_row = geglu_half > 0 ? geglu_natural_row(static_cast<int>(row), geglu_half) : row;
  const int nchunks = K >> 3;
  const uint4* src = reinterpret_cast<const uint4*>(W + src_row * static_cast<long long>(K));

  // Row absmax over |w|. The 256-thread shape takes it on the fp16 pipe (packed max of
  // absolute values), leaving the ALU pipe, which the rounding and packing keep busy,
  // a little freer; the longer rows keep the integer max of the |w| bit patterns
  // (measured 2% faster on QKV, attn-out and FFN-up, 1% slower on FFN-down). Both give
  // the bit pattern of the largest |w| of finite fp16 values.
  uint4 v[CPT];
  uint32_t m = 0;
  __half2 hm = __halves2half2(__ushort_as_half(0), __ushort_as_half(0));
#pragma unroll
  for (int i = 0; i < CPT; ++i) {
    const int c = threadIdx.x + i * T;
    if (c < nchunks) {
      v[i] = ld_stream_v4(src + c);
      if constexpr (T <= 256) {
        const __half2 a = __habs2(*reinterpret_cast<const __half2*>(&v[i].x));
        const __half2 b = __habs2(*reinterpret_cast<const __half2*>(&v[i].y));
        const __half2 cz = __habs2(*reinterpret_cast<const __half2*>(&v[i].z));
        const __half2 dw = __habs2(*reinterpret_cast<const __half2*>(&v[i].w));
        hm = __hmax2(hm, __hmax2(__hmax2(a, b), __hmax2(cz, dw)));
      } else {
        m = __vimax3_u16x2(m, v[i].x & 0x7fff7fffu, v[i].y & 0x7fff7fffu);
        m = __vimax3_u16x2(m, v[i].z & 0x7fff7fffu, v[i].w & 0x7fff7fffu);
      }
    } else {
      v[i] = make_uint4(0, 0, 0, 0);
    }
  }
  if constexpr (T <= 256) m = *reinterpret_cast<const uint32_t*>(&hm);
  m = max(m & 0xffffu, m >> 16);
  m = __reduce_max_sync(0xffffffffu, m);

  __shared__ uint32_t warp_max[T / 32];
  const int warp = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) warp_max[warp] = m;
  __syncthreads();
  uint32_t a_bits = warp_max[0];
#pragma unroll
  for (int i = 1; i < T / 32; ++i) a_bits = max(a_bits, warp_max[i]);

  // a2: s = fp16_rn(fp32(a) / d)
  const float af = __half2float(__ushort_as_half(static_cast<unsigned short>(a_bits)));
  const __half s = __float2half_rn(__fdiv_rn(af, static_cast<float>(D)));
  const float sf = __half2float(s);
  if (threadIdx.x == 0) scale[row] = s;

  const bool zero_row = (sf == 0.0f);
  const bool exact_all = sf < 0x1p-14f;  // subnormal scale: the clamp can fire
  const float r = zero_row ? 0.0f : __frcp_rn(sf);

#pragma unroll
  for (int i = 0; i < CPT; ++i) {
    const int c = threadIdx.x + i * T;
    if (c >= nchunks) continue;
    uint32_t u[8];
    if (zero_row) {
#pragma unroll
      for (int j = 0; j < 8; ++j) u[j] = 0;
    } else {
      chunk_codes<BITS>(v[i], sf, r, exact_all, u);
    }
    if constexpr (BITS == 4) {
      reinterpret_cast<uint32_t*>(packed + row * static_cast<long long>(K / 2))[c] = pack_int4_word(u);
    } else {
      const uint2 out = make_uint2(low_bytes4(u[0], u[1], u[2], u[3]), low_bytes4(u[4], u[5], u[6], u[7]));
      reinterpret_cast<uint2*>(packed + row * static_cast<long long>(K))[c] = out;
    }
  }
}

// ---------------------------------------------------------------- zero-point INT4
// Asymmetric variant (GLM-130B paper card, "Pitfalls": a zero-point INT4 quantizer
// scored better on LAMBADA but was not adopted; the card gives no formula). Per row:
//   lo = min(0, min W), hi = max(0, max W), s = fp16_rn(fl32(fl32(hi - lo) / 15)),
//   z = clamp(rint(fl32(-lo / s)), 0, 15), q = clamp(RNE(w / s) + z, 0, 15) unsigned,
// q = 0 and z = 0 where s == 0. Codes are packed like the symmetric ones (low nibble =
// even k). RNE(w / s) is exact, by the same fma candidate and comparison fix-up as
// quantize_kernel (|w / s| <= 16 here).
__device__ __forceinline__ void zp_chunk_codes(const uint4 v, float sf, float r, bool exact_all, int z,
                                               uint32_t (&q)[8]) {
  const uint32_t words[4] = {v.x, v.y, v.z, v.w};
  float w[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&words[i]));
    w[2 * i] = f.x;
    w[2 * i + 1] = f.y;
  }
  constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
  constexpr float kMargin = 0.5f - 0x1p-15f;
  float kf[8];
  bool near = exact_all;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    kf[i] = fmaf(w[i], r, kMagic) - kMagic;
    near |= fabsf(fmaf(w[i], r, -kf[i])) >= kMargin;
  }
  if (near) {
#pragma unroll
    for (int i = 0; i < 8; ++i) kf[i] = static_cast<float>(exact_code_d<16>(w[i], sf, kf[i]));
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) q[i] = static_cast<uint32_t>(min(max(static_cast<int>(kf[i]) + z, 0), 15));
}

template <int CPT, int T>
__global__ void __launch_bounds__(T) quantize_zp_kernel(const __half* __restrict__ W, int K,
                                                        uint8_t* __restrict__ packed, __half* __restrict__ scale,
                                                        uint8_t* __restrict__ zero) {
  const long long row = blockIdx.x;
  const int nchunks = K >> 3;
  const uint4* src = reinterpret_cast<const uint4*>(W + row * static_cast<long long>(K));
  uint4 v[CPT];
  __half2 mn = __float2half2_rn(0.0f), mx = mn;      // the range includes zero
#pragma unroll
  for (int i = 0; i < CPT; ++i) {
    const int c = threadIdx.x + i * T;
    v[i] = make_uint4(0, 0, 0, 0);
    if (c < nchunks) {
      v[i] = ld_stream_v4(src + c);
      const uint32_t words[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const __half2 h = *reinterpret_cast<const __half2*>(&words[j]);
        mn = __hmin2(mn, h);
        mx = __hmax2(mx, h);
      }
    }
  }
  float lo = fminf(__low2float(mn), __high2float(mn));
  float hi = fmaxf(__low2float(mx), __high2float(mx));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, off));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, off));
  }
  __shared__ float warp_lo[T / 32], warp_hi[T / 32];
  const int warp = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) {
    warp_lo[warp] = lo;
    warp_hi[warp] = hi;
  }
  __syncthreads();
  lo = warp_lo[0];
  hi = warp_hi[0];
#pragma unroll
  for (int i = 1; i < T / 32; ++i) {
    lo = fminf(lo, warp_lo[i]);
    hi = fmaxf(hi, warp_hi[i]);
  }
  const __half s = __float2half_rn(__fdiv_rn(hi - lo, 15.0f));
  const float sf = __half2float(s);
  const bool zero_row = (sf == 0.0f);
  const int z = zero_row ? 0 : min(max(static_cast<int>(rintf(__fdiv_rn(-lo, sf))), 0), 15);
  if (threadIdx.x == 0) {
    scale[row] = s;
    zero[row] = static_cast<uint8_t>(z);
  }
  const bool exact_all = sf < 0x1p-14f;  // subnormal scale
  const float r = zero_row ? 0.0f : __frcp_rn(sf);
#pragma unroll
  for (int i = 0; i < CPT; ++i) {
    const int c = threadIdx.x + i * T;
    if (c >= nchunks) continue;
    uint32_t q[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (!zero_row) zp_chunk_codes(v[i], sf, r, exact_all, z, q);
    uint32_t word = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) word |= q[j] << (4 * j);
    reinterpret_cast<uint32_t*>(packed + row * static_cast<long long>(K / 2))[c] = word;
  }
}

}  // namespace glmq
