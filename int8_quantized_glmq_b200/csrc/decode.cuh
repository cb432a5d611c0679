// Decode-regime W4A16 / W8A16 GEMM: Y[M,N] = fp16( s[n] * sum_k X[m,k] q[n,k] ), M <= 16.
//
// GLM-130B paper card (wikillm.com), "Method": linear_forward dequantizes the
// weights at run time (weight = quant * scale[:, None]) and multiplies FP16
// activations by them; paperlayer summary, "INT4 Quantization for RTX
// 3090s/2080s": weights are converted to FP16 at run time, activations stay FP16.
// The scale multiplies whole rows of W, so it is applied once per output in the
// epilogue instead of once per weight (equal in exact arithmetic).
//
// With M <= 16 the packed weights are the whole working set: the kernel is an
// HBM stream. Design:
//  * Work units are (row tile of 256 rows, K part) pairs, enumerated K-part major;
//    each persistent CTA takes one contiguous range of units, so the load is
//    balanced to within one unit and a CTA changes K part (and so restages its
//    activation slice) at most a few times. The number of K parts is the smallest
//    that both fits the activation slice in shared memory and spreads the units
//    evenly over the SMs.
//  * Warp 16 is the producer: one lane issues, per stage, one 2-D TMA tile load of
//    256 rows x 128 bytes (128-byte swizzle, 32 KB) into a kDecodeStages-deep
//    ring, with an L2 evict-first hint. Rows past N and bytes past K are
//    zero-filled by the TMA unit.
//  * Warps 0..15 are consumers: warp w owns rows 16w .. 16w+15 of the tile and
//    reads the whole stage's K segment for them. Codes are dequantized in
//    registers with exponent-bias tricks (a code c becomes the fp16 number
//    1024 + (c ^ 8) by OR-ing it into the mantissa) and feed mma.sync m16n8k16
//    as the A operand straight from registers, X being the B operand. The K order
//    inside each MMA is permuted identically on both operands so that each 32-bit
//    packed word feeds two MMAs without a byte shuffle; the permutation is applied
//    once, when the consumers stage the activation slice into shared memory in
//    exactly the order the B fragments are read.
//  * A warp's sums stay in registers for the whole unit, so a unit ends without
//    any cross-warp reduction or barrier: the warp scales, rounds and stores its
//    own 16 rows. When a tile is split over several K parts each warp instead adds
//    its partial sums into an fp32 scratch buffer with fire-and-forget
//    red.global.add, and a small stream-ordered finalize kernel
//    (decode_finalize_kernel) scales, rounds and stores Y and returns the scratch
//    to zero for the next call.
#pragma once

#include <cuda.h>

#include "epilogue.cuh"
#include "glmq_ptx.cuh"

namespace glmq {

constexpr int kDecodeConsumerWarps = 16;
constexpr int kDecodeThreads = (kDecodeConsumerWarps + 1) * 32;
constexpr int kDecodeStages = 6;
constexpr int kDecodeRows = 16 * kDecodeConsumerWarps;                // rows per tile (256)
constexpr int kDecodeSegB = 128;         // packed bytes per row per stage (one TMA box width)
constexpr int kDecodeStageBytes = kDecodeRows * kDecodeSegB;          // 32 KB: one TMA box per stage
// ring + barriers; the activation slice follows
constexpr int kDecodeFixedSmem = kDecodeStages * kDecodeStageBytes + 256;

template <int BITS, int MP, int CHAINS = 2, int ZP = 0>
struct DecodeCfg {
  static_assert(CHAINS == 2 || CHAINS == 4, "accumulator chains");
  static_assert(ZP == 0 || BITS == 4, "zero-point codes are INT4");
  static constexpr int kZP = ZP;   // 1: zero-point INT4 codes (unsigned, per-row zero point)
  // biased dequantization: low nibbles give the fp16 integer kLowBase + (value), high
  // nibbles kHighBase + 16 (value); symmetric codes carry their own +8 offset in the XOR
  static constexpr uint32_t kXorLo = ZP ? 0x64006400u : 0x64086408u;
  static constexpr uint32_t kXorHi = ZP ? 0x64006400u : 0x64806480u;
  static constexpr float kLowBias = ZP ? 1024.0f : 1032.0f;    // per unit of x in a low-nibble slot
  static constexpr float kHighBias = ZP ? 1024.0f : 1152.0f;   // per unit of x / 16 in a high-nibble slot
  static constexpr int kBits = BITS;
  static constexpr int kMP = MP;                    // token capacity of the activation layout (M <= MP)
  static constexpr int kNB = (MP + 7) / 8;          // n8 token blocks of the MMA
  static constexpr int KPB = (BITS == 4) ? 2 : 1;   // codes per byte
  static constexpr int SEGK = kDecodeSegB * KPB;    // k per segment
  static constexpr int SK = SEGK;                   // k per stage (one segment)
  static constexpr int TB = kDecodeSegB / 4;        // packed bytes per thread per row per segment (32)
  static constexpr int TK = TB * KPB;               // k per thread per segment
  static constexpr int TW = TB / 4;                 // 32-bit words per thread per row per segment (8)
  static constexpr int XU = TK / 8;                 // 16-byte activation units per thread per segment
  static constexpr int kChains = CHAINS;            // independent MMA accumulator chains per token block
};

struct DecodeArgs {
  const __half* X;
  const __half* scale;
  __half* Y;
  float* ws;          // fp32 [M, N] scratch, zero on entry (used when parts > 1)
  const uint8_t* zero;  // zero-point codes: uint8 [N] per-row zero point, else NULL
  const __half* bias; // fp16 [N] in the natural row order of W, or NULL (epilogue.cuh)
  int geglu;          // 1: packed rows in the GeGLU layout, Y is [M, N / 2]
  int M;
  int N;
  int K;
  int KPP;            // k per part (multiple of SK)
  int parts;
  int tiles;
  int units;          // parts * tiles
  // The next decode call on the stream (glmq_gemm_decode_prefetch), planned the same
  // way: while this call's ring drains, its producer prefetches into L2 the stages the
  // next call's CTAs load first. nxt_grid == 0: no next call.
  int nxt_grid;
  int nxt_units;
  int nxt_tiles;
  int nxt_KPP;
  int nxt_K;
};

// INT4, biased form: one packed word (8 codes, k = 0..7 of the word) -> 4 half2
// registers holding the pairs (0,4), (1,5), (2,6), (3,7). A code nibble OR-ed into
// the mantissa of 1024 gives an exact fp16 integer: for symmetric codes (XOR 0x6408 /
// 0x6480) low nibbles give 1032 + q and high nibbles 1152 + 16 q; for zero-point codes
// (XOR 0x6400) 1024 + c and 1024 + 16 c. The MMA's B operand holds x for low-nibble
// slots and x / 16 for high-nibble slots, so every product is (code value) * x plus a
// bias depending only on x, and the accumulated bias is removed per segment (see
// decode_segment). Four LOP3 and one shift per 8 codes.
template <uint32_t XLO, uint32_t XHI>
__device__ __forceinline__ void dequant_int4_word_biased(uint32_t w, uint32_t (&p)[4]) {
  const uint32_t w8 = w >> 8;
  p[0] = lop3_and_xor(w, 0x000F000Fu, XLO);
  p[1] = lop3_and_xor(w, 0x00F000F0u, XHI);
  p[2] = lop3_and_xor(w8, 0x000F000Fu, XLO);
  p[3] = lop3_and_xor(w8, 0x00F000F0u, XHI);
}

// INT8: one word (4 codes, k = 0..3) -> half2 pairs (0,1), (2,3).
__device__ __forceinline__ void dequant_int8_word(uint32_t w, uint32_t (&p)[2]) {
  const __half2 kBias = __halves2half2(__ushort_as_half(0xE480), __ushort_as_half(0xE480));  // -1152
  const uint32_t x = w ^ 0x80808080u;
  uint32_t lo = prmt(x, 0x64646464u, 0x4140u);
  uint32_t hi = prmt(x, 0x64646464u, 0x4342u);
  __half2 a = __hadd2(*reinterpret_cast<__half2*>(&lo), kBias);
  __half2 b = __hadd2(*reinterpret_cast<__half2*>(&hi), kBias);
  p[0] = *reinterpret_cast<uint32_t*>(&a);
  p[1] = *reinterpret_cast<uint32_t*>(&b);
}

__device__ __forceinline__ void tma_load_2d_hint(void* smem_dst, const CUtensorMap* map, int x, int y, uint64_t* bar,
                                                 uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint "
      "[%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// L2 prefetch of one TMA box (a hint: no shared memory is written, nothing waits).
__device__ __forceinline__ void tma_prefetch_2d(const CUtensorMap* map, int x, int y) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(x), "r"(y)
               : "memory");
}

// Index (in 16-byte units) of the activation unit read by lane (n, c) for unit jj of
// segment sg of the current K part. Consecutive lanes of a token read consecutive
// units; the token stride is the compile-time capacity MP, so within a stage every
// fragment address is a per-lane base plus an immediate.
template <class C>
__host__ __device__ constexpr uint32_t x_unit(int sg, int jj, int n, int c) {
  return static_cast<uint32_t>(((sg * C::XU + jj) * C::kMP + n) * 4 + c);
}

// One stage of one consumer warp: its segment (TK codes per lane) of rows ra and
// ra + 8, against the staged activations. kTail: some lanes' codes lie past K.
template <class C, bool kTail>
__device__ __forceinline__ void decode_segment(uint32_t box, uint32_t xseg, uint32_t wlane, uint32_t xlane0,
                                               uint32_t xlane1, bool valid, const float* bias_seg, int c,
                                               float (&acc)[C::kChains][C::kNB][4]) {
  constexpr uint32_t kJStride = static_cast<uint32_t>(C::kMP) * 64u;   // bytes between consecutive jj
  uint32_t wa[C::TW], wb[C::TW];
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    uint4 va = make_uint4(0, 0, 0, 0), vb = make_uint4(0, 0, 0, 0);
    if (!kTail || valid) {
      // 128-byte swizzle: lane offsets for q = 0 / 1 are precomputed in wlane (low / high 16 bits)
      const uint32_t off = q ? (wlane >> 16) : (wlane & 0xFFFFu);
      va = lds_v4(box + off);
      vb = lds_v4(box + off + 8 * kDecodeSegB);
    }
    wa[4 * q + 0] = va.x; wa[4 * q + 1] = va.y; wa[4 * q + 2] = va.z; wa[4 * q + 3] = va.w;
    wb[4 * q + 0] = vb.x; wb[4 * q + 1] = vb.y; wb[4 * q + 2] = vb.z; wb[4 * q + 3] = vb.w;
  }
  if constexpr (C::kBits == 4) {
#pragma unroll
    for (int j = 0; j < C::TW; ++j) {
      uint4 bf[C::kNB];
#pragma unroll
      for (int nb = 0; nb < C::kNB; ++nb) {
        bf[nb] = make_uint4(0, 0, 0, 0);
        if (!kTail || valid) bf[nb] = lds_v4(xseg + (nb ? xlane1 : xlane0) + j * kJStride);
      }
      uint32_t pa[4], pb[4];
      dequant_int4_word_biased<C::kXorLo, C::kXorHi>(wa[j], pa);
      dequant_int4_word_biased<C::kXorLo, C::kXorHi>(wb[j], pb);
      const int h0 = (C::kChains == 4) ? 2 * (j & 1) : 0;
#pragma unroll
      for (int nb = 0; nb < C::kNB; ++nb) {
        mma_16816(acc[h0][nb], pa[0], pb[0], pa[1], pb[1], bf[nb].x, bf[nb].y);
        mma_16816(acc[h0 + 1][nb], pa[2], pb[2], pa[3], pb[3], bf[nb].z, bf[nb].w);
      }
    }
    // remove the bias this segment added: bias_seg[t] = sum_k (1032 or 1152) * B[k][t]
#pragma unroll
    for (int nb = 0; nb < C::kNB; ++nb) {
      const float2 b = *reinterpret_cast<const float2*>(bias_seg + 8 * nb + 2 * c);
      acc[0][nb][0] -= b.x;
      acc[0][nb][2] -= b.x;
      acc[0][nb][1] -= b.y;
      acc[0][nb][3] -= b.y;
    }
  } else {
#pragma unroll
    for (int j2 = 0; j2 < C::TW / 2; ++j2) {
      uint4 bf[C::kNB];
#pragma unroll
      for (int nb = 0; nb < C::kNB; ++nb) {
        bf[nb] = make_uint4(0, 0, 0, 0);
        if (!kTail || valid) bf[nb] = lds_v4(xseg + (nb ? xlane1 : xlane0) + j2 * kJStride);
      }
      uint32_t pa0[2], pb0[2], pa1[2], pb1[2];
      dequant_int8_word(wa[2 * j2], pa0);
      dequant_int8_word(wb[2 * j2], pb0);
      dequant_int8_word(wa[2 * j2 + 1], pa1);
      dequant_int8_word(wb[2 * j2 + 1], pb1);
      const int h0 = (C::kChains == 4) ? 2 * (j2 & 1) : 0;
#pragma unroll
      for (int nb = 0; nb < C::kNB; ++nb) {
        mma_16816(acc[h0][nb], pa0[0], pb0[0], pa0[1], pb0[1], bf[nb].x, bf[nb].y);
        mma_16816(acc[h0 + 1][nb], pa1[0], pb1[0], pa1[1], pb1[1], bf[nb].z, bf[nb].w);
      }
    }
  }
}

// Copies the activation slice X[:, pk0 : pk0 + plen] into shared memory in the order
// the B fragments are read (x_unit), INT4 slots permuted and high-nibble slots
// divided by 16 (see dequant_int4_word_biased). Units of tokens >= M and of k past
// plen are not written (no fragment of a real token reads them).
// With issued != 0 every thread adds 1 to that shared counter once its first batch of
// global loads has been issued (or at once when it has none).
template <class C>
__device__ __forceinline__ void stage_activations(const __half* __restrict__ X, int K, int M, int pk0, int plen,
                                                  uint8_t* xbuf, int ct, uint32_t issued = 0) {
  constexpr int kCT = kDecodeConsumerWarps * 32;
  constexpr int kBatch = 8;
  const int nseg = (plen + C::SEGK - 1) / C::SEGK;
  const int total = nseg * C::XU * C::kMP * 4;                  // 16-byte units of the slice
  if (issued != 0 && ct >= total) shared_count_add(issued);
  for (int d0 = ct; d0 < total; d0 += kCT * kBatch) {
    uint4 v[kBatch];
    bool live[kBatch];
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      const int d = d0 + b * kCT;
      const int cc = d & 3;
      const int n = (d >> 2) % C::kMP;
      const int rest = (d >> 2) / C::kMP;
      const int jj = rest % C::XU;
      const int sg = rest / C::XU;
      const int kr = sg * C::SEGK + cc * C::TK + jj * 8;        // part-relative k of the 8 values
      live[b] = d < total && n < M && kr < plen;
      v[b] = make_uint4(0, 0, 0, 0);
      if (live[b]) v[b] = __ldg(reinterpret_cast<const uint4*>(X + static_cast<long long>(n) * K + pk0 + kr));
    }
    if (issued != 0 && d0 == ct) shared_count_add(issued);
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      if (!live[b]) continue;
      uint4 o;
      if constexpr (C::kBits == 4) {
        // low-nibble slots (x0,x4), (x2,x6) as is; high-nibble slots (x1,x5), (x3,x7) divided by 16
        const __half2 kSixteenth = __halves2half2(__ushort_as_half(0x2C00), __ushort_as_half(0x2C00));
        o.x = prmt(v[b].x, v[b].z, 0x5410u);
        uint32_t hy = prmt(v[b].x, v[b].z, 0x7632u);
        o.z = prmt(v[b].y, v[b].w, 0x5410u);
        uint32_t hw = prmt(v[b].y, v[b].w, 0x7632u);
        __half2 sy = __hmul2(*reinterpret_cast<__half2*>(&hy), kSixteenth);
        __half2 sw = __hmul2(*reinterpret_cast<__half2*>(&hw), kSixteenth);
        o.y = *reinterpret_cast<uint32_t*>(&sy);
        o.w = *reinterpret_cast<uint32_t*>(&sw);
      } else {
        o = v[b];
      }
      *reinterpret_cast<uint4*>(xbuf + 16u * static_cast<uint32_t>(d0 + b * kCT)) = o;
    }
  }
}

// ---------------------------------------------------------------- the kernel
template <class C>
__global__ void __launch_bounds__(kDecodeThreads, 1)
    decode_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_next,
                  const DecodeArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* wring = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kDecodeStages * kDecodeStageBytes);
  uint64_t* empty = full + kDecodeStages;
  uint32_t* x_issued = reinterpret_cast<uint32_t*>(empty + kDecodeStages);   // inside the fixed 256 bytes
  uint8_t* xbuf = smem + kDecodeFixedSmem;
  // INT4 only: per (segment, token) bias of the biased dequantization, after the activation slice;
  // zero-point codes: then per-token sums of x over the part
  float* bias_s = reinterpret_cast<float*>(xbuf + 2 * C::kMP * a.KPP);
  float* sx_s = bias_s + (a.KPP / C::SEGK) * 16;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int M = a.M, N = a.N, K = a.K;
  const int G = gridDim.x;
  const int u_begin = static_cast<int>((static_cast<long long>(blockIdx.x) * a.units) / G);
  const int u_end = static_cast<int>((static_cast<long long>(blockIdx.x + 1) * a.units) / G);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kDecodeStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kDecodeConsumerWarps);
    }
    *x_issued = 0;
    fence_barrier_init();
  }
  __syncthreads();
  // everything above touches only shared memory; X, W, Y and the scratch may belong
  // to the previous kernel in the stream
  griddep_wait();
  if (threadIdx.x == 0) griddep_launch_dependents();

  if (warp == kDecodeConsumerWarps) {
    // ------------------------------------------------------------ producer warp
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      uint32_t armed[kDecodeStages] = {};
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      // The consumers stage the first part's activations as soon as they start. Let
      // their loads enter the memory system before the weight stream fills the ring
      // (behind ~200 KB per SM of TMA traffic they would arrive microseconds later).
      // Only an ordering hint: the wait is bounded and the stream starts either way.
      const uint32_t issued_u32 = smem_u32(x_issued);
      for (int i = 0; i < 4096 && shared_count_read(issued_u32) < static_cast<uint32_t>(kDecodeConsumerWarps * 32);
           ++i)
        __nanosleep(32);
      int pref_part = u_begin < u_end ? u_begin / a.tiles : -1;
      for (int u = u_begin; u < u_end && ok; ++u) {
        const int p = u / a.tiles;
        const int t = u - p * a.tiles;
        const int pk0 = p * a.KPP;
        const int plen = min(a.KPP, K - pk0);
        const int nst = (plen + C::SK - 1) / C::SK;
        if (p != pref_part) {
          // a later part: bring its activation slice into L2 while the ring still holds
          // the previous part's stages (rows of X are 128-byte aligned: K % 64 == 0)
          for (int n = 0; n < M; ++n)
            bulk_prefetch_l2(a.X + static_cast<long long>(n) * K + pk0, static_cast<uint32_t>(plen) * 2u);
          pref_part = p;
        }
        for (int ks = 0; ks < nst; ++ks) {
          if (!mbar_wait(&empty[stage], phase ^ 1)) { ok = false; break; }
          const int xb0 = (pk0 + ks * C::SK) / C::KPB;            // first packed byte of the stage
          mbar_arrive_expect_tx(&full[stage], static_cast<uint32_t>(kDecodeStageBytes));
          armed[stage] = phase + 1;
          tma_load_2d_hint(wring + stage * kDecodeStageBytes, &tmap_w, xb0, t * kDecodeRows, &full[stage], pol);
          if (++stage == kDecodeStages) { stage = 0; phase ^= 1; }
        }
      }
      if (ok && a.nxt_grid > 0) {
        // Every load of this CTA is issued; its consumers still work through up to a
        // full ring. Meanwhile bring the next call's first ring fill into L2: next CTA b
        // (b = this CTA, this CTA + G, ...) starts with the first kDecodeStages stages
        // of its units. The next call's weights do not depend on this call's output.
        for (int b = blockIdx.x; b < a.nxt_grid; b += G) {
          const int ub = static_cast<int>((static_cast<long long>(b) * a.nxt_units) / a.nxt_grid);
          const int ue = static_cast<int>((static_cast<long long>(b + 1) * a.nxt_units) / a.nxt_grid);
          int left = kDecodeStages;
          for (int u = ub; u < ue && left > 0; ++u) {
            const int p = u / a.nxt_tiles;
            const int t = u - p * a.nxt_tiles;
            const int pk0 = p * a.nxt_KPP;
            const int plen = min(a.nxt_KPP, a.nxt_K - pk0);
            const int nst = (plen + C::SK - 1) / C::SK;
            for (int ks = 0; ks < nst && left > 0; ++ks, --left)
              tma_prefetch_2d(&tmap_next, (pk0 + ks * C::SK) / C::KPB, t * kDecodeRows);
          }
        }
      }
      // never leave while TMA writes into this CTA's shared memory may be in flight
      bool drained = true;
      for (int s = 0; s < kDecodeStages; ++s)
        if (armed[s] && !mbar_wait(&full[s], armed[s] - 1)) drained = false;
      if (!ok || !drained) report_error(kErrDecodeProducerWait);
    }
    return;
  }

  // -------------------------------------------------------------- consumer warps
  const int r = lane >> 2;
  const int c = lane & 3;
  const int ct = threadIdx.x;                // 0 .. 511
  constexpr int kCT = kDecodeConsumerWarps * 32;
  const uint32_t wring_u32 = smem_u32(wring);
  const uint32_t xbuf_u32 = smem_u32(xbuf);
  const int ra = 16 * warp + r;              // this lane's rows: ra and ra + 8 (same ra & 7)
  // per-lane byte offsets: packed row ra, 16-byte units 2c and 2c+1 under the 128-byte swizzle
  const uint32_t wlane = static_cast<uint32_t>(ra * kDecodeSegB + (((2 * c) ^ (ra & 7)) << 4)) |
                         (static_cast<uint32_t>(ra * kDecodeSegB + (((2 * c + 1) ^ (ra & 7)) << 4)) << 16);
  // activation units of this lane's tokens (clamped to a real token; results past M are discarded)
  const uint32_t xlane0 = 16u * x_unit<C>(0, 0, min(r, M - 1), c);
  const uint32_t xlane1 = 16u * x_unit<C>(0, 0, min(r + 8, M - 1), c);
  const bool split = a.parts > 1;
  int stage = 0;
  uint32_t phase = 0;
  int cur_part = -1;
  bool ok = true;

  for (int u = u_begin; u < u_end; ++u) {
    const int p = u / a.tiles;
    const int t = u - p * a.tiles;
    const int pk0 = p * a.KPP;
    const int plen = min(a.KPP, K - pk0);
    if (p != cur_part) {
      // stage this part's activations in fragment order (all consumers, then barrier).
      // Thread i fills shared 16-byte unit i (conflict-free stores); each thread first
      // issues all its global loads of a batch through the read-only path, then stores.
      named_barrier_sync(1, kCT);
      stage_activations<C>(a.X, K, M, pk0, plen, xbuf, ct, cur_part < 0 ? smem_u32(x_issued) : 0u);
      if constexpr (C::kBits == 4) {
        // per (segment, token) bias sum_k (1032 or 1152) * B[k], one warp per real pair
        // (lane = 8-value chunk of the 256-k segment), read back from the staged slice
        static_assert(C::SEGK == 256, "one lane per 8-value chunk of a segment");
        named_barrier_sync(1, kCT);
        const int nseg = a.KPP / C::SEGK;
        const int pseg = (plen + C::SEGK - 1) / C::SEGK;
        for (int i = ct; i < nseg * 16; i += kCT) {                // entries the pair loop never writes
          if ((i & 15) >= M || (i >> 4) >= pseg) bias_s[i] = 0.0f;
        }
        for (int pair = warp; pair < pseg * M; pair += kDecodeConsumerWarps) {
          const int sg = pair / M;
          const int n = pair - sg * M;
          float bias = 0.0f;
          if (sg * C::SEGK + lane * 8 < plen) {
            const uint4 o = *reinterpret_cast<const uint4*>(xbuf + 16u * x_unit<C>(sg, lane & 7, n, lane >> 3));
            const float2 fx = __half22float2(*reinterpret_cast<const __half2*>(&o.x));
            const float2 fy = __half22float2(*reinterpret_cast<const __half2*>(&o.y));
            const float2 fz = __half22float2(*reinterpret_cast<const __half2*>(&o.z));
            const float2 fw = __half22float2(*reinterpret_cast<const __half2*>(&o.w));
            bias = C::kLowBias * ((fx.x + fx.y) + (fz.x + fz.y)) + C::kHighBias * ((fy.x + fy.y) + (fw.x + fw.y));
          }
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) bias += __shfl_xor_sync(0xffffffffu, bias, off);
          if (lane == 0) bias_s[sg * 16 + n] = bias;
        }
        if constexpr (C::kZP) {
          // per-token sum of x over the part, for the zero-point term z[n] * sum_k x[m,k]
          // (high-nibble slots hold x / 16)
          const int units = pseg * C::XU * 4;
          for (int n = warp; n < M; n += kDecodeConsumerWarps) {
            float sx = 0.0f;
            for (int i = lane; i < units; i += 32) {
              const int sg = i / (C::XU * 4);
              const int rem = i - sg * (C::XU * 4);
              const int jj = rem >> 2, cc = rem & 3;
              if (sg * C::SEGK + cc * C::TK + jj * 8 < plen) {
                const uint4 o = *reinterpret_cast<const uint4*>(xbuf + 16u * x_unit<C>(sg, jj, n, cc));
                const float2 fx = __half22float2(*reinterpret_cast<const __half2*>(&o.x));
                const float2 fy = __half22float2(*reinterpret_cast<const __half2*>(&o.y));
                const float2 fz = __half22float2(*reinterpret_cast<const __half2*>(&o.z));
                const float2 fw = __half22float2(*reinterpret_cast<const __half2*>(&o.w));
                sx += ((fx.x + fx.y) + (fz.x + fz.y)) + 16.0f * ((fy.x + fy.y) + (fw.x + fw.y));
              }
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) sx += __shfl_xor_sync(0xffffffffu, sx, off);
            if (lane == 0) sx_s[n] = sx;
          }
        }
      }
      cur_part = p;
      named_barrier_sync(1, kCT);
    }

    float acc[C::kChains][C::kNB][4];
#pragma unroll
    for (int h = 0; h < C::kChains; ++h)
#pragma unroll
      for (int nb = 0; nb < C::kNB; ++nb)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[h][nb][i] = 0.0f;

    const int nst = (plen + C::SK - 1) / C::SK;
    for (int ks = 0; ks < nst; ++ks) {
      if (ok && !mbar_wait_warp(&full[stage], phase)) ok = false;
      if (ok) {
        const uint32_t box = wring_u32 + stage * kDecodeStageBytes;
        const uint32_t xseg = xbuf_u32 + 16u * x_unit<C>(ks, 0, 0, 0);
        const float* bias_seg = bias_s + ks * 16;
        const int kseg = pk0 + ks * C::SK;                        // absolute k of this stage
        if (kseg + C::SK <= K) {
          decode_segment<C, false>(box, xseg, wlane, xlane0, xlane1, true, bias_seg, c, acc);
        } else {
          const bool valid = kseg + c * C::TK < K;
          decode_segment<C, true>(box, xseg, wlane, xlane0, xlane1, valid, bias_seg, c, acc);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[stage]);
      if (++stage == kDecodeStages) { stage = 0; phase ^= 1; }
    }

    // ---- unit epilogue, per warp: rows ra and ra + 8, tokens 8 nb + 2 c (+1)
    const int row_a = t * kDecodeRows + ra;
    const int row_b = row_a + 8;
    const bool live_a = row_a < N, live_b = row_b < N;
    const float sa = (!split && live_a) ? __half2float(a.scale[row_a]) : 0.0f;
    const float sb = (!split && live_b) ? __half2float(a.scale[row_b]) : 0.0f;
    const float ba = (!split && live_a) ? epilogue_bias(a.bias, a.geglu, row_a, N) : 0.0f;
    float za = 0.0f, zb = 0.0f;
    if constexpr (C::kZP) {
      za = live_a ? static_cast<float>(a.zero[row_a]) : 0.0f;
      zb = live_b ? static_cast<float>(a.zero[row_b]) : 0.0f;
    }
    const float bb = (!split && live_b) ? epilogue_bias(a.bias, a.geglu, row_b, N) : 0.0f;
#pragma unroll
    for (int nb = 0; nb < C::kNB; ++nb) {
#pragma unroll
      for (int h = 1; h < C::kChains; ++h)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[0][nb][i] += acc[h][nb][i];
      if constexpr (C::kZP) {
        // the MMAs saw the unsigned codes: remove z[row] * sum_k x[m,k] (this part's k)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int m = 8 * nb + 2 * c + (i & 1);
          if (m < M) acc[0][nb][i] -= ((i < 2) ? za : zb) * sx_s[m];
        }
      }
      if (!split && a.geglu) {
        // rows row_a (first GeGLU half) and row_b (second half) of the same output column
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int m = 8 * nb + 2 * c + i;
          if (m < M && live_a) {
            const float ua = sa * acc[0][nb][i] + ba, ub = sb * acc[0][nb][i + 2] + bb;
            a.Y[static_cast<long long>(m) * (N >> 1) + geglu_column(row_a)] = __float2half_rn(gelu_exact(ua) * ub);
          }
        }
        continue;
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int m = 8 * nb + 2 * c + (i & 1);
        const int row = (i < 2) ? row_a : row_b;
        if (m < M && row < N) {
          const long long idx = static_cast<long long>(m) * N + row;
          if (split) atomicAdd(a.ws + idx, acc[0][nb][i]);   // result unused: a reduction
          else a.Y[idx] = __float2half_rn(((i < 2) ? sa : sb) * acc[0][nb][i] + ((i < 2) ? ba : bb));
        }
      }
    }
  }
  if (!ok && lane == 0) report_error(kErrDecodeConsumerWait);
}

}  // namespace glmq
