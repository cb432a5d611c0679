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
//    balanced to within one unit. K parts exist only to spread the units evenly
//    over the SMs (tiles split over parts cost a round trip of fp32 partial sums).
//  * A stage is one 256-k segment of one tile: 256 weight rows x 128 packed bytes
//    (32 KB), the matching activations of the MP token rows (in the order the
//    MMA fragments read them) and a per-token bias for the biased dequantization.
//    The ring has kStages stages (5 or 6, whatever fits in shared memory).
//  * Warp 16 is the producer: one lane issues, per stage, two 2-D TMA tile loads:
//    the stage's activations X[0 : MP, k0 : k0 + SK] (rows past M and values past K
//    are zero-filled by the TMA unit) into the stage's activation slot, and the weight
//    box (128-byte swizzle, L2 evict-first hint; rows past N and bytes past K
//    zero-filled).
//  * Warps 17.. are activation warps (one for M <= 2, three for larger M; warp 17 + i
//    takes the stages with sequence number i mod their count, each only after the
//    previous phase of its ring stage has been handed on). Once a slot's raw
//    activations have landed the warp
//    rewrites them in place into fragment order, dividing the high-nibble slots by 16
//    (see below), with a lane-to-unit mapping under which both the reads and the
//    writes of shared memory are free of bank conflicts; the per-token bias of the
//    stage is then one short MMA chain on the slot's fragments (for M <= 2, where most
//    of that chain's columns would be padding, a warp reduction of the lanes' sums).
//  * Warps 0..15 are consumers: warp w owns rows 16w .. 16w+15 of the tile and
//    reads the whole stage's K segment for them. Codes are dequantized in
//    registers with exponent-bias tricks (a code c becomes the fp16 number
//    1024 + (c ^ 8) by OR-ing it into the mantissa) and feed mma.sync m16n8k16
//    as the A operand straight from registers, X being the B operand. The K order
//    inside each MMA is permuted identically on both operands so that each 32-bit
//    packed word feeds two MMAs without a byte shuffle; the activation producers
//    apply the permutation to X.
//  * A warp's sums stay in registers for the whole unit, so a unit ends without
//    any cross-warp reduction or barrier: the warp scales, rounds and stores its
//    own 16 rows. When a tile is split over several K parts each warp instead adds
//    its partial sums into an fp32 scratch buffer with fire-and-forget
//    red.global.add, and a small stream-ordered finalize kernel
//    (decode_finalize_kernel) scales, rounds and stores Y and returns the scratch
//    to zero for the next call.
//  * Every wait is bounded. A warp whose wait gives up reports it and stops: it
//    neither consumes nor releases further stages, so a stage is never refilled
//    while a copy into it may still be in flight, and the weight producer still
//    waits for each of its own copies to land before its CTA exits.
#pragma once

#include <cuda.h>

#include "epilogue.cuh"
#include "glmq_ptx.cuh"

namespace glmq {

#ifndef DECODE_WAIT_P
#define DECODE_WAIT_P mbar_wait
#endif
#ifndef DECODE_WAIT_X
#define DECODE_WAIT_X mbar_wait_warp
#endif
#ifndef DECODE_WAIT_C
#define DECODE_WAIT_C mbar_wait_warp
#endif

constexpr int kDecodeConsumerWarps = 16;
constexpr int kDecodeProducerWarp = 16;                               // weight TMA
constexpr int kDecodeXWarp0 = 17;                                     // activation warps 17..
constexpr int kDecodeRows = 16 * kDecodeConsumerWarps;                // rows per tile (256)
constexpr int kDecodeSegB = 128;         // packed bytes per row per stage (one TMA box width)
constexpr int kDecodeStageBytes = kDecodeRows * kDecodeSegB;          // 32 KB: one TMA box per stage
constexpr int kDecodeSmemLimit = 232448;  // opt-in shared memory per block on sm_100
constexpr int kDecodeMaxStages = 6;

template <int BITS, int MP, int CHAINS = 2, int ZP = 0>
struct DecodeCfg {
  static_assert(CHAINS == 2 || CHAINS == 4, "accumulator chains");
  static_assert(ZP == 0 || BITS == 4, "zero-point codes are INT4");
  static_assert(MP == 1 || MP == 2 || MP == 4 || MP == 8 || MP == 16, "token capacity");
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
  static constexpr int SK = kDecodeSegB * KPB;      // k per stage
  static constexpr int TB = kDecodeSegB / 4;        // packed bytes per thread per row per stage (32)
  static constexpr int TK = TB * KPB;               // k per thread per stage
  static constexpr int TW = TB / 4;                 // 32-bit words per thread per row per stage (8)
  static constexpr int XU = TK / 8;                 // 16-byte activation units per thread per stage
  static constexpr int kChains = CHAINS;            // independent MMA accumulator chains per token block
  // activation warps: one keeps up with the small slots of M <= 2; three for M >= 4 (at
  // most 20 warps in all, so ptxas still allows 96 registers per thread)
  static constexpr int kXWarps = MP >= 4 ? 3 : 1;
  // M <= 4: the activation warp also waits for the stage's weight box before releasing
  // the stage, so the consumers wait on one barrier per stage instead of two (measured
  // about 5 us faster per four-call M=1 or M=4 group; slower at M=16, where three
  // activation warps take turns and the consumers keep both waits)
  static constexpr bool kGateW = MP <= 4;
  static constexpr int kThreads = (kDecodeConsumerWarps + 1 + kXWarps) * 32;
  static constexpr int X_UNITS = XU * MP * 4;       // 16-byte units in a stage's activation slot
  static constexpr int X_BYTES = X_UNITS * 16;
  // per stage and token: the bias of the biased dequantization (INT4), then (zero point)
  // the sum of x over the stage
  static constexpr int B_FLOATS = ZP ? 32 : 16;
  static constexpr int STAGE_TOTAL = kDecodeStageBytes + X_BYTES + B_FLOATS * 4 + 4 * 8;
  static constexpr int kStages = (kDecodeSmemLimit - 1024) / STAGE_TOTAL < kDecodeMaxStages
                                     ? (kDecodeSmemLimit - 1024) / STAGE_TOTAL : kDecodeMaxStages;
  static constexpr int SMEM_BYTES = kStages * STAGE_TOTAL + 1024;   // + alignment slack
  static_assert(kStages >= 4, "pipeline depth");
  static_assert(SMEM_BYTES <= kDecodeSmemLimit, "shared memory");
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
  int nxt_stages;     // ring depth of the next call's kernel configuration
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

// Index (in 16-byte units) of activation unit (jj, n, c) in a stage's activation slot:
// the 8 values of token n that lane c multiplies with its codes jj*8 .. jj*8+7 (k =
// c*TK + jj*8 .. +7 of the stage). Consecutive lanes of a token read consecutive
// units; the token stride is the compile-time capacity MP, so within a stage every
// fragment address is a per-lane base plus an immediate.
template <class C>
__host__ __device__ constexpr uint32_t x_unit(int jj, int n, int c) {
  return static_cast<uint32_t>((jj * C::kMP + n) * 4 + c);
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


// Rewrites one stage's activation slot in place, called by all 32 lanes of an
// activation warp once the slot's raw activations have landed. Raw layout (the TMA
// box): token n's SK values at n * SK * 2 bytes, i.e. 16-byte unit (n, kr / 8) for the
// 8 values from k0 + kr. Fragment layout: unit x_unit(jj, n, c) holds the 8 values lane
// c multiplies with its codes jj*8 .. jj*8+7, i.e. kr = c * TK + jj * 8; INT4 values are
// permuted to the MMA k order (0,4),(1,5),(2,6),(3,7) with the high-nibble slots (1,5)
// and (3,7) divided by 16 (exact: a power of two); INT8 values keep their order.
// Every lane first reads all its units, the warp synchronizes, then every lane writes
// them back, so the permutation can be done in place. Lane (p, l) = (L / 8, L % 8)
// handles, for its i-th unit, jj = l (INT4) and a rotation of the remaining indices by
// (i, p), chosen so that within each 8-lane phase of a 16-byte access the raw units
// read fall in 8 distinct bank groups (distinct raw unit index mod 8) and so do the
// fragment units written (distinct (4n + c) mod 8).
// Unit (jj, n, c) of lane `lane`'s i-th unit in transform_activation_stage.
template <class C>
__device__ __forceinline__ void transform_unit(int i, int lane, int& jj, int& n, int& c) {
  constexpr int MP = C::kMP;
  const int p = lane >> 3, l = lane & 7;
  if constexpr (C::kBits == 4) {
    if constexpr (MP == 1) {
      jj = lane & 7; n = 0; c = lane >> 3;
    } else {
      const int z = i * 4 + p, q = (l + (z & 7)) & 7;
      jj = l; n = 2 * (z >> 3) + (q >> 2); c = q & 3;
    }
  } else {
    if constexpr (MP == 1) {
      jj = lane & 3; n = 0; c = (lane >> 2) & 3;
    } else {
      const int z = i * 4 + p, w = ((l & 3) + (z & 3)) & 3;
      jj = l & 3; n = 2 * (z >> 2) + (w >> 1); c = 2 * (w & 1) + (l >> 2);
    }
  }
}

template <class C>
__device__ __forceinline__ void transform_activation_stage(uint32_t slot, int lane, float (&bsum)[2],
                                                           float (&ssum)[2]) {
  constexpr int MP = C::kMP;
  constexpr int RAW_UNITS = C::SK / 8;                    // 16-byte units per token row
  constexpr int PER = (C::kBits == 4) ? MP : (MP == 1 ? 1 : MP / 2);
  const bool live = !(C::kBits == 8 && MP == 1) || lane < 16;
  uint4 v[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    int jj, n, c;
    transform_unit<C>(i, lane, jj, n, c);
    if (live) v[i] = lds_v4(slot + 16u * static_cast<uint32_t>(n * RAW_UNITS + (c * C::TK + jj * 8) / 8));
  }
  __syncwarp();
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    int jj, n, c;
    transform_unit<C>(i, lane, jj, n, c);
    uint4 o = v[i];
    if constexpr (C::kBits == 4) {
      const __half2 kSixteenth = __halves2half2(__ushort_as_half(0x2C00), __ushort_as_half(0x2C00));
      o.x = prmt(v[i].x, v[i].z, 0x5410u);
      uint32_t hy = prmt(v[i].x, v[i].z, 0x7632u);
      o.z = prmt(v[i].y, v[i].w, 0x5410u);
      uint32_t hw = prmt(v[i].y, v[i].w, 0x7632u);
      __half2 sy = __hmul2(*reinterpret_cast<__half2*>(&hy), kSixteenth);
      __half2 sw = __hmul2(*reinterpret_cast<__half2*>(&hw), kSixteenth);
      o.y = *reinterpret_cast<uint32_t*>(&sy);
      o.w = *reinterpret_cast<uint32_t*>(&sw);
    }
    if (live) sts_v4(slot + 16u * x_unit<C>(jj, n, c), o);
    if constexpr (C::kBits == 4 && MP <= 2) {
      // this unit's share of the token's bias (and sum of x): see stage_sums_mma
      const float2 fx = __half22float2(*reinterpret_cast<const __half2*>(&o.x));
      const float2 fy = __half22float2(*reinterpret_cast<const __half2*>(&o.y));
      const float2 fz = __half22float2(*reinterpret_cast<const __half2*>(&o.z));
      const float2 fw = __half22float2(*reinterpret_cast<const __half2*>(&o.w));
      const float lo = (fx.x + fx.y) + (fz.x + fz.y), hi = (fy.x + fy.y) + (fw.x + fw.y);
      const float b = C::kLowBias * lo + C::kHighBias * hi, sx = lo + 16.0f * hi;
      bsum[0] += n == 0 ? b : 0.0f;
      bsum[1] += n == 1 ? b : 0.0f;
      ssum[0] += n == 0 ? sx : 0.0f;
      ssum[1] += n == 1 ? sx : 0.0f;
    }
  }
}

// INT4: the per-token sums a stage's activation slot needs, written into its bias slot:
// bias[t] = sum_k (kLowBias or kHighBias) * B[k][t] over the stage (what the biased
// dequantization adds to every output of token t), and, for zero-point codes,
// sx[t] = sum_k x[t,k] (B holds x in low-nibble slots, x / 16 in high ones). They are
// computed on the tensor cores with the same fragments the consumers read: a constant
// A operand whose rows 0..7 hold the bias coefficients of each slot and rows 8..15
// the sum-of-x coefficients (1 low, 16 high), times the slot's B fragments. Row 0 of
// the product holds bias[t] and row 8 sx[t] for the 8 tokens of each n8 block. Called
// by all 32 lanes of the warp after the slot is written and the warp synchronized.
template <class C>
__device__ __forceinline__ void stage_sums_mma(uint32_t xslot_u32, float* bslot, int M, int lane) {
  constexpr uint32_t kJStride = static_cast<uint32_t>(C::kMP) * 64u;
  const __half2 lo = __float2half2_rn(C::kLowBias), hi = __float2half2_rn(C::kHighBias);
  const __half2 one = __float2half2_rn(1.0f), sixteen = __float2half2_rn(16.0f);
  const uint32_t a0 = *reinterpret_cast<const uint32_t*>(&lo), a2 = *reinterpret_cast<const uint32_t*>(&hi);
  const uint32_t a1 = *reinterpret_cast<const uint32_t*>(&one), a3 = *reinterpret_cast<const uint32_t*>(&sixteen);
  const int r = lane >> 2, c = lane & 3;
  // four independent accumulator chains per n8 block keep the chain latency short
  float d[C::kNB][4][4];
#pragma unroll
  for (int nb = 0; nb < C::kNB; ++nb)
#pragma unroll
    for (int h = 0; h < 4; ++h)
#pragma unroll
      for (int i = 0; i < 4; ++i) d[nb][h][i] = 0.0f;
#pragma unroll
  for (int j = 0; j < C::XU; ++j) {
#pragma unroll
    for (int nb = 0; nb < C::kNB; ++nb) {
      const uint4 bf = lds_v4(xslot_u32 + 16u * x_unit<C>(0, min(8 * nb + r, M - 1), c) + j * kJStride);
      mma_16816(d[nb][2 * (j & 1)], a0, a1, a2, a3, bf.x, bf.y);
      mma_16816(d[nb][2 * (j & 1) + 1], a0, a1, a2, a3, bf.z, bf.w);
    }
  }
#pragma unroll
  for (int nb = 0; nb < C::kNB; ++nb) {
    float dd[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) dd[i] = (d[nb][0][i] + d[nb][1][i]) + (d[nb][2][i] + d[nb][3][i]);
    const int t = 8 * nb + 2 * c;
    if (r == 0 && t < M) {
      bslot[t] = dd[0];
      if constexpr (C::kZP) bslot[16 + t] = dd[2];
    }
    if (r == 0 && t + 1 < M) {
      bslot[t + 1] = dd[1];
      if constexpr (C::kZP) bslot[16 + t + 1] = dd[3];
    }
  }
}

// ---------------------------------------------------------------- the kernel
template <class C>
__global__ void __launch_bounds__(C::kThreads, 1)
    decode_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x,
                  const __grid_constant__ CUtensorMap tmap_next, const DecodeArgs a) {
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* wring = smem;                                           // S x 32 KB weight boxes
  uint8_t* xring = smem + S * kDecodeStageBytes;                   // S activation slots
  float* bring = reinterpret_cast<float*>(xring + S * C::X_BYTES); // S bias slots
  uint64_t* fullw = reinterpret_cast<uint64_t*>(bring + S * C::B_FLOATS);   // weight box landed (1 + tx)
  uint64_t* fullr = fullw + S;                                     // raw activations landed (1 + tx)
  uint64_t* fullx = fullr + S;                                     // activation slot rewritten (1)
  uint64_t* empty = fullx + S;                                     // stage released (16 consumer warps)

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int M = a.M, N = a.N, K = a.K;
  const int G = gridDim.x;
  const int u_begin = static_cast<int>((static_cast<long long>(blockIdx.x) * a.units) / G);
  const int u_end = static_cast<int>((static_cast<long long>(blockIdx.x + 1) * a.units) / G);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&fullw[s], 1);
      mbar_init(&fullr[s], 1);
      mbar_init(&fullx[s], 1);
      mbar_init(&empty[s], kDecodeConsumerWarps);
    }
    fence_barrier_init();
  }
  // bias slots of tokens no activation producer writes (M <= token < 16) read as zero
  for (int i = threadIdx.x; i < S * C::B_FLOATS; i += C::kThreads) bring[i] = 0.0f;
  __syncthreads();
  // everything above touches only shared memory; X, W, Y and the scratch may belong
  // to the previous kernel in the stream
  griddep_wait();
  if (threadIdx.x == 0) griddep_launch_dependents();

  if (warp == kDecodeProducerWarp) {
    // ------------------------------------------------------------ weight producer
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      uint32_t armed[S] = {};
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int u = u_begin; u < u_end && ok; ++u) {
        const int p = u / a.tiles;
        const int t = u - p * a.tiles;
        const int pk0 = p * a.KPP;
        const int plen = min(a.KPP, K - pk0);
        const int nst = (plen + C::SK - 1) / C::SK;
        for (int ks = 0; ks < nst; ++ks) {
          if (!DECODE_WAIT_P(&empty[stage], phase ^ 1)) { ok = false; break; }
          const int k0 = pk0 + ks * C::SK;
          mbar_arrive_expect_tx(&fullr[stage], static_cast<uint32_t>(C::X_BYTES));
          tma_load_2d(xring + stage * C::X_BYTES, &tmap_x, k0, 0, &fullr[stage]);
          mbar_arrive_expect_tx(&fullw[stage], static_cast<uint32_t>(kDecodeStageBytes));
          armed[stage] = phase + 1;
          tma_load_2d_hint(wring + stage * kDecodeStageBytes, &tmap_w, k0 / C::KPB, t * kDecodeRows, &fullw[stage],
                           pol);
          if (++stage == S) { stage = 0; phase ^= 1; }
        }
      }
      if (ok && a.nxt_grid > 0) {
        // Every load of this CTA is issued; its consumers still work through up to a
        // full ring. Meanwhile bring the next call's first ring fill into L2: next CTA b
        // (b = this CTA, this CTA + G, ...) starts with the first nxt_stages stages
        // of its units. The next call's weights do not depend on this call's output.
        for (int b = blockIdx.x; b < a.nxt_grid; b += G) {
          const int ub = static_cast<int>((static_cast<long long>(b) * a.nxt_units) / a.nxt_grid);
          const int ue = static_cast<int>((static_cast<long long>(b + 1) * a.nxt_units) / a.nxt_grid);
          int left = a.nxt_stages;
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
      for (int s = 0; s < S; ++s)
        if (armed[s] && (!mbar_wait_drain(&fullw[s], armed[s] - 1) || !mbar_wait_drain(&fullr[s], armed[s] - 1)))
          drained = false;
      if (!ok || !drained) report_error(kErrDecodeProducerWait);
    }
    return;
  }

  if (warp >= kDecodeXWarp0) {
    // ------------------------------------------------------------ activation producers
    const int xw = warp - kDecodeXWarp0;
    int q = 0;                    // stage sequence number of this CTA
    bool ok = true;
    for (int u = u_begin; u < u_end && ok; ++u) {
      const int p = u / a.tiles;
      const int pk0 = p * a.KPP;
      const int plen = min(a.KPP, K - pk0);
      const int nst = (plen + C::SK - 1) / C::SK;
      for (int ks = 0; ks < nst; ++ks, ++q) {
        if (C::kXWarps > 1 && q % C::kXWarps != xw) continue;
        const int stage = q % S;
        const uint32_t phase = static_cast<uint32_t>(q / S) & 1u;
        if (C::kXWarps > 1 && S % C::kXWarps != 0 && q >= S) {
          // Successive phases of this stage fall to different warps (3 warps, 5 stages
          // at MP = 16). A parity wait on phase n + 1 passes at once while phase n is
          // still incomplete, so first wait until the stage's previous phase has been
          // released to the consumers: fullr is then at the phase waited on below.
          if (!DECODE_WAIT_X(&fullx[stage], phase ^ 1u)) { ok = false; break; }
        }
        if (!DECODE_WAIT_X(&fullr[stage], phase)) { ok = false; break; }
        const uint32_t slot = smem_u32(xring + stage * C::X_BYTES);
        float bsum[2] = {0.0f, 0.0f}, ssum[2] = {0.0f, 0.0f};
        transform_activation_stage<C>(slot, lane, bsum, ssum);
        __syncwarp();
        if constexpr (C::kBits == 4 && C::kMP <= 2) {
          float* bs = bring + stage * C::B_FLOATS;
#pragma unroll
          for (int t = 0; t < C::kMP; ++t) {
            float b = bsum[t], sx = ssum[t];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
              b += __shfl_xor_sync(0xffffffffu, b, off);
              if constexpr (C::kZP) sx += __shfl_xor_sync(0xffffffffu, sx, off);
            }
            if (lane == 0) {
              bs[t] = b;
              if constexpr (C::kZP) bs[16 + t] = sx;
            }
          }
          __syncwarp();
        } else if constexpr (C::kBits == 4) {
          stage_sums_mma<C>(slot, bring + stage * C::B_FLOATS, M, lane);
          __syncwarp();
        }
        if constexpr (C::kGateW) {
          // this warp also gates the weight box: once it has landed, order the TMA's
          // writes before the generic loads of the consumers that acquire fullx
          if (!DECODE_WAIT_X(&fullw[stage], phase)) { ok = false; break; }
          fence_proxy_async_smem();
        }
        if (lane == 0) mbar_arrive(&fullx[stage]);
      }
    }
    if (!ok && lane == 0) report_error(kErrDecodeProducerWait);
    return;
  }

  // -------------------------------------------------------------- consumer warps
  const int r = lane >> 2;
  const int c = lane & 3;
  const uint32_t wring_u32 = smem_u32(wring);
  const uint32_t xring_u32 = smem_u32(xring);
  const int ra = 16 * warp + r;              // this lane's rows: ra and ra + 8 (same ra & 7)
  // per-lane byte offsets: packed row ra, 16-byte units 2c and 2c+1 under the 128-byte swizzle
  const uint32_t wlane = static_cast<uint32_t>(ra * kDecodeSegB + (((2 * c) ^ (ra & 7)) << 4)) |
                         (static_cast<uint32_t>(ra * kDecodeSegB + (((2 * c + 1) ^ (ra & 7)) << 4)) << 16);
  // activation units of this lane's tokens (clamped to a real token; results past M are discarded)
  const uint32_t xlane0 = 16u * x_unit<C>(0, min(r, M - 1), c);
  const uint32_t xlane1 = 16u * x_unit<C>(0, min(r + 8, M - 1), c);
  const bool split = a.parts > 1;
  int stage = 0;
  uint32_t phase = 0;
  bool ok = true;

  for (int u = u_begin; u < u_end && ok; ++u) {
    const int p = u / a.tiles;
    const int t = u - p * a.tiles;
    const int pk0 = p * a.KPP;
    const int plen = min(a.KPP, K - pk0);

    float acc[C::kChains][C::kNB][4];
#pragma unroll
    for (int h = 0; h < C::kChains; ++h)
#pragma unroll
      for (int nb = 0; nb < C::kNB; ++nb)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[h][nb][i] = 0.0f;
    float sxa[C::kNB][2] = {};   // zero point: sum of x over the unit for tokens 8 nb + 2 c (+1)

    const int nst = (plen + C::SK - 1) / C::SK;
    for (int ks = 0; ks < nst; ++ks) {
      if (!DECODE_WAIT_C(&fullx[stage], phase) || (!C::kGateW && !DECODE_WAIT_C(&fullw[stage], phase))) {
        ok = false;
        break;
      }
      const uint32_t box = wring_u32 + stage * kDecodeStageBytes;
      const uint32_t xseg = xring_u32 + stage * C::X_BYTES;
      const float* bias_seg = bring + stage * C::B_FLOATS;
      const int kseg = pk0 + ks * C::SK;                        // absolute k of this stage
      if (kseg + C::SK <= K) {
        decode_segment<C, false>(box, xseg, wlane, xlane0, xlane1, true, bias_seg, c, acc);
      } else {
        const bool valid = kseg + c * C::TK < K;
        decode_segment<C, true>(box, xseg, wlane, xlane0, xlane1, valid, bias_seg, c, acc);
      }
      if constexpr (C::kZP) {
#pragma unroll
        for (int nb = 0; nb < C::kNB; ++nb) {
          const float2 v = *reinterpret_cast<const float2*>(bias_seg + 16 + 8 * nb + 2 * c);
          sxa[nb][0] += v.x;
          sxa[nb][1] += v.y;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[stage]);
      if (++stage == S) { stage = 0; phase ^= 1; }
    }
    if (!ok) break;

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
        // the MMAs saw the unsigned codes: remove z[row] * sum_k x[m,k] (this unit's k)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[0][nb][i] -= ((i < 2) ? za : zb) * sxa[nb][i & 1];
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
