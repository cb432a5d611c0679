// Prefill-regime W4A16 / W8A16 GEMM on the 5th-generation tensor cores (tcgen05).
//
//   Y[m,n] = fp16( s[n] * sum_k X[m,k] q[n,k] )
//
// GLM-130B paper card (wikillm.com), "Method": linear_forward with weight =
// quant * scale[:, None] and FP16 activations; paperlayer summary, "INT4
// Quantization for RTX 3090s/2080s": weights are converted to FP16 at run time.
// With M up to a 2048-token prompt the product is a dense contraction, so it runs
// on tcgen05.mma (kind::f16, fp32 accumulation in tensor memory).
//
// The MMA is issued "swapped": the 128 weight rows of a tile are the MMA's M
// dimension (operand A) and BN tokens its N dimension (operand B), so the per-row
// scale s[n] belongs to one TMEM lane and is applied once per output in the
// epilogue. Warp roles (persistent CTAs, one per SM, static round-robin tiles,
// the BN-token tiles of one weight tile consecutive so the packed rows are read
// from HBM once and then hit in L2):
//   warp 20      TMA producer: 2-D tensor copies of the X tile (BN x 64 fp16,
//                128-byte swizzle) and of the packed weight tile (128 rows of
//                32 / 64 bytes, 32- / 64-byte swizzle) into a kStages ring;
//   warps 0..15  dequantizers, four independent groups of 128 threads (one weight
//                row per thread = one TMEM lane); group g takes every fourth K
//                block, so four K blocks are dequantized at once. A thread turns its
//                row's 64 codes into fp16 and writes them with one tcgen05.st into
//                one of 8 A slots in tensor memory (the A operand never touches
//                shared memory, which then carries only the X and packed tiles);
//   warp 21      MMA issuer: the warp runs the issue loop and its elected lane
//                issues 4 tcgen05.mma (K=16, A from TMEM, X from shared memory)
//                per 64-wide K block and commits the A slot and the stage;
//   warps 16..19 epilogue: tcgen05.ld of its 32 TMEM lanes, times s[n], fp16
//                stores. Two accumulators when they fit beside the A slots
//                (BN <= 128), else one, which the next tile's MMAs wait for.
// Work units are (tile, K part) pairs. Large problems use one part per tile; when
// there are fewer tiles than SMs (small M), tiles are split over K parts so every
// SM has work, each unit adds its fp32 partial tile into a scratch buffer with
// red.global.add and a stream-ordered finalize kernel scales, rounds and stores Y.
// No TMA multicast is used anywhere.
#pragma once

#include <cuda.h>

#include "epilogue.cuh"
#include "glmq_ptx.cuh"

namespace glmq {

constexpr int kPrefillDequantWarps = 16;
constexpr int kPrefillDequantGroups = 4;     // groups of 4 warps; group g dequantizes K blocks g, g+4, ...
constexpr int kPrefillEpilogueWarp0 = 16;
constexpr int kPrefillProducerWarp = 20;
constexpr int kPrefillMmaWarp = 21;
constexpr int kPrefillThreads = 22 * 32;
constexpr int kPrefillSmemBudget = 232448 - 1024 /*alignment*/ - 512 /*barriers*/;

template <int BITS, int BN, int ZP = 0>
struct PrefillCfg {
  static constexpr int kZP = ZP;   // 1: zero-point INT4 codes (unsigned, per-row zero point)
  static constexpr int kBits = BITS;
  static constexpr int kBN = BN;
  static constexpr int BM = 128;
  static constexpr int BK = 64;
  static constexpr int X_BYTES = BN * BK * 2;           // B operand tile
  static constexpr int WROW = BK * BITS / 8;            // packed bytes per row per K block (32 or 64)
  static constexpr int W_BYTES = BM * WROW;
  static constexpr int STAGE_BYTES = X_BYTES + W_BYTES;
  // The stage count is a multiple of the dequantizer groups, so each stage (and each A
  // slot) is only ever waited on by the one group that reads every phase of it.
  static constexpr int kStageSets = kPrefillSmemBudget / (kPrefillDequantGroups * STAGE_BYTES);
  static constexpr int kStages = kPrefillDequantGroups * (kStageSets < 2 ? kStageSets : 2);
  // TMEM: one or two fp32 accumulators of BN columns and the dequantized A operand in
  // NA slots of one 64-k block (32 columns) each: two accumulators whenever at least
  // one A slot per dequantizer group fits beside them (at most two per group).
  static constexpr int kAccBufs = (512 - 2 * BN) / 32 >= kPrefillDequantGroups ? 2 : 1;
  static constexpr int ACC_COLS = kAccBufs * BN;
  static constexpr int kSlotsFit = (512 - ACC_COLS) / 32;
  static constexpr int NA = kSlotsFit >= 2 * kPrefillDequantGroups ? 2 * kPrefillDequantGroups
                                                                     : kPrefillDequantGroups;
  static constexpr int A_COLS = NA * 32;
  static constexpr int TMEM_COLS = 512;
  static constexpr int SMEM_BYTES = kStages * STAGE_BYTES + 1024 /*align*/ + 512 /*barriers*/;
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "UMMA N for M=128");
  static_assert(X_BYTES % 1024 == 0, "swizzle atoms stay 1024-byte aligned");
  static_assert(kStages >= kPrefillDequantGroups, "one stage per dequantizer group at least");
  static_assert(ACC_COLS + A_COLS <= TMEM_COLS, "tensor memory budget");
  // kind::f16, fp32 accumulator, fp16 A and B, both K-major, N = BN, M = 128
  static constexpr uint32_t IDESC = (1u << 4) | (uint32_t(BN >> 3) << 17) | (uint32_t(BM >> 4) << 24);
};

struct PrefillArgs {
  const __half* scale;
  __half* Y;
  float* ws;      // fp32 [M, N] scratch, zero on entry (used when parts > 1)
  const uint8_t* xs;  // skinny kernel only: activation tiles pre-swizzled by skinny_pack_x_kernel
  const __half* bias; // fp16 [N] in the natural row order of W, or NULL (epilogue.cuh)
  int geglu;          // 1: packed rows in the GeGLU layout, Y is [M, N / 2]
  const uint8_t* zero;  // zero-point codes: uint8 [N] per-row zero point, else NULL
  int M;
  int N;
  int K;
  int tiles_m;
  int tiles;
  int parts;      // K parts per split tile
  int kbp;        // K blocks per part
  // prefill kernel: tiles 0 .. full-1 are whole units (units 0 .. full-1); tiles full ..
  // tiles-1 are split over the parts, K-part major. full = 0: every tile is split
  // (parts == 1: none is). The skinny kernel uses full = 0.
  int full;
  int units;      // full + (tiles - full) * parts
};

// Work unit u of the prefill kernel: tile t (= nt * tiles_m + mt), its K blocks
// [kb0, kb1), and whether its sums go through the scratch (split tiles).
struct PrefillUnit {
  int t;
  int kb0;
  int kb1;
  bool split;
};
__device__ __forceinline__ PrefillUnit prefill_unit(const PrefillArgs& a, int u, int num_kb) {
  PrefillUnit w;
  if (u < a.full) {
    w.t = u;
    w.kb0 = 0;
    w.kb1 = num_kb;
    w.split = false;
    return w;
  }
  const int rest = a.tiles - a.full;
  const int v = u - a.full;
  const int p = v / rest;
  w.t = a.full + (v - p * rest);
  w.kb0 = p * a.kbp;
  w.kb1 = min(num_kb, w.kb0 + a.kbp);
  w.split = a.parts > 1;
  return w;
}

// Epilogue of one TMEM lane (packed weight row n) for tokens m0 .. m0 + mend - 1,
// called by all 32 lanes of an epilogue warp (the GeGLU pair of row n, n % 16 < 8,
// is row n + 8, 8 lanes up in the same warp). Lanes with n >= N pass s = 0.
template <int kChunk>
__device__ __forceinline__ void tmem_lane_epilogue(const PrefillArgs& a, int n, float s, const uint32_t (&v)[32],
                                                   int m0, int mend) {
  const bool live = n < a.N;
  const float b = live ? epilogue_bias(a.bias, a.geglu, n, a.N) : 0.0f;
  if (!a.geglu) {
    if (!live) return;
    __half* yp = a.Y + static_cast<long long>(m0) * a.N + n;
#pragma unroll
    for (int j = 0; j < kChunk; ++j)
      if (j < mend) yp[static_cast<long long>(j) * a.N] = __float2half_rn(s * __uint_as_float(v[j]) + b);
    return;
  }
  const int F = a.N >> 1;
  const bool first_half = live && (n & 15) < 8;
  __half* yp = a.Y + static_cast<long long>(m0) * F + geglu_column(n);
#pragma unroll
  for (int j = 0; j < kChunk; ++j) {
    const float u = s * __uint_as_float(v[j]) + b;
    const float ub = __shfl_down_sync(0xffffffffu, u, 8);
    if (first_half && j < mend) yp[static_cast<long long>(j) * F] = __float2half_rn(gelu_exact(u) * ub);
  }
}

// ---------------------------------------------------------------- tcgen05 / TMA wrappers
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t smem_addr) {
  // K-major, 128-byte swizzle: LBO = 1 (16 B units, unused), SBO = 1024 B between
  // 8-row groups, descriptor version 1, layout type 2 (SWIZZLE_128B).
  return static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu) | (1ull << 16) | (64ull << 32) | (1ull << 46) |
         (2ull << 61);
}

__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// ---------------------------------------------------------------- warp-wide MMA issue
// The tcgen05 kernels issue their MMAs from a whole warp: every lane runs the issue
// loop (so its addresses and descriptors are warp-uniform values) and the MMA and
// commit instructions are predicated on one elected lane. Measured on B200 with 16
// back-to-back M=128, K=16 MMAs: about 12 cycles per MMA at N=16 and the full tensor
// rate from N=64 up, against 70-93 cycles per MMA when a single lane runs the loop
// inside a lane-0 branch.
__device__ __forceinline__ uint32_t elect_one_sync() {
  uint32_t leader;
  asm volatile(
      "{\n\t.reg .pred P;\n\t.reg .b32 x;\n\t"
      "elect.sync x|P, 0xffffffff;\n\t"
      "selp.u32 %0, 1, 0, P;\n\t}"
      : "=r"(leader));
  return leader;
}

// umma_f16 issued by the elected lane only (leader != 0 in exactly one lane).
template <uint32_t kAccumulate>
__device__ __forceinline__ void umma_f16_elected(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                                 uint32_t leader) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.ne.b32 e, %5, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "n"(kAccumulate), "r"(leader)
      : "memory");
}

// umma_commit issued by the elected lane only.
__device__ __forceinline__ void umma_commit_elected(uint64_t* bar, uint32_t leader) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "setp.ne.b32 e, %1, 0;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(smem_u32(bar)),
      "r"(leader)
      : "memory");
}

// tcgen05.mma kind::f16 with the A operand in TMEM and B in shared memory, the B
// descriptor given as its two 32-bit halves (an issuing loop offsets the low half,
// which holds the start address, with plain 32-bit adds). Issued by the elected lane
// only (leader != 0 in exactly one lane of the issuing warp).
template <uint32_t kAccumulate>
__device__ __forceinline__ void umma_f16_tmem_a_lh(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo, uint32_t b_hi,
                                                   uint32_t idesc, uint32_t leader) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t.reg .b64 bd;\n\t"
      "setp.ne.b32 p, %5, 0;\n\t"
      "setp.ne.b32 e, %6, 0;\n\t"
      "mov.b64 bd, {%2, %3};\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], bd, %4, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "r"(b_lo), "r"(b_hi), "r"(idesc), "n"(kAccumulate), "r"(leader)
      : "memory");
}

// Writes 32 consecutive 32-bit TMEM columns of this warp's 32 lanes (lane i: row i of
// the warp's lane quarter). Asynchronous: tcgen05.wait::st before reusing v.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
      "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]),
      "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]),
      "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}


__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
        "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
        "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}


// INT4 word (8 codes) -> fp16 values. A code nibble c OR-ed into the mantissa of 1024
// (low nibbles: XOR constant xlo) or of 1024 at 16x weight (high nibbles: xhi) gives
// an exact fp16 integer; adding b0 (low) or scaling by 1/16 and adding b1 (high)
// leaves the code's value. Symmetric codes: xlo = 0x6408 (1024 + (c ^ 8) = 1032 + q),
// xhi = 0x6480, b0 = -1032, b1 = -72. Zero-point codes: xlo = xhi = 0x6400,
// b0 = -(1024 + z), b1 = -(64 + z), giving c - z.
__device__ __forceinline__ void dequant_int4_pairs(uint32_t w, uint32_t xlo, uint32_t xhi, __half2 b0, __half2 b1,
                                                   __half2 (&r)[4]) {
  const __half2 kOne16 = __halves2half2(__ushort_as_half(0x2C00), __ushort_as_half(0x2C00));  // 1/16
  const uint32_t w8 = w >> 8;
  uint32_t h0 = lop3_and_xor(w, 0x000F000Fu, xlo);   // (0, 4)
  uint32_t h1 = lop3_and_xor(w, 0x00F000F0u, xhi);   // (1, 5) * 16
  uint32_t h2 = lop3_and_xor(w8, 0x000F000Fu, xlo);  // (2, 6)
  uint32_t h3 = lop3_and_xor(w8, 0x00F000F0u, xhi);  // (3, 7) * 16
  r[0] = __hadd2(*reinterpret_cast<__half2*>(&h0), b0);
  r[1] = __hfma2(*reinterpret_cast<__half2*>(&h1), kOne16, b1);
  r[2] = __hadd2(*reinterpret_cast<__half2*>(&h2), b0);
  r[3] = __hfma2(*reinterpret_cast<__half2*>(&h3), kOne16, b1);
}

struct Int4Dequant {
  uint32_t xlo, xhi;
  __half2 b0, b1;
};

__device__ __forceinline__ Int4Dequant int4_dequant_symmetric() {
  return {0x64086408u, 0x64806480u, __halves2half2(__ushort_as_half(0xE408), __ushort_as_half(0xE408)),   // -1032
          __halves2half2(__ushort_as_half(0xD480), __ushort_as_half(0xD480))};                             // -72
}

__device__ __forceinline__ Int4Dequant int4_dequant_zero_point(int z) {
  return {0x64006400u, 0x64006400u, __float2half2_rn(-(1024.0f + static_cast<float>(z))),
          __float2half2_rn(-(64.0f + static_cast<float>(z)))};
}

// k order 0..7 of the word
__device__ __forceinline__ uint4 dequant_int4_natural(uint32_t w, const Int4Dequant& d) {
  __half2 r[4];
  dequant_int4_pairs(w, d.xlo, d.xhi, d.b0, d.b1, r);
  const uint32_t p0 = *reinterpret_cast<uint32_t*>(&r[0]), p1 = *reinterpret_cast<uint32_t*>(&r[1]);
  const uint32_t p2 = *reinterpret_cast<uint32_t*>(&r[2]), p3 = *reinterpret_cast<uint32_t*>(&r[3]);
  return make_uint4(prmt(p0, p1, 0x5410u), prmt(p2, p3, 0x5410u), prmt(p0, p1, 0x7632u), prmt(p2, p3, 0x7632u));
}
// k order (0,4,1,5,2,6,3,7): no byte shuffle
__device__ __forceinline__ uint4 dequant_int4_paired(uint32_t w, const Int4Dequant& d) {
  __half2 r[4];
  dequant_int4_pairs(w, d.xlo, d.xhi, d.b0, d.b1, r);
  return make_uint4(*reinterpret_cast<uint32_t*>(&r[0]), *reinterpret_cast<uint32_t*>(&r[1]),
                    *reinterpret_cast<uint32_t*>(&r[2]), *reinterpret_cast<uint32_t*>(&r[3]));
}
__device__ __forceinline__ uint2 dequant_int8_natural(uint32_t w) {
  const __half2 kBias = __halves2half2(__ushort_as_half(0xE480), __ushort_as_half(0xE480));  // -1152
  const uint32_t x = w ^ 0x80808080u;
  uint32_t lo = prmt(x, 0x64646464u, 0x4140u);
  uint32_t hi = prmt(x, 0x64646464u, 0x4342u);
  __half2 a = __hadd2(*reinterpret_cast<__half2*>(&lo), kBias);
  __half2 b = __hadd2(*reinterpret_cast<__half2*>(&hi), kBias);
  return make_uint2(*reinterpret_cast<uint32_t*>(&a), *reinterpret_cast<uint32_t*>(&b));
}

// ---------------------------------------------------------------- the kernel
template <class C>
__global__ void __launch_bounds__(kPrefillThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                   const PrefillArgs a) {
  constexpr int S = C::kStages;
  constexpr int NA = C::NA;
  constexpr int NB = C::kAccBufs;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * C::STAGE_BYTES);
  uint64_t* full = bars;                  // X and W tiles landed            (count 1 + tx)
  uint64_t* empty = bars + S;             // stage's MMAs done               (tcgen05.commit)
  uint64_t* afull = bars + 2 * S;         // A slot written                  (count 4 warps)
  uint64_t* aempty = afull + NA;          // A slot's MMAs done              (tcgen05.commit)
  uint64_t* accfull = aempty + NA;        // accumulator ready               (tcgen05.commit), x NB
  uint64_t* accempty = accfull + NB;      // accumulator drained             (count 4 warps), x NB
  uint64_t* final_bar = accempty + NB;    // all MMAs done, on the failure path (tcgen05.commit)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(final_bar + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int num_kb = a.K / C::BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < NA; ++i) {
      mbar_init(&afull[i], kPrefillDequantWarps / kPrefillDequantGroups);
      mbar_init(&aempty[i], 1);
    }
    for (int b = 0; b < NB; ++b) {
      mbar_init(&accfull[b], 1);
      mbar_init(&accempty[b], 4);
    }
    mbar_init(final_bar, 1);
    fence_barrier_init();
  }
  if (warp == kPrefillMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(C::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int G = gridDim.x;
  bool ok = true;

  if (warp == kPrefillProducerWarp) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t armed[S] = {};
      int stage = 0;
      uint32_t phase = 0;
      for (int u = blockIdx.x; u < a.units && ok; u += G) {
        const PrefillUnit w = prefill_unit(a, u, num_kb);
        const int nt = w.t / a.tiles_m;
        const int mt = w.t - nt * a.tiles_m;
        for (int kb = w.kb0; kb < w.kb1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1)) { ok = false; break; }
          uint8_t* st = smem + stage * C::STAGE_BYTES;
          mbar_arrive_expect_tx(&full[stage], C::X_BYTES + C::W_BYTES);
          armed[stage] = phase + 1;
          tma_load_2d(st, &tmap_x, kb * C::BK, mt * C::kBN, &full[stage]);
          tma_load_2d(st + C::X_BYTES, &tmap_w, kb * C::WROW, nt * C::BM, &full[stage]);
          if (++stage == S) { stage = 0; phase ^= 1; }
        }
      }
      bool drained = true;
      for (int s = 0; s < S; ++s)
        if (armed[s] && !mbar_wait_drain(&full[s], armed[s] - 1)) drained = false;
      if (!ok || !drained) report_error(kErrPrefillWait);
    }
  } else if (warp < kPrefillDequantWarps) {
    // ------------------------------------------------------------ dequantizers
    // Group g (warps 4g .. 4g+3, TMEM lanes 32 (w % 4) ...) takes the K blocks with
    // sequence number % 4 == g: stage seq % S and A slot seq % NA are then always the
    // group's own, so each barrier it waits on is one whose every phase it takes.
    const int row = ((warp & 3) << 5) + lane;        // tile row = TMEM lane
    const int grp = warp >> 2;
    const uint32_t lane_addr = static_cast<uint32_t>((warp & 3) * 32) << 16;
    int seq = 0;                         // K-block sequence number across this CTA's units
    for (int u = blockIdx.x; u < a.units && ok; u += G) {
      const PrefillUnit w = prefill_unit(a, u, num_kb);
      Int4Dequant dq = int4_dequant_symmetric();
      if constexpr (C::kZP) {
        const int wrow = (w.t / a.tiles_m) * C::BM + row;
        dq = int4_dequant_zero_point(wrow < a.N ? a.zero[wrow] : 0);
      }
      for (int kb = w.kb0; kb < w.kb1; ++kb, ++seq) {
        if ((seq & (kPrefillDequantGroups - 1)) != grp) continue;
        const int stage = seq % S;
        const int slot = seq % NA;
        if (!mbar_wait_warp(&full[stage], (seq / S) & 1)) { ok = false; break; }
        const uint32_t w_tile = smem_u32(smem + stage * C::STAGE_BYTES + C::X_BYTES);
        uint32_t h[32];                   // the row's 64 fp16 values, natural k order
        if constexpr (C::kBits == 4) {
          // 32-byte rows, 32-byte swizzle: 16-byte unit u sits at u ^ ((row >> 2) & 1)
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const uint4 v = lds_v4(w_tile + row * 32 + ((hh ^ ((row >> 2) & 1)) << 4));
            const uint32_t words[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint4 o = dequant_int4_natural(words[j], dq);
              h[16 * hh + 4 * j + 0] = o.x;
              h[16 * hh + 4 * j + 1] = o.y;
              h[16 * hh + 4 * j + 2] = o.z;
              h[16 * hh + 4 * j + 3] = o.w;
            }
          }
        } else {
          // 64-byte rows, 64-byte swizzle: unit u sits at u ^ ((row >> 1) & 3)
#pragma unroll
          for (int uu = 0; uu < 4; ++uu) {
            const uint4 v = lds_v4(w_tile + row * 64 + ((uu ^ ((row >> 1) & 3)) << 4));
            const uint2 d0 = dequant_int8_natural(v.x), d1 = dequant_int8_natural(v.y);
            const uint2 d2 = dequant_int8_natural(v.z), d3 = dequant_int8_natural(v.w);
            h[8 * uu + 0] = d0.x; h[8 * uu + 1] = d0.y; h[8 * uu + 2] = d1.x; h[8 * uu + 3] = d1.y;
            h[8 * uu + 4] = d2.x; h[8 * uu + 5] = d2.y; h[8 * uu + 6] = d3.x; h[8 * uu + 7] = d3.y;
          }
        }
        if (!mbar_wait_warp(&aempty[slot], ((seq / NA) & 1) ^ 1)) { ok = false; break; }
        tc_fence_after();
        tmem_st32(tmem_base + lane_addr + C::ACC_COLS + slot * 32, h);
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&afull[slot]);
      }
    }
    if (!ok && lane == 0) report_error(kErrPrefillWait);
  } else if (warp == kPrefillMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the loop; the elected lane issues the MMAs (A from TMEM, the X
    // tile from shared memory) and commits.
    const uint32_t leader = elect_one_sync();
    int seq = 0;
    int it = 0;
    uint32_t acc_armed[NB] = {};
    const uint64_t desc0 = umma_desc_sw128(0);
    const uint32_t desc_hi = static_cast<uint32_t>(desc0 >> 32);
    // low descriptor half of stage 0's X tile (start address >> 4)
    const uint32_t x_lo_base = static_cast<uint32_t>(desc0) | ((smem_u32(smem) >> 4) & 0x3FFFu);
    constexpr uint32_t kStageLo = C::STAGE_BYTES >> 4;
    for (int u = blockIdx.x; u < a.units && ok; u += G, ++it) {
      const PrefillUnit w = prefill_unit(a, u, num_kb);
      const int kb0 = w.kb0;
      const int kb1 = w.kb1;
      const int ab = it % NB;
      const uint32_t aphase = (it / NB) & 1;
      if (!mbar_wait_warp(&accempty[ab], aphase ^ 1)) { ok = false; break; }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + ab * C::kBN;
      for (int kb = kb0; kb < kb1; ++kb, ++seq) {
        const int stage = seq % S;
        const int slot = seq % NA;
        if (!mbar_wait_warp(&afull[slot], (seq / NA) & 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t a_tmem = tmem_base + C::ACC_COLS + slot * 32;
        const uint32_t x_lo = x_lo_base + stage * kStageLo;
        // k sub-block kk: A columns kk * 8, X start address + kk * 32 bytes
        if (kb == kb0) umma_f16_tmem_a_lh<0>(d_tmem, a_tmem, x_lo, desc_hi, C::IDESC, leader);
        else umma_f16_tmem_a_lh<1>(d_tmem, a_tmem, x_lo, desc_hi, C::IDESC, leader);
        umma_f16_tmem_a_lh<1>(d_tmem, a_tmem + 8, x_lo + 2, desc_hi, C::IDESC, leader);
        umma_f16_tmem_a_lh<1>(d_tmem, a_tmem + 16, x_lo + 4, desc_hi, C::IDESC, leader);
        umma_f16_tmem_a_lh<1>(d_tmem, a_tmem + 24, x_lo + 6, desc_hi, C::IDESC, leader);
        umma_commit_elected(&aempty[slot], leader);
        umma_commit_elected(&empty[stage], leader);
      }
      if (!ok) break;
      umma_commit_elected(&accfull[ab], leader);
      acc_armed[ab] = aphase + 1;
    }
    // make sure no MMA is still reading shared memory or writing TMEM before the CTA
    // exits and the allocation is released
    bool drained = true;
    for (int b = 0; b < NB; ++b)
      if (acc_armed[b] && !mbar_wait_drain_warp(&accfull[b], acc_armed[b] - 1)) drained = false;
    if (!ok) {
      // a wait gave up mid-unit: MMAs may have been issued after the last commit above
      umma_commit_elected(final_bar, leader);
      if (!mbar_wait_drain_warp(final_bar, 0)) drained = false;
    }
    if ((!ok || !drained) && lane == 0) report_error(kErrPrefillWait);
  } else {
    // ------------------------------------------------------------ epilogue warps 16..19
    const int quarter = warp & 3;   // TMEM lanes 32*quarter .. 32*quarter+31
    int it = 0;
    for (int u = blockIdx.x; u < a.units && ok; u += G, ++it) {
      const int ab = it % NB;
      const uint32_t aphase = (it / NB) & 1;
      if (!mbar_wait_warp(&accfull[ab], aphase)) { ok = false; break; }
      tc_fence_after();
      const PrefillUnit w = prefill_unit(a, u, num_kb);
      const bool split = w.split;
      const int nt = w.t / a.tiles_m;
      const int mt = w.t - nt * a.tiles_m;
      const int n = nt * C::BM + quarter * 32 + lane;
      const float s = (n < a.N) ? __half2float(a.scale[n]) : 0.0f;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + ab * C::kBN;
      constexpr int kChunk = (C::kBN < 32) ? C::kBN : 32;
#pragma unroll 1
      for (int cb = 0; cb < C::kBN / kChunk; ++cb) {
        const int m0 = mt * C::kBN + cb * kChunk;
        if (m0 >= a.M) break;   // warp-uniform
        uint32_t v[32];
        if constexpr (kChunk == 16) tmem_ld16(t_row + cb * kChunk, v);
        else tmem_ld32(t_row + cb * kChunk, v);
        const int mend = min(kChunk, a.M - m0);
        if (split) {
          if (n < a.N) {
            float* wp = a.ws + static_cast<long long>(m0) * a.N + n;
#pragma unroll
            for (int j = 0; j < kChunk; ++j)
              if (j < mend) atomicAdd(wp + static_cast<long long>(j) * a.N, __uint_as_float(v[j]));
          }
        } else {
          tmem_lane_epilogue<kChunk>(a, n, s, v, m0, mend);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&accempty[ab]);
    }
    if (!ok && lane == 0) report_error(kErrPrefillWait);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kPrefillMmaWarp) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(C::TMEM_COLS)
                 : "memory");
  }
}

}  // namespace glmq
