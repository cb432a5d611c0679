// Tensor-core W4A16 / W8A16 GEMM for a skinny activation matrix (M <= 64 tokens):
//
//   Y[m,n] = fp16( s[n] * sum_k X[m,k] q[n,k] )
//
// GLM-130B paper card (wikillm.com), "Method": linear_forward with weight =
// quant * scale[:, None] and FP16 activations; paperlayer summary, "INT4
// Quantization for RTX 3090s/2080s": weights are converted to FP16 at run time.
//
// With few tokens the packed weights are the working set, so the kernel is built
// around a wide weight stream and cheap dequantization:
//  * Stages hold one TMA box of 128 weight rows x 128 packed bytes (256 k for INT4,
//    128 k for INT8; 128-byte swizzle) plus the matching activation tiles
//    (BN tokens x 64 k each). Wide box rows matter: the TMA path serves a roughly
//    fixed number of box rows per microsecond, so 128-byte rows stream several
//    times faster than the 32-byte rows of a 64-wide K block, and the activation
//    tiles do not take box rows at all: a small pre-pass (skinny_pack_x_kernel)
//    writes X once per call as the exact shared-memory image of every tile (128-byte
//    swizzle, INT4 k order, zero rows past M), and each stage fetches its tiles with
//    one contiguous bulk copy.
//  * The dequantized weights never touch shared memory: they are the MMA's A
//    operand in tensor memory. Four dequantizer groups of 128 threads (thread =
//    weight row = TMEM lane) take the 64-wide K blocks of the stream round-robin
//    (group g: blocks g, g+4, ...), turn 64 codes into fp16 in registers and write
//    them with one tcgen05.st into a ring of A slots.
//  * One thread issues tcgen05.mma (kind::f16, A from TMEM, B from shared memory,
//    fp32 accumulator in TMEM); the epilogue warps read the accumulator with
//    tcgen05.ld, multiply by s[n] and store fp16 (or add into the split-K scratch).
//  * INT4 codes are dequantized in the order (0,4,1,5,2,6,3,7) within each group
//    of 8, which costs no byte shuffle; the pre-pass writes the activations in the
//    same order (the MMA's k order is immaterial when both operands share it).
//  * Work units are (128-row tile, K part) pairs exactly as in the prefill kernel,
//    with the same split-K scratch and finalize kernel.
// No TMA multicast is used anywhere.
#pragma once

#include <cuda.h>

#include "glmq_ptx.cuh"
#include "prefill.cuh"

namespace glmq {

constexpr int kSkinnyDequantWarps = 16;    // 4 groups of 4 warps
constexpr int kSkinnyGroups = 4;
constexpr int kSkinnyEpilogueWarp0 = 16;   // warps 16..19
constexpr int kSkinnyProducerWarp = 20;
constexpr int kSkinnyMmaWarp = 21;
constexpr int kSkinnyThreads = 22 * 32;
constexpr int kSkinnyASlots = 8;           // A operand slots in TMEM (one 64-wide K block each)
static_assert((kSkinnyASlots & (kSkinnyASlots - 1)) == 0, "slot index by mask");
#ifndef SKINNY_ACC_CHAINS
#define SKINNY_ACC_CHAINS 1
#endif
// Independent accumulators per tile (consecutive MMAs of a K block alternate between
// them and the epilogue sums them). One by default: two measured no faster here.
constexpr int kSkinnyAccChains = SKINNY_ACC_CHAINS;

template <int BITS, int BN, int ZP = 0>
struct SkinnyCfg {
  static constexpr int kZP = ZP;   // 1: zero-point INT4 codes (unsigned, per-row zero point)
  static constexpr int kBits = BITS;
  static constexpr int kBN = BN;
  static constexpr int BM = 128;
  static constexpr int WB = 128;                          // packed bytes per row per stage
  static constexpr int KPB = (BITS == 4) ? 2 : 1;
  static constexpr int SK = WB * KPB;                     // k per stage
  static constexpr int KB = SK / 64;                      // 64-wide K blocks per stage (4 or 2)
  static constexpr int W_BYTES = BM * WB;                 // 16 KB
  static constexpr int XT_BYTES = BN * 128;               // one activation tile (BN x 64 fp16)
  static constexpr int STAGE_BYTES = W_BYTES + KB * XT_BYTES;
  static constexpr int kStages = (kPrefillSmemBudget / STAGE_BYTES) < kPrefillMaxStages
                                     ? (kPrefillSmemBudget / STAGE_BYTES) : kPrefillMaxStages;
  static constexpr int ACC_COLS = 2 * kSkinnyAccChains * BN;   // 2 tiles x chains x BN fp32 columns
  static constexpr int TMEM_COLS = 512;
  static constexpr int SMEM_BYTES = kStages * STAGE_BYTES + 1024 /*align*/ + 512 /*barriers*/;
  static_assert(BN == 16 || BN == 32 || BN == 64, "skinny token tiles");
  static_assert(XT_BYTES % 1024 == 0, "swizzle atoms stay 1024-byte aligned");
  static_assert(kStages >= 3, "pipeline depth");
  static_assert(ACC_COLS + kSkinnyASlots * 32 <= TMEM_COLS, "tensor memory budget");
  // kind::f16, fp32 accumulator, fp16 A (tensor memory) and B (shared memory), K-major, N = BN, M = 128
  static constexpr uint32_t IDESC = (1u << 4) | (uint32_t(BN >> 3) << 17) | (uint32_t(BM >> 4) << 24);
};

__device__ __forceinline__ void umma_f16_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                                uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// The same MMA with the B descriptor given as its two 32-bit halves (the issuing loop
// offsets the low half, which holds the start address, with plain 32-bit adds).
template <uint32_t kAccumulate>
__device__ __forceinline__ void umma_f16_tmem_a_lh(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo, uint32_t b_hi,
                                                   uint32_t idesc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 bd;\n\t"
      "setp.ne.b32 p, %5, 0;\n\t"
      "mov.b64 bd, {%2, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], bd, %4, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "r"(b_lo), "r"(b_hi), "r"(idesc), "r"(kAccumulate)
      : "memory");
}

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

// Pre-pass: X fp16 [M, K] -> the shared-memory image of every activation tile the
// skinny kernel reads: for 64-wide K block b, BN rows (tokens) of 128 bytes with the
// 128-byte swizzle (16-byte unit u of row r at (u ^ (r & 7)) * 16), rows >= M zero,
// INT4 values of each 8-group in the order (0,4,1,5,2,6,3,7). Tiles of consecutive
// K blocks are contiguous, so a stage's tiles are one contiguous range.
template <class C>
__global__ void __launch_bounds__(256) skinny_pack_x_kernel(const __half* __restrict__ X, int M, int K,
                                                            uint8_t* __restrict__ xs) {
  const long long total = static_cast<long long>(K / 64) * C::kBN * 8;     // 16-byte units
  for (long long i = blockIdx.x * 256LL + threadIdx.x; i < total; i += static_cast<long long>(gridDim.x) * 256) {
    const int u = static_cast<int>(i & 7);
    const long long rk = i >> 3;
    const int r = static_cast<int>(rk % C::kBN);
    const long long kb = rk / C::kBN;
    uint4 o = make_uint4(0, 0, 0, 0);
    if (r < M) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(X + static_cast<long long>(r) * K + kb * 64 + 8 * u));
      if constexpr (C::kBits == 4) {
        o = make_uint4(prmt(v.x, v.z, 0x5410u), prmt(v.x, v.z, 0x7632u), prmt(v.y, v.w, 0x5410u),
                       prmt(v.y, v.w, 0x7632u));
      } else {
        o = v;
      }
    }
    *reinterpret_cast<uint4*>(xs + kb * C::XT_BYTES + r * 128 + ((u ^ (r & 7)) << 4)) = o;
  }
}

// Valid 64-wide K blocks of the stage that starts at k0.
__device__ __forceinline__ int skinny_stage_kblocks(int k0, int K, int KB) { return min(KB, (K - k0) >> 6); }

template <class C>
__global__ void __launch_bounds__(kSkinnyThreads, 1)
    skinny_kernel(const __grid_constant__ CUtensorMap tmap_w, const PrefillArgs a) {
  constexpr int S = C::kStages;
  constexpr int NA = kSkinnyASlots;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * C::STAGE_BYTES);
  uint64_t* full = bars;                  // stage bytes landed            (count 1 + tx)
  uint64_t* empty = bars + S;             // stage's MMAs done             (tcgen05.commit)
  uint64_t* afull = bars + 2 * S;         // A slot written                (count 4 warps)
  uint64_t* aempty = afull + NA;          // A slot's MMAs done            (tcgen05.commit)
  uint64_t* accfull = aempty + NA;        // accumulator ready             (tcgen05.commit), x2
  uint64_t* accempty = accfull + 2;       // accumulator drained           (count 4 warps), x2
  uint64_t* final_bar = accempty + 2;     // all MMAs done, on the failure path (tcgen05.commit)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(final_bar + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int K = a.K;
  const int num_st = (K + C::SK - 1) / C::SK;     // stages along K
  const int G = gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < NA; ++i) {
      mbar_init(&afull[i], kSkinnyDequantWarps / kSkinnyGroups);
      mbar_init(&aempty[i], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accfull[b], 1);
      mbar_init(&accempty[b], 4);
    }
    mbar_init(final_bar, 1);
    fence_barrier_init();
  }
  if (warp == kSkinnyMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(C::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  bool ok = true;

  if (warp == kSkinnyProducerWarp) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t armed[S] = {};
      int stage = 0;
      uint32_t phase = 0;
      for (int u = blockIdx.x; u < a.units && ok; u += G) {
        const int p = u / a.tiles;
        const int t = u - p * a.tiles;
        const int nt = t / a.tiles_m;
        const int mt = t - nt * a.tiles_m;
        const int st1 = min(num_st, (p + 1) * a.kbp);
        for (int ks = p * a.kbp; ks < st1; ++ks) {
          if (!mbar_wait_suspend(&empty[stage], phase ^ 1)) { ok = false; break; }
          const int k0 = ks * C::SK;
          const int nkb = skinny_stage_kblocks(k0, K, C::KB);
          uint8_t* st = smem + stage * C::STAGE_BYTES;
          mbar_arrive_expect_tx(&full[stage], C::W_BYTES + nkb * C::XT_BYTES);
          armed[stage] = phase + 1;
          tma_load_2d(st, &tmap_w, k0 / C::KPB, nt * C::BM, &full[stage]);
          bulk_g2s(st + C::W_BYTES, a.xs + (static_cast<long long>(mt) * (K / 64) + k0 / 64) * C::XT_BYTES,
                   static_cast<uint32_t>(nkb * C::XT_BYTES), &full[stage]);
          if (++stage == S) { stage = 0; phase ^= 1; }
        }
      }
      bool drained = true;
      for (int s = 0; s < S; ++s)
        if (armed[s] && !mbar_wait_drain_suspend(&full[s], armed[s] - 1)) drained = false;
      if (!ok || !drained) report_error(kErrPrefillWait);
    }
  } else if (warp < kSkinnyDequantWarps) {
    // ------------------------------------------------------------ dequantizer groups
    const int grp = warp >> 2;                      // K blocks with sequence number % 4 == grp
    const int row = ((warp & 3) << 5) + lane;       // weight row of the tile = TMEM lane
    const uint32_t lane_addr = static_cast<uint32_t>((warp & 3) * 32) << 16;
    int stage = 0;
    uint32_t phase = 0;
    int kseq = 0;
    for (int u = blockIdx.x; u < a.units && ok; u += G) {
      const int p = u / a.tiles;
      const int st1 = min(num_st, (p + 1) * a.kbp);
      Int4Dequant dq = int4_dequant_symmetric();
      if constexpr (C::kZP) {
        const int wrow = ((u - p * a.tiles) / a.tiles_m) * C::BM + row;
        dq = int4_dequant_zero_point(wrow < a.N ? a.zero[wrow] : 0);
      }
      for (int ks = p * a.kbp; ks < st1 && ok; ++ks) {
        const int nkb = skinny_stage_kblocks(ks * C::SK, K, C::KB);
        bool waited = false;
        for (int j = 0; j < nkb; ++j, ++kseq) {
          if ((kseq & (kSkinnyGroups - 1)) != grp) continue;
          if (!waited) {
            if (!mbar_wait_warp_suspend(&full[stage], phase)) { ok = false; break; }
            waited = true;
          }
          const int slot = kseq % NA;
          if (!mbar_wait_warp_suspend(&aempty[slot], ((kseq / NA) & 1) ^ 1)) { ok = false; break; }
          tc_fence_after();
          uint8_t* st = smem + stage * C::STAGE_BYTES;
          const uint32_t w_tile = smem_u32(st);
          uint32_t h[32];
          if constexpr (C::kBits == 4) {
            // bytes [32j, 32j+32) of this row: 16-byte units 2j and 2j+1, 128-byte swizzle
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              const uint32_t unit = static_cast<uint32_t>((2 * j + q) ^ (row & 7));
              const uint4 v = lds_v4(w_tile + row * 128 + (unit << 4));
              const uint32_t words[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
              for (int wv = 0; wv < 4; ++wv) {
                const uint4 o = dequant_int4_paired(words[wv], dq);
                h[16 * q + 4 * wv + 0] = o.x;
                h[16 * q + 4 * wv + 1] = o.y;
                h[16 * q + 4 * wv + 2] = o.z;
                h[16 * q + 4 * wv + 3] = o.w;
              }
            }
          } else {
            // bytes [64j, 64j+64) of this row: units 4j .. 4j+3
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint32_t unit = static_cast<uint32_t>((4 * j + q) ^ (row & 7));
              const uint4 v = lds_v4(w_tile + row * 128 + (unit << 4));
              const uint2 d0 = dequant_int8_natural(v.x), d1 = dequant_int8_natural(v.y);
              const uint2 d2 = dequant_int8_natural(v.z), d3 = dequant_int8_natural(v.w);
              h[8 * q + 0] = d0.x; h[8 * q + 1] = d0.y; h[8 * q + 2] = d1.x; h[8 * q + 3] = d1.y;
              h[8 * q + 4] = d2.x; h[8 * q + 5] = d2.y; h[8 * q + 6] = d3.x; h[8 * q + 7] = d3.y;
            }
          }
          tmem_st32(tmem_base + lane_addr + C::ACC_COLS + slot * 32, h);
          asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&afull[slot]);
        }
        if (++stage == S) { stage = 0; phase ^= 1; }
      }
    }
    if (!ok && lane == 0) report_error(kErrPrefillWait);
  } else if (warp == kSkinnyMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    // A single thread issues every MMA, so its instruction stream is kept short: the B
    // descriptors of a stage come from one base by 32-bit adds to the low half (start
    // address in 16-byte units) and the accumulate flag is a compile-time constant per
    // K block. Its waits suspend in hardware like the other roles' (polling took issue
    // slots from the dequantizer warps sharing its scheduler and was slower).
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int kseq = 0;
      int it = 0;
      uint32_t acc_armed[2] = {};
      const uint64_t desc0 = umma_desc_sw128(0);
      const uint32_t desc_hi = static_cast<uint32_t>(desc0 >> 32);
      for (int u = blockIdx.x; u < a.units && ok; u += G, ++it) {
        const int p = u / a.tiles;
        const int st0 = p * a.kbp;
        const int st1 = min(num_st, st0 + a.kbp);
        const int ab = it & 1;
        const uint32_t aphase = (it >> 1) & 1;
        if (!mbar_wait_suspend(&accempty[ab], aphase ^ 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + ab * kSkinnyAccChains * C::kBN;
        bool first = true;
        for (int ks = st0; ks < st1 && ok; ++ks) {
          const int nkb = skinny_stage_kblocks(ks * C::SK, K, C::KB);
          // low descriptor half of the stage's first activation tile (start address >> 4)
          const uint32_t b_lo0 = static_cast<uint32_t>(desc0) |
                                 ((smem_u32(smem + stage * C::STAGE_BYTES + C::W_BYTES) >> 4) & 0x3FFFu);
          for (int j = 0; j < nkb; ++j, ++kseq) {
            const int slot = kseq & (NA - 1);
            if (!mbar_wait_suspend(&afull[slot], (kseq / NA) & 1)) { ok = false; break; }
            tc_fence_after();
            const uint32_t b_lo = b_lo0 + static_cast<uint32_t>(j * (C::XT_BYTES >> 4));
            const uint32_t a_tmem = tmem_base + C::ACC_COLS + slot * 32;
            // k sub-block kk: A columns kk * 8, B start address + kk * 32 bytes
            if (first) {
              umma_f16_tmem_a_lh<0>(d_tmem, a_tmem, b_lo, desc_hi, C::IDESC);
              umma_f16_tmem_a_lh<(kSkinnyAccChains > 1) ? 0 : 1>(d_tmem + (1 % kSkinnyAccChains) * C::kBN,
                                                                    a_tmem + 8, b_lo + 2, desc_hi, C::IDESC);
              first = false;
            } else {
              umma_f16_tmem_a_lh<1>(d_tmem, a_tmem, b_lo, desc_hi, C::IDESC);
              umma_f16_tmem_a_lh<1>(d_tmem + (1 % kSkinnyAccChains) * C::kBN, a_tmem + 8, b_lo + 2, desc_hi,
                                    C::IDESC);
            }
            umma_f16_tmem_a_lh<1>(d_tmem + (2 % kSkinnyAccChains) * C::kBN, a_tmem + 16, b_lo + 4, desc_hi, C::IDESC);
            umma_f16_tmem_a_lh<1>(d_tmem + (3 % kSkinnyAccChains) * C::kBN, a_tmem + 24, b_lo + 6, desc_hi, C::IDESC);
            umma_commit(&aempty[slot]);
          }
          if (!ok) break;
          umma_commit(&empty[stage]);
          if (++stage == S) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        umma_commit(&accfull[ab]);
        acc_armed[ab] = aphase + 1;
      }
      bool drained = true;
      for (int b = 0; b < 2; ++b)
        if (acc_armed[b] && !mbar_wait_drain_suspend(&accfull[b], acc_armed[b] - 1)) drained = false;
      if (!ok) {
        // a wait gave up mid-unit: MMAs may have been issued after the last commit above
        umma_commit(final_bar);
        if (!mbar_wait_drain_suspend(final_bar, 0)) drained = false;
      }
      if (!ok || !drained) report_error(kErrPrefillWait);
    }
  } else {
    // ------------------------------------------------------------ epilogue warps 16..19
    const int quarter = warp & 3;
    const bool split = a.parts > 1;
    int it = 0;
    for (int u = blockIdx.x; u < a.units && ok; u += G, ++it) {
      const int ab = it & 1;
      const uint32_t aphase = (it >> 1) & 1;
      if (!mbar_wait_warp_suspend(&accfull[ab], aphase)) { ok = false; break; }
      tc_fence_after();
      const int t = u % a.tiles;
      const int nt = t / a.tiles_m;
      const int mt = t - nt * a.tiles_m;
      const int n = nt * C::BM + quarter * 32 + lane;
      const float s = (n < a.N) ? __half2float(a.scale[n]) : 0.0f;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + ab * kSkinnyAccChains * C::kBN;
      constexpr int kChunk = (C::kBN < 32) ? C::kBN : 32;
#pragma unroll 1
      for (int cb = 0; cb < C::kBN / kChunk; ++cb) {
        const int m0 = mt * C::kBN + cb * kChunk;
        if (m0 >= a.M) break;   // warp-uniform
        uint32_t v[32];
        if constexpr (kChunk == 16) tmem_ld16(t_row + cb * kChunk, v);
        else tmem_ld32(t_row + cb * kChunk, v);
#pragma unroll
        for (int h = 1; h < kSkinnyAccChains; ++h) {
          uint32_t w[32];
          if constexpr (kChunk == 16) tmem_ld16(t_row + h * C::kBN + cb * kChunk, w);
          else tmem_ld32(t_row + h * C::kBN + cb * kChunk, w);
#pragma unroll
          for (int jj = 0; jj < kChunk; ++jj) v[jj] = __float_as_uint(__uint_as_float(v[jj]) + __uint_as_float(w[jj]));
        }
        const int mend = min(kChunk, a.M - m0);
        if (split) {
          if (n < a.N) {
            float* wp = a.ws + static_cast<long long>(m0) * a.N + n;
#pragma unroll
            for (int jj = 0; jj < kChunk; ++jj)
              if (jj < mend) atomicAdd(wp + static_cast<long long>(jj) * a.N, __uint_as_float(v[jj]));
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
  if (warp == kSkinnyMmaWarp) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(C::TMEM_COLS)
                 : "memory");
  }
}

}  // namespace glmq
