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
//  * Two rings. The weight ring holds TMA boxes of 128 weight rows x 128 packed
//    bytes (256 k for INT4, 128 k for INT8; 128-byte swizzle). Wide box rows
//    matter: the TMA path serves a roughly fixed number of box rows per
//    microsecond, so 128-byte rows stream several times faster than the 32-byte
//    rows of a 64-wide K block. The activation ring holds the matching activation
//    tiles (BN tokens x 64 k each), which take no box rows: a small pre-pass
//    (skinny_pack_x_kernel) writes X once per call as the exact shared-memory image
//    of every tile (128-byte swizzle, INT4 k order, zero rows past M), and a second
//    producer warp fetches a stage's tiles with one contiguous bulk copy.
//  * A weight box is released as soon as the dequantizers hold its codes in
//    registers; only the activation tiles wait for the MMAs. The weight ring's
//    round trip is therefore about one TMA latency, and with most of shared memory
//    given to it (8 to 13 boxes) enough bytes stay in flight to stream at HBM rate.
//  * The dequantized weights never touch shared memory: they are the MMA's A
//    operand in tensor memory. Four dequantizer groups of 128 threads (thread =
//    weight row = TMEM lane) take the 64-wide K blocks of the stream round-robin
//    (group g: blocks g, g+4, ...), turn 64 codes into fp16 in registers and write
//    them with one tcgen05.st into a ring of A slots. The four slots of one slot
//    group are filled together and handed to the MMA warp with one barrier.
//  * One warp runs the MMA loop and its elected lane issues tcgen05.mma (kind::f16,
//    A from TMEM, B from shared memory, fp32 accumulator in TMEM); the epilogue
//    warps read the accumulator with tcgen05.ld, multiply by s[n] and store fp16
//    (or add into the split-K scratch).
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

// Slot groups of 4 K blocks (32 TMEM columns each) hold the MMA's A operand; three
// fit beside two accumulators of up to 64 columns. Each slot group has its own crew
// of 4 dequantizer warps (one per TMEM lane quarter).
constexpr int kSkinnySlotGroups = 3;
constexpr int kSkinnyGroupBlocks = 4;
constexpr int kSkinnyDequantWarps = 4 * kSkinnySlotGroups;   // warps 0..11
constexpr int kSkinnyEpilogueWarp0 = 12;   // warps 12..15
constexpr int kSkinnyProducerWarp = 16;    // weight boxes
constexpr int kSkinnyMmaWarp = 17;
constexpr int kSkinnyXWarp = 18;           // activation tiles
constexpr int kSkinnyThreads = 19 * 32;
constexpr int kSkinnyMaxCrewWStages = 5;

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
  static constexpr int XS_BYTES = KB * XT_BYTES;          // one stage's activation tiles
  // Weight boxes: a ring of kCrewWStages boxes per crew (each box is waited on by the one
  // crew that reads it, so no wait can run a phase ahead of its barrier, whatever order
  // the copies land in); activation tiles: the rest of shared memory, at least three
  // slot groups' worth.
  static constexpr int kMinXStages = 3 * (4 / KB);
  static constexpr int kCrewWFit = (kPrefillSmemBudget - kMinXStages * XS_BYTES) / (kSkinnySlotGroups * W_BYTES);
  static constexpr int kCrewWStages = kCrewWFit < kSkinnyMaxCrewWStages ? kCrewWFit : kSkinnyMaxCrewWStages;
  static constexpr int kWStages = kSkinnySlotGroups * kCrewWStages;
  static constexpr int kXFit = (kPrefillSmemBudget - kWStages * W_BYTES) / XS_BYTES;
  static constexpr int kXStages = kXFit < 12 ? kXFit : 12;
  static constexpr int ACC_COLS = 2 * BN;                      // 2 tiles x BN fp32 columns
  static constexpr int TMEM_COLS = 512;
  static constexpr int SMEM_BYTES = kWStages * W_BYTES + kXStages * XS_BYTES + 1024 /*align*/ + 512 /*barriers*/;
  static_assert(kCrewWStages >= 2 && kXStages >= kMinXStages, "pipeline depth");
  static_assert(2 * kWStages + 2 * kXStages + 2 * kSkinnySlotGroups + 5 < 512 / 8, "barrier area");
  static_assert(BN == 16 || BN == 32 || BN == 64, "skinny token tiles");
  static_assert(XT_BYTES % 1024 == 0, "swizzle atoms stay 1024-byte aligned");
  static_assert(ACC_COLS + kSkinnySlotGroups * kSkinnyGroupBlocks * 32 <= TMEM_COLS, "tensor memory budget");
  static_assert(KB == 2 || KB == 4, "a slot group spans one INT4 stage or two INT8 stages");
  // kind::f16, fp32 accumulator, fp16 A (tensor memory) and B (shared memory), K-major, N = BN, M = 128
  static constexpr uint32_t IDESC = (1u << 4) | (uint32_t(BN >> 3) << 17) | (uint32_t(BM >> 4) << 24);
};

// One 64-wide K block: 4 MMAs (K = 16 each). Sub-block kk reads A columns kk * 8 of
// the slot and B from the tile's start address + kk * 32 bytes (+2 in the low
// descriptor half). kFirst: the block opens the accumulator (no accumulate).
template <bool kFirst, class C>
__device__ __forceinline__ void skinny_mma_block(uint32_t d, uint32_t a, uint32_t b_lo, uint32_t b_hi, uint32_t leader) {
  umma_f16_tmem_a_lh<kFirst ? 0u : 1u>(d, a, b_lo, b_hi, C::IDESC, leader);
  umma_f16_tmem_a_lh<1>(d, a + 8, b_lo + 2, b_hi, C::IDESC, leader);
  umma_f16_tmem_a_lh<1>(d, a + 16, b_lo + 4, b_hi, C::IDESC, leader);
  umma_f16_tmem_a_lh<1>(d, a + 24, b_lo + 6, b_hi, C::IDESC, leader);
}

// Threads per block of the pre-pass: one such block fits on an SM beside a skinny CTA
// (4 warps of at most 32 registers in the registers the skinny CTA leaves free).
constexpr int kPackThreads = 128;

// Pre-pass: X fp16 [M, K] -> the shared-memory image of every activation tile the
// skinny kernel reads: for 64-wide K block b, BN rows (tokens) of 128 bytes with the
// 128-byte swizzle (16-byte unit u of row r at (u ^ (r & 7)) * 16), rows >= M zero,
// INT4 values of each 8-group in the order (0,4,1,5,2,6,3,7). Tiles of consecutive
// K blocks are contiguous, so a stage's tiles are one contiguous range.
template <class C>
__global__ void __launch_bounds__(kPackThreads) skinny_pack_x_kernel(const __half* __restrict__ X, int M, int K,
                                                                     uint8_t* __restrict__ xs) {
  // Launched with a grid dependency: wait for the kernels before this one (X, and the
  // weights the skinny kernel reads without a wait of its own, are written by them),
  // then let the skinny kernel launch, so that its CTAs start streaming weights beside
  // this pass. The trigger must follow the wait: a dependent may launch as soon as
  // every block of this grid has triggered.
  griddep_wait();
  griddep_launch_dependents();
  const long long total = static_cast<long long>(K / 64) * C::kBN * 8;     // 16-byte units
  const long long stride = static_cast<long long>(gridDim.x) * kPackThreads;
  constexpr int U = 4;   // units per thread and pass, their loads in flight together
  for (long long i0 = static_cast<long long>(blockIdx.x) * kPackThreads + threadIdx.x; i0 < total;
       i0 += U * stride) {
    uint4 v[U];
#pragma unroll
    for (int q = 0; q < U; ++q) {
      const long long i = i0 + q * stride;
      const long long rk = i >> 3;
      const int r = static_cast<int>(rk % C::kBN);
      v[q] = make_uint4(0, 0, 0, 0);
      if (i < total && r < M)
        v[q] = __ldg(reinterpret_cast<const uint4*>(X + static_cast<long long>(r) * K + (rk / C::kBN) * 64 +
                                                     8 * static_cast<int>(i & 7)));
    }
#pragma unroll
    for (int q = 0; q < U; ++q) {
      const long long i = i0 + q * stride;
      if (i >= total) break;
      const int u = static_cast<int>(i & 7);
      const long long rk = i >> 3;
      const int r = static_cast<int>(rk % C::kBN);
      const long long kb = rk / C::kBN;
      uint4 o = v[q];
      if constexpr (C::kBits == 4)
        o = make_uint4(prmt(v[q].x, v[q].z, 0x5410u), prmt(v[q].x, v[q].z, 0x7632u), prmt(v[q].y, v[q].w, 0x5410u),
                       prmt(v[q].y, v[q].w, 0x7632u));
      *reinterpret_cast<uint4*>(xs + kb * C::XT_BYTES + r * 128 + ((u ^ (r & 7)) << 4)) = o;
    }
  }
}

// Valid 64-wide K blocks of the stage that starts at k0.
__device__ __forceinline__ int skinny_stage_kblocks(int k0, int K, int KB) { return min(KB, (K - k0) >> 6); }

template <class C>
__global__ void __launch_bounds__(kSkinnyThreads, 1)
    skinny_kernel(const __grid_constant__ CUtensorMap tmap_w, const PrefillArgs a) {
  constexpr int SW = C::kWStages;
  constexpr int SX = C::kXStages;
  constexpr int NG = kSkinnySlotGroups;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* wring = smem;                                  // SW weight boxes
  uint8_t* xring = smem + SW * C::W_BYTES;                // SX stages of activation tiles
  uint64_t* bars = reinterpret_cast<uint64_t*>(xring + SX * C::XS_BYTES);
  uint64_t* wfull = bars;                 // weight box landed                  (count 1 + tx)
  uint64_t* wempty = wfull + SW;          // weight box read into registers     (count 4 warps)
  uint64_t* xfull = wempty + SW;          // activation tiles landed            (count 1 + tx)
  uint64_t* xempty = xfull + SX;          // activation tiles' MMAs done        (tcgen05.commit)
  uint64_t* afull = xempty + SX;          // slot group written                 (count 4 warps)
  uint64_t* aempty = afull + NG;          // slot group's MMAs done             (tcgen05.commit)
  uint64_t* accfull = aempty + NG;        // accumulator ready                  (tcgen05.commit), x2
  uint64_t* accempty = accfull + 2;       // accumulator drained                (count 4 warps), x2
  uint64_t* final_bar = accempty + 2;     // all MMAs done, on the failure path (tcgen05.commit)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(final_bar + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int K = a.K;
  const int num_st = (K + C::SK - 1) / C::SK;     // stages along K
  const int G = gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SW; ++s) {
      mbar_init(&wfull[s], 1);
      mbar_init(&wempty[s], 4);
    }
    for (int s = 0; s < SX; ++s) {
      mbar_init(&xfull[s], 1);
      mbar_init(&xempty[s], 1);
    }
    for (int i = 0; i < NG; ++i) {
      mbar_init(&afull[i], 4);
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
    // ------------------------------------------------------------ weight boxes (TMA)
    // Stage i of a unit belongs to slot group (gsg + i / (4 / KB)) and so to that
    // group's crew; each crew's boxes cycle through its own kCrewWStages entries.
    if (lane == 0) {
      constexpr int SC = C::kCrewWStages;
      uint32_t armed[SW] = {};
      int cnt[NG] = {};        // boxes issued to each crew so far
      int gsg = 0;
      for (int u = blockIdx.x; u < a.units && ok; u += G) {
        const int p = u / a.tiles;
        const int nt = (u - p * a.tiles) / a.tiles_m;
        const int st0 = p * a.kbp;
        const int st1 = min(num_st, st0 + a.kbp);
        for (int ks = st0; ks < st1; ++ks) {
          const int crew = (gsg + (ks - st0) / (4 / C::KB)) % NG;
          const int n = cnt[crew]++;
          const int r = crew * SC + n % SC;
          const uint32_t ph = (n / SC) & 1;
          if (!mbar_wait(&wempty[r], ph ^ 1)) { ok = false; break; }
          mbar_arrive_expect_tx(&wfull[r], C::W_BYTES);
          armed[r] = ph + 1;
          tma_load_2d(wring + r * C::W_BYTES, &tmap_w, ks * C::WB, nt * C::BM, &wfull[r]);
        }
        gsg += (((min(K, st1 * C::SK) - st0 * C::SK) >> 6) + 3) >> 2;
      }
      bool drained = true;
      for (int s = 0; s < SW; ++s)
        if (armed[s] && !mbar_wait_drain(&wfull[s], armed[s] - 1)) drained = false;
      if (!ok || !drained) report_error(kErrPrefillWait);
    }
  } else if (warp == kSkinnyXWarp) {
    // ------------------------------------------------------------ activation tiles (bulk copies)
    // The activation image is written by the pre-pass, which may still be running: this
    // is the one role that waits for the grid dependency before its first access.
    griddep_wait();
    if (lane == 0) {
      uint32_t armed[SX] = {};
      int r = 0;
      uint32_t ph = 0;
      for (int u = blockIdx.x; u < a.units && ok; u += G) {
        const int p = u / a.tiles;
        const int mt = (u - p * a.tiles) % a.tiles_m;
        const int st1 = min(num_st, (p + 1) * a.kbp);
        for (int ks = p * a.kbp; ks < st1; ++ks) {
          const int k0 = ks * C::SK;
          const int nkb = skinny_stage_kblocks(k0, K, C::KB);
          if (!mbar_wait(&xempty[r], ph ^ 1)) { ok = false; break; }
          mbar_arrive_expect_tx(&xfull[r], nkb * C::XT_BYTES);
          armed[r] = ph + 1;
          bulk_g2s(xring + r * C::XS_BYTES, a.xs + (static_cast<long long>(mt) * (K / 64) + k0 / 64) * C::XT_BYTES,
                   static_cast<uint32_t>(nkb * C::XT_BYTES), &xfull[r]);
          if (++r == SX) { r = 0; ph ^= 1; }
        }
      }
      bool drained = true;
      for (int s = 0; s < SX; ++s)
        if (armed[s] && !mbar_wait_drain(&xfull[s], armed[s] - 1)) drained = false;
      if (!ok || !drained) report_error(kErrPrefillWait);
    }
  } else if (warp < kSkinnyDequantWarps) {
    // ------------------------------------------------------------ dequantizer crews
    // The K blocks of a work unit are numbered b = 0, 1, ...; block b sits in stage
    // b / KB of the unit (position b % KB there) and in slot group b / 4 (slot b % 4).
    // Slot groups are numbered across units; slot group q uses TMEM slot group q % 3
    // and is dequantized by crew q % 3 (warps 4c .. 4c+3, TMEM lanes 32 (w % 4) ...),
    // which writes all of its blocks (one INT4 stage or two INT8 stages): a warp
    // synchronises once per stage and per slot group, not once per block. A crew reads
    // its weight boxes from its own ring, in order, and releases each box as soon as
    // its rows' codes are in registers; the slot group is released by the MMAs.
    constexpr int kUnits = C::kBits == 4 ? 2 : 4;   // 16-byte units of a row per block
    const int crew = warp >> 2;                     // = the TMEM slot group it fills
    const int row = ((warp & 3) << 5) + lane;       // weight row of the tile = TMEM lane
    const uint32_t lane_addr = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t slots = tmem_base + lane_addr + C::ACC_COLS + crew * (kSkinnyGroupBlocks * 32);
    int wn = 0;    // boxes this crew has read (its ring position)
    int gsg = 0;   // slot groups of the earlier units
    for (int u = blockIdx.x; u < a.units && ok; u += G) {
      const int p = u / a.tiles;
      const int st0 = p * a.kbp;
      const int st1 = min(num_st, st0 + a.kbp);
      const int nb = (min(K, st1 * C::SK) - st0 * C::SK) >> 6;   // K blocks of the unit
      const int ngr = (nb + 3) >> 2;
      Int4Dequant dq = int4_dequant_symmetric();
      if constexpr (C::kZP) {
        const int wrow = ((u - p * a.tiles) / a.tiles_m) * C::BM + row;
        dq = int4_dequant_zero_point(wrow < a.N ? a.zero[wrow] : 0);
      }
      for (int g = ((crew - gsg) % NG + NG) % NG; g < ngr; g += NG) {
        const int gq = gsg + g;                     // slot-group sequence number; gq % NG == crew
        const int b0 = kSkinnyGroupBlocks * g;
        const int nblk = min(kSkinnyGroupBlocks, nb - b0);
        for (int i = 0; i < nblk; i += C::KB) {     // the group's stages
          const int r = crew * C::kCrewWStages + wn % C::kCrewWStages;   // this crew's next box
          const uint32_t wph = (wn / C::kCrewWStages) & 1;
          ++wn;
          const int nks = min(C::KB, nblk - i);     // blocks of this stage
          if (!mbar_wait_warp(&wfull[r], wph)) { ok = false; break; }
          const uint32_t w_row = smem_u32(wring + r * C::W_BYTES) + row * 128;
          uint4 raw[C::KB * kUnits];                // the row's 128 bytes of the box
#pragma unroll
          for (int v = 0; v < C::KB * kUnits; ++v)
            raw[v] = lds_v4(w_row + ((static_cast<uint32_t>(v) ^ static_cast<uint32_t>(row & 7)) << 4));
          if (i == 0) {
            if (!mbar_wait_warp(&aempty[crew], ((gq / NG) & 1) ^ 1)) { ok = false; break; }
            tc_fence_after();
          }
#pragma unroll
          for (int jj = 0; jj < C::KB; ++jj) {
            if (jj < nks) {
              uint32_t h[32];
              if constexpr (C::kBits == 4) {
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                  const uint32_t words[4] = {raw[2 * jj + q].x, raw[2 * jj + q].y, raw[2 * jj + q].z, raw[2 * jj + q].w};
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
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                  const uint4 w4 = raw[4 * jj + q];
                  const uint2 d0 = dequant_int8_natural(w4.x), d1 = dequant_int8_natural(w4.y);
                  const uint2 d2 = dequant_int8_natural(w4.z), d3 = dequant_int8_natural(w4.w);
                  h[8 * q + 0] = d0.x; h[8 * q + 1] = d0.y; h[8 * q + 2] = d1.x; h[8 * q + 3] = d1.y;
                  h[8 * q + 4] = d2.x; h[8 * q + 5] = d2.y; h[8 * q + 6] = d3.x; h[8 * q + 7] = d3.y;
                }
              }
              // tcgen05.st is asynchronous: h is reused by the next block only after this
              // store has completed
              tmem_st32(slots + (i + jj) * 32, h);
              asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
            }
          }
          // The box is released only after the dequantization above has consumed every
          // loaded register, so the loads have returned before the producer may refill it.
          __syncwarp();
          if (lane == 0) mbar_arrive(&wempty[r]);
        }
        if (!ok) break;
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&afull[crew]);
      }
      gsg += ngr;
    }
    // a crew that gave up may have stores in flight: none may reach TMEM after release
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
    if (!ok && lane == 0) report_error(kErrPrefillWait);
  } else if (warp == kSkinnyMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the issue loop, so the B descriptors (one base per activation
    // stage plus 32-bit adds to the low half, which holds the start address in 16-byte
    // units) and the TMEM addresses are warp-uniform; the elected lane issues the MMAs
    // and commits. One wait per slot group, then its 16 MMAs back to back.
    const uint32_t leader = elect_one_sync();
    int gst = 0, gsg = 0, it = 0;
    uint32_t acc_armed[2] = {};
    const uint64_t desc0 = umma_desc_sw128(0);
    const uint32_t desc_hi = static_cast<uint32_t>(desc0 >> 32);
    // low descriptor half of activation stage 0's first tile (start address >> 4)
    const uint32_t b_lo_base = static_cast<uint32_t>(desc0) | ((smem_u32(xring) >> 4) & 0x3FFFu);
    constexpr uint32_t kStageLo = C::XS_BYTES >> 4;
    constexpr uint32_t kTileLo = C::XT_BYTES >> 4;
    for (int u = blockIdx.x; u < a.units && ok; u += G, ++it) {
      const int p = u / a.tiles;
      const int st0 = p * a.kbp;
      const int st1 = min(num_st, st0 + a.kbp);
      const int nb = (min(K, st1 * C::SK) - st0 * C::SK) >> 6;
      const int ngr = (nb + 3) >> 2;
      const int ab = it & 1;
      const uint32_t aphase = (it >> 1) & 1;
      if (!mbar_wait_warp(&accempty[ab], aphase ^ 1)) { ok = false; break; }
      tc_fence_after();
      const uint32_t d = tmem_base + ab * C::kBN;
      for (int g = 0; g < ngr; ++g) {
        const int gq = gsg + g;
        const int sg = gq % NG;
        const int b0 = 4 * g;                       // first block; it opens an activation stage
        const int sq0 = gst + b0 / C::KB;
        const int x0 = sq0 % SX;
        if (!mbar_wait_warp(&afull[sg], (gq / NG) & 1)) { ok = false; break; }
        if (!mbar_wait_warp(&xfull[x0], (sq0 / SX) & 1)) { ok = false; break; }
        const uint32_t a_g = tmem_base + C::ACC_COLS + sg * (kSkinnyGroupBlocks * 32);
        const uint32_t lo0 = b_lo_base + x0 * kStageLo;
        if (b0 + 4 <= nb) {
          // whole slot group: one INT4 stage, or two INT8 stages
          if constexpr (C::KB == 4) {
            tc_fence_after();
            if (g == 0) skinny_mma_block<true, C>(d, a_g, lo0, desc_hi, leader);
            else skinny_mma_block<false, C>(d, a_g, lo0, desc_hi, leader);
            skinny_mma_block<false, C>(d, a_g + 32, lo0 + kTileLo, desc_hi, leader);
            skinny_mma_block<false, C>(d, a_g + 64, lo0 + 2 * kTileLo, desc_hi, leader);
            skinny_mma_block<false, C>(d, a_g + 96, lo0 + 3 * kTileLo, desc_hi, leader);
            umma_commit_elected(&aempty[sg], leader);
            umma_commit_elected(&xempty[x0], leader);
          } else {
            const int x1 = (x0 + 1 == SX) ? 0 : x0 + 1;
            if (!mbar_wait_warp(&xfull[x1], ((sq0 + 1) / SX) & 1)) { ok = false; break; }
            tc_fence_after();
            const uint32_t lo1 = b_lo_base + x1 * kStageLo;
            if (g == 0) skinny_mma_block<true, C>(d, a_g, lo0, desc_hi, leader);
            else skinny_mma_block<false, C>(d, a_g, lo0, desc_hi, leader);
            skinny_mma_block<false, C>(d, a_g + 32, lo0 + kTileLo, desc_hi, leader);
            skinny_mma_block<false, C>(d, a_g + 64, lo1, desc_hi, leader);
            skinny_mma_block<false, C>(d, a_g + 96, lo1 + kTileLo, desc_hi, leader);
            umma_commit_elected(&aempty[sg], leader);
            umma_commit_elected(&xempty[x0], leader);
            umma_commit_elected(&xempty[x1], leader);
          }
        } else {
          // the unit's last, partial slot group
          tc_fence_after();
          for (int b = b0; b < nb; ++b) {
            const int sq = gst + b / C::KB;
            const int x = sq % SX;
            if (b > b0 && b % C::KB == 0) {
              if (!mbar_wait_warp(&xfull[x], (sq / SX) & 1)) { ok = false; break; }
              tc_fence_after();
            }
            const uint32_t lo = b_lo_base + x * kStageLo + (b % C::KB) * kTileLo;
            if (b == 0) skinny_mma_block<true, C>(d, a_g + (b - b0) * 32, lo, desc_hi, leader);
            else skinny_mma_block<false, C>(d, a_g + (b - b0) * 32, lo, desc_hi, leader);
            if (b % C::KB == C::KB - 1 || b == nb - 1) umma_commit_elected(&xempty[x], leader);
          }
          if (!ok) break;
          umma_commit_elected(&aempty[sg], leader);
        }
      }
      if (!ok) break;
      umma_commit_elected(&accfull[ab], leader);
      acc_armed[ab] = aphase + 1;
      gst += st1 - st0;
      gsg += ngr;
    }
    bool drained = true;
    for (int b = 0; b < 2; ++b)
      if (acc_armed[b] && !mbar_wait_drain_warp(&accfull[b], acc_armed[b] - 1)) drained = false;
    if (!ok) {
      // a wait gave up mid-unit: MMAs may have been issued after the last commit above
      umma_commit_elected(final_bar, leader);
      if (!mbar_wait_drain_warp(final_bar, 0)) drained = false;
    }
    if ((!ok || !drained) && lane == 0) report_error(kErrPrefillWait);
  } else {
    // ------------------------------------------------------------ epilogue warps 12..15
    griddep_wait();   // (its first output follows the activations anyway)
    const int quarter = warp & 3;
    const bool split = a.parts > 1;
    int it = 0;
    for (int u = blockIdx.x; u < a.units && ok; u += G, ++it) {
      const int ab = it & 1;
      const uint32_t aphase = (it >> 1) & 1;
      if (!mbar_wait_warp(&accfull[ab], aphase)) { ok = false; break; }
      tc_fence_after();
      const int t = u % a.tiles;
      const int nt = t / a.tiles_m;
      const int mt = t - nt * a.tiles_m;
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
