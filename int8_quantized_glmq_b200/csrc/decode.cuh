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
//  * persistent CTAs (one per SM), each owning the row tiles b, b+G, b+2G, ...
//    (R = 16*ROWG rows per tile), processed in groups of up to kTileGroup tiles;
//  * warp 8 is a producer: it copies the packed rows of each stage (R rows x
//    SB bytes) with cp.async.bulk into a kStages-deep shared-memory ring (row
//    pitch padded so the consumers' 16-byte reads are bank-conflict free), with
//    an L2 evict-first hint, and the activation rows of the current K pass into
//    a padded X buffer (double-buffered when X does not fit at once);
//  * warps 0..7 are consumers: warp w takes segment w (SEGB bytes per row) of
//    every stage for all R rows, dequantizes codes in registers with exponent
//    bias tricks (a code c becomes the fp16 number 1024 + (c ^ 8) by OR-ing it
//    into the mantissa, then one subtraction), and feeds mma.sync m16n8k16 with
//    the weights as the A operand straight from registers and X as B. The K
//    order inside each MMA is permuted identically on both operands so that
//    each 32-bit packed word feeds two MMAs without a byte shuffle;
//  * the 8 consumer warps each hold a K-slice partial of every output; they add
//    it into a per-tile fp32 accumulator in shared memory with red.shared.add
//    (no barrier), and after the last K pass the tile is scaled by s[n],
//    rounded to fp16 and stored.
#pragma once

#include "glmq_ptx.cuh"

namespace glmq {

constexpr int kDecodeConsumerWarps = 8;
constexpr int kDecodeThreads = (kDecodeConsumerWarps + 1) * 32;
constexpr int kDecodeStages = 4;
constexpr int kTileGroup = 8;

template <int BITS, int NB, int SEGB, int ROWG>
struct DecodeCfg {
  static constexpr int kBits = BITS;
  static constexpr int kNB = NB;            // n8 token blocks: 1 for M <= 8, 2 for M <= 16
  static constexpr int kSegB = SEGB;        // packed bytes per row per consumer warp per stage
  static constexpr int kRowG = ROWG;        // 16-row groups per tile
  static constexpr int R = 16 * ROWG;       // rows per tile
  static constexpr int SB = SEGB * kDecodeConsumerWarps;  // packed bytes per row per stage
  static constexpr int KPB = (BITS == 4) ? 2 : 1;         // codes per byte
  static constexpr int SK = SB * KPB;       // k per stage
  static constexpr int SEGK = SEGB * KPB;   // k per segment
  static constexpr int TB = SEGB / 4;       // packed bytes per thread per row per segment
  static constexpr int TK = TB * KPB;       // k per thread per segment
  static constexpr int TW = TB / 4;         // 32-bit words per thread per row per segment
  static constexpr int WPAD = (SEGB == 128) ? 16 : 64;
  static constexpr int WPITCH = SB + WPAD;
  static constexpr int STAGE_BYTES = R * WPITCH;
  // X row pitch must shift a token's bank group by this many 16-byte units.
  static constexpr int XSHIFT = (BITS == 4) ? ((SEGB == 128) ? 4 : 2) : ((SEGB == 128) ? 2 : 1);
  static constexpr int ACC_BYTES = kTileGroup * R * 16 * 4;
  static constexpr int FIXED_SMEM = kDecodeStages * STAGE_BYTES + ACC_BYTES + 256;
  static_assert(TB == 16 || TB == 32, "thread slice is one or two 16-byte loads");
  static_assert(R <= 64, "producer lanes cover at most two rows each");
};

// Byte offset of element k inside a padded X row: 16 bytes of padding after every 128.
__host__ __device__ constexpr uint32_t x_off(uint32_t k) { return 2u * k + (k >> 6) * 16u; }

__host__ __device__ constexpr uint32_t x_pitch(uint32_t kp, int xshift) {
  const uint32_t base = x_off(kp);
  const uint32_t want = static_cast<uint32_t>(xshift) * 16u;
  return base + ((want + 128u - (base & 127u)) & 127u);
}

struct DecodeArgs {
  const __half* X;
  const uint8_t* packed;
  const __half* scale;
  __half* Y;
  int M;
  int N;
  int K;
  int KP;       // k per pass (multiple of SK)
  int passes;
  int XP;       // X row pitch in shared memory (bytes)
  int xbufs;    // 1 (X resident for the whole kernel) or 2 (double-buffered passes)
  int tiles;
};

// ---------------------------------------------------------------- dequantization
// INT4: one packed word (8 codes, k = 0..7 of the word) -> 4 half2 registers
// holding the pairs (0,4), (1,5), (2,6), (3,7).
__device__ __forceinline__ void dequant_int4_word(uint32_t w, uint32_t (&p)[4]) {
  const __half2 kBias0 = __halves2half2(__ushort_as_half(0xE408), __ushort_as_half(0xE408));  // -1032
  const __half2 kOne16 = __halves2half2(__ushort_as_half(0x2C00), __ushort_as_half(0x2C00));  // 1/16
  const __half2 kBias1 = __halves2half2(__ushort_as_half(0xD480), __ushort_as_half(0xD480));  // -72
  const uint32_t w8 = w >> 8;
  uint32_t h0 = lop3_and_xor(w, 0x000F000Fu, 0x64086408u);
  uint32_t h1 = lop3_and_xor(w, 0x00F000F0u, 0x64806480u);
  uint32_t h2 = lop3_and_xor(w8, 0x000F000Fu, 0x64086408u);
  uint32_t h3 = lop3_and_xor(w8, 0x00F000F0u, 0x64806480u);
  __half2 r0 = __hadd2(*reinterpret_cast<__half2*>(&h0), kBias0);
  __half2 r1 = __hfma2(*reinterpret_cast<__half2*>(&h1), kOne16, kBias1);
  __half2 r2 = __hadd2(*reinterpret_cast<__half2*>(&h2), kBias0);
  __half2 r3 = __hfma2(*reinterpret_cast<__half2*>(&h3), kOne16, kBias1);
  p[0] = *reinterpret_cast<uint32_t*>(&r0);
  p[1] = *reinterpret_cast<uint32_t*>(&r1);
  p[2] = *reinterpret_cast<uint32_t*>(&r2);
  p[3] = *reinterpret_cast<uint32_t*>(&r3);
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

// ---------------------------------------------------------------- the kernel
template <class C>
__global__ void __launch_bounds__(kDecodeThreads, 1) decode_kernel(const DecodeArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* wring = smem;
  float* acc_s = reinterpret_cast<float*>(smem + kDecodeStages * C::STAGE_BYTES);
  uint8_t* xbuf = smem + kDecodeStages * C::STAGE_BYTES + C::ACC_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(xbuf + a.xbufs * a.M * a.XP);
  uint64_t* full = bars;
  uint64_t* empty = bars + kDecodeStages;
  uint64_t* xfull = bars + 2 * kDecodeStages;
  uint64_t* xempty = xfull + 2;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int M = a.M, N = a.N, K = a.K;
  const long long row_bytes = static_cast<long long>(K) / C::KPB;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kDecodeStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kDecodeConsumerWarps);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&xfull[b], 1);
      mbar_init(&xempty[b], kDecodeConsumerWarps);
    }
    fence_barrier_init();
  }
  if (warp < kDecodeConsumerWarps) {
    for (int i = threadIdx.x; i < kTileGroup * C::R * 16; i += kDecodeConsumerWarps * 32) acc_s[i] = 0.0f;
  }
  __syncthreads();

  const int G = gridDim.x;
  const int multi = a.passes > 1;

  if (warp == kDecodeConsumerWarps) {
    // ------------------------------------------------------------ producer warp
    const uint64_t pol = policy_evict_first();
    int stage = 0;
    uint32_t phase = 0;
    int xb = 0;
    uint32_t xphase = 0;
    bool x_loaded = false;
    bool ok = true;
    // parity + 1 of the last phase each barrier was armed with (0 = never armed)
    uint32_t armed[kDecodeStages] = {};
    uint32_t xarmed[2] = {};
    for (int g0 = blockIdx.x; g0 < a.tiles && ok; g0 += G * kTileGroup) {
      for (int p = 0; p < a.passes && ok; ++p) {
        const int pk0 = p * a.KP;
        const int plen = min(a.KP, K - pk0);
        if (multi || !x_loaded) {
          if (multi && !mbar_wait_warp(&xempty[xb], xphase ^ 1)) { ok = false; break; }
          if (lane == 0) mbar_arrive_expect_tx(&xfull[xb], static_cast<uint32_t>(M) * plen * 2u);
          xarmed[xb] = xphase + 1;
          __syncwarp();
          const int pieces_per_row = plen >> 6;
          uint8_t* xdst = xbuf + xb * M * a.XP;
          for (int i = lane; i < M * pieces_per_row; i += 32) {
            const int n = i / pieces_per_row;
            const int pc = i - n * pieces_per_row;
            bulk_g2s(xdst + n * a.XP + x_off(pc * 64),
                     a.X + static_cast<long long>(n) * K + pk0 + pc * 64, 128u, &xfull[xb]);
          }
          x_loaded = true;
          if (multi) { xb ^= 1; if (xb == 0) xphase ^= 1; }
        }
        const int nst = (plen + C::SK - 1) / C::SK;
        for (int tt = 0; tt < kTileGroup && ok; ++tt) {
          const int tile = g0 + tt * G;
          if (tile >= a.tiles) break;
          const int row0 = tile * C::R;
          for (int ks = 0; ks < nst; ++ks) {
            if (!mbar_wait_warp(&empty[stage], phase ^ 1)) { ok = false; break; }
            const int k0 = pk0 + ks * C::SK;
            const uint32_t bytes = static_cast<uint32_t>(min(C::SB, static_cast<int>((K - k0) / C::KPB)));
            if (lane == 0) mbar_arrive_expect_tx(&full[stage], bytes * C::R);
            armed[stage] = phase + 1;
            __syncwarp();
            uint8_t* dst = wring + stage * C::STAGE_BYTES;
#pragma unroll
            for (int i = lane; i < C::R; i += 32) {
              const long long grow = min(row0 + i, N - 1);
              bulk_g2s_stream(dst + i * C::WPITCH, a.packed + grow * row_bytes + k0 / C::KPB, bytes,
                              &full[stage], pol);
            }
            if (++stage == kDecodeStages) { stage = 0; phase ^= 1; }
          }
        }
      }
    }
    // Do not leave while copies into this CTA's shared memory may be in flight:
    // wait (bounded) until the last phase armed on every barrier has landed.
    bool drained = true;
#pragma unroll
    for (int s = 0; s < kDecodeStages; ++s)
      if (armed[s] && !mbar_wait(&full[s], armed[s] - 1)) drained = false;
    for (int b = 0; b < 2; ++b)
      if (xarmed[b] && !mbar_wait(&xfull[b], xarmed[b] - 1)) drained = false;
    if ((!ok || !drained) && lane == 0) report_error(kErrDecodeProducerWait);
    return;
  }

  // -------------------------------------------------------------- consumer warps
  const int r = lane >> 2;
  const int c = lane & 3;
  int stage = 0;
  uint32_t phase = 0;
  int xb = 0;
  uint32_t xphase = 0;
  bool x_ready = false;
  bool ok = true;
  const uint32_t wring_u32 = smem_u32(wring);
  const uint32_t acc_u32 = smem_u32(acc_s);

  for (int g0 = blockIdx.x; g0 < a.tiles; g0 += G * kTileGroup) {
    for (int p = 0; p < a.passes; ++p) {
      const int pk0 = p * a.KP;
      const int plen = min(a.KP, K - pk0);
      const int xcur = multi ? xb : 0;
      if (ok && (multi || !x_ready)) {
        if (!mbar_wait_warp(&xfull[xcur], xphase)) ok = false;
        x_ready = true;
      }
      const uint32_t xrow[2] = {
          smem_u32(xbuf + xcur * M * a.XP + min(r, M - 1) * a.XP),
          smem_u32(xbuf + xcur * M * a.XP + min(r + 8, M - 1) * a.XP)};
      const int nst = (plen + C::SK - 1) / C::SK;
      for (int tt = 0; tt < kTileGroup; ++tt) {
        const int tile = g0 + tt * G;
        if (tile >= a.tiles) break;
        float acc[C::kRowG][C::kNB][4];
#pragma unroll
        for (int g = 0; g < C::kRowG; ++g)
#pragma unroll
          for (int nb = 0; nb < C::kNB; ++nb)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[g][nb][i] = 0.0f;

        for (int ks = 0; ks < nst; ++ks) {
          if (ok && !mbar_wait_warp(&full[stage], phase)) ok = false;
          const int kl = ks * C::SK + warp * C::SEGK;  // pass-relative k of this warp's segment
          if (ok && pk0 + kl < K) {
            const bool valid = pk0 + kl + c * C::TK < K;
            const uint32_t wbase = wring_u32 + stage * C::STAGE_BYTES + warp * C::kSegB + c * C::TB;
            // packed words of this thread: rows (16g + r) and (16g + r + 8)
            uint32_t wa[C::kRowG][C::TW], wb[C::kRowG][C::TW];
#pragma unroll
            for (int g = 0; g < C::kRowG; ++g) {
#pragma unroll
              for (int q = 0; q < C::TW / 4; ++q) {
                uint4 va = make_uint4(0, 0, 0, 0), vb = make_uint4(0, 0, 0, 0);
                if (valid) {
                  va = lds_v4(wbase + (16 * g + r) * C::WPITCH + 16 * q);
                  vb = lds_v4(wbase + (16 * g + r + 8) * C::WPITCH + 16 * q);
                }
                wa[g][4 * q + 0] = va.x; wa[g][4 * q + 1] = va.y; wa[g][4 * q + 2] = va.z; wa[g][4 * q + 3] = va.w;
                wb[g][4 * q + 0] = vb.x; wb[g][4 * q + 1] = vb.y; wb[g][4 * q + 2] = vb.z; wb[g][4 * q + 3] = vb.w;
              }
            }
            const uint32_t xk = kl + c * C::TK;  // pass-relative k of this thread's slice
            if constexpr (C::kBits == 4) {
#pragma unroll
              for (int j = 0; j < C::TW; ++j) {
                uint32_t bf[C::kNB][4];
#pragma unroll
                for (int nb = 0; nb < C::kNB; ++nb) {
                  uint4 xv = make_uint4(0, 0, 0, 0);
                  if (valid) xv = lds_v4(xrow[nb] + x_off(xk + 8 * j));
                  bf[nb][0] = prmt(xv.x, xv.z, 0x5410u);  // (x0, x4)
                  bf[nb][1] = prmt(xv.x, xv.z, 0x7632u);  // (x1, x5)
                  bf[nb][2] = prmt(xv.y, xv.w, 0x5410u);  // (x2, x6)
                  bf[nb][3] = prmt(xv.y, xv.w, 0x7632u);  // (x3, x7)
                }
#pragma unroll
                for (int g = 0; g < C::kRowG; ++g) {
                  uint32_t pa[4], pb[4];
                  dequant_int4_word(wa[g][j], pa);
                  dequant_int4_word(wb[g][j], pb);
#pragma unroll
                  for (int nb = 0; nb < C::kNB; ++nb) {
                    mma_16816(acc[g][nb], pa[0], pb[0], pa[1], pb[1], bf[nb][0], bf[nb][1]);
                    mma_16816(acc[g][nb], pa[2], pb[2], pa[3], pb[3], bf[nb][2], bf[nb][3]);
                  }
                }
              }
            } else {
#pragma unroll
              for (int j2 = 0; j2 < C::TW / 2; ++j2) {
                uint32_t bf[C::kNB][4];
#pragma unroll
                for (int nb = 0; nb < C::kNB; ++nb) {
                  uint4 xv = make_uint4(0, 0, 0, 0);
                  if (valid) xv = lds_v4(xrow[nb] + x_off(xk + 8 * j2));
                  bf[nb][0] = xv.x; bf[nb][1] = xv.y; bf[nb][2] = xv.z; bf[nb][3] = xv.w;
                }
#pragma unroll
                for (int g = 0; g < C::kRowG; ++g) {
#pragma unroll
                  for (int h = 0; h < 2; ++h) {
                    uint32_t pa[2], pb[2];
                    dequant_int8_word(wa[g][2 * j2 + h], pa);
                    dequant_int8_word(wb[g][2 * j2 + h], pb);
#pragma unroll
                    for (int nb = 0; nb < C::kNB; ++nb)
                      mma_16816(acc[g][nb], pa[0], pb[0], pa[1], pb[1], bf[nb][2 * h], bf[nb][2 * h + 1]);
                  }
                }
              }
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&empty[stage]);
          if (++stage == kDecodeStages) { stage = 0; phase ^= 1; }
        }
        // add this warp's K-slice partial into the tile accumulator
        const uint32_t tbase = acc_u32 + tt * (C::R * 16 * 4);
#pragma unroll
        for (int g = 0; g < C::kRowG; ++g) {
#pragma unroll
          for (int nb = 0; nb < C::kNB; ++nb) {
            const int t0 = 8 * nb + 2 * c;
            const int ra = 16 * g + r;
            if (t0 < M) {
              red_shared_add_f32(tbase + (ra * 16 + t0) * 4, acc[g][nb][0]);
              red_shared_add_f32(tbase + ((ra + 8) * 16 + t0) * 4, acc[g][nb][2]);
            }
            if (t0 + 1 < M) {
              red_shared_add_f32(tbase + (ra * 16 + t0 + 1) * 4, acc[g][nb][1]);
              red_shared_add_f32(tbase + ((ra + 8) * 16 + t0 + 1) * 4, acc[g][nb][3]);
            }
          }
        }
      }
      if (multi) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&xempty[xcur]);
        xb ^= 1;
        if (xb == 0) xphase ^= 1;
      }
    }
    // epilogue of the tile group: scale, round to fp16, store
    named_barrier_sync(1, kDecodeConsumerWarps * 32);
    const int ct = threadIdx.x;
    for (int tt = 0; tt < kTileGroup; ++tt) {
      const int tile = g0 + tt * G;
      if (tile >= a.tiles) break;
      const int row0 = tile * C::R;
      float* tacc = acc_s + tt * C::R * 16;
      for (int i = ct; i < M * C::R; i += kDecodeConsumerWarps * 32) {
        const int m = i / C::R;
        const int rr = i - m * C::R;
        const int grow = row0 + rr;
        const float v = tacc[rr * 16 + m];
        tacc[rr * 16 + m] = 0.0f;
        if (grow < N) {
          const float s = __half2float(a.scale[grow]);
          a.Y[static_cast<long long>(m) * N + grow] = __float2half_rn(s * v);
        }
      }
    }
    named_barrier_sync(1, kDecodeConsumerWarps * 32);
  }
  if (!ok && lane == 0) report_error(kErrDecodeConsumerWait);
}

}  // namespace glmq
