// glmq C ABI: argument validation, per-device set-up and kernel dispatch.
// The operations and their readings are documented in include/glmq.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <mutex>

#include "glmq.h"
#include "decode.cuh"
#include "finalize.cuh"
#include "prefill.cuh"
#include "quantize.cuh"
#include "skinny.cuh"

namespace {

using namespace glmq;

thread_local int t_last_cuda_error = 0;

struct DeviceInfo {
  bool init = false;
  bool supported = false;
  int sms = 0;
  int smem_optin = 0;
};

constexpr int kMaxDevices = 64;
DeviceInfo g_devices[kMaxDevices];
std::mutex g_mutex;

glmq_status cuda_fail(cudaError_t e) {
  t_last_cuda_error = static_cast<int>(e);
  return GLMQ_ERR_CUDA;
}

// Kernels enqueued by this library since it was loaded (glmq_kernel_launches).
std::atomic<unsigned long long> g_kernel_launches{0};

// Status of the kernel launch just made on this thread; an accepted launch is counted.
glmq_status launched() {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e);
  g_kernel_launches.fetch_add(1, std::memory_order_relaxed);
  return GLMQ_OK;
}

// Launches kernel<<<grid, block, smem, s>>>(args...) with programmatic stream
// serialization: it may begin (its shared-memory prologue) while the previous kernel
// in the stream drains, and waits for that kernel (griddep_wait) before it touches
// anything an earlier kernel may write. (The finalize pass and the skinny kernel read
// per-layer constants earlier; finalize.cuh and launch_skinny_cfg state why that is
// safe.) Counted like launched().
template <typename... KArgs, typename... Args>
glmq_status launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args...);
  if (e != cudaSuccess) return cuda_fail(e);
  return launched();
}

// Current device's properties (queried once per device). Returns an error
// status when the device is unusable.
glmq_status current_device(const DeviceInfo** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= kMaxDevices) return GLMQ_ERR_UNSUPPORTED_DEVICE;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceInfo& d = g_devices[dev];
  if (!d.init) {
    int major = 0, minor = 0;
    if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess) return cuda_fail(e);
    if ((e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess) return cuda_fail(e);
    if ((e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return cuda_fail(e);
    if ((e = cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess)
      return cuda_fail(e);
    d.supported = (major == 10 && minor == 0);
    d.init = true;
  }
  if (!d.supported) return GLMQ_ERR_UNSUPPORTED_DEVICE;
  *out = &d;
  return GLMQ_OK;
}

// Per-device, per-kernel opt-in to large dynamic shared memory. The attribute is
// raised only when a launch needs more than was granted before, so steady-state
// calls make no extra CUDA runtime call. Entries are keyed by the kernel's
// address (every instantiation of a kernel template has the same type).
struct SmemGrant {
  const void* fn;
  int dev;
  int bytes;
};
constexpr int kMaxGrants = 256;
SmemGrant g_grants[kMaxGrants];
int g_num_grants = 0;

template <class Kernel>
glmq_status allow_smem(Kernel kernel, int bytes) {
  const void* fn = reinterpret_cast<const void*>(kernel);
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= kMaxDevices) return GLMQ_ERR_UNSUPPORTED_DEVICE;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (bytes > g_devices[dev].smem_optin) return GLMQ_ERR_BAD_SHAPE;
  SmemGrant* g = nullptr;
  for (int i = 0; i < g_num_grants; ++i)
    if (g_grants[i].fn == fn && g_grants[i].dev == dev) g = &g_grants[i];
  if (g && bytes <= g->bytes) return GLMQ_OK;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return cuda_fail(e);
  if (!g && g_num_grants < kMaxGrants) g = &g_grants[g_num_grants++];
  if (g) *g = SmemGrant{fn, dev, bytes};
  return GLMQ_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

glmq_status check_common(int64_t N, int64_t K, int bits) {
  if (bits != 4 && bits != 8) return GLMQ_ERR_BAD_BITS;
  if (N < 0 || N > 0x7fffffffLL) return GLMQ_ERR_BAD_SHAPE;
  if (K <= 0 || (K % 64) != 0 || K > GLMQ_MAX_K) return GLMQ_ERR_BAD_SHAPE;
  return GLMQ_OK;
}

glmq_status check_gemm(const void* X, int64_t M, const void* packed, const void* scale, int64_t N, int64_t K,
                       int bits, void* Y) {
  glmq_status st = check_common(N, K, bits);
  if (st != GLMQ_OK) return st;
  if (M < 0 || M > 0x7fffffffLL) return GLMQ_ERR_BAD_SHAPE;
  if (M == 0 || N == 0) return GLMQ_OK;
  if (M * N > (int64_t(1) << 46)) return GLMQ_ERR_BAD_SHAPE;
  if (!X || !packed || !scale || !Y) return GLMQ_ERR_NULL_POINTER;
  if (!aligned16(X) || !aligned16(packed) || !aligned16(scale) || !aligned16(Y)) return GLMQ_ERR_MISALIGNED;
  return GLMQ_OK;
}

// ---------------------------------------------------------------- quantize
template <int BITS, int CPT, int T>
glmq_status launch_quantize_cpt(const void* W, int64_t N, int64_t K, void* packed, void* scale, int geglu_half,
                                cudaStream_t s) {
  quantize_kernel<BITS, CPT, T><<<static_cast<unsigned>(N), T, 0, s>>>(
      static_cast<const __half*>(W), static_cast<int>(K), static_cast<uint8_t*>(packed), static_cast<__half*>(scale),
      geglu_half);
  return launched();
}

// Block size and chunks per thread from the row length (K <= GLMQ_MAX_K: at most
// 8192 chunks of 8 values): 256 threads up to 6 chunks each, then 512 or 1024
// threads with at most 8 chunks each.
template <int BITS>
glmq_status launch_quantize(const void* W, int64_t N, int64_t K, void* packed, void* scale, int geglu_half,
                            cudaStream_t s) {
  const int64_t chunks = K / 8;
  if (chunks <= 256) return launch_quantize_cpt<BITS, 1, 256>(W, N, K, packed, scale, geglu_half, s);
  if (chunks <= 512) return launch_quantize_cpt<BITS, 2, 256>(W, N, K, packed, scale, geglu_half, s);
  if (chunks <= 1024) return launch_quantize_cpt<BITS, 4, 256>(W, N, K, packed, scale, geglu_half, s);
  if (chunks <= 1536) return launch_quantize_cpt<BITS, 6, 256>(W, N, K, packed, scale, geglu_half, s);
  if (chunks <= 2048) return launch_quantize_cpt<BITS, 4, 512>(W, N, K, packed, scale, geglu_half, s);
  if (chunks <= 3072) return launch_quantize_cpt<BITS, 6, 512>(W, N, K, packed, scale, geglu_half, s);
  if (chunks <= 4096) return launch_quantize_cpt<BITS, 8, 512>(W, N, K, packed, scale, geglu_half, s);
  if (chunks <= 6144) return launch_quantize_cpt<BITS, 6, 1024>(W, N, K, packed, scale, geglu_half, s);
  return launch_quantize_cpt<BITS, 8, 1024>(W, N, K, packed, scale, geglu_half, s);
}

template <int CPT, int T>
glmq_status launch_quantize_zp_cpt(const void* W, int64_t N, int64_t K, void* packed, void* scale, void* zero,
                                   cudaStream_t s) {
  quantize_zp_kernel<CPT, T><<<static_cast<unsigned>(N), T, 0, s>>>(
      static_cast<const __half*>(W), static_cast<int>(K), static_cast<uint8_t*>(packed), static_cast<__half*>(scale),
      static_cast<uint8_t*>(zero));
  return launched();
}

// Same block-size choice as launch_quantize.
glmq_status launch_quantize_zp(const void* W, int64_t N, int64_t K, void* packed, void* scale, void* zero,
                               cudaStream_t s) {
  const int64_t chunks = K / 8;
  if (chunks <= 256) return launch_quantize_zp_cpt<1, 256>(W, N, K, packed, scale, zero, s);
  if (chunks <= 512) return launch_quantize_zp_cpt<2, 256>(W, N, K, packed, scale, zero, s);
  if (chunks <= 1024) return launch_quantize_zp_cpt<4, 256>(W, N, K, packed, scale, zero, s);
  if (chunks <= 1536) return launch_quantize_zp_cpt<6, 256>(W, N, K, packed, scale, zero, s);
  if (chunks <= 2048) return launch_quantize_zp_cpt<4, 512>(W, N, K, packed, scale, zero, s);
  if (chunks <= 3072) return launch_quantize_zp_cpt<6, 512>(W, N, K, packed, scale, zero, s);
  if (chunks <= 4096) return launch_quantize_zp_cpt<8, 512>(W, N, K, packed, scale, zero, s);
  if (chunks <= 6144) return launch_quantize_zp_cpt<6, 1024>(W, N, K, packed, scale, zero, s);
  return launch_quantize_zp_cpt<8, 1024>(W, N, K, packed, scale, zero, s);
}

// ---------------------------------------------------------------- TMA descriptors
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

glmq_status make_map_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t inner, uint64_t outer,
                        uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = encode_tiled_fn();
  if (!fn) return cuda_fail(cudaErrorInitializationError);
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_stride_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cuda_fail(cudaErrorInvalidValue);
  return GLMQ_OK;
}

// ---------------------------------------------------------------- decode scratch
// fp32 [M, N] partial sums for decode calls whose tiles are split over several K
// parts. Allocated once per device on first use (grown when a larger problem
// arrives) and zeroed at allocation; the finalize kernel returns it to zero.
struct DecodeScratch {
  float* ws = nullptr;
  size_t ws_elems = 0;
  uint8_t* xs = nullptr;     // skinny kernel's activation image
  size_t xs_bytes = 0;
};
DecodeScratch g_scratch[kMaxDevices];

glmq_status decode_scratch(size_t ws_elems, float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  std::lock_guard<std::mutex> lock(g_mutex);
  DecodeScratch& sc = g_scratch[dev];
  if (sc.ws_elems < ws_elems) {
    if (sc.ws) cudaFree(sc.ws);
    sc.ws = nullptr;
    sc.ws_elems = 0;
    if ((e = cudaMalloc(&sc.ws, ws_elems * sizeof(float))) != cudaSuccess) return cuda_fail(e);
    if ((e = cudaMemset(sc.ws, 0, ws_elems * sizeof(float))) != cudaSuccess) return cuda_fail(e);
    sc.ws_elems = ws_elems;
  }
  *out = sc.ws;
  return GLMQ_OK;
}

// Per-call options of a GEMM call: the fused epilogue (epilogue.cuh: optional bias,
// optional GeGLU), zero-point codes, and the decode kernel's next-call prefetch hint.
struct Epi {
  const __half* bias = nullptr;
  int geglu = 0;
  const uint8_t* zero = nullptr;   // zero-point INT4 codes: per-row zero points
  const void* next_packed = nullptr;   // glmq_gemm_decode_prefetch: the next call's weights
  int next_M = 0, next_N = 0, next_K = 0;
};

// Launches finalize_epilogue_kernel: one thread per output column of every token row.
// Columns (packed rows of W) n0 .. N-1 only: the rows of the tiles that were split.
glmq_status launch_finalize_epi(float* ws, const __half* scale, const Epi& e, __half* Y, int M, int N,
                                cudaStream_t s, int n0 = 0) {
  const int width = e.geglu ? N / 2 : N;
  const int j0 = e.geglu ? n0 / 2 : n0;
  const dim3 grid(static_cast<unsigned>((width - j0 + 255) / 256), static_cast<unsigned>(std::min(M, 65535)));
  return launch_pdl(finalize_epilogue_kernel, grid, dim3(256), 0, s, ws, scale, e.bias, e.geglu, Y, M, N, j0);
}

// Launches decode_finalize_kernel: one thread per group of 4 columns and block of
// kFinalizeRows token rows (per column and row when N is not a multiple of 4), all in
// one pass (rows beyond the grid's y extent loop).
// Columns n0 .. N-1 only (n0 a multiple of 16): the rows of the tiles that were split.
glmq_status launch_finalize(float* ws, const __half* scale, __half* Y, int M, int N, cudaStream_t s, int n0 = 0) {
  const bool vec = (N % 4) == 0;
  const int groups = vec ? (N - n0) / 4 : N - n0;
  const int rows = vec ? (M + kFinalizeRows - 1) / kFinalizeRows : M;
  const dim3 grid(static_cast<unsigned>((groups + 255) / 256), static_cast<unsigned>(std::min(rows, 65535)));
  if (vec) return launch_pdl(decode_finalize_kernel<4>, grid, dim3(256), 0, s, ws, scale, Y, M, N, n0);
  return launch_pdl(decode_finalize_kernel<1>, grid, dim3(256), 0, s, ws, scale, Y, M, N, n0);
}

// Per-device buffer for the skinny kernel's pre-swizzled activation tiles (grown on
// demand; fully rewritten by every call before it is read, so never cleared).
glmq_status skinny_x_scratch(size_t bytes, uint8_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  std::lock_guard<std::mutex> lock(g_mutex);
  DecodeScratch& sc = g_scratch[dev];
  if (sc.xs_bytes < bytes) {
    if (sc.xs) cudaFree(sc.xs);
    sc.xs = nullptr;
    sc.xs_bytes = 0;
    if ((e = cudaMalloc(&sc.xs, bytes)) != cudaSuccess) return cuda_fail(e);
    sc.xs_bytes = bytes;
  }
  *out = sc.xs;
  return GLMQ_OK;
}

// ---------------------------------------------------------------- decode
struct DecodePlan {
  int KPP, parts, tiles, units, smem, grid, stages;
};

// Stages of the largest per-CTA share when `units` (tile, K part) units, enumerated
// K-part major (part p holds units p*tiles .. p*tiles + tiles - 1), are split into G
// contiguous ranges; every part has spp stages except the last, which has `last`.
long long max_cta_stages(long long tiles, int parts, int spp, int last, int G) {
  const long long units = tiles * parts;
  const long long last0 = (parts - 1) * tiles;      // first unit of the last part
  long long worst = 0;
  for (int b = 0; b < G; ++b) {
    const long long u0 = (b * units) / G, u1 = ((b + 1) * units) / G;
    const long long in_last = std::max(0LL, u1 - std::max(u0, last0));
    const long long w = (u1 - u0) * spp - in_last * (spp - last);
    worst = std::max(worst, w);
  }
  return worst;
}

// Choose the K-part length. Activations stream through the stages, so any split fits;
// parts only spread the (tile, part) units over the SMs. Among the part counts that
// split the K stages into parts of equal length (the last may be shorter), take the
// one whose most loaded CTA has the least work relative to a perfect spread,
// preferring fewer parts (each split tile costs a round trip of fp32 partial sums
// through the scratch buffer and a finalize launch).
template <class C>
bool plan_decode(const DeviceInfo& dev, int N, int K, DecodePlan* pl) {
  if (C::SMEM_BYTES > dev.smem_optin) return false;
  const int stages = (K + C::SK - 1) / C::SK;
  const long long tiles = (static_cast<long long>(N) + kDecodeRows - 1) / kDecodeRows;
  if (stages < 1 || tiles < 1 || tiles * stages > 0x7fffffffLL) return false;
  int parts = 1;
  double best = -1.0;
  for (int P = 1; P <= stages && P <= 32; ++P) {
    const int spp = (stages + P - 1) / P;
    if ((stages + spp - 1) / spp != P) continue;      // not a distinct split
    const long long units = tiles * P;
    const int G = static_cast<int>(units < dev.sms ? units : dev.sms);
    const int last = stages - (P - 1) * spp;
    const double eff = static_cast<double>(tiles * stages) /
                       (static_cast<double>(dev.sms) * max_cta_stages(tiles, P, spp, last, G));
    if (eff > best + 0.02) {
      best = eff;
      parts = P;
    }
  }
  const int spp = (stages + parts - 1) / parts;
  pl->KPP = spp * C::SK;
  pl->parts = (stages + spp - 1) / spp;
  pl->tiles = static_cast<int>(tiles);
  pl->units = pl->parts * pl->tiles;
  pl->grid = pl->units < dev.sms ? pl->units : dev.sms;
  pl->smem = C::SMEM_BYTES;
  pl->stages = C::kStages;
  return true;
}

// The decode plan of a call with M tokens (the kernel configuration launch_decode picks).
template <int BITS>
bool plan_decode_for(const DeviceInfo& dev, int M, int N, int K, DecodePlan* pl) {
  if (M <= 1) return plan_decode<DecodeCfg<BITS, 1>>(dev, N, K, pl);
  if (M <= 2) return plan_decode<DecodeCfg<BITS, 2>>(dev, N, K, pl);
  if (M <= 4) return plan_decode<DecodeCfg<BITS, 4>>(dev, N, K, pl);
  if (M <= 8) return plan_decode<DecodeCfg<BITS, 8>>(dev, N, K, pl);
  return plan_decode<DecodeCfg<BITS, 16>>(dev, N, K, pl);
}

template <class C>
glmq_status launch_decode_cfg(const DeviceInfo& dev, const void* X, int M, const void* packed, const void* scale,
                              int N, int K, void* Y, cudaStream_t s, const Epi& e = Epi()) {
  DecodePlan pl;
  if (!plan_decode<C>(dev, N, K, &pl)) return GLMQ_ERR_BAD_SHAPE;
  CUtensorMap tw;
  const uint64_t row_bytes = uint64_t(K) / C::KPB;
  glmq_status st = make_map_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, packed, row_bytes, N, row_bytes, kDecodeSegB,
                               kDecodeRows, CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != GLMQ_OK) return st;
  // the activations: box of SK values x MP token rows (rows past M read as zero)
  CUtensorMap tx;
  st = make_map_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, X, K, M, uint64_t(K) * 2, C::SK, C::kMP,
                   CU_TENSOR_MAP_SWIZZLE_NONE);
  if (st != GLMQ_OK) return st;
  // next-call hint: the same map and plan the next decode call will use
  CUtensorMap tn = tw;
  DecodePlan npl = {};
  if (e.next_packed) {
    if (!plan_decode_for<C::kBits>(dev, e.next_M, e.next_N, e.next_K, &npl)) return GLMQ_ERR_BAD_SHAPE;
    const uint64_t nrow = uint64_t(e.next_K) / C::KPB;
    st = make_map_2d(&tn, CU_TENSOR_MAP_DATA_TYPE_UINT8, e.next_packed, nrow, e.next_N, nrow, kDecodeSegB, kDecodeRows,
                     CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != GLMQ_OK) return st;
  }
  DecodeArgs a;
  a.X = static_cast<const __half*>(X);
  a.scale = static_cast<const __half*>(scale);
  a.Y = static_cast<__half*>(Y);
  a.ws = nullptr;
  a.zero = e.zero;
  a.bias = e.bias;
  a.geglu = e.geglu;
  a.M = M;
  a.N = N;
  a.K = K;
  a.KPP = pl.KPP;
  a.parts = pl.parts;
  a.tiles = pl.tiles;
  a.units = pl.units;
  a.nxt_grid = e.next_packed ? npl.grid : 0;
  a.nxt_units = npl.units;
  a.nxt_tiles = npl.tiles;
  a.nxt_KPP = npl.KPP;
  a.nxt_K = e.next_K;
  a.nxt_stages = npl.stages;
  if (pl.parts > 1 && (st = decode_scratch(static_cast<size_t>(M) * N, &a.ws)) != GLMQ_OK) return st;
  if ((st = allow_smem(decode_kernel<C>, pl.smem)) != GLMQ_OK) return st;
  if ((st = launch_pdl(decode_kernel<C>, dim3(pl.grid), dim3(C::kThreads), pl.smem, s, tw, tx, tn, a)) != GLMQ_OK)
    return st;
  if (pl.parts > 1) {
    st = (e.bias || e.geglu) ? launch_finalize_epi(a.ws, a.scale, e, a.Y, M, N, s)
                             : launch_finalize(a.ws, a.scale, a.Y, M, N, s);
    if (st != GLMQ_OK) return st;
  }
  return GLMQ_OK;
}

template <int BITS, int ZP = 0>
glmq_status launch_decode(const DeviceInfo& dev, const void* X, int M, const void* packed, const void* scale, int N,
                          int K, void* Y, cudaStream_t s, const Epi& e = Epi()) {
  if (M <= 1) return launch_decode_cfg<DecodeCfg<BITS, 1, 2, ZP>>(dev, X, M, packed, scale, N, K, Y, s, e);
  if (M <= 2) return launch_decode_cfg<DecodeCfg<BITS, 2, 2, ZP>>(dev, X, M, packed, scale, N, K, Y, s, e);
  if (M <= 4) return launch_decode_cfg<DecodeCfg<BITS, 4, 2, ZP>>(dev, X, M, packed, scale, N, K, Y, s, e);
  if (M <= 8) return launch_decode_cfg<DecodeCfg<BITS, 8, 2, ZP>>(dev, X, M, packed, scale, N, K, Y, s, e);
  return launch_decode_cfg<DecodeCfg<BITS, 16, 2, ZP>>(dev, X, M, packed, scale, N, K, Y, s, e);
}

// ---------------------------------------------------------------- prefill
// With at least as many tiles as SMs, whole tiles fill waves = tiles / sms rounds of
// the persistent CTAs, and a last, partial round would keep the CTAs that have a tile
// in it busy for a whole tile time while the others idle. Instead, the tiles from the
// weight-row band that contains tile waves * sms on (a band is tiles_m tiles, so the
// split tiles cover whole rows of W and the finalize pass covers only those rows) are
// split over P K parts: the first (tiles before the band) stay whole. The split units
// fill the CTAs left idle in the last whole round and then at most one more round of
// 1/P of a tile: about waves + 1/P tile times instead of waves + 1. Taken when P >= 2
// and the tile time saved (at ~10 TFLOP/s per SM) is above the ~5 us of a finalize
// launch. Sets *full and *parts; leaves them alone otherwise.
void plan_tail_split(int tiles, int tiles_m, int num_steps, int min_steps_per_part, int sms, double tile_flops,
                     int* full, int* parts) {
  if (tiles < sms || tiles % sms == 0) return;
  const int waves = tiles / sms;
  const int whole = (waves * sms / tiles_m) * tiles_m;
  const int rest = tiles - whole;
  const int idle = waves * sms - whole;            // CTAs without a whole tile in the last whole round
  int P = (sms + idle) / rest;
  if (P > num_steps / min_steps_per_part) P = num_steps / min_steps_per_part;
  if (P > 16) P = 16;
  if (P < 2) return;
  if (tile_flops * (1.0 - 1.0 / P) < 5e-6 * 1e13) return;
  *full = whole;
  *parts = P;
}

// Choose K parts for `tiles` tiles of `num_steps` K steps each: only when there are
// fewer tiles than SMs, the split that spreads (tile, part) units most evenly,
// preferring fewer parts (each split tile costs a round trip of fp32 partial sums
// through the scratch buffer and a finalize launch).
int plan_parts(int tiles, int num_steps, int min_steps_per_part, int sms) {
  int parts = 1;
  if (tiles < sms) {
    double best = 0.0;
    for (int P = 1; P <= 16 && P * min_steps_per_part <= num_steps; ++P) {
      const int units = tiles * P;
      const int grid = units < sms ? units : sms;
      const double eff = (static_cast<double>(units) / grid) / ((units + grid - 1) / grid) *
                         (static_cast<double>(grid) / sms);
      if (eff > best + 0.02) {
        best = eff;
        parts = P;
      }
    }
  }
  return parts;
}

template <class C>
glmq_status launch_prefill_cfg(const DeviceInfo& dev, const void* X, int M, const void* packed, const void* scale,
                               int N, int K, void* Y, cudaStream_t s, const Epi& e) {
  CUtensorMap tx, tw;
  glmq_status st = make_map_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, X, K, M, uint64_t(K) * 2, C::BK, C::kBN,
                               CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != GLMQ_OK) return st;
  const uint64_t row_bytes = uint64_t(K) * C::kBits / 8;
  st = make_map_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, packed, row_bytes, N, row_bytes, C::WROW, C::BM,
                   C::kBits == 4 ? CU_TENSOR_MAP_SWIZZLE_32B : CU_TENSOR_MAP_SWIZZLE_64B);
  if (st != GLMQ_OK) return st;
  PrefillArgs a;
  a.scale = static_cast<const __half*>(scale);
  a.Y = static_cast<__half*>(Y);
  a.ws = nullptr;
  a.xs = nullptr;
  a.bias = e.bias;
  a.geglu = e.geglu;
  a.zero = e.zero;
  a.M = M;
  a.N = N;
  a.K = K;
  a.tiles_m = (M + C::kBN - 1) / C::kBN;
  const long long tiles = static_cast<long long>((N + C::BM - 1) / C::BM) * a.tiles_m;
  if (tiles > 0x7fffffffLL / 64) return GLMQ_ERR_BAD_SHAPE;
  a.tiles = static_cast<int>(tiles);
  const int num_kb = K / C::BK;
  int parts = plan_parts(a.tiles, num_kb, 4, dev.sms);
  a.full = 0;
  if (parts == 1) {
    const double tile_flops = 2.0 * C::BM * C::kBN * K;
    plan_tail_split(a.tiles, a.tiles_m, num_kb, 4, dev.sms, tile_flops, &a.full, &parts);
  }
  a.kbp = (num_kb + parts - 1) / parts;
  a.parts = (num_kb + a.kbp - 1) / a.kbp;
  a.units = a.full + (a.tiles - a.full) * a.parts;
  if (a.parts > 1 && (st = decode_scratch(static_cast<size_t>(M) * N, &a.ws)) != GLMQ_OK) return st;
  if (C::SMEM_BYTES > dev.smem_optin) return GLMQ_ERR_BAD_SHAPE;
  if ((st = allow_smem(prefill_kernel<C>, C::SMEM_BYTES)) != GLMQ_OK) return st;
  const int grid = a.units < dev.sms ? a.units : dev.sms;
  prefill_kernel<C><<<grid, kPrefillThreads, C::SMEM_BYTES, s>>>(tx, tw, a);
  if ((st = launched()) != GLMQ_OK) return st;
  if (a.parts > 1) {
    // the split tiles are the weight-row bands from full / tiles_m on
    const int n0 = (a.full / a.tiles_m) * C::BM;
    st = (e.bias || e.geglu) ? launch_finalize_epi(a.ws, a.scale, e, a.Y, M, N, s, n0)
                             : launch_finalize(a.ws, a.scale, a.Y, M, N, s, n0);
    if (st != GLMQ_OK) return st;
  }
  return GLMQ_OK;
}

template <class C>
glmq_status launch_skinny_cfg(const DeviceInfo& dev, const void* X, int M, const void* packed, const void* scale,
                              int N, int K, void* Y, cudaStream_t s, const Epi& e) {
  if (M > C::kBN) return GLMQ_ERR_BAD_SHAPE;   // one token tile: the activation image holds BN rows
  CUtensorMap tw;
  const uint64_t row_bytes = uint64_t(K) / C::KPB;
  glmq_status st = make_map_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, packed, row_bytes, N, row_bytes, C::WB, C::BM,
                               CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != GLMQ_OK) return st;
  PrefillArgs a;
  a.scale = static_cast<const __half*>(scale);
  a.Y = static_cast<__half*>(Y);
  a.ws = nullptr;
  uint8_t* xs = nullptr;
  if ((st = skinny_x_scratch(static_cast<size_t>(K / 64) * C::XT_BYTES, &xs)) != GLMQ_OK) return st;
  a.xs = xs;
  a.bias = e.bias;
  a.geglu = e.geglu;
  a.zero = e.zero;
  a.M = M;
  a.N = N;
  a.K = K;
  a.tiles_m = (M + C::kBN - 1) / C::kBN;
  const long long tiles = static_cast<long long>((N + C::BM - 1) / C::BM) * a.tiles_m;
  if (tiles > 0x7fffffffLL / 64) return GLMQ_ERR_BAD_SHAPE;
  a.tiles = static_cast<int>(tiles);
  const int num_st = (K + C::SK - 1) / C::SK;
  const int parts = plan_parts(a.tiles, num_st, 2, dev.sms);
  a.kbp = (num_st + parts - 1) / parts;          // stages per part
  a.parts = (num_st + a.kbp - 1) / a.kbp;
  a.full = 0;
  a.units = a.tiles * a.parts;
  if (a.parts > 1 && (st = decode_scratch(static_cast<size_t>(M) * N, &a.ws)) != GLMQ_OK) return st;
  if (C::SMEM_BYTES > dev.smem_optin) return GLMQ_ERR_BAD_SHAPE;
  if ((st = allow_smem(skinny_kernel<C>, C::SMEM_BYTES)) != GLMQ_OK) return st;
  const int grid = a.units < dev.sms ? a.units : dev.sms;
  // Both launches carry a grid dependency. The pre-pass (one small block per SM at most,
  // so a skinny CTA fits beside it) waits for the kernels before it and then lets the
  // skinny kernel launch; the skinny kernel's weight producer streams weight boxes while
  // the pre-pass runs, and only its activation producer (and epilogue) wait for the
  // pre-pass. Reading the weights, scales and zero points early is safe: the skinny
  // kernel launches only after the pre-pass has passed its grid-dependency wait, i.e.
  // after every earlier kernel has completed, and the pre-pass writes none of them.
  {
    const long long units16 = static_cast<long long>(K / 64) * C::kBN * 8;
    const int blocks = static_cast<int>(std::min<long long>((units16 + kPackThreads - 1) / kPackThreads, dev.sms));
    if ((st = launch_pdl(skinny_pack_x_kernel<C>, dim3(blocks), dim3(kPackThreads), 0, s,
                         static_cast<const __half*>(X), M, K, xs)) != GLMQ_OK)
      return st;
  }
  if ((st = launch_pdl(skinny_kernel<C>, dim3(grid), dim3(kSkinnyThreads), C::SMEM_BYTES, s, tw, a)) != GLMQ_OK)
    return st;
  if (a.parts > 1) {
    st = (e.bias || e.geglu) ? launch_finalize_epi(a.ws, a.scale, e, a.Y, M, N, s)
                             : launch_finalize(a.ws, a.scale, a.Y, M, N, s);
    if (st != GLMQ_OK) return st;
  }
  return GLMQ_OK;
}

template <int BITS, int ZP = 0>
glmq_status launch_prefill(const DeviceInfo& dev, const void* X, int M, const void* packed, const void* scale, int N,
                           int K, void* Y, cudaStream_t s, const Epi& e = Epi()) {
  // up to 64 tokens: the skinny kernel (wide weight stream, A operand in tensor memory)
  if (M <= 16) return launch_skinny_cfg<SkinnyCfg<BITS, 16, ZP>>(dev, X, M, packed, scale, N, K, Y, s, e);
  if (M <= 32) return launch_skinny_cfg<SkinnyCfg<BITS, 32, ZP>>(dev, X, M, packed, scale, N, K, Y, s, e);
  if (M <= 64) return launch_skinny_cfg<SkinnyCfg<BITS, 64, ZP>>(dev, X, M, packed, scale, N, K, Y, s, e);
  // tensor-core prefill: 128-token tiles with two accumulators up to M = 128; above 256
  // tokens INT4 uses 192-token tiles, whose two accumulators still fit in TMEM beside
  // four A slots (measured faster than 256-token tiles with one accumulator: B200, INT4,
  // M = 512 and 2048 on the four GLM shapes); otherwise 256-token tiles
  if (M <= 128) return launch_prefill_cfg<PrefillCfg<BITS, 128, ZP>>(dev, X, M, packed, scale, N, K, Y, s, e);
  if (BITS == 4 && M > 256)
    return launch_prefill_cfg<PrefillCfg<BITS, 192, ZP>>(dev, X, M, packed, scale, N, K, Y, s, e);
  return launch_prefill_cfg<PrefillCfg<BITS, 256, ZP>>(dev, X, M, packed, scale, N, K, Y, s, e);
}

// ---------------------------------------------------------------- decode without allocation
// Callers that must not allocate device memory (see glmq_gemm_decode_noalloc in
// glmq.h) get the decode kernel with its split-K partial sums kept in this fixed
// array instead of the lazily allocated scratch. It is static storage: every GPU
// that loads the library holds it until the process exits. Host code must not use
// the array's name as a device address: the address is obtained per device with
// cudaGetSymbolAddress.
constexpr size_t kNoAllocScratchFloats = size_t(1) << 20;   // 4 MiB per device
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchFloats];
float* g_noalloc_scratch_ptr[kMaxDevices];

// Device address of g_noalloc_scratch on the current device (looked up once per device).
glmq_status noalloc_scratch(float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= kMaxDevices) return GLMQ_ERR_UNSUPPORTED_DEVICE;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_noalloc_scratch_ptr[dev]) {
    void* p = nullptr;
    if ((e = cudaGetSymbolAddress(&p, g_noalloc_scratch)) != cudaSuccess) return cuda_fail(e);
    g_noalloc_scratch_ptr[dev] = static_cast<float*>(p);
  }
  *out = g_noalloc_scratch_ptr[dev];
  return GLMQ_OK;
}

template <class C>
glmq_status launch_decode_noalloc_cfg(const DeviceInfo& dev, const void* X, int M, const void* packed,
                                      const void* scale, int N, int K, void* Y, cudaStream_t s) {
  DecodePlan pl;
  if (!plan_decode<C>(dev, N, K, &pl)) return GLMQ_ERR_BAD_SHAPE;
  CUtensorMap tw;
  const uint64_t row_bytes = uint64_t(K) / C::KPB;
  glmq_status st = make_map_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, packed, row_bytes, N, row_bytes, kDecodeSegB,
                               kDecodeRows, CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != GLMQ_OK) return st;
  CUtensorMap tx;
  st = make_map_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, X, K, M, uint64_t(K) * 2, C::SK, C::kMP,
                   CU_TENSOR_MAP_SWIZZLE_NONE);
  if (st != GLMQ_OK) return st;
  DecodeArgs a;
  a.X = static_cast<const __half*>(X);
  a.scale = static_cast<const __half*>(scale);
  a.Y = static_cast<__half*>(Y);
  a.ws = nullptr;
  a.M = M;
  a.N = N;
  a.K = K;
  a.KPP = pl.KPP;
  a.parts = pl.parts;
  a.tiles = pl.tiles;
  a.units = pl.units;
  a.bias = nullptr;
  a.geglu = 0;
  a.zero = nullptr;
  a.nxt_grid = a.nxt_units = a.nxt_tiles = a.nxt_KPP = a.nxt_K = a.nxt_stages = 0;
  cudaError_t e;
  if (pl.parts > 1) {
    if ((st = noalloc_scratch(&a.ws)) != GLMQ_OK) return st;
    // The partial sums must start at zero. Every call shares the array, and a call
    // whose kernel gave up a bounded wait (glmq_last_device_error) can leave partial
    // sums behind, so each call clears its own region on its stream instead of relying
    // on the previous call's finalize pass having returned it to zero.
    if ((e = cudaMemsetAsync(a.ws, 0, static_cast<size_t>(M) * N * sizeof(float), s)) != cudaSuccess)
      return cuda_fail(e);
  }
  if ((st = allow_smem(decode_kernel<C>, pl.smem)) != GLMQ_OK) return st;
  if ((st = launch_pdl(decode_kernel<C>, dim3(pl.grid), dim3(C::kThreads), pl.smem, s, tw, tx, tw, a)) != GLMQ_OK)
    return st;
  if (pl.parts > 1) {
    if ((st = launch_finalize(a.ws, a.scale, a.Y, M, N, s)) != GLMQ_OK) return st;
  }
  return GLMQ_OK;
}

template <int BITS>
glmq_status launch_decode_noalloc(const DeviceInfo& dev, const void* X, int M, const void* packed, const void* scale,
                                  int N, int K, void* Y, cudaStream_t s) {
  if (M <= 1) return launch_decode_noalloc_cfg<DecodeCfg<BITS, 1>>(dev, X, M, packed, scale, N, K, Y, s);
  if (M <= 2) return launch_decode_noalloc_cfg<DecodeCfg<BITS, 2>>(dev, X, M, packed, scale, N, K, Y, s);
  if (M <= 4) return launch_decode_noalloc_cfg<DecodeCfg<BITS, 4>>(dev, X, M, packed, scale, N, K, Y, s);
  if (M <= 8) return launch_decode_noalloc_cfg<DecodeCfg<BITS, 8>>(dev, X, M, packed, scale, N, K, Y, s);
  return launch_decode_noalloc_cfg<DecodeCfg<BITS, 16>>(dev, X, M, packed, scale, N, K, Y, s);
}

enum class Route { kAuto, kDecode, kPrefill };

glmq_status gemm_entry(Route route, const void* X, int64_t M, const void* packed, const void* scale, int64_t N,
                       int64_t K, int bits, void* Y, void* stream, const Epi& e = Epi()) {
  glmq_status st = check_gemm(X, M, packed, scale, N, K, bits, Y);
  if (st != GLMQ_OK) return st;
  if (route == Route::kDecode && M > GLMQ_DECODE_MAX_M) return GLMQ_ERR_BAD_SHAPE;
  if (M == 0 || N == 0) return GLMQ_OK;
  const DeviceInfo* dev = nullptr;
  if ((st = current_device(&dev)) != GLMQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool decode = route == Route::kDecode || (route == Route::kAuto && M <= GLMQ_DECODE_AUTO_MAX_M);
  const int m = static_cast<int>(M), n = static_cast<int>(N), k = static_cast<int>(K);
  if (decode) {
    if (e.zero) return launch_decode<4, 1>(*dev, X, m, packed, scale, n, k, Y, s, e);
    return bits == 4 ? launch_decode<4>(*dev, X, m, packed, scale, n, k, Y, s, e)
                     : launch_decode<8>(*dev, X, m, packed, scale, n, k, Y, s, e);
  }
  if (e.zero) return launch_prefill<4, 1>(*dev, X, m, packed, scale, n, k, Y, s, e);
  return bits == 4 ? launch_prefill<4>(*dev, X, m, packed, scale, n, k, Y, s, e)
                   : launch_prefill<8>(*dev, X, m, packed, scale, n, k, Y, s, e);
}

glmq_status quantize_entry(const void* W, int64_t N, int64_t K, int bits, void* packed, void* scale, void* stream,
                           bool geglu) {
  glmq_status st = check_common(N, K, bits);
  if (st != GLMQ_OK) return st;
  if (geglu && (N % 16) != 0) return GLMQ_ERR_BAD_SHAPE;
  if (N == 0) return GLMQ_OK;
  if (!W || !packed || !scale) return GLMQ_ERR_NULL_POINTER;
  if (!aligned16(W) || !aligned16(packed) || !aligned16(scale)) return GLMQ_ERR_MISALIGNED;
  const DeviceInfo* dev = nullptr;
  if ((st = current_device(&dev)) != GLMQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int half = geglu ? static_cast<int>(N / 2) : 0;
  return bits == 4 ? launch_quantize<4>(W, N, K, packed, scale, half, s)
                   : launch_quantize<8>(W, N, K, packed, scale, half, s);
}

}  // namespace

extern "C" {

int glmq_abi_version(void) { return GLMQ_ABI_VERSION; }

size_t glmq_packed_bytes(int64_t N, int64_t K, int bits) {
  if (check_common(N, K, bits) != GLMQ_OK) return 0;
  return static_cast<size_t>(N) * static_cast<size_t>(K) * static_cast<size_t>(bits) / 8u;
}

glmq_status glmq_quantize(const void* W, int64_t N, int64_t K, int bits, void* packed, void* scale, void* stream) {
  return quantize_entry(W, N, K, bits, packed, scale, stream, false);
}

glmq_status glmq_quantize_geglu(const void* W, int64_t N, int64_t K, int bits, void* packed, void* scale,
                                void* stream) {
  return quantize_entry(W, N, K, bits, packed, scale, stream, true);
}

glmq_status glmq_gemm(const void* X, int64_t M, const void* packed, const void* scale, int64_t N, int64_t K, int bits,
                      void* Y, void* stream) {
  return gemm_entry(Route::kAuto, X, M, packed, scale, N, K, bits, Y, stream);
}

glmq_status glmq_gemm_decode(const void* X, int64_t M, const void* packed, const void* scale, int64_t N, int64_t K,
                             int bits, void* Y, void* stream) {
  return gemm_entry(Route::kDecode, X, M, packed, scale, N, K, bits, Y, stream);
}

glmq_status glmq_gemm_decode_prefetch(const void* X, int64_t M, const void* packed, const void* scale, int64_t N,
                                      int64_t K, int bits, void* Y, const void* next_packed, int64_t next_M,
                                      int64_t next_N, int64_t next_K, void* stream) {
  Epi e;
  if (next_packed) {
    if (next_M < 1 || next_M > GLMQ_DECODE_MAX_M || next_N < 1) return GLMQ_ERR_BAD_SHAPE;
    glmq_status st = check_common(next_N, next_K, bits);
    if (st != GLMQ_OK) return st;
    if (!aligned16(next_packed)) return GLMQ_ERR_MISALIGNED;
    e.next_packed = next_packed;
    e.next_M = static_cast<int>(next_M);
    e.next_N = static_cast<int>(next_N);
    e.next_K = static_cast<int>(next_K);
  }
  return gemm_entry(Route::kDecode, X, M, packed, scale, N, K, bits, Y, stream, e);
}

glmq_status glmq_gemm_prefill(const void* X, int64_t M, const void* packed, const void* scale, int64_t N, int64_t K,
                              int bits, void* Y, void* stream) {
  return gemm_entry(Route::kPrefill, X, M, packed, scale, N, K, bits, Y, stream);
}

glmq_status glmq_gemm_fused(const void* X, int64_t M, const void* packed, const void* scale, const void* bias,
                            int64_t N, int64_t K, int bits, int epilogue, void* Y, void* stream) {
  if (epilogue != GLMQ_EPILOGUE_NONE && epilogue != GLMQ_EPILOGUE_GEGLU) return GLMQ_ERR_BAD_SHAPE;
  const bool geglu = epilogue == GLMQ_EPILOGUE_GEGLU;
  if (geglu && (N % 16) != 0) return GLMQ_ERR_BAD_SHAPE;
  if (bias && (reinterpret_cast<uintptr_t>(bias) & 1u) != 0) return GLMQ_ERR_MISALIGNED;
  Epi e;
  e.bias = static_cast<const __half*>(bias);
  e.geglu = geglu ? 1 : 0;
  return gemm_entry(Route::kAuto, X, M, packed, scale, N, K, bits, Y, stream, e);
}

glmq_status glmq_quantize_zp(const void* W, int64_t N, int64_t K, void* packed, void* scale, void* zero,
                             void* stream) {
  glmq_status st = check_common(N, K, 4);
  if (st != GLMQ_OK) return st;
  if (N == 0) return GLMQ_OK;
  if (!W || !packed || !scale || !zero) return GLMQ_ERR_NULL_POINTER;
  if (!aligned16(W) || !aligned16(packed) || !aligned16(scale)) return GLMQ_ERR_MISALIGNED;
  const DeviceInfo* dev = nullptr;
  if ((st = current_device(&dev)) != GLMQ_OK) return st;
  return launch_quantize_zp(W, N, K, packed, scale, zero, static_cast<cudaStream_t>(stream));
}

glmq_status glmq_gemm_zp(const void* X, int64_t M, const void* packed, const void* scale, const void* zero,
                         int64_t N, int64_t K, void* Y, void* stream) {
  if (!zero && M > 0 && N > 0) return GLMQ_ERR_NULL_POINTER;
  Epi e;
  e.zero = static_cast<const uint8_t*>(zero);
  return gemm_entry(Route::kAuto, X, M, packed, scale, N, K, 4, Y, stream, e);
}

glmq_status glmq_gemm_decode_noalloc(const void* X, int64_t M, const void* packed, const void* scale, int64_t N,
                                     int64_t K, int bits, void* Y, void* stream) {
  glmq_status st = check_gemm(X, M, packed, scale, N, K, bits, Y);
  if (st != GLMQ_OK) return st;
  if (M > GLMQ_DECODE_MAX_M) return GLMQ_ERR_BAD_SHAPE;
  if (static_cast<size_t>(M) * static_cast<size_t>(N) > kNoAllocScratchFloats) return GLMQ_ERR_BAD_SHAPE;
  if (M == 0 || N == 0) return GLMQ_OK;
  const DeviceInfo* dev = nullptr;
  if ((st = current_device(&dev)) != GLMQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int m = static_cast<int>(M), n = static_cast<int>(N), k = static_cast<int>(K);
  return bits == 4 ? launch_decode_noalloc<4>(*dev, X, m, packed, scale, n, k, Y, s)
                   : launch_decode_noalloc<8>(*dev, X, m, packed, scale, n, k, Y, s);
}

glmq_status glmq_set_wait_limit_ns(uint64_t limit_ns) {
  const unsigned long long v = limit_ns == 0 ? glmq::kWaitLimitNs : static_cast<unsigned long long>(limit_ns);
  const DeviceInfo* dev = nullptr;
  glmq_status st = current_device(&dev);
  if (st != GLMQ_OK) return st;
  const cudaError_t e = cudaMemcpyToSymbol(glmq::g_wait_limit_ns, &v, sizeof(v));
  if (e != cudaSuccess) return cuda_fail(e);
  return GLMQ_OK;
}

const char* glmq_status_string(int status) {
  switch (status) {
    case GLMQ_OK: return "ok";
    case GLMQ_ERR_NULL_POINTER: return "a required pointer is NULL";
    case GLMQ_ERR_BAD_BITS: return "bits must be 4 or 8";
    case GLMQ_ERR_BAD_SHAPE: return "unsupported shape (need K > 0, K % 64 == 0, K <= 65536, sizes in range)";
    case GLMQ_ERR_MISALIGNED: return "a pointer is not 16-byte aligned";
    case GLMQ_ERR_CUDA: return "a CUDA runtime call failed";
    case GLMQ_ERR_DEVICE: return "a kernel reported a device-side error";
    case GLMQ_ERR_UNSUPPORTED_DEVICE: return "the current device is not an sm_100 (B200-class) GPU";
    default: return "unknown glmq status";
  }
}

int glmq_last_cuda_error(void) { return t_last_cuda_error; }

uint64_t glmq_kernel_launches(void) { return g_kernel_launches.load(std::memory_order_relaxed); }

glmq_status glmq_last_device_error(void* stream, uint32_t* flags) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  unsigned int word = 0;
  if ((e = cudaMemcpyFromSymbol(&word, glmq::g_device_status, sizeof(word))) != cudaSuccess) return cuda_fail(e);
  if (flags) *flags = word;
  if (word == 0) return GLMQ_OK;
  const unsigned int zero = 0;
  if ((e = cudaMemcpyToSymbol(glmq::g_device_status, &zero, sizeof(zero))) != cudaSuccess) return cuda_fail(e);
  // a kernel that gave up may have left decode scratch non-zero: restore the invariant
  int dev = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return cuda_fail(e);
  {
    std::lock_guard<std::mutex> lock(g_mutex);
    DecodeScratch& sc = g_scratch[dev];
    if (sc.ws && (e = cudaMemset(sc.ws, 0, sc.ws_elems * sizeof(float))) != cudaSuccess) return cuda_fail(e);
  }
  return GLMQ_ERR_DEVICE;
}

}  // extern "C"
