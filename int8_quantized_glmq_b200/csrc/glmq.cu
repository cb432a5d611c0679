// glmq C ABI: argument validation, per-device set-up and kernel dispatch.
// The operations and their readings are documented in include/glmq.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "glmq.h"
#include "decode.cuh"
#include "prefill.cuh"
#include "quantize.cuh"

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

// Per-device, per-kernel opt-in to large dynamic shared memory.
template <class Kernel>
glmq_status allow_smem(Kernel kernel, int bytes) {
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return cuda_fail(e);
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
template <int BITS, int CPT>
glmq_status launch_quantize_cpt(const void* W, int64_t N, int64_t K, void* packed, void* scale, cudaStream_t s) {
  quantize_kernel<BITS, CPT><<<static_cast<unsigned>(N), kQuantThreads, 0, s>>>(
      static_cast<const __half*>(W), static_cast<int>(K), static_cast<uint8_t*>(packed), static_cast<__half*>(scale));
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? GLMQ_OK : cuda_fail(e);
}

template <int BITS>
glmq_status launch_quantize(const void* W, int64_t N, int64_t K, void* packed, void* scale, cudaStream_t s) {
  const int64_t need = (K / 8 + kQuantThreads - 1) / kQuantThreads;  // 16-byte chunks per thread
  if (need <= 1) return launch_quantize_cpt<BITS, 1>(W, N, K, packed, scale, s);
  if (need <= 2) return launch_quantize_cpt<BITS, 2>(W, N, K, packed, scale, s);
  if (need <= 4) return launch_quantize_cpt<BITS, 4>(W, N, K, packed, scale, s);
  if (need <= 6) return launch_quantize_cpt<BITS, 6>(W, N, K, packed, scale, s);
  if (need <= 8) return launch_quantize_cpt<BITS, 8>(W, N, K, packed, scale, s);
  if (need <= 12) return launch_quantize_cpt<BITS, 12>(W, N, K, packed, scale, s);
  if (need <= 16) return launch_quantize_cpt<BITS, 16>(W, N, K, packed, scale, s);
  if (need <= 24) return launch_quantize_cpt<BITS, 24>(W, N, K, packed, scale, s);
  return launch_quantize_cpt<BITS, 32>(W, N, K, packed, scale, s);
}

// ---------------------------------------------------------------- decode
template <class C>
glmq_status launch_decode_cfg(const DeviceInfo& dev, const void* X, int M, const void* packed, const void* scale,
                              int N, int K, void* Y, cudaStream_t s) {
  const int barrier_bytes = 128;
  const int avail = dev.smem_optin - (kDecodeStages * C::STAGE_BYTES + C::ACC_BYTES + barrier_bytes);
  DecodeArgs a;
  a.X = static_cast<const __half*>(X);
  a.packed = static_cast<const uint8_t*>(packed);
  a.scale = static_cast<const __half*>(scale);
  a.Y = static_cast<__half*>(Y);
  a.M = M;
  a.N = N;
  a.K = K;
  const int k_round = (K + C::SK - 1) / C::SK * C::SK;
  const int xp1 = static_cast<int>(x_pitch(k_round, C::XSHIFT));
  if (static_cast<long long>(M) * xp1 <= avail) {
    a.KP = k_round;
    a.passes = 1;
    a.XP = xp1;
    a.xbufs = 1;
  } else {
    int kp = 0;
    for (int cand = C::SK; cand < k_round; cand += C::SK) {
      if (2LL * M * x_pitch(cand, C::XSHIFT) <= avail) kp = cand; else break;
    }
    if (kp == 0) return GLMQ_ERR_BAD_SHAPE;
    a.KP = kp;
    a.passes = (K + kp - 1) / kp;
    a.XP = static_cast<int>(x_pitch(kp, C::XSHIFT));
    a.xbufs = 2;
  }
  a.tiles = (N + C::R - 1) / C::R;
  const int smem = kDecodeStages * C::STAGE_BYTES + C::ACC_BYTES + a.xbufs * M * a.XP + barrier_bytes;
  glmq_status st = allow_smem(decode_kernel<C>, smem);
  if (st != GLMQ_OK) return st;
  const int grid = a.tiles < dev.sms ? a.tiles : dev.sms;
  decode_kernel<C><<<grid, kDecodeThreads, smem, s>>>(a);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? GLMQ_OK : cuda_fail(e);
}

template <int BITS>
glmq_status launch_decode(const DeviceInfo& dev, const void* X, int M, const void* packed, const void* scale, int N,
                          int K, void* Y, cudaStream_t s) {
  if (M <= 8) return launch_decode_cfg<DecodeCfg<BITS, 1, 128, 2>>(dev, X, M, packed, scale, N, K, Y, s);
  return launch_decode_cfg<DecodeCfg<BITS, 2, 64, 2>>(dev, X, M, packed, scale, N, K, Y, s);
}

// ---------------------------------------------------------------- prefill
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

template <class C>
glmq_status launch_prefill_cfg(const DeviceInfo& dev, const void* X, int M, const void* packed, const void* scale,
                               int N, int K, void* Y, cudaStream_t s) {
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
  a.M = M;
  a.N = N;
  a.K = K;
  a.tiles_m = (M + C::kBN - 1) / C::kBN;
  const long long tiles = static_cast<long long>((N + C::BM - 1) / C::BM) * a.tiles_m;
  if (tiles > 0x7fffffffLL) return GLMQ_ERR_BAD_SHAPE;
  a.tiles = static_cast<int>(tiles);
  if (C::SMEM_BYTES > dev.smem_optin) return GLMQ_ERR_BAD_SHAPE;
  st = allow_smem(prefill_kernel<C>, C::SMEM_BYTES);
  if (st != GLMQ_OK) return st;
  const int grid = a.tiles < dev.sms ? a.tiles : dev.sms;
  prefill_kernel<C><<<grid, kPrefillThreads, C::SMEM_BYTES, s>>>(tx, tw, a);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? GLMQ_OK : cuda_fail(e);
}

template <int BITS>
glmq_status launch_prefill(const DeviceInfo& dev, const void* X, int M, const void* packed, const void* scale, int N,
                           int K, void* Y, cudaStream_t s) {
  if (M <= 32) return launch_prefill_cfg<PrefillCfg<BITS, 32>>(dev, X, M, packed, scale, N, K, Y, s);
  if (M <= 64) return launch_prefill_cfg<PrefillCfg<BITS, 64>>(dev, X, M, packed, scale, N, K, Y, s);
  if (M <= 128) return launch_prefill_cfg<PrefillCfg<BITS, 128>>(dev, X, M, packed, scale, N, K, Y, s);
  return launch_prefill_cfg<PrefillCfg<BITS, 256>>(dev, X, M, packed, scale, N, K, Y, s);
}

enum class Route { kAuto, kDecode, kPrefill };

glmq_status gemm_entry(Route route, const void* X, int64_t M, const void* packed, const void* scale, int64_t N,
                       int64_t K, int bits, void* Y, void* stream) {
  glmq_status st = check_gemm(X, M, packed, scale, N, K, bits, Y);
  if (st != GLMQ_OK) return st;
  if (route == Route::kDecode && M > GLMQ_DECODE_MAX_M) return GLMQ_ERR_BAD_SHAPE;
  if (M == 0 || N == 0) return GLMQ_OK;
  const DeviceInfo* dev = nullptr;
  if ((st = current_device(&dev)) != GLMQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool decode = route == Route::kDecode || (route == Route::kAuto && M <= GLMQ_DECODE_MAX_M);
  const int m = static_cast<int>(M), n = static_cast<int>(N), k = static_cast<int>(K);
  if (decode) {
    return bits == 4 ? launch_decode<4>(*dev, X, m, packed, scale, n, k, Y, s)
                     : launch_decode<8>(*dev, X, m, packed, scale, n, k, Y, s);
  }
  return bits == 4 ? launch_prefill<4>(*dev, X, m, packed, scale, n, k, Y, s)
                   : launch_prefill<8>(*dev, X, m, packed, scale, n, k, Y, s);
}

}  // namespace

extern "C" {

int glmq_abi_version(void) { return GLMQ_ABI_VERSION; }

size_t glmq_packed_bytes(int64_t N, int64_t K, int bits) {
  if (check_common(N, K, bits) != GLMQ_OK) return 0;
  return static_cast<size_t>(N) * static_cast<size_t>(K) * static_cast<size_t>(bits) / 8u;
}

glmq_status glmq_quantize(const void* W, int64_t N, int64_t K, int bits, void* packed, void* scale, void* stream) {
  glmq_status st = check_common(N, K, bits);
  if (st != GLMQ_OK) return st;
  if (N == 0) return GLMQ_OK;
  if (!W || !packed || !scale) return GLMQ_ERR_NULL_POINTER;
  if (!aligned16(W) || !aligned16(packed) || !aligned16(scale)) return GLMQ_ERR_MISALIGNED;
  const DeviceInfo* dev = nullptr;
  if ((st = current_device(&dev)) != GLMQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return bits == 4 ? launch_quantize<4>(W, N, K, packed, scale, s) : launch_quantize<8>(W, N, K, packed, scale, s);
}

glmq_status glmq_gemm(const void* X, int64_t M, const void* packed, const void* scale, int64_t N, int64_t K, int bits,
                      void* Y, void* stream) {
  return gemm_entry(Route::kAuto, X, M, packed, scale, N, K, bits, Y, stream);
}

glmq_status glmq_gemm_decode(const void* X, int64_t M, const void* packed, const void* scale, int64_t N, int64_t K,
                             int bits, void* Y, void* stream) {
  return gemm_entry(Route::kDecode, X, M, packed, scale, N, K, bits, Y, stream);
}

glmq_status glmq_gemm_prefill(const void* X, int64_t M, const void* packed, const void* scale, int64_t N, int64_t K,
                              int bits, void* Y, void* stream) {
  return gemm_entry(Route::kPrefill, X, M, packed, scale, N, K, bits, Y, stream);
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

glmq_status glmq_last_device_error(void* stream, uint32_t* flags) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  unsigned int word = 0;
  if ((e = cudaMemcpyFromSymbol(&word, glmq::g_device_status, sizeof(word))) != cudaSuccess) return cuda_fail(e);
  if (flags) *flags = word;
  if (word == 0) return GLMQ_OK;
  const unsigned int zero = 0;
  if ((e = cudaMemcpyToSymbol(glmq::g_device_status, &zero, sizeof(zero))) != cudaSuccess) return cuda_fail(e);
  return GLMQ_ERR_DEVICE;
}

}  // extern "C"
