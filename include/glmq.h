/*
 * glmq: weight-only INT4 / INT8 quantization and the dequantizing linear layer
 * (W4A16 / W8A16) for GLM-130B projection shapes, on NVIDIA B200 (sm_100a).
 *
 * The operations are those of the GLM-130B paper's weight-only quantization
 * ("GLM-130B: An Open Bilingual Pre-trained Model"):
 *   - wikillm.com paper card, "Method": every output row of a linear layer gets
 *     one scale, its absolute maximum divided by 7; weights are rounded to
 *     integers in [-7, 7], two INT4 values per byte; at run time the weights are
 *     dequantized (quant * scale[:, None]) and multiplied by FP16 activations.
 *   - same card, "Paper vs code", quantization-scale bullet: the divisor is
 *     2^(b-1) - 1 (7 for INT4, 127 for INT8) and the scale is computed per
 *     output row in FP16.
 *   - paperlayer.ai summary, "INT4 Quantization for RTX 3090s/2080s": only the
 *     linear-layer weights are quantized, activations stay FP16 and weights are
 *     converted to FP16 at run time.
 *
 * Readings this library fixes where the pages are silent:
 *   scale  s[n] = fp16_rn( fp32(max_k |W[n,k]|) / d ),  d = 7 (INT4) or 127 (INT8)
 *   code   q[n,k] = clamp( round_half_even( fp32(W[n,k]) / fp32(s[n]) ), -d, d ),
 *          and q[n,:] = 0 on a row whose scale rounds to 0
 *   INT4   byte j of row n = (q[n,2j] & 0xF) | ((q[n,2j+1] & 0xF) << 4)
 *          (low nibble = even k, 4-bit two's complement; 0x8 never occurs)
 *   INT8   byte k of row n = q[n,k] as a two's-complement int8
 *   linear Y[m,n] = fp16_rn( s[n] * sum_k X[m,k] * q[n,k] ), products exact,
 *          sum accumulated in fp32 (the scale factors out of the k-sum).
 *
 * Conventions for every entry point:
 *   - All tensors are dense, row-major, in DEVICE memory of the current CUDA
 *     device, allocated and owned by the caller; the library never allocates,
 *     frees or retains them. Every pointer must be 16-byte aligned.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *     stream). Calls only enqueue work on that stream and return without
 *     synchronizing; results are visible after the stream reaches that point.
 *   - Arguments are validated before anything is enqueued; a call that returns
 *     an error status has enqueued nothing. No entry point aborts or throws.
 *   - Shapes: N >= 0 rows (out_features), K in_features with K > 0,
 *     K % 64 == 0 and K <= GLMQ_MAX_K; M >= 0 activation rows. N == 0 or
 *     M == 0 is an empty problem: GLMQ_OK, nothing is enqueued, pointers may
 *     be NULL.
 *   - Inputs are finite fp16 values; NaN or Inf inputs are outside the contract.
 *   - Calls that overlap on the GPU and write the same output race.
 *   - Library-owned device state, one instance per device: the fp32 scratch of
 *     GEMM calls whose tiles are split over K parts (see glmq_gemm), the skinny
 *     kernel's activation image (16 < M <= 64), the fixed array of
 *     glmq_gemm_decode_noalloc, and the device status word. GEMM calls that use
 *     one of these buffers must not overlap on the GPU: issue them on one stream,
 *     or order the streams. Quantize calls use none of them.
 */
#ifndef GLMQ_H
#define GLMQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define GLMQ_API __attribute__((visibility("default")))
#else
#define GLMQ_API
#endif

#define GLMQ_ABI_VERSION 1
#define GLMQ_MAX_K 65536
/* Largest M the decode (register-dequant GEMV) kernel accepts (glmq_gemm_decode). */
#define GLMQ_DECODE_MAX_M 16
/* glmq_gemm sends M <= GLMQ_DECODE_AUTO_MAX_M to the decode kernel and larger M to the
 * tcgen05 tensor-core kernels (a skinny variant up to 64 tokens, the prefill kernel
 * above), which split tiles over K when there are fewer tiles than SMs. */
#define GLMQ_DECODE_AUTO_MAX_M 16

typedef enum glmq_status {
  GLMQ_OK = 0,
  GLMQ_ERR_NULL_POINTER = 1,      /* a required pointer is NULL                       */
  GLMQ_ERR_BAD_BITS = 2,          /* bits is not 4 or 8                                */
  GLMQ_ERR_BAD_SHAPE = 3,         /* a size is negative, K % 64 != 0, K > GLMQ_MAX_K,
                                     or a size exceeds a kernel's limit               */
  GLMQ_ERR_MISALIGNED = 4,        /* a pointer is not 16-byte aligned                 */
  GLMQ_ERR_CUDA = 5,              /* a CUDA runtime call failed (see glmq_last_cuda_error) */
  GLMQ_ERR_DEVICE = 6,            /* a kernel reported a device-side error            */
  GLMQ_ERR_UNSUPPORTED_DEVICE = 7 /* the current device is not compute capability 10.0 */
} glmq_status;

/* The ABI version this library was built with (GLMQ_ABI_VERSION). */
GLMQ_API int glmq_abi_version(void);

/* Bytes of packed weight storage for an [N, K] weight at `bits` bits:
 * N*K/2 for INT4, N*K for INT8. Returns 0 for invalid arguments. Host-only. */
GLMQ_API size_t glmq_packed_bytes(int64_t N, int64_t K, int bits);

/*
 * One-shot weight quantization (paper card, "Method": quantize_linear_int4;
 * "Paper vs code": per-row absmax / (2^(b-1)-1), FP16 scale).
 *   W       in : fp16 [N, K], row n = output feature n
 *   packed  out: uint8 [N, K*bits/8] (glmq_packed_bytes(N, K, bits) bytes)
 *   scale   out: fp16 [N]
 * Packed codes and scales are a pure function of W (bit-for-bit reproducible).
 * Limits: N <= 2^31 - 1.
 */
GLMQ_API glmq_status glmq_quantize(const void* W, int64_t N, int64_t K, int bits, void* packed, void* scale,
                          void* stream);

/*
 * Dequantizing linear layer (paper card, "Method": linear_forward):
 *   Y[m,n] = fp16_rn( s[n] * sum_k X[m,k] * q[n,k] ), fp32 accumulation.
 *   X       in : fp16 [M, K] activations
 *   packed  in : codes from glmq_quantize (same N, K, bits)
 *   scale   in : fp16 [N]
 *   Y       out: fp16 [M, N]; must not overlap any input
 * Dispatch: M <= GLMQ_DECODE_AUTO_MAX_M runs the decode kernel (HBM-bound stream
 * of the packed weights, register dequantization, warp-level MMA); larger M runs
 * the tcgen05 tensor-core kernel. Both give results within the documented accuracy.
 * Either kernel may split tiles over K parts; it then accumulates fp32 partial sums
 * in a per-device scratch buffer that the library allocates on first use (call once
 * outside stream capture before capturing) and runs a second, finalize kernel.
 */
GLMQ_API glmq_status glmq_gemm(const void* X, int64_t M, const void* packed, const void* scale, int64_t N,
                      int64_t K, int bits, void* Y, void* stream);

/* glmq_gemm forced onto the decode kernel. Requires M <= GLMQ_DECODE_MAX_M. */
GLMQ_API glmq_status glmq_gemm_decode(const void* X, int64_t M, const void* packed, const void* scale,
                             int64_t N, int64_t K, int bits, void* Y, void* stream);

/*
 * glmq_gemm_decode with a prefetch hint for the NEXT decode call on the same stream
 * (a decode step runs the layers' projections back to back, and a layer's weights do
 * not depend on the previous layer's output). Y is computed exactly as by
 * glmq_gemm_decode (same kernel and plan; the hint only adds L2 prefetches).
 *   next_packed in : codes of the next call's weight, uint8 [next_N, next_K*bits/8], same
 *                    bits as this call, 16-byte aligned; NULL = no hint (plain
 *                    glmq_gemm_decode)
 *   next_M         : the next call's token count, 1..GLMQ_DECODE_MAX_M
 *   next_N, next_K : the next call's shape (limits as glmq_gemm)
 * While this call's pipeline drains, its kernel prefetches into L2 the weight tiles the
 * next call's kernel loads first (the first ring fill of each of its CTAs). Only reads
 * of next_packed are issued, and only as L2 prefetches; nothing is written. The hint
 * pays when the next call follows directly (no other large traffic in between).
 * Errors: as glmq_gemm_decode; GLMQ_ERR_BAD_SHAPE for next_M outside 1..16, next_N < 1
 * or a bad next_K; GLMQ_ERR_BAD_BITS never (bits is shared); GLMQ_ERR_MISALIGNED for an
 * unaligned next_packed.
 */
GLMQ_API glmq_status glmq_gemm_decode_prefetch(const void* X, int64_t M, const void* packed, const void* scale,
                                               int64_t N, int64_t K, int bits, void* Y, const void* next_packed,
                                               int64_t next_M, int64_t next_N, int64_t next_K, void* stream);

/* glmq_gemm forced onto the tensor-core prefill kernel (any M >= 0). */
GLMQ_API glmq_status glmq_gemm_prefill(const void* X, int64_t M, const void* packed, const void* scale,
                              int64_t N, int64_t K, int bits, void* Y, void* stream);

/*
 * One-shot quantization like glmq_quantize, with the packed rows (and scales) stored
 * in the layout the fused GeGLU epilogue reads (GLM-130B paper card, "Method": the
 * feed-forward block is a GeGLU; FFN-up holds both GLU branches, rows 0 .. N/2-1 the
 * first and N/2 .. N-1 the second). Packed row 16g + r holds row 8g + r of W for
 * r < 8 and row N/2 + 8g + r - 8 for r >= 8.
 *   Same arguments and codes as glmq_quantize; only the row order differs.
 *   Requires N % 16 == 0, else GLMQ_ERR_BAD_SHAPE.
 */
GLMQ_API glmq_status glmq_quantize_geglu(const void* W, int64_t N, int64_t K, int bits, void* packed, void* scale,
                                         void* stream);

/* Epilogues of glmq_gemm_fused. */
#define GLMQ_EPILOGUE_NONE 0
#define GLMQ_EPILOGUE_GEGLU 1

/*
 * glmq_gemm with a fused epilogue (paper card, "Paper vs code": biases stay FP16;
 * "Method": GeGLU feed-forward block).
 *   bias      in : fp16 [N] in the natural row order of W, or NULL; 2-byte aligned.
 *   epilogue     : GLMQ_EPILOGUE_NONE:  Y [M, N],   Y = fp16( s[n] * sum_k X q + bias[n] )
 *                  GLMQ_EPILOGUE_GEGLU: Y [M, N/2], with U = s * sum_k X q + bias over the
 *                  N = 2F rows, Y[m,j] = fp16( GELU(U[m,j]) * U[m,F+j] ), GELU(u) =
 *                  0.5 u (1 + erf(u / sqrt 2)); packed and scale must come from
 *                  glmq_quantize_geglu, and N % 16 == 0.
 * Other arguments, dispatch, scratch and errors as glmq_gemm; an unknown epilogue
 * value is GLMQ_ERR_BAD_SHAPE.
 */
GLMQ_API glmq_status glmq_gemm_fused(const void* X, int64_t M, const void* packed, const void* scale,
                                     const void* bias, int64_t N, int64_t K, int bits, int epilogue, void* Y,
                                     void* stream);

/*
 * Zero-point (asymmetric) INT4 quantization (GLM-130B paper card, "Pitfalls": a
 * zero-point INT4 quantizer scored better on LAMBADA than the absmax one, which the
 * authors kept as cheaper; the card gives no formula). Per output row:
 *   lo = min(0, min_k W), hi = max(0, max_k W)          (fp16 values)
 *   s  = fp16_rn( fl32( fl32(hi - lo) / 15 ) )
 *   z  = clamp( rint( fl32(-lo / s) ), 0, 15 )           (0 where s == 0)
 *   q  = clamp( rint( fl32(w / s) ) + z, 0, 15 )         (0 where s == 0), unsigned
 *   W   in : fp16 [N, K]
 *   packed out: uint8 [N, K/2], two unsigned codes per byte, low nibble = even k
 *   scale  out: fp16 [N];  zero out: uint8 [N]
 * Limits and errors as glmq_quantize (bits is 4). Results are bit-for-bit reproducible.
 */
GLMQ_API glmq_status glmq_quantize_zp(const void* W, int64_t N, int64_t K, void* packed, void* scale, void* zero,
                                      void* stream);

/*
 * Dequantizing linear layer for zero-point codes from glmq_quantize_zp:
 *   Y[m,n] = fp16_rn( s[n] * sum_k X[m,k] * (q[n,k] - z[n]) ), fp32 accumulation.
 * Arguments, dispatch, scratch and errors as glmq_gemm with bits = 4; zero must not be
 * NULL (GLMQ_ERR_NULL_POINTER).
 */
GLMQ_API glmq_status glmq_gemm_zp(const void* X, int64_t M, const void* packed, const void* scale, const void* zero,
                                  int64_t N, int64_t K, void* Y, void* stream);

/*
 * glmq_gemm_decode without any device allocation (the paper has no counterpart:
 * this is a deployment variant of the decode kernel).
 *
 * glmq_gemm_decode may allocate its split-K scratch with cudaMalloc on first use.
 * Some callers cannot let a library do that: a host framework whose caching
 * allocator or fixed-size arena owns the whole device-memory budget (an
 * allocation behind its back can fail, or push the framework out of memory), and
 * serving loops with a latency budget, where cudaMalloc can synchronize the device
 * and block in the driver. This entry point never allocates. Its scratch is a
 * fixed, statically allocated device array of GLMQ_NOALLOC_SCRATCH_FLOATS fp32
 * values (4 MiB) that every GPU which loads the library holds until the process
 * exits.
 *   - Same arguments, layout and results as glmq_gemm_decode (M <= 16).
 *   - Requires M * N <= GLMQ_NOALLOC_SCRATCH_FLOATS, else GLMQ_ERR_BAD_SHAPE and
 *     nothing is enqueued.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress, no allocation); make that first call before any
 *     stream capture on that device.
 *   - All calls share the one array, and it keeps the last call's contents: a call
 *     whose tiles are split over K parts clears the part it accumulates into, on its
 *     stream, before its kernel runs. Calls that overlap on the GPU (different
 *     streams, no ordering between them) race on the array and may produce wrong
 *     results.
 */
#define GLMQ_NOALLOC_SCRATCH_FLOATS (1u << 20)
GLMQ_API glmq_status glmq_gemm_decode_noalloc(const void* X, int64_t M, const void* packed, const void* scale,
                                              int64_t N, int64_t K, int bits, void* Y, void* stream);

/* Static description of a status code. Never NULL. */
GLMQ_API const char* glmq_status_string(int status);

/* The cudaError_t value (as int) of the last failed CUDA call in this thread,
 * 0 if none. */
GLMQ_API int glmq_last_cuda_error(void);

/*
 * Number of kernels this library has enqueued since it was loaded, over all
 * devices and threads: quantize, decode, tensor-core and finalize kernels. The
 * stream memset of glmq_gemm_decode_noalloc is not a kernel and is not counted.
 * A launch recorded into a CUDA graph during stream capture counts once, when it
 * is captured; replays of the graph do not count. Host-only; never fails.
 */
GLMQ_API uint64_t glmq_kernel_launches(void);

/*
 * Synchronizes `stream`, then reads and clears the current device's status
 * word, which kernels set when a bounded internal wait gives up (instead of
 * hanging). Returns GLMQ_OK if the word was 0, else GLMQ_ERR_DEVICE and, if
 * `flags` is not NULL, stores the word's bits there. For tests and debugging:
 * it blocks the calling thread.
 */
GLMQ_API glmq_status glmq_last_device_error(void* stream, uint32_t* flags);

/*
 * Failure-detection hook (the paper has no counterpart). Every internal wait of
 * the kernels on a pipeline barrier gives up after a wall-clock limit, 2 s by
 * default, sets a bit in the device status word (see glmq_last_device_error) and
 * lets the kernel finish without hanging; its outputs are then not valid. This sets
 * that limit, in nanoseconds, for kernels launched afterwards on the current
 * device; 0 restores the default. Tests lower it to make a normal call's waits run
 * out and check that the failure is reported. The waits by which a block makes sure
 * its own copies and tensor-core operations have finished before it exits always
 * keep the default limit, so a lowered limit never ends a block with work in flight.
 * Not for production use. Synchronous with respect to the host; must not be called
 * while kernels of this library run on the device.
 * Errors: GLMQ_ERR_UNSUPPORTED_DEVICE, GLMQ_ERR_CUDA.
 */
GLMQ_API glmq_status glmq_set_wait_limit_ns(uint64_t limit_ns);

#ifdef __cplusplus
}
#endif

#endif /* GLMQ_H */
