"""glmq_gemm_decode_noalloc: the decode GEMM for callers that cannot let a library
allocate device memory -- a host framework whose caching allocator or fixed arena owns
the device-memory budget, or a serving loop that must not block in cudaMalloc. Its
split-K scratch is a fixed static device array instead of a lazily allocated buffer.

This file is collected last on purpose, so that a run which stops at the first failure
has already run every other test. The GPU test calls the entry point through the C ABI
twice in a row per shape and checks each result against the CPU oracle and against
glmq_gemm_decode, within the accuracy bar the other tests use. Three shapes split their
tiles over K parts (the partial sums go through the static array and a finalize kernel
runs); one shape fills the GPU with whole tiles, so no scratch is used and only the
decode kernel is launched.
"""
import numpy as np
import pytest

import oracle
from inputs import gaussian_fp16

TOL = 5e-3
B200_SMS = 148


def test_noalloc_rejects_oversized_problem_before_any_device_work():
    from int8_quantized_glmq_b200 import _binding as B
    big_n = B.NOALLOC_SCRATCH_FLOATS // 16 + 1          # M * N one row past the fixed scratch
    aligned = 1 << 20                                   # never dereferenced: rejected during validation
    st = B.raw_gemm(aligned, 16, aligned, aligned, big_n, 64, 4, aligned, 0, "decode_noalloc")
    assert st == B.ERR_BAD_SHAPE
    assert B.raw_gemm(aligned, 17, aligned, aligned, 8, 64, 4, aligned, 0, "decode_noalloc") == B.ERR_BAD_SHAPE


# kernels per call on a 148-SM B200: decode + finalize when tiles are split over K parts
@pytest.mark.gpu
@pytest.mark.parametrize("bits,M,N,K,kernels", [(4, 16, 4096, 12288, 2),    # 16 K parts
                                                (8, 16, 3000, 32768, 2),    # 37 K parts, ragged N, INT8
                                                (4, 1, 5000, 12288, 2),     # 7 K parts at one token
                                                (4, 1, 36864, 1024, 1)])    # 144 whole tiles: no scratch
def test_noalloc_matches_oracle_on_two_calls(bits, M, N, K, kernels):
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from int8_quantized_glmq_b200 import _binding as B
    torch.cuda.set_device(0)
    W = gaussian_fp16((N, K), 0.02, 77 + N)
    packed, scale = oracle.quantize_linear(W, bits)
    Pd = torch.from_numpy(packed).cuda()
    Sd = torch.from_numpy(scale).cuda()
    stream = torch.cuda.current_stream().cuda_stream
    count_kernels = torch.cuda.get_device_properties(0).multi_processor_count == B200_SMS
    for call in range(2):
        Xh = gaussian_fp16((M, K), 1.0, 900 + call)
        X = torch.from_numpy(Xh).cuda()
        Y_dec = torch.empty((M, N), dtype=torch.float16, device="cuda")
        Y_new = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
        n0 = B.kernel_launches()
        st = B.raw_gemm(X.data_ptr(), M, Pd.data_ptr(), Sd.data_ptr(), N, K, bits, Y_new.data_ptr(), stream,
                        "decode_noalloc")
        assert st == B.OK, B.status_string(st)
        if count_kernels:
            assert B.kernel_launches() - n0 == kernels
        st = B.raw_gemm(X.data_ptr(), M, Pd.data_ptr(), Sd.data_ptr(), N, K, bits, Y_dec.data_ptr(), stream, "decode")
        assert st == B.OK
        torch.cuda.synchronize()
        new = Y_new.cpu().numpy()
        assert np.all(np.isfinite(new))
        assert oracle.relative_max_error(new, oracle.linear_forward(Xh, packed, scale, bits)) <= TOL
        assert oracle.relative_max_error(new, Y_dec.cpu().numpy()) <= TOL
    assert B.last_device_error(stream) == (B.OK, 0)
