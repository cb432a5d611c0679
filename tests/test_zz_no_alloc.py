"""glmq_gemm_decode_noalloc: the decode GEMM for callers that cannot allocate device
memory (graph capture, a framework-owned memory pool, no driver calls that may block
after start-up). It keeps its split-K scratch in a fixed static device array.

This file is collected last on purpose. The GPU test calls the new entry point
through the C ABI twice in a row and checks each result against glmq_gemm_decode,
within the accuracy bar the other tests use. It covers a shape whose tiles are split
over K parts (so the static scratch is used) and one whose tiles are not.
"""
import numpy as np
import pytest

import oracle
from inputs import gaussian_fp16

TOL = 5e-3


def test_noalloc_rejects_oversized_problem_before_any_device_work():
    from int8_quantized_glmq_b200 import _binding as B
    big_n = B.NOALLOC_SCRATCH_FLOATS // 16 + 1          # M * N one row past the fixed scratch
    aligned = 1 << 20                                   # never dereferenced: rejected during validation
    st = B.raw_gemm(aligned, 16, aligned, aligned, big_n, 64, 4, aligned, 0, "decode_noalloc")
    assert st == B.ERR_BAD_SHAPE
    assert B.raw_gemm(aligned, 17, aligned, aligned, 8, 64, 4, aligned, 0, "decode_noalloc") == B.ERR_BAD_SHAPE


@pytest.mark.gpu
@pytest.mark.parametrize("bits,M,N,K", [(4, 16, 4096, 12288),    # split over K parts: uses the static scratch
                                        (8, 16, 3000, 32768),    # split, ragged N, INT8
                                        (4, 1, 5000, 12288)])    # single K part: no scratch
def test_noalloc_matches_decode_on_two_calls(bits, M, N, K):
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
    for call in range(2):
        X = torch.from_numpy(gaussian_fp16((M, K), 1.0, 900 + call)).cuda()
        Y_ref = torch.empty((M, N), dtype=torch.float16, device="cuda")
        Y_new = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
        st = B.raw_gemm(X.data_ptr(), M, Pd.data_ptr(), Sd.data_ptr(), N, K, bits, Y_ref.data_ptr(), stream, "decode")
        assert st == B.OK
        st = B.raw_gemm(X.data_ptr(), M, Pd.data_ptr(), Sd.data_ptr(), N, K, bits, Y_new.data_ptr(), stream,
                        "decode_noalloc")
        assert st == B.OK, B.status_string(st)
        torch.cuda.synchronize()
        ref = Y_ref.cpu().numpy()
        new = Y_new.cpu().numpy()
        assert np.all(np.isfinite(new))
        assert oracle.relative_max_error(new, ref) <= TOL
    assert B.last_device_error(stream) == (B.OK, 0)
