"""GPU parity of the fused epilogues (glmq_gemm_fused, glmq_quantize_geglu) against the
epilogue oracle, through the C ABI.

Shapes are chosen to reach every code path: large N with a short K leaves one K part
per tile, so the decode, skinny and prefill kernels apply the epilogue themselves
(decode per lane, skinny and prefill across TMEM lanes of a warp); small N splits
tiles over K parts, so the finalize kernel applies it."""
import numpy as np
import pytest

import oracle
from gpu_helpers import to_dev, to_host, torch_cuda
from inputs import gaussian_fp16

pytestmark = pytest.mark.gpu

TOL = 5e-3
TIGHT = 2e-3


def glmq():
    torch_cuda()
    import int8_quantized_glmq_b200 as g
    return g


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("N,K", [(96, 512), (2048, 1024)])
def test_quantize_geglu_layout_bit_exact(bits, N, K):
    g = glmq()
    W = gaussian_fp16((N, K), 0.02, 100 + N)
    p_ref, s_ref = oracle.quantize_linear_geglu(W, bits)
    p, s = g.quantize(to_dev(W), bits, geglu=True)
    assert np.array_equal(to_host(s).view(np.uint16), s_ref.view(np.uint16))
    assert np.array_equal(to_host(p), p_ref)


def test_quantize_geglu_rejects_rows_not_multiple_of_16():
    g = glmq()
    from int8_quantized_glmq_b200 import _binding as B
    W = to_dev(gaussian_fp16((40, 64), 0.02, 1))
    with pytest.raises(B.GlmqError):
        g.quantize(W, 4, geglu=True)


# (M, N, K): decode / skinny / prefill, each with one K part (fused in the kernel) and
# with several K parts (fused in the finalize kernel)
CASES = [(1, 38400, 128), (5, 38400, 64), (16, 38400, 128), (40, 19200, 128), (300, 19200, 128),
         (1, 1024, 2048), (16, 512, 1024), (40, 1024, 1024), (300, 512, 1024)]


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("M,N,K", CASES)
def test_bias_epilogue(bits, M, N, K):
    g = glmq()
    W = gaussian_fp16((N, K), 0.05, 200 + M)
    b = gaussian_fp16((1, N), 0.5, 300 + M)[0]
    X = gaussian_fp16((M, K), 1.0, 400 + M)
    packed, s = oracle.quantize_linear(W, bits)
    Y = to_host(g.gemm_fused(to_dev(X), to_dev(packed), to_dev(s), bits, bias=to_dev(b)))
    ref = oracle.linear_bias_forward(X, packed, s, bits, b)
    err = oracle.relative_max_error(Y, ref)
    assert err <= TOL and err <= TIGHT, err


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("with_bias", [False, True])
@pytest.mark.parametrize("M,N,K", CASES)
def test_geglu_epilogue(bits, with_bias, M, N, K):
    g = glmq()
    W = gaussian_fp16((N, K), 0.08, 500 + M)
    b = gaussian_fp16((1, N), 0.5, 600 + M)[0] if with_bias else None
    X = gaussian_fp16((M, K), 1.0, 700 + M)
    p_nat, s_nat = oracle.quantize_linear(W, bits)
    packed, s = g.quantize(to_dev(W), bits, geglu=True)
    Y = to_host(g.gemm_fused(to_dev(X), packed, s, bits, bias=None if b is None else to_dev(b), epilogue="geglu"))
    assert Y.shape == (M, N // 2)
    ref = oracle.geglu_forward(X, p_nat, s_nat, bits, b)
    assert np.all(np.isfinite(Y))
    err = oracle.relative_max_error(Y, ref)
    assert err <= TOL and err <= TIGHT, err


def test_fused_none_without_bias_equals_gemm():
    g = glmq()
    W = gaussian_fp16((1024, 1024), 0.02, 9)
    X = to_dev(gaussian_fp16((4, 1024), 1.0, 10))
    packed, s = g.quantize(to_dev(W), 4)
    assert np.array_equal(to_host(g.gemm_fused(X, packed, s, 4)), to_host(g.gemm(X, packed, s, 4)))
