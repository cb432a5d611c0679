"""Prefill calls whose last round of tiles is split over K parts.

With at least as many tiles as SMs, the tensor-core kernel keeps the tiles of the
whole rounds of its persistent CTAs whole and splits the weight-row bands from the
last, partial round on over K parts (partial sums through the scratch, then a finalize
pass over those rows only). These shapes have 150 tiles on a 148-SM B200: 147 or 148
whole tiles and a split tail. Every output is compared with the oracle, so both the
whole tiles (written by the kernel) and the split rows (written by the finalize pass,
with the fused bias / GeGLU epilogue where asked) are checked, and the launch counter
shows that the finalize pass ran.
"""
import numpy as np
import pytest

import oracle
from gpu_helpers import record_error, to_dev, to_host, torch_cuda
from inputs import gaussian_fp16

TOL = 5e-3
# (bits, M, N, K): INT4 above M = 256 uses 192-token tiles (3 per 512 tokens, 50 row
# tiles of 128); INT8 above M = 128 uses 256-token tiles (2 per 300 tokens, 75 row tiles)
CASES = [(4, 512, 6400, 4096), (8, 300, 9600, 4096)]


def glmq():
    torch_cuda()
    import int8_quantized_glmq_b200 as g
    return g


@pytest.mark.gpu
@pytest.mark.parametrize("bits,M,N,K", CASES)
def test_tail_split_prefill_matches_oracle(bits, M, N, K):
    g = glmq()
    W = gaussian_fp16((N, K), 0.02, 7100 + bits)
    X = gaussian_fp16((M, K), 1.0, 7200 + bits)
    packed, s = oracle.quantize_linear(W, bits)
    Xd, pd, sd = to_dev(X), to_dev(packed), to_dev(s)
    g.gemm(Xd, pd, sd, bits)                         # scratch allocated outside the count
    n0 = g.kernel_launches()
    Y = to_host(g.gemm(Xd, pd, sd, bits))
    assert g.kernel_launches() - n0 == 2             # the tensor-core kernel and the finalize pass
    err = record_error(f"prefill_tail/int{bits}/M{M}_N{N}_K{K}", oracle.relative_max_error(
        Y, oracle.linear_forward(X, packed, s, bits)))
    assert err <= TOL, err
    assert g.last_device_error()[0] == 0


@pytest.mark.gpu
def test_tail_split_prefill_fused_epilogues():
    g = glmq()
    M, N, K = 512, 6400, 4096
    W = gaussian_fp16((N, K), 0.08, 7300)
    b = gaussian_fp16((1, N), 0.5, 7301)[0]
    X = gaussian_fp16((M, K), 1.0, 7302)
    p_nat, s_nat = oracle.quantize_linear(W, 4)
    Xd = to_dev(X)
    Y = to_host(g.gemm_fused(Xd, to_dev(p_nat), to_dev(s_nat), 4, bias=to_dev(b)))
    err = oracle.relative_max_error(Y, oracle.linear_bias_forward(X, p_nat, s_nat, 4, b))
    assert err <= TOL, err
    packed, s = g.quantize(to_dev(W), 4, geglu=True)
    Y = to_host(g.gemm_fused(Xd, packed, s, 4, bias=to_dev(b), epilogue="geglu"))
    assert Y.shape == (M, N // 2)
    ref = oracle.geglu_forward(X, p_nat, s_nat, 4, b)
    assert np.all(np.isfinite(Y))
    err = oracle.relative_max_error(Y, ref)
    assert err <= TOL, err


@pytest.mark.gpu
def test_tail_split_prefill_zero_point():
    g = glmq()
    M, N, K = 512, 6400, 4096
    W = gaussian_fp16((N, K), 0.02, 7400)
    X = gaussian_fp16((M, K), 1.0, 7401)
    p, s, z = oracle.quantize_linear_zp(W)
    Y = to_host(g.gemm_zp(to_dev(X), to_dev(p), to_dev(s), to_dev(z)))
    err = oracle.relative_max_error(Y, oracle.linear_forward_zp(X, p, s, z))
    assert err <= TOL, err
