"""GPU parity of the zero-point INT4 variant (glmq_quantize_zp, glmq_gemm_zp) against
its oracle, through the C ABI: codes, scales and zero points bit-exact; Y within the
accuracy bar on every kernel (decode, skinny, prefill; with and without K splits)."""
import numpy as np
import pytest

import oracle
from gpu_helpers import edge_case_weight, to_dev, to_host, torch_cuda
from inputs import gaussian_fp16, tiny_weight
from inputs.synthetic import outlier_activations

pytestmark = pytest.mark.gpu

TOL = 5e-3
TIGHT = 2e-3


def glmq():
    torch_cuda()
    import int8_quantized_glmq_b200 as g
    return g


def check_quantize_zp(W):
    g = glmq()
    p_ref, s_ref, z_ref = oracle.quantize_linear_zp(W)
    p, s, z = g.quantize_zp(to_dev(W))
    assert np.array_equal(to_host(s).view(np.uint16), s_ref.view(np.uint16)), "scales differ"
    assert np.array_equal(to_host(z), z_ref), "zero points differ"
    p = to_host(p)
    if not np.array_equal(p, p_ref):
        bad = np.argwhere(p != p_ref)
        raise AssertionError(f"{len(bad)} packed bytes differ, first at {bad[0]}")
    return p_ref, s_ref, z_ref


@pytest.mark.parametrize("shape", [(256, 512), (96, 64), (300, 12288), (64, 32768), (40, 65536)])
def test_quantize_zp_bit_exact(shape):
    check_quantize_zp(gaussian_fp16(shape, 0.02, 11 + shape[1]))


def test_quantize_zp_tiny_config_and_edge_rows():
    check_quantize_zp(tiny_weight())
    W = edge_case_weight(64, 512)
    W[5] = np.float16(0.25)                         # constant positive row
    W[6] = np.float16(-3.0)                         # constant negative row
    rng = np.random.default_rng(3)
    W[7] = (rng.random(512) * 0.05).astype(np.float16)          # skewed positive
    check_quantize_zp(W)


CASES = [(1, 1024, 12288), (4, 512, 4096), (16, 1024, 12288), (1, 38400, 128), (16, 38400, 128),
         (40, 1024, 4096), (40, 19200, 128), (300, 512, 4096), (300, 19200, 128)]


@pytest.mark.parametrize("M,N,K", CASES)
def test_gemm_zp(M, N, K):
    g = glmq()
    W = gaussian_fp16((N, K), 0.02, 30 + M)
    X = gaussian_fp16((M, K), 1.0, 40 + M)
    packed, s, z = oracle.quantize_linear_zp(W)
    Y = to_host(g.gemm_zp(to_dev(X), to_dev(packed), to_dev(s), to_dev(z)))
    ref = oracle.linear_forward_zp(X, packed, s, z)
    err = oracle.relative_max_error(Y, ref)
    assert err <= TOL and err <= TIGHT, err


@pytest.mark.parametrize("M", [1, 16, 40, 300])
def test_gemm_zp_outlier_activations(M):
    g = glmq()
    W = gaussian_fp16((512, 12288), 0.02, 50 + M)
    X = outlier_activations(M, 12288, 60 + M)
    packed, s, z = oracle.quantize_linear_zp(W)
    Y = to_host(g.gemm_zp(to_dev(X), to_dev(packed), to_dev(s), to_dev(z)))
    ref = oracle.linear_forward_zp(X, packed, s, z)
    err = oracle.relative_max_error(Y, ref)
    assert err <= TOL and err <= TIGHT, err
