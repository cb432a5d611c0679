"""Parity at the full GLM-130B projection shapes (QKV 12288->36864, attn-out
12288->12288, FFN-up 12288->65536, FFN-down 32768->12288), in the launch
configuration the benchmark times.

The GPU quantizes and multiplies the whole projection; the oracle recomputes a
sample of output features (rows of W) one by one: the first and last 64 rows
(tile edges) and 128 random rows. Quantization works row by row, so a row's
codes do not depend on the other rows; each sampled output column of Y depends
only on its row of W.
"""
import numpy as np
import pytest

import oracle
from gpu_helpers import record_error, to_dev, to_host, torch_cuda
from inputs import GLM_PROJECTIONS, PROJECTION_ORDER, decode_activations, prefill_activations, projection_weight

pytestmark = pytest.mark.gpu

TOL = 5e-3


def sample_rows(N: int, seed: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    rows = np.concatenate([np.arange(64), np.arange(N - 64, N), rng.choice(N, 128, replace=False)])
    return np.unique(rows)


@pytest.fixture(scope="module", params=PROJECTION_ORDER)
def projection(request):
    torch = torch_cuda()
    import int8_quantized_glmq_b200 as glmq
    name = request.param
    idx = PROJECTION_ORDER.index(name)
    N, K = GLM_PROJECTIONS[name]
    W = projection_weight(name, seed=1000 + idx)
    Wd = to_dev(W)
    out = {"name": name, "N": N, "K": K, "rows": sample_rows(N, idx)}
    for bits in (4, 8):
        packed, scale = glmq.quantize(Wd, bits)
        torch.cuda.synchronize()
        out[bits] = (packed, scale)
    out["W_rows"] = W[out["rows"]]
    del Wd, W
    torch.cuda.empty_cache()
    yield out
    del out
    torch.cuda.empty_cache()


@pytest.mark.parametrize("bits", [4, 8])
def test_quantize_full_projection_sampled_rows(projection, bits):
    rows = projection["rows"]
    packed, scale = projection[bits]
    p_ref, s_ref = oracle.quantize_linear(projection["W_rows"], bits)
    p = to_host(packed[to_dev(rows.astype(np.int64))])
    s = to_host(scale)[rows]
    assert np.array_equal(s.view(np.uint16), s_ref.view(np.uint16))
    assert np.array_equal(p, p_ref)


def _check_gemm(projection, bits, M, seed):
    import int8_quantized_glmq_b200 as glmq
    K = projection["K"]
    rows = projection["rows"]
    X = decode_activations(M, K, seed) if M <= 16 else prefill_activations(M, K, seed)
    packed, scale = projection[bits]
    Y = glmq.gemm(to_dev(X), packed, scale, bits)
    Ys = to_host(Y[:, to_dev(rows.astype(np.int64))])
    p_rows, s_rows = oracle.quantize_linear(projection["W_rows"], bits)
    Y_ref = oracle.linear_forward_rows(X, p_rows, s_rows, bits)
    err = record_error(f"full/{projection['name']}/int{bits}/M={M}", oracle.relative_max_error(Ys, Y_ref))
    assert err <= TOL, err


@pytest.mark.parametrize("M", [1, 4, 16])
def test_decode_int4_full_projection(projection, M):
    _check_gemm(projection, 4, M, 2000 + M)


@pytest.mark.parametrize("M", [17, 32, 64])
def test_skinny_int4_full_projection(projection, M):
    """16 < M <= 64: the tcgen05 skinny kernel (A operand in tensor memory)."""
    _check_gemm(projection, 4, M, 5000 + M)


def test_prefill_int4_full_projection(projection):
    _check_gemm(projection, 4, 2048, 3000)


@pytest.mark.parametrize("M", [1, 64, 2048])
def test_int8_full_projection(projection, M):
    _check_gemm(projection, 8, M, 4000 + M)
