"""Accuracy headroom at the longest rows the library accepts (K = 65536) and at the
FFN-down row length (K = 32768), with plain N(0, 1) activations and with the pages'
activation-outlier profile, on every route: decode (M <= 16), skinny (16 < M <= 64)
and prefill, INT4 and INT8.

The decode kernel accumulates biased products, (1032 + q) x and (1152 + 16 q) x / 16,
in fp32 and removes the bias once per 256-k segment, so its fp32 sums are larger than
the signal; the error grows with K and with activation outliers. Each case records
its observed relative max error (see GLMQ_ERROR_REPORT in conftest.py) and must stay
within the 5e-3 bar.
"""
import numpy as np
import pytest

import oracle
from gpu_helpers import record_error, to_dev, to_host, torch_cuda
from inputs import gaussian_fp16
from inputs.synthetic import outlier_activations

pytestmark = pytest.mark.gpu

TOL = 5e-3
N = 1024


@pytest.fixture(scope="module", params=[(4, 65536), (8, 65536), (4, 32768)], ids=lambda p: f"int{p[0]}-K{p[1]}")
def layer(request):
    torch_cuda()
    bits, K = request.param
    W = gaussian_fp16((N, K), 0.02, 6100 + K + bits)
    packed, scale = oracle.quantize_linear(W, bits)
    yield {"bits": bits, "K": K, "packed": packed, "scale": scale, "dev": (to_dev(packed), to_dev(scale))}


@pytest.mark.parametrize("acts", ["gaussian", "outliers"])
@pytest.mark.parametrize("M,route", [(1, "decode"), (16, "decode"), (64, "prefill"), (256, "prefill")])
def test_error_headroom(layer, M, route, acts):
    import int8_quantized_glmq_b200 as g
    bits, K = layer["bits"], layer["K"]
    X = gaussian_fp16((M, K), 1.0, 6200 + M) if acts == "gaussian" else outlier_activations(M, K, 6300 + M)
    Pd, Sd = layer["dev"]
    Y = to_host(g.gemm(to_dev(X), Pd, Sd, bits, route=route))
    ref = oracle.linear_forward(X, layer["packed"], layer["scale"], bits)
    assert np.all(np.isfinite(Y))
    kernel = "decode" if route == "decode" else ("skinny" if M <= 64 else "prefill")
    err = record_error(f"headroom/{kernel}/int{bits}/K={K}/M={M}/{acts}", oracle.relative_max_error(Y, ref))
    assert err <= TOL, err
