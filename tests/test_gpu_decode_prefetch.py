"""GPU checks of glmq_gemm_decode_prefetch: the decode GEMM that also prefetches the
next call's first weight tiles into L2.

The hint only issues L2 prefetches, so Y is what glmq_gemm_decode computes. Tiles
split over K parts add fp32 partial sums atomically, in an order that can differ from
run to run for either call, so the two outputs may differ by one fp16 ulp there (or,
near zero, by the absolute fp32 reordering error); every case checks that bound and the
oracle's accuracy bar. The cases
cover next calls with other M (other kernel configurations and K-part plans), other N
and K, the same weights again, INT8, a chain of hinted calls in a CUDA graph (the way
a decode step uses it), and next weights whose last tile is ragged.
"""
import numpy as np
import pytest

import oracle
from gpu_helpers import to_dev, to_host, torch_cuda
from inputs import gaussian_fp16

pytestmark = pytest.mark.gpu


def glmq():
    torch_cuda()
    import int8_quantized_glmq_b200 as g
    return g


def assert_within_one_ulp(a, b):
    """|a - b| <= one fp16 ulp, or, for outputs near zero (where the partial sums cancel
    and their fp32 reordering error is absolute), <= 1e-4 of the largest output."""
    a64, b64 = a.astype(np.float64), b.astype(np.float64)
    ulp = np.spacing(np.maximum(np.abs(a), np.abs(b)).astype(np.float16)).astype(np.float64)
    bound = np.maximum(ulp, 1e-4 * np.max(np.abs(b64)))
    assert np.all(np.abs(a64 - b64) <= bound), float(np.max(np.abs(a64 - b64) / bound))


def _layer(g, N, K, bits, seed):
    W = gaussian_fp16((N, K), 0.02, seed)
    p, s = g.quantize(to_dev(W), bits)
    return W, p, s


# (M, N, K) of this call, (next_M, next_N, next_K) of the hinted next call
CASES = [
    ((1, 4096, 2048), (16, 2048, 4096)),
    ((4, 2048, 4096), (1, 4096, 2048)),
    ((16, 1024, 1024), (4, 3000, 1024)),        # next N ragged (last tile partial)
    ((1, 38400, 128), (1, 38400, 128)),
    ((7, 1536, 3072), (7, 1536, 3072)),
]


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("cur,nxt", CASES)
def test_prefetch_hint_leaves_output_unchanged(bits, cur, nxt):
    g = glmq()
    M, N, K = cur
    nM, nN, nK = nxt
    W, p, s = _layer(g, N, K, bits, 900 + N)
    _, pn, _ = _layer(g, nN, nK, bits, 901 + nN)
    Xh = gaussian_fp16((M, K), 1.0, 902 + M)
    X = to_dev(Xh)
    Y_plain = to_host(g.gemm_decode(X, p, s, bits))
    Y_hint = to_host(g.gemm_decode_prefetch(X, p, s, bits, next_packed=pn, next_M=nM))
    assert_within_one_ulp(Y_hint, Y_plain)
    pr, sr = oracle.quantize_linear(W, bits)
    assert oracle.relative_max_error(Y_hint, oracle.linear_forward(Xh, pr, sr, bits)) <= 2e-3


def test_prefetch_hint_against_oracle():
    g = glmq()
    W, p, s = _layer(g, 2048, 1024, 4, 910)
    _, pn, _ = _layer(g, 1024, 2048, 4, 911)
    X = gaussian_fp16((3, 1024), 1.0, 912)
    Y = to_host(g.gemm_decode_prefetch(to_dev(X), p, s, 4, next_packed=pn, next_M=3))
    pr, sr = oracle.quantize_linear(W, 4)
    assert oracle.relative_max_error(Y, oracle.linear_forward(X, pr, sr, 4)) <= 2e-3


def test_hinted_chain_in_a_graph_matches_plain_calls():
    """Four projections of different shapes, each call hinting the next (the last the
    first), captured in a CUDA graph and replayed; outputs match the plain calls'."""
    torch = torch_cuda()
    g = glmq()
    shapes = [(3072, 1024), (1024, 1024), (4096, 1024), (1024, 2048)]
    layers = [_layer(g, N, K, 4, 920 + i) for i, (N, K) in enumerate(shapes)]
    Ms = [1, 4, 16, 2]
    xs = [to_dev(gaussian_fp16((m, K), 1.0, 930 + i)) for i, (m, (_, K)) in enumerate(zip(Ms, shapes))]
    ref = [to_host(g.gemm_decode(x, p, s, 4)) for x, (_, p, s) in zip(xs, layers)]
    ys = [torch.empty((m, N), dtype=torch.float16, device="cuda") for m, (N, _) in zip(Ms, shapes)]

    def step():
        for i, (x, (_, p, s)) in enumerate(zip(xs, layers)):
            j = (i + 1) % len(layers)
            g.gemm_decode_prefetch(x, p, s, 4, next_packed=layers[j][1], next_M=Ms[j], out=ys[i])

    step()                                          # sizes the scratch outside capture
    torch.cuda.synchronize()
    cs = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=cs):
        step()
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    for y, r in zip(ys, ref):
        assert_within_one_ulp(to_host(y), r)
    st, flags = g.last_device_error()
    assert st == 0, f"device status {flags:#x}"
    del graph
