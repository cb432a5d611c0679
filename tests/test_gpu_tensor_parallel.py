"""GPU parity of the tensor-parallel shards (int8_quantized_glmq_b200.tensor_parallel)
with the library's GEMM as the local step, through the C ABI.

The GLM-130B paper card ("Paper vs code") runs the INT4 model 4-way model-parallel.
With one GPU the four ranks are emulated one after another, each running its own
shard: no collective runs and no kernel waits on another. The host concatenates the
column-parallel outputs and sums the row-parallel partials, which is what the
all-gather and the all-reduce compute (the collectives themselves, and the fp16
rounding of the reduction, are covered by the gloo tests on CPU).
"""
import numpy as np
import pytest

import oracle
from gpu_helpers import to_dev, to_host, torch_cuda
from inputs import GLM_PROJECTIONS, decode_activations, gaussian_fp16, projection_weight

pytestmark = pytest.mark.gpu

TOL = 5e-3
T = 4


def modules():
    torch_cuda()
    import int8_quantized_glmq_b200 as g
    from int8_quantized_glmq_b200 import tensor_parallel as tp
    return g, tp


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("M", [1, 16, 64])
def test_column_parallel_shards(bits, M):
    g, tp = modules()
    N, K = 2048, 1024
    W = gaussian_fp16((N, K), 0.02, 700 + M)
    X = gaussian_fp16((M, K), 1.0, 710 + M)
    p, s = g.quantize(to_dev(W), bits)
    parts = [to_host(tp.ColumnParallelLinear(p, s, bits, r, T).forward(to_dev(X))) for r in range(T)]
    assert all(part.shape == (M, N // T) for part in parts)
    pn, sn = oracle.quantize_linear(W, bits)
    assert oracle.relative_max_error(np.concatenate(parts, axis=1), oracle.linear_forward(X, pn, sn, bits)) <= TOL


@pytest.mark.parametrize("M", [1, 64])
def test_column_parallel_geglu_shards_with_bias(M):
    g, tp = modules()
    N, K = 1024, 512
    W = gaussian_fp16((N, K), 0.05, 720 + M)
    b = gaussian_fp16((1, N), 0.5, 721 + M)[0]
    X = gaussian_fp16((M, K), 1.0, 722 + M)
    p, s = g.quantize(to_dev(W), 4, geglu=True)
    parts = [to_host(tp.ColumnParallelLinear(p, s, 4, r, T, bias=to_dev(b), epilogue="geglu").forward(to_dev(X)))
             for r in range(T)]
    pn, sn = oracle.quantize_linear(W, 4)
    ref = oracle.geglu_forward(X, pn, sn, 4, b)
    assert oracle.relative_max_error(np.concatenate(parts, axis=1), ref) <= TOL


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("M", [1, 16, 64])
def test_row_parallel_partials(bits, M):
    g, tp = modules()
    N, K = 1024, 4096
    W = gaussian_fp16((N, K), 0.02, 730 + M)
    b = gaussian_fp16((1, N), 0.5, 731 + M)[0]
    X = gaussian_fp16((M, K), 1.0, 732 + M)
    p, s = g.quantize(to_dev(W), bits)
    pn, sn = oracle.quantize_linear(W, bits)
    Xd = to_dev(X)
    kb = K // T * bits // 8
    acc = np.zeros((M, N), dtype=np.float32)
    for r in range(T):
        layer = tp.RowParallelLinear(p, s, bits, r, T, bias=to_dev(b))
        part = to_host(layer.partial(layer.local_input(Xd)))
        Xr = X[:, r * K // T:(r + 1) * K // T]
        pr = pn[:, r * kb:(r + 1) * kb]
        ref_r = oracle.linear_bias_forward(Xr, pr, sn, bits, b) if r == 0 else oracle.linear_forward(Xr, pr, sn, bits)
        assert oracle.relative_max_error(part, ref_r) <= TOL
        acc += part.astype(np.float32)
    assert oracle.relative_max_error(acc.astype(np.float16), oracle.linear_bias_forward(X, pn, sn, bits, b)) <= TOL


def _sample_rows(N, seed):
    rng = np.random.default_rng(seed)
    return np.unique(np.concatenate([np.arange(32), np.arange(N - 32, N), rng.choice(N, 64, replace=False)]))


@pytest.mark.parametrize("M", [1, 16])
def test_glm_attn_out_row_parallel_int4(M):
    """attn-out 12288 -> 12288 split 4 ways over K (3072 per rank), sampled output rows."""
    g, tp = modules()
    N, K = GLM_PROJECTIONS["attn_out"]
    W = projection_weight("attn_out", seed=1001)
    rows = _sample_rows(N, 5)
    p, s = g.quantize(to_dev(W), 4)
    pn, sn = oracle.quantize_linear(W[rows], 4)
    X = decode_activations(M, K, 740 + M)
    Xd = to_dev(X)
    ridx = to_dev(rows.astype(np.int64))
    kb = K // T // 2
    acc = np.zeros((M, rows.size), dtype=np.float32)
    for r in range(T):
        layer = tp.RowParallelLinear(p, s, 4, r, T)
        part = to_host(layer.partial(layer.local_input(Xd))[:, ridx])
        ref_r = oracle.linear_forward(X[:, r * K // T:(r + 1) * K // T], pn[:, r * kb:(r + 1) * kb], sn, 4)
        assert oracle.relative_max_error(part, ref_r) <= TOL
        acc += part.astype(np.float32)
    assert oracle.relative_max_error(acc.astype(np.float16), oracle.linear_forward(X, pn, sn, 4)) <= TOL


@pytest.mark.parametrize("M", [1, 16])
def test_glm_qkv_column_parallel_int4(M):
    """QKV 12288 -> 36864 split 4 ways over N (9216 rows per rank), sampled rows of each shard."""
    g, tp = modules()
    N, K = GLM_PROJECTIONS["qkv"]
    W = projection_weight("qkv", seed=1000)
    p, s = g.quantize(to_dev(W), 4)
    X = decode_activations(M, K, 750 + M)
    Xd = to_dev(X)
    n = N // T
    for r in range(T):
        Y = tp.ColumnParallelLinear(p, s, 4, r, T).forward(Xd)
        rows = _sample_rows(n, 10 + r)
        pn, sn = oracle.quantize_linear(W[r * n + rows], 4)
        got = to_host(Y[:, to_dev(rows.astype(np.int64))])
        assert oracle.relative_max_error(got, oracle.linear_forward(X, pn, sn, 4)) <= TOL


@pytest.mark.parametrize("M", [1, 20])
def test_row_parallel_pieces_match_the_whole_partial(M):
    """The overlapped forward runs the local GEMM in pieces of output rows (chunk_rows):
    each piece, computed through the C ABI on its row slice of the shard, matches the
    columns of the whole partial (up to the fp32 summation order of a different K split)."""
    g, tp = modules()
    N, K = 1536, 2048
    W = gaussian_fp16((N, K), 0.02, 900 + M)
    X = gaussian_fp16((M, K), 1.0, 910 + M)
    p, s = g.quantize(to_dev(W), 4)
    layer = tp.RowParallelLinear(p, s, 4, 1, T)
    Xl = layer.local_input(to_dev(X))
    whole = to_host(layer.partial(Xl))
    pieces = tp.chunk_rows(N, 4)
    assert len(pieces) > 1
    for n0, n1 in pieces:
        assert oracle.relative_max_error(to_host(layer.partial(Xl, n0, n1)), whole[:, n0:n1]) <= 1e-3
