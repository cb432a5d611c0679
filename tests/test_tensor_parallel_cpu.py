"""Tensor-parallel sharding of the quantized linear layers, on CPU.

The GLM-130B paper card ("Paper vs code") runs the INT4 model 4-way model-parallel.
These tests check the host side of that split with the oracle standing in for the
local GEMM (the library's GEMM needs a GPU; its own parity is covered by the GPU
tests): shard slicing, bias placement, the GeGLU-packed column split, and the
all-gather / all-reduce run by two and by four gloo ranks on 127.0.0.1.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from inputs import gaussian_fp16  # noqa: E402
from int8_quantized_glmq_b200 import tensor_parallel as tp  # noqa: E402


def oracle_local(X, packed, scale, bits, bias=None, epilogue="none"):
    """The local GEMM of one shard, computed by the oracle (natural or GeGLU row layout)."""
    Xn, p, s = X.numpy(), packed.numpy(), scale.numpy()
    b = None if bias is None else bias.numpy()
    if epilogue == "geglu":
        inv = np.argsort(oracle.geglu_row_order(p.shape[0]))      # packed row of each natural row
        return torch.from_numpy(oracle.geglu_forward(Xn, p[inv], s[inv], bits, b))
    if b is None:
        return torch.from_numpy(oracle.linear_forward(Xn, p, s, bits))
    return torch.from_numpy(oracle.linear_bias_forward(Xn, p, s, bits, b))


def _layer(N, K, bits, seed, geglu=False):
    W = gaussian_fp16((N, K), 0.02, seed)
    p, s = oracle.quantize_linear_geglu(W, bits) if geglu else oracle.quantize_linear(W, bits)
    pn, sn = oracle.quantize_linear(W, bits)
    return torch.from_numpy(p), torch.from_numpy(s), pn, sn


@pytest.mark.parametrize("bits", [4, 8])
def test_column_shards_reproduce_the_unsharded_layer(bits):
    N, K, T = 256, 384, 4
    p, s, pn, sn = _layer(N, K, bits, 11)
    X = gaussian_fp16((3, K), 1.0, 12)
    parts = [tp.ColumnParallelLinear(p, s, bits, r, T, local=oracle_local).forward(torch.from_numpy(X))
             for r in range(T)]
    Y = torch.cat(parts, dim=1).numpy()
    assert np.array_equal(Y.view(np.uint16), oracle.linear_forward(X, pn, sn, bits).view(np.uint16))


def test_geglu_column_shards_with_bias():
    N, K, T = 512, 256, 4                       # F = 256 outputs, 64 per rank
    p, s, pn, sn = _layer(N, K, 4, 21, geglu=True)
    b = gaussian_fp16((1, N), 0.5, 22)[0]
    X = gaussian_fp16((5, K), 1.0, 23)
    parts = []
    for r in range(T):
        layer = tp.ColumnParallelLinear(p, s, 4, r, T, bias=torch.from_numpy(b), epilogue="geglu",
                                        local=oracle_local)
        assert layer.packed.shape[0] == N // T and layer.bias.shape[0] == N // T
        parts.append(layer.forward(torch.from_numpy(X)))
    Y = torch.cat(parts, dim=1).numpy()
    ref = oracle.geglu_forward(X, pn, sn, 4, b)
    assert Y.shape == (5, N // 2)
    assert np.array_equal(Y.view(np.uint16), ref.view(np.uint16))


def test_row_shards_keep_the_unsharded_codes_and_scales():
    N, K, T = 64, 1024, 4
    for bits in (4, 8):
        p, s, pn, sn = _layer(N, K, bits, 31)
        codes = oracle.unpack(pn, bits, K)
        for r in range(T):
            layer = tp.RowParallelLinear(p, s, bits, r, T, local=oracle_local)
            assert layer.K_local == K // T
            assert np.array_equal(oracle.unpack(layer.packed.numpy(), bits, K // T),
                                  codes[:, r * K // T:(r + 1) * K // T])
            assert np.array_equal(layer.scale.numpy().view(np.uint16), sn.view(np.uint16))


@pytest.mark.parametrize("bits", [4, 8])
def test_row_partials_sum_to_the_unsharded_layer(bits):
    N, K, T = 192, 1024, 4
    p, s, pn, sn = _layer(N, K, bits, 41)
    b = gaussian_fp16((1, N), 0.5, 42)[0]
    X = gaussian_fp16((4, K), 1.0, 43)
    acc = np.zeros((4, N), dtype=np.float32)
    for r in range(T):
        layer = tp.RowParallelLinear(p, s, bits, r, T, bias=torch.from_numpy(b), local=oracle_local)
        assert (layer.bias is not None) == (r == 0)            # the bias is added once
        acc += layer.partial(layer.local_input(torch.from_numpy(X))).numpy().astype(np.float32)
    ref = oracle.linear_bias_forward(X, pn, sn, bits, b)
    assert oracle.relative_max_error(acc.astype(np.float16), ref) <= 5e-3
    # without the bias on rank 0 the sum would be off by b: a check that it is there
    no_bias = oracle.linear_forward(X, pn, sn, bits).astype(np.float64)
    assert np.abs(acc - no_bias - b.astype(np.float64)).max() <= 5e-3 * np.abs(ref.astype(np.float64)).max()


def test_shard_validation():
    p = torch.zeros((48, 64), dtype=torch.uint8)
    s = torch.zeros((48,), dtype=torch.float16)
    with pytest.raises(ValueError):
        tp.column_shard(p, s, 0, 5)                            # 48 rows over 5 ranks
    with pytest.raises(ValueError):
        tp.row_shard(p, s, 4, 0, 4)                            # K = 128: 32 values per rank
    with pytest.raises(ValueError):
        tp.ColumnParallelLinear(p, s, 4, 0, 2, epilogue="geglu", local=oracle_local)   # 24-row GeGLU shard
    with pytest.raises(ValueError):
        tp.ColumnParallelLinear(p, s, 4, 0, 1, epilogue="relu", local=oracle_local)
    pk, sk = tp.row_shard(p, s, 4, 1, 2)                       # K = 128: 64 values per rank
    assert pk.shape == (48, 32) and sk is s


def test_single_rank_is_the_plain_layer():
    N, K = 64, 256
    p, s, pn, sn = _layer(N, K, 4, 51)
    X = gaussian_fp16((2, K), 1.0, 52)
    ref = oracle.linear_forward(X, pn, sn, 4)
    col = tp.ColumnParallelLinear(p, s, 4, 0, 1, local=oracle_local).forward(torch.from_numpy(X), gather=True)
    row = tp.RowParallelLinear(p, s, 4, 0, 1, local=oracle_local).forward(torch.from_numpy(X))
    assert np.array_equal(col.numpy().view(np.uint16), ref.view(np.uint16))
    assert np.array_equal(row.numpy().view(np.uint16), ref.view(np.uint16))


def _free_port():
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def _rank_main(rank, world, port, out_q):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        out = {}
        for N, M in ((128, 3), (768, 20)):        # 768 rows at M = 20: three overlapped row pieces
            K = 512
            p, s, _, _ = _layer(N, K, 4, 61 + N)
            b = torch.from_numpy(gaussian_fp16((1, N), 0.5, 62 + N)[0])
            X = torch.from_numpy(gaussian_fp16((M, K), 1.0, 63 + N))
            col = tp.ColumnParallelLinear(p, s, 4, rank, world, bias=b, local=oracle_local)
            row = tp.RowParallelLinear(p, s, 4, rank, world, bias=b, local=oracle_local)
            out[N] = (col.forward(X, gather=True).numpy(), row.forward(row.local_input(X)).numpy())
        out_q.put((rank, out))
    finally:
        dist.destroy_process_group()


def test_chunk_rows():
    assert tp.chunk_rows(768, 4) == [(0, 256), (256, 512), (512, 768)]
    assert tp.chunk_rows(12288, 4) == [(0, 3072), (3072, 6144), (6144, 9216), (9216, 12288)]
    assert tp.chunk_rows(300, 4) == [(0, 256), (256, 300)]
    assert tp.chunk_rows(100, 1) == [(0, 100)]
    assert tp.chunk_rows(0, 4) == []


@pytest.mark.parametrize("world", [2, 4])           # 4: the INT4 model's 4-way split
def test_gloo_ranks_gather_and_reduce(world):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for pr in procs:
        pr.start()
    got = sorted((q.get(timeout=120) for _ in range(world)), key=lambda t: t[0])
    for pr in procs:
        pr.join(timeout=60)
        if pr.is_alive():
            pr.kill()
            pytest.fail("a rank did not finish")
        assert pr.exitcode == 0

    for N, M in ((128, 3), (768, 20)):
        K = 512
        W = gaussian_fp16((N, K), 0.02, 61 + N)
        pn, sn = oracle.quantize_linear(W, 4)
        b = gaussian_fp16((1, N), 0.5, 62 + N)[0]
        X = gaussian_fp16((M, K), 1.0, 63 + N)
        ref = oracle.linear_bias_forward(X, pn, sn, 4, b)
        # the ranks' fp16 partials (rank 0 adds the bias), as the oracle computes them
        kl = K // world
        parts = [oracle.linear_bias_forward(X[:, :kl], pn[:, :kl // 2], sn, 4, b)]
        parts += [oracle.linear_forward(X[:, r * kl:(r + 1) * kl], pn[:, r * kl // 2:(r + 1) * kl // 2], sn, 4)
                  for r in range(1, world)]
        exact = np.sum([pt.astype(np.float64) for pt in parts], axis=0)
        for _, out in got:
            Yc, Yr = out[N]
            assert np.array_equal(Yc.view(np.uint16), ref.view(np.uint16))        # column: identical
            assert oracle.relative_max_error(Yr, ref) <= 5e-3
            if world == 2:
                # one fp16 rounding of the sum of the two partials (exact in fp32)
                two = (parts[0].astype(np.float32) + parts[1].astype(np.float32)).astype(np.float16)
                assert np.array_equal(Yr.view(np.uint16), two.view(np.uint16))
            else:
                # world - 1 fp16 roundings of partial sums, in the collective's order
                bound = (world - 1) * 2.0 ** -11 * np.abs(exact).max() * 2
                assert np.abs(Yr.astype(np.float64) - exact).max() <= bound
