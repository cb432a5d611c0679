"""Back-to-back decode calls: every bounded wait completes and every output is right.

Each barrier of a ring stage must have one waiting warp that takes every phase in
order: a parity wait cannot tell phase n from phase n + 2, so a warp that waits on a
phase before the previous one has completed passes at once and reads a slot whose
copy is still in flight. Such a race is rare and needs load: it shows up as a wrong
output and, later, as a wait that runs out (GLMQ_ERR_DEVICE from
glmq_last_device_error). Here several thousand decode calls run back to back from one
CUDA graph: M = 16, 4 and 1 mixed (the ring has 5 stages at M = 16 and 6 below, with
one or three activation warps), on an unsplit and a split-K shape, plus zero-point
INT4 codes at M = 16. The device status word is read after every replay, and the
outputs are checked against the oracle.
"""
import numpy as np
import pytest

import oracle
from gpu_helpers import record_error, to_dev, to_host, torch_cuda
from inputs import gaussian_fp16

TOL = 5e-3
SHAPES = [(36864, 4096), (12288, 12288)]   # (N, K): 144 unsplit tiles; 48 tiles in K parts
MS = (16, 4, 16, 1)
REPEATS = 25                               # per graph: 25 x (4 x 2 + 1) = 225 calls
REPLAYS = 12


@pytest.mark.gpu
def test_back_to_back_decode_calls_complete_every_wait():
    torch = torch_cuda()
    import int8_quantized_glmq_b200 as glmq
    from int8_quantized_glmq_b200 import _binding as B
    weights = []
    for i, (N, K) in enumerate(SHAPES):
        W = gaussian_fp16((N, K), 0.02, 6100 + i)
        packed, scale = glmq.quantize(to_dev(W), 4)
        rows = np.unique(np.concatenate([np.arange(32), np.arange(N - 32, N),
                                         np.random.default_rng(6110 + i).choice(N, 64, replace=False)]))
        weights.append((N, K, packed, scale, W[rows], rows))
        del W
    # zero-point INT4 codes on the split shape (the same ring of 5 stages at M = 16)
    Nz, Kz = SHAPES[1]
    Wz = gaussian_fp16((Nz, Kz), 0.02, 6120)
    pzd, szd, zzd = glmq.quantize_zp(to_dev(Wz))
    zrows = weights[1][5]
    wz_rows = Wz[zrows]
    del Wz
    xz = gaussian_fp16((16, Kz), 1.0, 6130)
    xzd = to_dev(xz)
    yz = torch.empty((16, Nz), dtype=torch.float16, device="cuda")
    xs = {(m, i): gaussian_fp16((m, K), 1.0, 6200 + 10 * m + i) for i, (N, K, *_) in enumerate(weights)
          for m in set(MS)}
    xd = {key: to_dev(x) for key, x in xs.items()}
    ys = {(m, i): torch.empty((m, N), dtype=torch.float16, device="cuda") for i, (N, *_) in enumerate(weights)
          for m in set(MS)}
    assert glmq.last_device_error() == (B.OK, 0)

    def calls():
        for _ in range(REPEATS):
            for m in MS:
                for i, (N, K, packed, scale, *_rest) in enumerate(weights):
                    glmq.gemm_decode(xd[(m, i)], packed, scale, 4, out=ys[(m, i)])
            glmq.gemm_zp(xzd, pzd, szd, zzd, out=yz)

    calls()                                   # lazily allocated scratch, before capture
    torch.cuda.synchronize()
    assert glmq.last_device_error() == (B.OK, 0)
    stream = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        calls()
    for r in range(REPLAYS):
        graph.replay()
        torch.cuda.synchronize()
        assert glmq.last_device_error() == (B.OK, 0), f"replay {r}"
    del graph

    for i, (N, K, packed, scale, w_rows, rows) in enumerate(weights):
        p_ref, s_ref = oracle.quantize_linear(w_rows, 4)
        for m in set(MS):
            Y = to_host(ys[(m, i)])[:, rows]
            err = oracle.relative_max_error(Y, oracle.linear_forward(xs[(m, i)], p_ref, s_ref, 4))
            record_error(f"back_to_back/N{N}_K{K}/M{m}", err)
            assert err <= TOL, (N, K, m, err)
    pz_rows, sz_rows, zz_rows = oracle.quantize_linear_zp(wz_rows)
    assert np.array_equal(pz_rows, to_host(pzd)[zrows])
    err = oracle.relative_max_error(to_host(yz)[:, zrows], oracle.linear_forward_zp(xz, pz_rows, sz_rows, zz_rows))
    record_error(f"back_to_back/zero_point/N{Nz}_K{Kz}/M16", err)
    assert err <= TOL, err
