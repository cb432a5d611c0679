"""Parity of the 70-layer INT4 sweep (GLM-130B paper card, "Method": INT4 linear weights
of about 70 GB; "Hyperparameters": 70 layers), in the launch configuration the
benchmark times: every projection of every layer quantized once on the GPU and
resident in HBM, and one CUDA graph running the M=1 decode GEMM through all 280 of
them in layer order.

For layers 0, 35 and 69 the test regenerates each projection's fp16 weights on the
device with the sweep's own seeded generator, and then checks:
  * every row's packed codes and scale against the oracle, bit-exact (the whole layer,
    in row blocks);
  * the decode output the graph wrote for that layer (the graph keeps those layers'
    outputs in their own buffers) on sampled output features, within the 5e-3 bar.
A wrong layer, scale or pointer anywhere in the graph's order would show up at one of
these layers, or in the layer count the graph launches.
"""
import numpy as np
import pytest

import oracle
from gpu_helpers import record_error, to_host, torch_cuda
from inputs import GLM_PROJECTIONS, PROJECTION_ORDER

pytestmark = pytest.mark.gpu

TOL = 5e-3
CHECKED_LAYERS = (0, 35, 69)
ROW_BLOCK = 4096


def test_sweep_layers_match_the_oracle():
    torch = torch_cuda()
    import bench
    import int8_quantized_glmq_b200 as glmq
    free, _ = torch.cuda.mem_get_info()
    if free < 75e9:
        pytest.skip("the 70-layer sweep needs about 70 GB free on the device")
    sw = bench.Sweep(torch, glmq, bench.SWEEP_LAYERS, keep=CHECKED_LAYERS)
    assert sw.kernels_per_replay >= 4 * bench.SWEEP_LAYERS     # one decode launch per call (+ finalize)
    sw.graph.replay()
    torch.cuda.synchronize()
    rng = np.random.default_rng(70)
    for layer in CHECKED_LAYERS:
        for p, name in enumerate(PROJECTION_ORDER):
            N, K = GLM_PROJECTIONS[name]
            W = torch.empty((N, K), dtype=torch.float16, device="cuda")
            bench.sweep_weight(torch, layer, p, W)
            packed, scale = sw.quant[layer][p]
            for n0 in range(0, N, ROW_BLOCK):
                n1 = min(N, n0 + ROW_BLOCK)
                p_ref, s_ref = oracle.quantize_linear(to_host(W[n0:n1]), 4)
                assert np.array_equal(to_host(scale[n0:n1]).view(np.uint16), s_ref.view(np.uint16)), \
                    (layer, name, n0)
                assert np.array_equal(to_host(packed[n0:n1]), p_ref), (layer, name, n0)
            rows = np.unique(np.concatenate([np.arange(32), np.arange(N - 32, N), rng.choice(N, 192, replace=False)]))
            X = to_host(sw.xs[name])
            p_rows, s_rows = oracle.quantize_linear(to_host(W[torch.from_numpy(rows).cuda()]), 4)
            Y = to_host(sw.kept[(layer, name)])[:, rows]
            err = record_error(f"sweep/layer{layer}/{name}/M=1", oracle.relative_max_error(
                Y, oracle.linear_forward(X, p_rows, s_rows, 4)))
            assert err <= TOL, (layer, name, err)
            del W
    del sw
    torch.cuda.empty_cache()
