"""GPU parity against the CPU oracle, through the C ABI (via the ctypes binding).

Packed codes and scales must be bit-exact. Y must satisfy
max|Y - Y_ref| / max|Y_ref| <= 5e-3 (the accuracy bar for the linear layer);
the kernels actually land far inside it, so a tighter check (2e-3) is applied too.
"""
import numpy as np
import pytest

import oracle
from gpu_helpers import edge_case_weight, to_dev, to_host, torch_cuda
from inputs import gaussian_fp16, tiny_activations, tiny_weight

pytestmark = pytest.mark.gpu

TOL = 5e-3
TIGHT = 2e-3


def glmq():
    torch_cuda()
    import int8_quantized_glmq_b200 as g
    return g


def gpu_quantize(W, bits):
    g = glmq()
    packed, scale = g.quantize(to_dev(W), bits)
    return to_host(packed), to_host(scale)


def check_quantize(W, bits):
    p_ref, s_ref = oracle.quantize_linear(W, bits)
    p, s = gpu_quantize(W, bits)
    assert np.array_equal(s.view(np.uint16), s_ref.view(np.uint16)), "scales differ"
    if not np.array_equal(p, p_ref):
        bad = np.argwhere(p != p_ref)
        r, c = bad[0]
        raise AssertionError(f"{len(bad)} packed bytes differ, first at row {r} byte {c}: "
                             f"gpu {p[r, c]:#04x} oracle {p_ref[r, c]:#04x}")
    return p_ref, s_ref


def check_gemm(X, packed, scale, bits, route):
    g = glmq()
    Y = to_host(g.gemm(to_dev(X), to_dev(packed), to_dev(scale), bits, route=route))
    Y_ref = oracle.linear_forward(X, packed, scale, bits)
    err = oracle.relative_max_error(Y, Y_ref)
    assert err <= TOL, err
    assert err <= TIGHT, err
    return err


# ---------------------------------------------------------------- quantize

@pytest.mark.parametrize("bits", [4, 8])
def test_quantize_tiny_config(bits):
    check_quantize(tiny_weight(), bits)


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("K", [64, 192, 2048, 2112, 12288])
def test_quantize_edge_rows_ragged(bits, K):
    check_quantize(edge_case_weight(37, K), bits)


@pytest.mark.parametrize("bits", [4, 8])
def test_quantize_max_k(bits):
    W = gaussian_fp16((5, 65536), 0.02, 31)
    W[1, 777] = 3.0
    check_quantize(W, bits)


@pytest.mark.parametrize("bits", [4, 8])
def test_quantize_single_row_and_deterministic(bits):
    W = gaussian_fp16((1, 512), 0.02, 3)
    p1, s1 = gpu_quantize(W, bits)
    p2, s2 = gpu_quantize(W, bits)
    assert np.array_equal(p1, p2) and np.array_equal(s1.view(np.uint16), s2.view(np.uint16))
    check_quantize(W, bits)


# ---------------------------------------------------------------- decode kernel (M <= 16)

@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("M", list(range(1, 17)))
def test_decode_tiny_config_all_m(bits, M):
    W = tiny_weight()
    packed, scale = check_quantize(W, bits)
    X = gaussian_fp16((M, W.shape[1]), 1.0, 100 + M)
    check_gemm(X, packed, scale, bits, "decode")


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("M,N,K", [(1, 1, 64), (3, 33, 128), (5, 95, 4160), (8, 64, 12288),
                                   (16, 70, 2112), (16, 40, 32768), (4, 300, 8256), (9, 31, 65536)])
def test_decode_ragged_shapes(bits, M, N, K):
    W = gaussian_fp16((N, K), 0.02, N + K)
    packed, scale = oracle.quantize_linear(W, bits)
    X = gaussian_fp16((M, K), 1.0, M + 1)
    check_gemm(X, packed, scale, bits, "decode")


FP16_OVERFLOW = 65520.0   # |y| >= 65520 rounds to +-inf in fp16 (round to nearest even)


def check_edge_rows(Y, X, packed, scale, bits):
    """Per output column: +-inf exactly where the exact result overflows fp16 (both sides
    round to nearest), elsewhere within the tolerance of that column's finite magnitude."""
    K = X.shape[1]
    Y64 = X.astype(np.float64) @ oracle.dequantize(packed, scale, bits, K).T
    Y = Y.astype(np.float64)
    near = np.abs(np.abs(Y64) - FP16_OVERFLOW) < 0.005 * FP16_OVERFLOW
    over = (np.abs(Y64) >= FP16_OVERFLOW) & ~near
    assert np.array_equal(Y[over], np.sign(Y64[over]) * np.inf)
    fin = ~over & ~near
    assert np.all(np.isfinite(Y[fin & (np.abs(Y64) < FP16_OVERFLOW * 0.99)]))
    for n in range(Y.shape[1]):
        col = fin[:, n] & np.isfinite(Y[:, n])
        if not col.any():
            continue
        ref = Y64[col, n]
        err = np.max(np.abs(Y[col, n] - ref))
        assert err <= TOL * max(np.max(np.abs(ref)), 1e-30) + 2 ** -24, n


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("route,M", [("decode", 7), ("decode", 16), ("prefill", 7), ("prefill", 200)])
def test_edge_rows_including_fp16_overflow(bits, route, M):
    W = edge_case_weight(45, 512)
    packed, scale = oracle.quantize_linear(W, bits)
    X = gaussian_fp16((M, 512), 1.0, 9)
    g = glmq()
    Y = to_host(g.gemm(to_dev(X), to_dev(packed), to_dev(scale), bits, route=route))
    check_edge_rows(Y, X, packed, scale, bits)


def test_decode_closed_form_unit_vectors():
    """X = e_k gives Y[:, n] = fp16(s[n] q[n, k]) exactly."""
    W = gaussian_fp16((128, 1024), 0.02, 5)
    packed, scale = oracle.quantize_linear(W, 4)
    ks = [0, 1, 7, 8, 63, 64, 255, 1023]
    X = np.zeros((len(ks), 1024), dtype=np.float16)
    for i, k in enumerate(ks):
        X[i, k] = 1
    g = glmq()
    Y = to_host(g.gemm(to_dev(X), to_dev(packed), to_dev(scale), 4, route="decode"))
    assert np.array_equal(Y, oracle.linear_forward(X, packed, scale, 4))


# ---------------------------------------------------------------- prefill kernel (tensor cores)

@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("M", [1, 4, 16, 17, 31, 32, 33, 63, 64, 65, 127, 128, 129, 255, 256, 257, 600])
def test_prefill_tiny_config_m_sweep(bits, M):
    W = tiny_weight()
    packed, scale = oracle.quantize_linear(W, bits)
    X = gaussian_fp16((M, W.shape[1]), 1.0, 200 + M)
    check_gemm(X, packed, scale, bits, "prefill")


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("M,N,K", [(64, 1, 64), (100, 129, 64), (300, 200, 1088), (2048, 130, 512),
                                   (48, 383, 12288), (512, 256, 32768)])
def test_prefill_ragged_shapes(bits, M, N, K):
    W = gaussian_fp16((N, K), 0.02, 3 * N + K)
    packed, scale = oracle.quantize_linear(W, bits)
    X = gaussian_fp16((M, K), 1.0, M + 2)
    check_gemm(X, packed, scale, bits, "prefill")


def test_prefill_closed_form_unit_vectors():
    W = gaussian_fp16((256, 1024), 0.02, 6)
    packed, scale = oracle.quantize_linear(W, 4)
    ks = list(range(0, 1024, 37))
    X = np.zeros((len(ks), 1024), dtype=np.float16)
    for i, k in enumerate(ks):
        X[i, k] = 1
    g = glmq()
    Y = to_host(g.gemm(to_dev(X), to_dev(packed), to_dev(scale), 4, route="prefill"))
    assert np.array_equal(Y, oracle.linear_forward(X, packed, scale, 4))


def test_auto_dispatch_matches_both_kernels():
    W = gaussian_fp16((96, 512), 0.02, 8)
    packed, scale = oracle.quantize_linear(W, 4)
    g = glmq()
    for M in (16, 17):
        X = gaussian_fp16((M, 512), 1.0, M)
        Y = to_host(g.gemm(to_dev(X), to_dev(packed), to_dev(scale), 4))
        assert oracle.relative_max_error(Y, oracle.linear_forward(X, packed, scale, 4)) <= TIGHT


@pytest.mark.parametrize("bits,M", [(4, 1), (4, 16), (8, 4)])
def test_chained_calls_read_the_previous_output(bits, M):
    """Three back-to-back calls on one stream, each call's X being the previous call's Y.

    The decode and finalize kernels may begin while the kernel before them is still
    running and must wait for it before reading its output. With N = K = 4096 these
    calls split tiles over K parts, so the chain alternates decode and finalize
    kernels. Reference: the oracle chain (Y rounded to fp16 between layers)."""
    import torch
    g = glmq()
    K = 4096
    layers = [oracle.quantize_linear(gaussian_fp16((K, K), 0.02, 500 + i), bits) for i in range(3)]
    dev = [(to_dev(p), to_dev(s)) for p, s in layers]
    X = gaussian_fp16((M, K), 1.0, 600 + M)
    x = to_dev(X)
    torch.cuda.synchronize()
    for p, s in dev:
        x = g.gemm(x, p, s, bits)                    # no host work between the launches
    Y = to_host(x)
    ref = X
    for p, s in layers:
        ref = oracle.linear_forward(ref, p, s, bits)
    assert np.all(np.isfinite(Y))
    assert oracle.relative_max_error(Y, ref) <= TOL


def test_kernel_launch_counter_counts_each_kernel():
    g = glmq()
    W = gaussian_fp16((512, 1024), 0.02, 3)
    n0 = g.kernel_launches()
    packed, scale = g.quantize(to_dev(W), 4)
    assert g.kernel_launches() == n0 + 1
    n1 = g.kernel_launches()
    g.gemm(to_dev(gaussian_fp16((1, 1024), 1.0, 4)), packed, scale, 4)
    assert g.kernel_launches() - n1 in (1, 2)          # the kernel, plus a finalize kernel when K is split


def test_no_device_error_reported():
    g = glmq()
    W = gaussian_fp16((64, 256), 0.02, 1)
    packed, scale = g.quantize(to_dev(W), 4)
    g.gemm(to_dev(gaussian_fp16((2, 256), 1.0, 2)), packed, scale, 4)
    g.gemm(to_dev(gaussian_fp16((40, 256), 1.0, 2)), packed, scale, 4)
    st, flags = g.last_device_error()
    assert st == 0 and flags == 0
