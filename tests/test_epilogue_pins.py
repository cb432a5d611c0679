"""Pins for the epilogue oracle (oracle/glmq_epilogue.py), against things other than
itself: the normal CDF of an independent library, exact identities of GELU, brute
force in pure-Python loops, and closed forms of the bias add."""
import math

import numpy as np
import pytest

import oracle
from inputs import gaussian_fp16


def test_gelu_matches_normal_cdf_of_scipy():
    scipy_special = pytest.importorskip("scipy.special")
    x = np.linspace(-12.0, 12.0, 4001)
    ref = x * scipy_special.ndtr(x)                 # x * Phi(x), independent implementation
    assert np.max(np.abs(oracle.gelu(x) - ref)) <= 1e-14 * np.max(np.abs(ref)) + 1e-300


def test_gelu_identities_and_values():
    x = np.linspace(-6.0, 6.0, 1201)
    # Phi(x) + Phi(-x) = 1  =>  gelu(x) - gelu(-x) = x  (exact up to rounding)
    assert np.max(np.abs(oracle.gelu(x) - oracle.gelu(-x) - x)) < 1e-15 * 8
    assert oracle.gelu(np.array([0.0]))[0] == 0.0
    # Phi(1) = 0.841344746068542948585...
    assert abs(oracle.gelu(np.array([1.0]))[0] - 0.8413447460685429) < 1e-15
    assert abs(oracle.gelu(np.array([-1.0]))[0] - (-0.15865525393145705)) < 1e-15
    g = oracle.gelu(np.array([40.0, -40.0]))
    assert g[0] == 40.0 and abs(g[1]) < 1e-300          # Phi(40) rounds to 1 and Phi(-40) to ~0


def test_geglu_row_order_small_example_and_permutation():
    order = oracle.geglu_row_order(32)
    assert order.tolist() == [0, 1, 2, 3, 4, 5, 6, 7, 16, 17, 18, 19, 20, 21, 22, 23,
                              8, 9, 10, 11, 12, 13, 14, 15, 24, 25, 26, 27, 28, 29, 30, 31]
    for N in (16, 48, 65536):
        o = oracle.geglu_row_order(N)
        assert np.array_equal(np.sort(o), np.arange(N))
        p = np.arange(N)
        pair_a, pair_b = o[p % 16 < 8], o[p % 16 >= 8]
        assert np.array_equal(pair_b - pair_a, np.full(N // 2, N // 2))   # a row j pairs with F + j
    with pytest.raises(ValueError):
        oracle.geglu_row_order(24)


@pytest.mark.parametrize("bits", [4, 8])
def test_bias_closed_forms(bits):
    W = gaussian_fp16((40, 128), 0.02, 21)
    packed, s = oracle.quantize_linear(W, bits)
    b = gaussian_fp16((1, 40), 0.5, 22)[0]
    Xz = np.zeros((3, 128), dtype=np.float16)
    assert np.array_equal(oracle.linear_bias_forward(Xz, packed, s, bits, b), np.tile(b, (3, 1)))
    X = gaussian_fp16((3, 128), 1.0, 23)
    Y0 = oracle.linear_bias_forward(X, packed, s, bits, np.zeros(40, dtype=np.float16))
    assert np.array_equal(Y0, oracle.linear_forward(X, packed, s, bits))
    # unit vector: U[:, n] = s[n] q[n, k] + b[n], exact in float64
    q = oracle.unpack(packed, bits, 128).astype(np.float64)
    e = np.zeros((1, 128), dtype=np.float16)
    e[0, 5] = 1.0
    U = oracle.linear_pre(e, packed, s, bits, b)
    assert np.array_equal(U[0], s.astype(np.float64) * q[:, 5] + b.astype(np.float64))


@pytest.mark.parametrize("bits", [4, 8])
def test_geglu_brute_force(bits):
    N, K, M = 16, 64, 2
    W = gaussian_fp16((N, K), 0.05, 31)
    b = gaussian_fp16((1, N), 0.3, 32)[0]
    X = gaussian_fp16((M, K), 1.0, 33)
    packed, s = oracle.quantize_linear(W, bits)
    q = oracle.unpack(packed, bits, K)
    Y = oracle.geglu_forward(X, packed, s, bits, b)
    F = N // 2
    for m in range(M):
        for j in range(F):
            ua = sum(float(X[m, k]) * float(s[j]) * int(q[j, k]) for k in range(K)) + float(b[j])
            ub = sum(float(X[m, k]) * float(s[F + j]) * int(q[F + j, k]) for k in range(K)) + float(b[F + j])
            y = 0.5 * ua * (1.0 + math.erf(ua / math.sqrt(2.0))) * ub
            assert Y[m, j] == np.float16(y), (m, j, Y[m, j], y)


def test_geglu_layout_quantizes_the_same_rows():
    W = gaussian_fp16((48, 64), 0.02, 41)
    p_nat, s_nat = oracle.quantize_linear(W, 4)
    p_g, s_g = oracle.quantize_linear_geglu(W, 4)
    order = oracle.geglu_row_order(48)
    assert np.array_equal(p_g, p_nat[order]) and np.array_equal(s_g.view(np.uint16), s_nat[order].view(np.uint16))
