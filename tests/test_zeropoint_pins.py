"""Pins for the zero-point INT4 oracle (oracle/glmq_zeropoint.py): a hand-worked
example, the invariants the readings imply, and pure-Python brute force."""
import numpy as np
import pytest

import oracle
from inputs import gaussian_fp16

H = np.float16


def test_hand_worked_two_rows():
    W = np.array([[-1.5, 0, 0.5, 1.0, 3.0, -0.25, 2.0, 1.5],
                  [1, 2, 3, 4, 5, 6, 7, 7.5]], dtype=H)
    packed, s, z = oracle.quantize_linear_zp(W)
    # row 0: lo -1.5, hi 3 -> s = fp16(4.5/15) = fp16(0.3) = 0.300048828125, z = rint(1.5/s) = 5
    # row 1: lo 0 (range includes zero), hi 7.5 -> s = 0.5, z = 0
    assert s.tolist() == [0.300048828125, 0.5]
    assert z.tolist() == [5, 0]
    assert oracle.unpack_u4(packed, 8).tolist() == [[0, 5, 7, 8, 15, 4, 12, 10], [2, 4, 6, 8, 10, 12, 14, 15]]
    assert packed.tolist() == [[0x50, 0x87, 0x4F, 0xAC], [0x42, 0x86, 0xCA, 0xFE]]
    e4 = np.zeros((1, 8), dtype=H)
    e4[0, 4] = 1.0
    # s * (q - z): 0.300048828125 * 10 = 3.00048828125 rounds to fp16 3.0; 0.5 * 10 = 5
    assert oracle.linear_forward_zp(e4, packed, s, z).tolist() == [[3.0, 5.0]]


def test_invariants():
    W = gaussian_fp16((64, 256), 0.02, 51)
    W[3] = 0                                             # all-zero row
    W[4] = H(0.01)                                       # constant row
    packed, s, z = oracle.quantize_linear_zp(W)
    q = oracle.unpack_u4(packed, 256).astype(np.int32)
    assert s[3] == 0 and z[3] == 0 and np.all(q[3] == 0)
    assert z[4] == 0 and np.all(q[4] == 15)              # range [0, 0.01]: every entry is the top code
    live = np.arange(64) != 3
    W64 = W.astype(np.float64)
    deq = (q - z[:, None].astype(np.int32)) * s.astype(np.float64)[:, None]
    assert np.all(np.abs(deq[live] - W64[live]) <= s.astype(np.float64)[live, None] / 2 * (1 + 1e-3))
    zero_pos = W == 0
    assert np.all((q == z[:, None])[zero_pos & live[:, None]])          # zero is exact
    rows = [n for n in range(64) if n not in (3, 4)]
    argmin = np.argmin(W64, axis=1)
    assert all(q[n, argmin[n]] == 0 for n in rows)       # the row minimum takes code 0
    assert np.array_equal(oracle.unpack_u4(oracle.pack_u4(q.astype(np.uint8)), 256), q)


def test_brute_force_linear():
    W = gaussian_fp16((6, 32), 0.05, 52)
    X = gaussian_fp16((3, 32), 1.0, 53)
    packed, s, z = oracle.quantize_linear_zp(W)
    q = oracle.unpack_u4(packed, 32)
    Y = oracle.linear_forward_zp(X, packed, s, z)
    for m in range(3):
        for n in range(6):
            y = sum(float(X[m, k]) * float(s[n]) * (int(q[n, k]) - int(z[n])) for k in range(32))
            assert Y[m, n] == H(y)


def test_more_accurate_than_symmetric_on_skewed_rows():
    # a row whose values are all positive: the symmetric quantizer spends half its codes
    rng = np.random.default_rng(54)
    W = (rng.random((32, 512)) * 0.05).astype(H)
    p4, s4 = oracle.quantize_linear(W, 4)
    pz, sz, zz = oracle.quantize_linear_zp(W)
    err_sym = np.abs(oracle.dequantize(p4, s4, 4, 512) - W.astype(np.float64)).mean()
    err_zp = np.abs(oracle.dequantize_zp(pz, sz, zz, 512) - W.astype(np.float64)).mean()
    assert err_zp < 0.6 * err_sym
