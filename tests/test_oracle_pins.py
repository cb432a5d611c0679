"""Pins for the CPU oracle, against things other than the oracle itself.

* hand-worked golden examples (tests/golden/, each value derived by hand);
* an exact-integer formulation of the rounding (fp16 values scaled by 2^24 are
  integers, so round-half-even of |w|/s is integer division plus a remainder test);
* the exact rational rounding of the scale, from the binary16 definition;
* pure-Python brute force with exact rationals on tiny layers;
* closed forms of the linear layer and invariants of the encoding.

Definitions pinned: GLM-130B paper card (wikillm.com), "Method" (INT4 pseudocode,
dequantizing linear) and "Paper vs code" (divisor 2^(b-1)-1, per-row FP16 scale).
"""
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from exact_fp16 import (Q24, fp16_to_fraction, fraction_to_fp16, positive_fp16_values,
                        round_half_even)
from golden_io import load_hand_example


# ---------------------------------------------------------------- golden examples

@pytest.mark.parametrize("name", ["hand_int4_4x8.txt", "hand_int8_4x8.txt"])
def test_hand_worked_example(name):
    g = load_hand_example(name)
    bits = g["bits"]
    W = g["W"].astype(np.float16)
    assert np.array_equal(W.astype(np.float64), g["W"]), "fixture W must be exact fp16"
    packed, s = oracle.quantize_linear(W, bits)
    assert np.array_equal(s.astype(np.float64), g["scale"])
    assert np.array_equal(oracle.unpack(packed, bits, W.shape[1]).astype(np.int64), g["q"])
    assert np.array_equal(packed, g["packed"])
    X = g["X"].astype(np.float16)
    Y = oracle.linear_forward(X, packed, s, bits)
    assert np.array_equal(Y.astype(np.float64), g["Y"])


# ---------------------------------------------------------------- the scale

@pytest.mark.parametrize("bits", [4, 8])
def test_scale_is_correctly_rounded_quotient_for_every_fp16(bits):
    """s = fp16(fp32(a)/d) equals the exactly rounded fp16(a/d) for every positive fp16 a."""
    d = (1 << (bits - 1)) - 1
    a = positive_fp16_values()
    s = oracle.row_scale(a, bits)
    expect = np.array([fraction_to_fp16(fp16_to_fraction(v) / d) for v in a], dtype=np.float16)
    assert np.array_equal(s.view(np.uint16), expect.view(np.uint16))


def test_scale_zero_only_for_tiny_rows():
    """s = 0 exactly when a/d rounds to 0 in fp16 (a <= 3*2^-24 for INT4)."""
    a = positive_fp16_values()
    s4 = oracle.row_scale(a, 4)
    zero = a[s4 == 0].astype(np.float64)
    assert np.array_equal(zero * Q24, np.array([1.0, 2.0, 3.0]))


# ---------------------------------------------------------------- the rounding of w/s

def exact_codes(w16: np.ndarray, s16: np.ndarray, d: int) -> np.ndarray:
    """RNE(w/s) clamped to [-d, d] by exact int64 arithmetic on 2^24-scaled values.

    Independent of the oracle: no floating-point division and no np.rint.
    """
    W = np.round(np.abs(w16.astype(np.float64)) * Q24).astype(np.int64)
    S = np.round(s16.astype(np.float64) * Q24).astype(np.int64)
    out = np.zeros(np.broadcast(W, S).shape, dtype=np.int64)
    live = np.broadcast_to(S, out.shape) > 0
    Wb = np.broadcast_to(W, out.shape)[live]
    Sb = np.broadcast_to(S, out.shape)[live]
    k = Wb // Sb
    r2 = 2 * (Wb - k * Sb)
    k = np.where(r2 > Sb, k + 1, np.where((r2 == Sb) & (k % 2 == 1), k + 1, k))
    k = np.minimum(k, d)
    out[live] = k
    sign = np.where(np.broadcast_to(w16, out.shape).astype(np.float64) < 0, -1, 1)
    return out * sign


def _check_rounding_for_absmax(a_vals: np.ndarray, bits: int):
    """For each absmax a: every fp16 w with |w| <= a, both signs, against exact_codes."""
    d = (1 << (bits - 1)) - 1
    pos = np.concatenate([[np.float16(0)], positive_fp16_values()])
    for start in range(0, len(a_vals), 64):
        a = a_vals[start:start + 64]
        lim = np.max(a)
        w = pos[pos <= lim]
        w = np.concatenate([w, -w[1:]])
        s = oracle.row_scale(a, bits)
        q = oracle.quantize_rows(np.broadcast_to(w, (len(a), len(w))).copy(), s, bits)
        ref = exact_codes(w[None, :], s[:, None], d)
        valid = np.abs(w[None, :].astype(np.float64)) <= a[:, None].astype(np.float64)
        bad = valid & (q.astype(np.int64) != ref)
        assert not bad.any(), (a[np.nonzero(bad)[0][0]], w[np.nonzero(bad)[1][0]])


@pytest.mark.parametrize("bits", [4, 8])
def test_rounding_exact_structured_subset(bits):
    """Strided absmax values across the whole fp16 range plus every subnormal and power of two."""
    pos = positive_fp16_values()
    pow2 = pos[(pos.view(np.uint16) & 0x3FF) == 0]
    picks = np.unique(np.concatenate([pos[:1100], pos[::211], pow2, pos[-3:]]))
    _check_rounding_for_absmax(picks, bits)


@pytest.mark.slow
@pytest.mark.parametrize("bits", [4, 8])
def test_rounding_exact_exhaustive(bits):
    """Every (w, a) fp16 pair with |w| <= a (about 10^9 pairs; GLMQ_SLOW=1)."""
    _check_rounding_for_absmax(positive_fp16_values(), bits)


# ---------------------------------------------------------------- brute force, tiny

def brute_force_quantize(Wf, bits):
    """Pure-Python exact quantize + pack of a small matrix of exact fp16 values."""
    d = (1 << (bits - 1)) - 1
    rows = []
    scales = []
    for row in Wf:
        a = max(abs(v) for v in row)
        s = fp16_to_fraction(fraction_to_fp16(a / d))
        codes = []
        for v in row:
            if s == 0:
                codes.append(0)
                continue
            k = round_half_even(v / s)
            codes.append(max(-d, min(d, k)))
        if bits == 4:
            b = [((codes[2 * j] & 0xF) | ((codes[2 * j + 1] & 0xF) << 4)) for j in range(len(codes) // 2)]
        else:
            b = [c & 0xFF for c in codes]
        rows.append(b)
        scales.append(s)
    return np.array(rows, dtype=np.uint8), scales


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("seed", [3, 4])
def test_brute_force_tiny_layer(bits, seed):
    rng = np.random.default_rng(seed)
    N, K, M = 6, 16, 3
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
    W[1, :] = 0
    W[2, 5] = np.float16(0.5)           # a strong outlier
    W[3, :] = np.float16(2.0 ** -24) * np.arange(K, dtype=np.float16)  # subnormal row
    Wf = [[fp16_to_fraction(v) for v in r] for r in W]
    bf_packed, bf_scales = brute_force_quantize(Wf, bits)
    packed, s = oracle.quantize_linear(W, bits)
    assert np.array_equal(packed, bf_packed)
    assert [fp16_to_fraction(v) for v in s] == bf_scales
    # Activations on a 2^-6 grid keep every float64 partial sum exact.
    X = (rng.integers(-256, 257, size=(M, K)) / 64.0).astype(np.float16)
    Y = oracle.linear_forward(X, packed, s, bits)
    q = oracle.unpack(packed, bits, K)
    for m in range(M):
        for n in range(N):
            exact = sum(fp16_to_fraction(X[m, k]) * bf_scales[n] * int(q[n, k]) for k in range(K))
            assert Y[m, n].view(np.uint16) == fraction_to_fp16(exact).view(np.uint16) or \
                (exact == 0 and float(Y[m, n]) == 0.0)


# ---------------------------------------------------------------- closed forms of the linear

@pytest.mark.parametrize("bits", [4, 8])
def test_linear_unit_vectors_and_row_sums(bits):
    rng = np.random.default_rng(11)
    N, K = 40, 64
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
    packed, s = oracle.quantize_linear(W, bits)
    q = oracle.unpack(packed, bits, K).astype(np.int64)
    sf = [fp16_to_fraction(v) for v in s]
    ks = [0, 1, 31, 63]
    X = np.zeros((len(ks) + 1, K), dtype=np.float16)
    for i, k in enumerate(ks):
        X[i, k] = 1
    X[-1, :] = 1
    Y = oracle.linear_forward(X, packed, s, bits)
    for i, k in enumerate(ks):
        expect = np.array([fraction_to_fp16(sf[n] * int(q[n, k])) for n in range(N)], dtype=np.float16)
        assert np.array_equal(Y[i].astype(np.float64), expect.astype(np.float64))
    rowsum = np.array([fraction_to_fp16(sf[n] * int(q[n].sum())) for n in range(N)], dtype=np.float16)
    assert np.array_equal(Y[-1].astype(np.float64), rowsum.astype(np.float64))


def test_linear_is_linear_in_x():
    """Y(2^j X) = 2^j Y(X) when nothing under/overflows (power-of-two scaling of activations)."""
    rng = np.random.default_rng(12)
    W = (rng.standard_normal((32, 128)) * 0.02).astype(np.float16)
    X = rng.standard_normal((3, 128)).astype(np.float16)
    packed, s = oracle.quantize_linear(W, 4)
    Y1 = oracle.linear_forward(X, packed, s, 4).astype(np.float64)
    Y4 = oracle.linear_forward((X.astype(np.float32) * 4).astype(np.float16), packed, s, 4).astype(np.float64)
    assert np.array_equal(Y4, 4 * Y1)


# ---------------------------------------------------------------- invariants of the encoding

@pytest.mark.parametrize("bits", [4, 8])
def test_invariants(bits):
    d = (1 << (bits - 1)) - 1
    rng = np.random.default_rng(5)
    N, K = 64, 256
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
    W[0] = 0
    W[1, 17] = -np.max(np.abs(W[1])) * np.float16(3)   # negative absmax element
    packed, s = oracle.quantize_linear(W, bits)
    q = oracle.unpack(packed, bits, K).astype(np.int64)
    # all-zero row -> scale 0 and codes 0
    assert s[0] == 0 and not q[0].any()
    # codes stay in [-d, d]
    assert q.min() >= -d and q.max() <= d
    # +-absmax maps to +-d on rows with a normal scale
    a = oracle.row_absmax(W)
    for n in range(1, N):
        at = np.nonzero(np.abs(W[n]) == a[n])[0]
        assert np.all(q[n, at] == np.sign(W[n, at].astype(np.float64)) * d)
    # |w - s q| <= s/2 element-wise (no clamp fires on these rows)
    err = np.abs(W.astype(np.float64) - s.astype(np.float64)[:, None] * q)
    assert np.all(err <= s.astype(np.float64)[:, None] / 2)
    # sign symmetry
    pn, sn = oracle.quantize_linear(-W, bits)
    assert np.array_equal(sn, s)
    assert np.array_equal(oracle.unpack(pn, bits, K).astype(np.int64), -q)
    # power-of-two scaling of W leaves the codes unchanged and scales s exactly
    p2, s2 = oracle.quantize_linear((W.astype(np.float32) * 8).astype(np.float16), bits)
    assert np.array_equal(p2, packed)
    assert np.array_equal(s2.astype(np.float64), 8 * s.astype(np.float64))
    if bits == 4:
        nib = np.concatenate([packed & 0xF, packed >> 4], axis=1)
        assert not np.any(nib == 0x8)


def test_pack_unpack_roundtrip():
    rng = np.random.default_rng(6)
    q = rng.integers(-7, 8, size=(9, 64)).astype(np.int8)
    assert np.array_equal(oracle.unpack(oracle.pack_int4(q), 4, 64), q)
    q8 = rng.integers(-127, 128, size=(9, 64)).astype(np.int8)
    assert np.array_equal(oracle.unpack(oracle.pack(q8, 8), 8, 64), q8)
    # nibble order: low nibble = even k
    one = np.zeros((1, 2), dtype=np.int8)
    one[0, 0], one[0, 1] = 1, -1
    assert oracle.pack_int4(one)[0, 0] == 0xF1


def test_relative_error_measure():
    R = np.array([[1.0, -4.0]])
    assert oracle.relative_max_error(R + np.array([[0.01, 0.0]]), R) == pytest.approx(0.0025)


def test_tiny_config_accuracy_of_int4_against_fp16():
    """W4A16 on the Tiny workload stays close to the unquantized fp64 product (sanity of scale)."""
    from inputs import tiny_weight, tiny_activations
    W = tiny_weight()
    X = tiny_activations()
    packed, s = oracle.quantize_linear(W, 4)
    Y = oracle.linear_forward(X, packed, s, 4).astype(np.float64)
    ref = X.astype(np.float64) @ W.astype(np.float64).T
    # absmax INT4 with 10x outliers loses precision; the error is bounded by sum |x| * s / 2
    bound = (np.abs(X.astype(np.float64)) @ (s.astype(np.float64)[:, None] / 2 * np.ones((1, 512))).T)
    assert np.all(np.abs(Y - ref) <= bound + np.abs(ref) * 2 ** -10 + 1e-3)
