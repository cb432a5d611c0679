"""Plain CPU oracle for GLM-130B weight-only INT4/INT8 quantization and the
dequantizing linear layer (W4A16 / W8A16).

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import or run this module. The product path
(the CUDA library and its Python binding) never calls it, and this module
imports nothing from the product package: the two share no code.

Everything here is written for obviousness, not speed: numpy only, one
definition per step, in the order and notation of the pages.

Source passages (GLM-130B: An Open Bilingual Pre-trained Model):
  * wikillm.com paper card, "Method": weight-only INT4 quantization with one
    absmax scale per output row, ``scale = max(abs(weight), dim=1) / 7``,
    ``quant = round(weight / scale[:, None])`` in [-7, 7], two INT4 values packed
    per byte; ``linear_forward``: ``weight = quant * scale[:, None]``,
    ``inputs @ weight.T`` with FP16 activations.
  * same card, "Paper vs code", quantization-scale bullet: the divisor is
    2^(b-1) - 1 (7 for INT4, 127 for INT8), per output row, the scale computed
    in FP16; rounding and int8 packing follow.
  * same card, "Results": INT8 weights as a second precision.
  * paperlayer.ai summary, "INT4 Quantization for RTX 3090s/2080s": weights are
    converted to FP16 at run time, activations stay FP16.

Readings where the pages are silent or loose (each also listed in the design
notes):
  R1 divisor d = 2^(b-1) - 1; codes lie in [-d, d]; -8 / -128 never occur.
  R2 scale s = fp16_rn( fp32(a) / fp32(d) ), a = row absmax (exact in fp16).
  R3 code q = clamp( rint( fp32(w) / fp32(s) ), -d, d ), IEEE fp32 quotient,
     round half to even; a row whose scale is 0 gets q = 0 everywhere.
  R4 INT4 packing: byte j of a row = (q[2j] & 0xF) | ((q[2j+1] & 0xF) << 4)
     (low nibble = even k, 4-bit two's complement). INT8: the int8 code as is.
  R5 linear: Y[m,n] = fp16_rn( sum_k X[m,k] * s[n] * q[n,k] ), products and sum
     in float64 (each s*q is exact in float64).
  R6 inputs are finite; non-finite weights or activations are out of contract.
"""
from __future__ import annotations

import numpy as np

# ---------------------------------------------------------------------------
# R1: the divisor
# ---------------------------------------------------------------------------


def divisor(bits: int) -> int:
    """d = 2^(bits-1) - 1 ("Paper vs code", quantization-scale bullet)."""
    if bits not in (4, 8):
        raise ValueError("bits must be 4 or 8")
    return (1 << (bits - 1)) - 1


# ---------------------------------------------------------------------------
# a1: row absmax (paper card, "Method": max(abs(weight), dim=1))
# ---------------------------------------------------------------------------


def row_absmax(W: np.ndarray) -> np.ndarray:
    """a[n] = max_k |W[n,k]| over fp16 values (exact: a max of fp16 magnitudes)."""
    W = np.asarray(W)
    assert W.dtype == np.float16 and W.ndim == 2
    return np.max(np.abs(W), axis=1)


# ---------------------------------------------------------------------------
# a2: the per-row scale ("Paper vs code": absmax / (2^(b-1)-1), in FP16)
# ---------------------------------------------------------------------------


def row_scale(a: np.ndarray, bits: int) -> np.ndarray:
    """s[n] = fp16_rn( fp32(a[n]) / fp32(d) )   (reading R2)."""
    d = np.float32(divisor(bits))
    return (np.asarray(a, dtype=np.float16).astype(np.float32) / d).astype(np.float16)


# ---------------------------------------------------------------------------
# a3: quantize (paper card, "Method": round(weight / scale[:, None]) in [-7, 7])
# ---------------------------------------------------------------------------


def quantize_rows(W: np.ndarray, s: np.ndarray, bits: int) -> np.ndarray:
    """q[n,k] = clamp(rint(fp32(W[n,k]) / fp32(s[n])), -d, d); q = 0 where s[n] == 0.

    ``np.rint`` rounds half to even; the fp32 division is IEEE round-to-nearest.
    """
    d = divisor(bits)
    W32 = np.asarray(W, dtype=np.float16).astype(np.float32)
    s32 = np.asarray(s, dtype=np.float16).astype(np.float32)
    q = np.zeros(W32.shape, dtype=np.int16)
    live = s32 != 0
    if np.any(live):
        quotient = W32[live] / s32[live][:, None]          # IEEE fp32 division
        q[live] = np.clip(np.rint(quotient), -d, d).astype(np.int16)
    return q.astype(np.int8)


# ---------------------------------------------------------------------------
# a4: packing ("Method": two INT4 values per byte; order is reading R4)
# ---------------------------------------------------------------------------


def pack_int4(q: np.ndarray) -> np.ndarray:
    """uint8 [N, K/2]: low nibble = q[:, 2j], high nibble = q[:, 2j+1]."""
    q = np.asarray(q, dtype=np.int8)
    assert q.ndim == 2 and q.shape[1] % 2 == 0
    nib = q.astype(np.int16) & 0xF                       # 4-bit two's complement
    lo = nib[:, 0::2]
    hi = nib[:, 1::2]
    return (lo | (hi << 4)).astype(np.uint8)


def pack(q: np.ndarray, bits: int) -> np.ndarray:
    """Packed weight bytes for ``bits``: [N, K/2] for INT4, [N, K] int8 bytes for INT8."""
    if bits == 4:
        return pack_int4(q)
    divisor(bits)
    return np.ascontiguousarray(np.asarray(q, dtype=np.int8)).view(np.uint8)


def quantize_linear(W: np.ndarray, bits: int):
    """One-shot weight quantization of a linear layer: returns (packed uint8, scale fp16)."""
    a = row_absmax(W)
    s = row_scale(a, bits)
    q = quantize_rows(W, s, bits)
    return pack(q, bits), s


# ---------------------------------------------------------------------------
# a5: unpack (inverse of R4; written independently of ``pack_int4``)
# ---------------------------------------------------------------------------


def unpack(packed: np.ndarray, bits: int, K: int) -> np.ndarray:
    """Codes int8 [N, K] from packed bytes (sign-extends each nibble for INT4)."""
    packed = np.asarray(packed, dtype=np.uint8)
    if bits == 8:
        return packed.view(np.int8).reshape(packed.shape[0], K)
    N = packed.shape[0]
    assert packed.shape[1] * 2 == K
    out = np.empty((N, K), dtype=np.int8)
    low = (packed & 0x0F).astype(np.int8)
    high = (packed >> 4).astype(np.int8)
    out[:, 0::2] = np.where(low >= 8, low - 16, low)
    out[:, 1::2] = np.where(high >= 8, high - 16, high)
    return out


# ---------------------------------------------------------------------------
# a6/a7: the dequantizing linear (paper card, "Method": linear_forward)
# ---------------------------------------------------------------------------


def dequantize(packed: np.ndarray, s: np.ndarray, bits: int, K: int) -> np.ndarray:
    """float64 weight = quant * scale[:, None] (exact in float64)."""
    q = unpack(packed, bits, K).astype(np.float64)
    return q * np.asarray(s, dtype=np.float16).astype(np.float64)[:, None]


def linear_forward(X: np.ndarray, packed: np.ndarray, s: np.ndarray, bits: int,
                   row_block: int = 4096) -> np.ndarray:
    """Y[m,n] = fp16_rn( sum_k float64(X[m,k]) * float64(s[n] * q[n,k]) )   (reading R5).

    Rows of W are processed in blocks only to bound host memory; each output
    element is one float64 dot product rounded once to fp16.
    """
    X = np.asarray(X)
    assert X.dtype == np.float16 and X.ndim == 2
    M, K = X.shape
    N = packed.shape[0]
    X64 = X.astype(np.float64)
    Y = np.empty((M, N), dtype=np.float16)
    for n0 in range(0, N, row_block):
        n1 = min(N, n0 + row_block)
        Wd = dequantize(packed[n0:n1], s[n0:n1], bits, K)
        Y[:, n0:n1] = (X64 @ Wd.T).astype(np.float16)
    return Y


def linear_forward_rows(X: np.ndarray, packed_rows: np.ndarray, s_rows: np.ndarray,
                        bits: int) -> np.ndarray:
    """The same definition for a sample of output features (selected rows of W)."""
    return linear_forward(X, packed_rows, s_rows, bits)


def relative_max_error(Y: np.ndarray, Y_ref: np.ndarray) -> float:
    """max|Y - Y_ref| / max|Y_ref| in float64 (the accuracy bar's measure)."""
    Y = np.asarray(Y, dtype=np.float64)
    R = np.asarray(Y_ref, dtype=np.float64)
    denom = float(np.max(np.abs(R))) if R.size else 0.0
    err = float(np.max(np.abs(Y - R))) if R.size else 0.0
    if denom == 0.0:
        return 0.0 if err == 0.0 else float("inf")
    return err / denom
