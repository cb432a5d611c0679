"""Plain CPU oracle for the fused epilogues of the GLM-130B projections: the fp16 bias
add, and the GeGLU of the feed-forward block.

TEST INFRASTRUCTURE, like :mod:`oracle.glmq_oracle`. Only ``tests/``,
``__graft_entry__.smoke()`` and the CPU legs of ``bench.py`` may import it. It shares no
code with the CUDA library, and numpy plus the standard library are its only tools.

Source passages (GLM-130B: An Open Bilingual Pre-trained Model):
  * wikillm.com paper card, "Method": the feed-forward block is a GeGLU. The FFN width
    is 32768 = 8/3 x 12288, so the FFN-up projection carries 2 x 32768 output rows
    (the two GLU branches) and FFN-down reads 32768 inputs.
  * same card, "Paper vs code": the quantized layers are QKV, attention output and
    both MLP projections; embeddings, norms and biases stay FP16.
  * paperlayer.ai summary, section B.3: GeGLU feed-forward network (GELU, Hendrycks
    and Gimpel, in the citation list).

Readings (the pages do not fix these; each is also listed in the design notes):
  E1 bias: Y[m,n] = fp16_rn( sum_k X[m,k] s[n] q[n,k] + b[n] ), b fp16 [N] in the
     natural row order of W, added before the single rounding.
  E2 GeGLU: the FFN-up output U (the E1 value before rounding, N = 2F rows) splits into
     halves a = U[:, :F] and b = U[:, F:]; Y[m,j] = fp16_rn( GELU(a[m,j]) * b[m,j] ),
     the GEGLU(x, W, V) = GELU(xW) * xV form with the GELU on the first half.
  E3 GELU is the exact form x * Phi(x) = 0.5 x (1 + erf(x / sqrt 2)).
  E4 layout for the fused kernel: glmq_quantize_geglu stores the packed rows in
     blocks of 16: packed row 16g + r holds natural row 8g + r (r < 8) or F + 8g + r - 8
     (r >= 8), so each GeGLU pair sits 8 rows apart in one 16-row block. The scale
     follows the same order; the bias stays in natural order.
"""
from __future__ import annotations

import math

import numpy as np

from .glmq_oracle import dequantize, quantize_linear


def linear_pre(X: np.ndarray, packed: np.ndarray, s: np.ndarray, bits: int, bias=None) -> np.ndarray:
    """float64 U[m,n] = sum_k X[m,k] * s[n] q[n,k] (+ b[n]): reading E1 before rounding."""
    X = np.asarray(X)
    assert X.dtype == np.float16 and X.ndim == 2
    K = X.shape[1]
    U = X.astype(np.float64) @ dequantize(packed, s, bits, K).T
    if bias is not None:
        U = U + np.asarray(bias, dtype=np.float16).astype(np.float64)[None, :]
    return U


def linear_bias_forward(X, packed, s, bits, bias) -> np.ndarray:
    """Y = fp16_rn(U) with the bias of reading E1."""
    return linear_pre(X, packed, s, bits, bias).astype(np.float16)


def gelu(x: np.ndarray) -> np.ndarray:
    """Exact GELU (reading E3) in float64, erf from the standard library."""
    x = np.asarray(x, dtype=np.float64)
    erf = np.vectorize(math.erf, otypes=[np.float64])
    return 0.5 * x * (1.0 + erf(x / math.sqrt(2.0)))


def geglu_forward(X, packed, s, bits, bias=None) -> np.ndarray:
    """Y[m,j] = fp16_rn( GELU(U[m,j]) * U[m,F+j] ), j < F = N/2 (reading E2).

    ``packed``, ``s`` and ``bias`` are in the natural row order of W."""
    U = linear_pre(X, packed, s, bits, bias)
    F = U.shape[1] // 2
    assert U.shape[1] == 2 * F
    return (gelu(U[:, :F]) * U[:, F:]).astype(np.float16)


def geglu_row_order(N: int) -> np.ndarray:
    """Natural row index held by each packed row in the GeGLU layout (reading E4)."""
    if N % 16 != 0:
        raise ValueError("the GeGLU layout needs N % 16 == 0")
    F = N // 2
    p = np.arange(N)
    g, r = p // 16, p % 16
    return np.where(r < 8, 8 * g + r, F + 8 * g + (r - 8))


def quantize_linear_geglu(W: np.ndarray, bits: int):
    """(packed, scale) of W with its rows stored in the GeGLU layout (reading E4)."""
    order = geglu_row_order(np.asarray(W).shape[0])
    return quantize_linear(np.asarray(W)[order], bits)
