"""Plain CPU oracle for the zero-point (asymmetric) INT4 variant of the weight-only
quantization and its dequantizing linear layer.

TEST INFRASTRUCTURE, like :mod:`oracle.glmq_oracle`. Only ``tests/``,
``__graft_entry__.smoke()`` and the CPU legs of ``bench.py`` may import it. It shares no
code with the CUDA library, and numpy is its only tool.

Source passage (GLM-130B: An Open Bilingual Pre-trained Model): wikillm.com paper card,
"Pitfalls". An asymmetric INT4 quantizer with a zero point scored better on LAMBADA
(80.63 against 79.47 for the symmetric absmax quantizer), but the symmetric one was
kept as cheaper. The card gives no formula.

Readings (each also listed in the design notes):
  Z1 range: lo = min(0, min_k W[n,k]), hi = max(0, max_k W[n,k]) (exact fp16 values;
     zero is inside the range, so an all-zero row gives s = 0 and a constant row is
     still representable).
  Z2 scale: s = fp16_rn( fp32(hi - lo) / 15 ), the difference and the quotient each
     rounded to nearest in IEEE fp32.
  Z3 zero point: z = clamp(rint(fp32(-lo) / fp32(s)), 0, 15), one uint8 per row;
     z = 0 where s == 0.
  Z4 codes: q = clamp(rint(fp32(w) / fp32(s)) + z, 0, 15), unsigned 4-bit, round half
     to even on the IEEE fp32 quotient; q = 0 where s == 0. Packed two per byte, low
     nibble = even k, as for the symmetric codes.
  Z5 linear: Y[m,n] = fp16_rn( sum_k X[m,k] * s[n] * (q[n,k] - z[n]) ), float64 sum.
"""
from __future__ import annotations

import numpy as np


def zp_range(W: np.ndarray):
    """(lo, hi) per row as float32: reading Z1."""
    W = np.asarray(W)
    assert W.dtype == np.float16 and W.ndim == 2
    W32 = W.astype(np.float32)
    lo = np.minimum(W32.min(axis=1), np.float32(0.0))
    hi = np.maximum(W32.max(axis=1), np.float32(0.0))
    return lo, hi


def zp_scale(lo: np.ndarray, hi: np.ndarray) -> np.ndarray:
    """s = fp16_rn( fl32(fl32(hi - lo) / 15) ): reading Z2."""
    return ((np.asarray(hi, np.float32) - np.asarray(lo, np.float32)) / np.float32(15.0)).astype(np.float16)


def zp_zero(lo: np.ndarray, s: np.ndarray) -> np.ndarray:
    """z = clamp(rint(fp32(-lo) / fp32(s)), 0, 15); 0 where s == 0: reading Z3."""
    s32 = np.asarray(s, np.float16).astype(np.float32)
    z = np.zeros(s32.shape, dtype=np.uint8)
    live = s32 != 0
    z[live] = np.clip(np.rint(-np.asarray(lo, np.float32)[live] / s32[live]), 0, 15).astype(np.uint8)
    return z


def zp_codes(W: np.ndarray, s: np.ndarray, z: np.ndarray) -> np.ndarray:
    """q = clamp(rint(fp32(w) / fp32(s)) + z, 0, 15); 0 where s == 0: reading Z4."""
    W32 = np.asarray(W, np.float16).astype(np.float32)
    s32 = np.asarray(s, np.float16).astype(np.float32)
    q = np.zeros(W32.shape, dtype=np.int16)
    live = s32 != 0
    if np.any(live):
        k = np.rint(W32[live] / s32[live][:, None])
        q[live] = np.clip(k + z[live][:, None].astype(np.float32), 0, 15).astype(np.int16)
    return q.astype(np.uint8)


def pack_u4(q: np.ndarray) -> np.ndarray:
    """uint8 [N, K/2]: low nibble = q[:, 2j], high nibble = q[:, 2j+1] (unsigned codes)."""
    q = np.asarray(q, dtype=np.uint8)
    assert q.ndim == 2 and q.shape[1] % 2 == 0 and np.all(q < 16)
    return (q[:, 0::2] | (q[:, 1::2] << 4)).astype(np.uint8)


def unpack_u4(packed: np.ndarray, K: int) -> np.ndarray:
    """Unsigned codes uint8 [N, K] from packed bytes (written independently of pack_u4)."""
    packed = np.asarray(packed, dtype=np.uint8)
    assert packed.shape[1] * 2 == K
    out = np.empty((packed.shape[0], K), dtype=np.uint8)
    out[:, 0::2] = packed & 0x0F
    out[:, 1::2] = packed >> 4
    return out


def quantize_linear_zp(W: np.ndarray):
    """One-shot zero-point INT4 quantization: (packed uint8 [N, K/2], scale fp16 [N], zero uint8 [N])."""
    lo, hi = zp_range(W)
    s = zp_scale(lo, hi)
    z = zp_zero(lo, s)
    return pack_u4(zp_codes(W, s, z)), s, z


def dequantize_zp(packed, s, z, K: int) -> np.ndarray:
    """float64 weight = s * (q - z) (exact in float64)."""
    q = unpack_u4(packed, K).astype(np.float64)
    return (q - np.asarray(z, np.float64)[:, None]) * np.asarray(s, np.float16).astype(np.float64)[:, None]


def linear_forward_zp(X: np.ndarray, packed, s, z, row_block: int = 4096) -> np.ndarray:
    """Y[m,n] = fp16_rn( sum_k X[m,k] * s[n] (q[n,k] - z[n]) ): reading Z5."""
    X = np.asarray(X)
    assert X.dtype == np.float16 and X.ndim == 2
    M, K = X.shape
    N = packed.shape[0]
    X64 = X.astype(np.float64)
    Y = np.empty((M, N), dtype=np.float16)
    for n0 in range(0, N, row_block):
        n1 = min(N, n0 + row_block)
        Y[:, n0:n1] = (X64 @ dequantize_zp(packed[n0:n1], s[n0:n1], z[n0:n1], K).T).astype(np.float16)
    return Y
