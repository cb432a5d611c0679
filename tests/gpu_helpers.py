"""Helpers for the GPU parity tests: host numpy <-> device tensors, edge-case weights,
and a record of the observed GEMM errors."""
import numpy as np

#: (case, relative max error) of every GEMM parity check that records itself; written
#: to the JSON file named by GLMQ_ERROR_REPORT at the end of the session (conftest.py)
OBSERVED_ERRORS = []


def record_error(case: str, err: float) -> float:
    OBSERVED_ERRORS.append((case, float(err)))
    return err


def torch_cuda():
    import torch
    if not torch.cuda.is_available():
        import pytest
        pytest.skip("needs a CUDA device")
    return torch


def to_dev(a: np.ndarray):
    torch = torch_cuda()
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def to_host(t) -> np.ndarray:
    return t.cpu().numpy()


def edge_case_weight(n_rows: int, K: int, seed: int = 7) -> np.ndarray:
    """fp16 [n_rows, K] mixing the rows that stress the quantizer's readings.

    Rows cycle through: zeros; a single huge outlier; subnormal magnitudes (scale
    subnormal, the clamp can fire); scales that round to zero; exact ties
    (dyadic values with absmax 7 / 14 / 127); negative absmax; N(0, 0.02) rows.
    """
    rng = np.random.default_rng(seed)
    W = np.zeros((n_rows, K), dtype=np.float32)
    for i in range(n_rows):
        kind = i % 9
        if kind == 0:
            continue                                           # all-zero row
        if kind == 1:
            W[i] = rng.standard_normal(K) * 0.02
            W[i, rng.integers(K)] = 60000.0                    # one huge outlier
        elif kind == 2:
            W[i] = rng.integers(-40, 41, K) * 2.0 ** -24        # subnormal values
        elif kind == 3:
            W[i] = rng.integers(-3, 4, K) * 2.0 ** -24          # scale rounds to 0 (INT4)
        elif kind == 4:
            W[i] = rng.integers(-14, 15, K) * 0.5               # ties with absmax 7: s = 1
            W[i, 0] = 7.0
        elif kind == 5:
            W[i] = rng.integers(-254, 255, K) * 0.5             # INT8 ties, absmax 127
            W[i, 1] = -127.0
        elif kind == 6:
            W[i] = rng.standard_normal(K) * 0.02
            W[i, 2] = -1.0                                      # negative absmax
        elif kind == 7:
            W[i] = rng.integers(-28, 29, K) * 0.5               # absmax 14: s = 2, ties at odd halves
            W[i, 3] = 14.0
        else:
            W[i] = rng.standard_normal(K) * 0.02
    return W.astype(np.float16)
