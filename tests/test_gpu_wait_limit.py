"""Failure detection without a GPU fault.

Every wait of the kernels on a pipeline barrier gives up after a wall-clock limit,
sets a bit in the device status word and lets the kernel finish. Here the limit is
lowered (glmq_set_wait_limit_ns) to 1 ns, so a normal call's waits run out while its
tiles are still on their way from HBM: the call must come back with GLMQ_ERR_DEVICE
and its kernel's flag bits from glmq_last_device_error, and with the default limit
restored the next call must again match the oracle, which also shows that the
split-K scratch was returned to zero. Nothing faults, traps or hangs: the waits by
which a block makes sure its own copies have landed (and, in the tensor-core
kernels, its own MMAs have finished) before it exits keep the default limit.
"""
import numpy as np
import pytest

import oracle
from gpu_helpers import to_dev, to_host, torch_cuda
from inputs import gaussian_fp16

TOL = 5e-3
DECODE_CONSUMER_WAIT = 1 << 0      # glmq_ptx.cuh: kErrDecodeConsumerWait
DECODE_PRODUCER_WAIT = 1 << 1      # kErrDecodeProducerWait
TCGEN05_WAIT = 1 << 2              # kErrPrefillWait: the skinny and prefill kernels


@pytest.mark.gpu
def test_waits_that_run_out_are_reported_and_the_next_call_is_correct():
    torch = torch_cuda()
    import int8_quantized_glmq_b200 as glmq
    from int8_quantized_glmq_b200 import _binding as B
    M, N, K = 16, 8192, 16384                      # tiles split over K parts: the scratch is used
    W = gaussian_fp16((N, K), 0.02, 4242)
    X = gaussian_fp16((M, K), 1.0, 4243)
    packed, scale = glmq.quantize(to_dev(W), 4)
    Xd = to_dev(X)
    assert glmq.last_device_error() == (B.OK, 0)
    try:
        glmq.set_wait_limit_ns(1)
        glmq.gemm_decode(Xd, packed, scale, 4)        # enqueued normally; its waits give up on the device
        st, flags = glmq.last_device_error()
    finally:
        glmq.set_wait_limit_ns(0)
    assert st == B.ERR_DEVICE
    assert flags & DECODE_CONSUMER_WAIT
    assert flags & ~(DECODE_CONSUMER_WAIT | DECODE_PRODUCER_WAIT) == 0
    assert glmq.last_device_error() == (B.OK, 0)       # reading cleared the word

    rows = np.unique(np.concatenate([np.arange(64), np.arange(N - 64, N),
                                     np.random.default_rng(5).choice(N, 128, replace=False)]))
    Y = to_host(glmq.gemm_decode(Xd, packed, scale, 4))
    p_ref, s_ref = oracle.quantize_linear(W[rows], 4)
    assert np.array_equal(to_host(packed)[rows], p_ref)
    err = oracle.relative_max_error(Y[:, rows], oracle.linear_forward(X, p_ref, s_ref, 4))
    assert err <= TOL, err
    assert glmq.last_device_error() == (B.OK, 0)


@pytest.mark.gpu
@pytest.mark.parametrize("M", [32, 256], ids=["skinny", "prefill"])
def test_tensor_core_kernels_report_waits_that_run_out(M):
    """The same for the tcgen05 kernels: 16 < M <= 64 runs the skinny kernel, M > 64 the
    prefill kernel; both split these tiles over K parts, so the scratch is used."""
    torch = torch_cuda()
    import int8_quantized_glmq_b200 as glmq
    from int8_quantized_glmq_b200 import _binding as B
    N, K = 8192, 16384
    W = gaussian_fp16((N, K), 0.02, 4252 + M)
    X = gaussian_fp16((M, K), 1.0, 4253 + M)
    packed, scale = glmq.quantize(to_dev(W), 4)
    Xd = to_dev(X)
    assert glmq.last_device_error() == (B.OK, 0)
    try:
        glmq.set_wait_limit_ns(1)
        glmq.gemm(Xd, packed, scale, 4, route="prefill")
        st, flags = glmq.last_device_error()
    finally:
        glmq.set_wait_limit_ns(0)
    assert st == B.ERR_DEVICE
    assert flags == TCGEN05_WAIT
    assert glmq.last_device_error() == (B.OK, 0)

    rows = np.unique(np.concatenate([np.arange(64), np.arange(N - 64, N),
                                     np.random.default_rng(6).choice(N, 128, replace=False)]))
    Y = to_host(glmq.gemm(Xd, packed, scale, 4, route="prefill"))
    p_ref, s_ref = oracle.quantize_linear(W[rows], 4)
    err = oracle.relative_max_error(Y[:, rows], oracle.linear_forward(X, p_ref, s_ref, 4))
    assert err <= TOL, err
    assert glmq.last_device_error() == (B.OK, 0)
