"""C-ABI checks that need no GPU: the library loads, exports every symbol the
header declares, and rejects bad arguments before touching a device.

Every call here returns during argument validation (bad bits, bad shape, NULL
or misaligned pointers, empty problems); none reaches a kernel launch, so the
file is safe to run on a machine with a GPU too.
"""
import ctypes
import os
import re

import pytest

import int8_quantized_glmq_b200 as glmq
from int8_quantized_glmq_b200 import _binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "glmq.h")


def header_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"GLMQ_API\s+[\w\s\*]+?\b(glmq_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    lib = glmq.lib()
    syms = header_symbols()
    assert len(syms) >= 9
    for s in syms:
        assert hasattr(lib, s), s
    assert set(syms) == set(B.SIGNATURES), "binding and header disagree"


def test_header_constants_match_binding():
    text = open(HEADER).read()
    assert int(re.search(r"#define GLMQ_DECODE_MAX_M (\d+)", text).group(1)) == B.DECODE_MAX_M
    assert int(re.search(r"#define GLMQ_DECODE_AUTO_MAX_M (\d+)", text).group(1)) == B.DECODE_AUTO_MAX_M
    assert int(re.search(r"#define GLMQ_MAX_K (\d+)", text).group(1)) == B.MAX_K
    for name, val in [("GLMQ_OK", B.OK), ("GLMQ_ERR_BAD_SHAPE", B.ERR_BAD_SHAPE),
                      ("GLMQ_ERR_MISALIGNED", B.ERR_MISALIGNED), ("GLMQ_ERR_DEVICE", B.ERR_DEVICE)]:
        assert int(re.search(name + r" = (\d+)", text).group(1)) == val


def test_abi_version_and_packed_bytes():
    assert glmq.abi_version() == 1
    assert glmq.packed_bytes(36864, 12288, 4) == 36864 * 12288 // 2
    assert glmq.packed_bytes(12288, 32768, 8) == 12288 * 32768
    assert glmq.packed_bytes(3, 100, 4) == 0          # K % 64 != 0
    assert glmq.packed_bytes(3, 64, 5) == 0           # bad bits
    assert glmq.packed_bytes(-1, 64, 4) == 0


def test_status_strings():
    for st in range(8):
        assert glmq.status_string(st)
    assert "unknown" in glmq.status_string(99)


ALIGNED = 1 << 20   # never dereferenced: every call below fails validation first


@pytest.mark.parametrize("bits,K,expect", [(5, 64, B.ERR_BAD_BITS), (4, 100, B.ERR_BAD_SHAPE),
                                           (4, 0, B.ERR_BAD_SHAPE), (8, 65536 + 64, B.ERR_BAD_SHAPE)])
def test_quantize_rejects_bad_arguments(bits, K, expect):
    assert B.raw_quantize(ALIGNED, 4, K, bits, ALIGNED, ALIGNED) == expect


def test_quantize_null_and_misaligned():
    assert B.raw_quantize(0, 4, 64, 4, ALIGNED, ALIGNED) == B.ERR_NULL_POINTER
    assert B.raw_quantize(ALIGNED, 4, 64, 4, 0, ALIGNED) == B.ERR_NULL_POINTER
    assert B.raw_quantize(ALIGNED + 8, 4, 64, 4, ALIGNED, ALIGNED) == B.ERR_MISALIGNED
    assert B.raw_quantize(ALIGNED, 4, 64, 4, ALIGNED, ALIGNED + 2) == B.ERR_MISALIGNED


def test_quantize_empty_is_ok_without_device():
    assert B.raw_quantize(0, 0, 64, 4, 0, 0) == B.OK


@pytest.mark.parametrize("route", ["auto", "decode", "prefill"])
def test_gemm_validation(route):
    g = lambda **kw: B.raw_gemm(kw.get("X", ALIGNED), kw.get("M", 4), kw.get("P", ALIGNED), kw.get("S", ALIGNED),
                                kw.get("N", 8), kw.get("K", 64), kw.get("bits", 4), kw.get("Y", ALIGNED),
                                0, route)
    assert g(bits=3) == B.ERR_BAD_BITS
    assert g(K=96) == B.ERR_BAD_SHAPE
    assert g(M=-1) == B.ERR_BAD_SHAPE
    assert g(N=-5) == B.ERR_BAD_SHAPE
    assert g(X=0) == B.ERR_NULL_POINTER
    assert g(Y=0) == B.ERR_NULL_POINTER
    assert g(S=ALIGNED + 4) == B.ERR_MISALIGNED
    assert g(P=ALIGNED + 1) == B.ERR_MISALIGNED
    assert g(M=0, X=0, Y=0) == B.OK           # empty problem: nothing enqueued
    assert g(N=0, P=0, S=0, Y=0) == B.OK


def test_decode_route_rejects_large_m():
    assert B.raw_gemm(ALIGNED, 17, ALIGNED, ALIGNED, 8, 64, 4, ALIGNED, 0, "decode") == B.ERR_BAD_SHAPE


def test_binding_rejects_cpu_tensors():
    torch = pytest.importorskip("torch")
    W = torch.zeros((4, 64), dtype=torch.float16)
    with pytest.raises(ValueError):
        glmq.quantize(W, 4)


def test_kernel_launch_counter_ignores_rejected_calls():
    n0 = glmq.kernel_launches()
    assert n0 >= 0
    assert B.raw_quantize(ALIGNED, 4, 100, 4, ALIGNED, ALIGNED) == B.ERR_BAD_SHAPE
    assert B.raw_gemm(ALIGNED, 4, ALIGNED, ALIGNED, 8, 64, 3, ALIGNED, 0, "auto") == B.ERR_BAD_BITS
    assert B.raw_gemm(0, 0, ALIGNED, ALIGNED, 8, 64, 4, 0, 0, "auto") == B.OK     # empty: nothing enqueued
    assert glmq.kernel_launches() == n0


def test_fused_entry_points_validate_before_device_work():
    g = lambda **kw: B.raw_gemm_fused(kw.get("X", ALIGNED), kw.get("M", 4), ALIGNED, ALIGNED, kw.get("bias", 0),
                                      kw.get("N", 32), 64, 4, kw.get("epi", B.EPILOGUE_NONE), ALIGNED, 0)
    assert g(epi=7) == B.ERR_BAD_SHAPE
    assert g(epi=B.EPILOGUE_GEGLU, N=24) == B.ERR_BAD_SHAPE       # GeGLU needs N % 16 == 0
    assert g(bias=ALIGNED + 1) == B.ERR_MISALIGNED
    assert g(X=0) == B.ERR_NULL_POINTER
    assert g(M=0, X=0) == B.OK
    assert B.raw_quantize_geglu(ALIGNED, 40, 64, 4, ALIGNED, ALIGNED) == B.ERR_BAD_SHAPE
    assert B.raw_quantize_geglu(ALIGNED, 48, 64, 3, ALIGNED, ALIGNED) == B.ERR_BAD_BITS
    assert B.raw_quantize_geglu(0, 0, 64, 4, 0, 0) == B.OK


def test_zero_point_entry_points_validate_before_device_work():
    assert B.raw_quantize_zp(ALIGNED, 4, 100, ALIGNED, ALIGNED, ALIGNED) == B.ERR_BAD_SHAPE
    assert B.raw_quantize_zp(ALIGNED, 4, 64, ALIGNED, ALIGNED, 0) == B.ERR_NULL_POINTER
    assert B.raw_quantize_zp(ALIGNED + 2, 4, 64, ALIGNED, ALIGNED, ALIGNED) == B.ERR_MISALIGNED
    assert B.raw_quantize_zp(0, 0, 64, 0, 0, 0) == B.OK
    assert B.raw_gemm_zp(ALIGNED, 4, ALIGNED, ALIGNED, 0, 8, 64, ALIGNED) == B.ERR_NULL_POINTER
    assert B.raw_gemm_zp(ALIGNED, 4, ALIGNED, ALIGNED, ALIGNED, 8, 96, ALIGNED) == B.ERR_BAD_SHAPE
    assert B.raw_gemm_zp(0, 0, ALIGNED, ALIGNED, 0, 8, 64, 0) == B.OK


def test_decode_prefetch_entry_validates_before_device_work():
    g = lambda **kw: B.raw_gemm_decode_prefetch(
        kw.get("X", ALIGNED), kw.get("M", 4), ALIGNED, ALIGNED, kw.get("N", 8), kw.get("K", 64), kw.get("bits", 4),
        kw.get("Y", ALIGNED), kw.get("NP", ALIGNED), kw.get("NM", 1), kw.get("NN", 8), kw.get("NK", 64), 0)
    assert g(NM=0) == B.ERR_BAD_SHAPE
    assert g(NM=17) == B.ERR_BAD_SHAPE                 # the next call must be a decode call too
    assert g(NN=0) == B.ERR_BAD_SHAPE
    assert g(NK=96) == B.ERR_BAD_SHAPE
    assert g(NP=ALIGNED + 8) == B.ERR_MISALIGNED
    assert g(bits=3) == B.ERR_BAD_BITS
    assert g(M=17) == B.ERR_BAD_SHAPE                  # this call is a decode call
    assert g(X=0) == B.ERR_NULL_POINTER
    assert g(M=0, X=0, Y=0) == B.OK                    # empty problem: nothing enqueued
    assert g(NP=0, NM=0, NN=0, NK=0, M=0, X=0, Y=0) == B.OK   # no hint: the hint fields are ignored
