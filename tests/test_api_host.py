"""The C ABI on the host (no GPU): library loads, every declared entry point is
exported, and every argument error is reported before any CUDA call."""
import ctypes
import os
import re

import pytest

qmm = pytest.importorskip("decode_gemv_qmm_b200")
lib = qmm.lib

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "qmm.h")


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"QMM_API\s+[\w\s\*]+?\b(qmm_\w+)\s*\(", text)))


def test_every_declared_symbol_is_exported():
    names = declared_symbols()
    assert len(names) >= 20
    for name in names:
        assert hasattr(lib, name), f"{name} declared in include/qmm.h but not exported"


def test_version_and_error_string():
    assert qmm.version().startswith("qmm ")
    assert isinstance(lib.qmm_last_error_string(), bytes)


P16 = 0x1000          # a 16-byte aligned, never dereferenced pointer value
P_ODD = 0x1004        # 4-byte but not 16-byte aligned


def st_name(st):
    return qmm.STATUS_NAMES[st]


@pytest.mark.parametrize("call,expect", [
    (lambda: lib.qmm_q8_gemv(1, 8, 64, 16, P16, P16, P16, 0), "QMM_ERR_BLOCK"),
    (lambda: lib.qmm_q8_gemv(1, 8, 65, 32, P16, P16, P16, 0), "QMM_ERR_SHAPE"),
    (lambda: lib.qmm_q8_gemv(9, 8, 64, 32, P16, P16, P16, 0), "QMM_ERR_SHAPE"),
    (lambda: lib.qmm_q8_gemv(-1, 8, 64, 32, P16, P16, P16, 0), "QMM_ERR_SHAPE"),
    (lambda: lib.qmm_q8_gemv(1, 8, 32768 + 32, 32, P16, P16, P16, 0), "QMM_ERR_SHAPE"),
    (lambda: lib.qmm_q8_gemv(1, 8, 64, 32, 0, P16, P16, 0), "QMM_ERR_NULL"),
    (lambda: lib.qmm_q8_gemv(1, 8, 64, 32, P_ODD, P16, P16, 0), "QMM_ERR_ALIGN"),
    (lambda: lib.qmm_q8_gemv(1, 8, 64, 32, P16, P_ODD, P16, 0), "QMM_ERR_ALIGN"),
    (lambda: lib.qmm_q8_gemv(1, 8, 64, 32, P16, P16, P16 + 2, 0), "QMM_ERR_ALIGN"),
    (lambda: lib.qmm_q8_gemv_ex(1, 8, 64, 32, P16, P16, P16, 6, 0), "QMM_ERR_SHAPE"),
    (lambda: lib.qmm_quantize_act_q8(2, 48, 32, P16, P16, P16, 0), "QMM_ERR_SHAPE"),
    (lambda: lib.qmm_quantize_act_q8(2, 64, 32, P16, P_ODD, P16, 0), "QMM_ERR_ALIGN"),
    (lambda: lib.qmm_q8q8_gemv(1, 8, 64, 32, P16, 0, P16, P16, 0), "QMM_ERR_NULL"),
    (lambda: lib.qmm_q8q8_gemv(1, 8, 64, 32, P16, P16, 0, P16, 0), "QMM_ERR_NULL"),
    (lambda: lib.qmm_q8q8_block_dots(1, 8, 64, 32, P16, P16, 0, 0), "QMM_ERR_NULL"),
    (lambda: lib.qmm_q8q8_gemv_fused(1, 8, 64, 32, P16, P16, 0, P16, P16, 0, 0), "QMM_ERR_NULL"),
    (lambda: lib.qmm_q8q8_gemv_fused(1, 8, 64, 32, P16, P16, P16, 0, P16, 0, 0), "QMM_ERR_NULL"),
    (lambda: lib.qmm_q8q8_gemv_fused(1, 8, 64, 32, P16, P16, P_ODD, P16, P16, 0, 0), "QMM_ERR_ALIGN"),
    (lambda: lib.qmm_q8q8_gemv_fused(9, 8, 64, 32, P16, P16, P16, P16, P16, 0, 0), "QMM_ERR_SHAPE"),
    (lambda: lib.qmm_q8q8_gemv_fused(1, 8, 64, 32, P16, P16, P16, P16, P16, 2, 0), "QMM_ERR_SHAPE"),
    (lambda: lib.qmm_q4_swiglu_gateup(9, 8, 64, 32, P16, P16, P16, P16, 0), "QMM_ERR_SHAPE"),
    (lambda: lib.qmm_q4_swiglu_gateup(8, 8, 64, 32, P16, P_ODD, P16, P16, 0), "QMM_ERR_ALIGN"),
    (lambda: lib.qmm_q4_gateup_unfused(8, 8, 64, 32, P16, P16, P16, 0, P16, P16, 0), "QMM_ERR_NULL"),
    (lambda: lib.qmm_quantize_act_q8_0(2, 64, 32, P16, P_ODD, 0), "QMM_ERR_ALIGN"),
    (lambda: lib.qmm_quantize_act_q8_0(2, 48, 32, P16, P16, 0), "QMM_ERR_SHAPE"),
    (lambda: lib.qmm_q8q8_gemv_q8_0(1, 8, 64, 32, P16, 0, P16, 0, 0), "QMM_ERR_NULL"),
    (lambda: lib.qmm_q8q8_gemv_q8_0(1, 8, 64, 32, P16, P_ODD, P16, 0, 0), "QMM_ERR_ALIGN"),
    (lambda: lib.qmm_q8q8_gemv_q8_0(9, 8, 64, 32, P16, P16, P16, 0, 0), "QMM_ERR_SHAPE"),
    (lambda: lib.qmm_q8_gemv_auto(1, 8, 64, 32, P16, P16, P16, 0, P16, 0, 0), "QMM_ERR_NULL"),
    (lambda: lib.qmm_q8_gemv_auto(1, 8, 64, 32, P16, P16, P16, P16, 0, 0, 0), "QMM_ERR_NULL"),
    (lambda: lib.qmm_q8_gemv_auto(1, 8, 64, 32, P16, P16, P16, P16, P16, 2, 0), "QMM_ERR_SHAPE"),
    (lambda: lib.qmm_q4_gemv(1, 8, 64, 32, 0, P16, P16, 0, 0), "QMM_ERR_NULL"),
    (lambda: lib.qmm_q4_gemv(1, 8, 64, 32, P16, P_ODD, P16, 0, 0), "QMM_ERR_ALIGN"),
    (lambda: lib.qmm_q4_gemv(9, 8, 64, 32, P16, P16, P16, 0, 0), "QMM_ERR_SHAPE"),
    (lambda: lib.qmm_q4_gemv(1, 8, 64, 32, P16, P16, P16, 8, 0), "QMM_ERR_SHAPE"),
    (lambda: lib.qmm_quant_matmul_prefill(2, 8, 8, 64, 32, P16, P16, P16, 0), "QMM_ERR_DTYPE"),
    (lambda: lib.qmm_quant_matmul_prefill(0, 8, 8, 64, 32, P16, P_ODD, P16, 0), "QMM_ERR_ALIGN"),
    (lambda: lib.qmm_quant_matmul_prefill(1, 8, -8, 64, 32, P16, P16, P16, 0), "QMM_ERR_SHAPE"),
    (lambda: lib.qmm_quant_matmul_prefill_ex(0, 8, 8, 64, 32, P16, P16, P16, 2, 0), "QMM_ERR_SHAPE"),
    (lambda: lib.qmm_prefill_plan(0, 1024, 4864, 896, 32, 0), "QMM_ERR_NULL"),
    (lambda: lib.qmm_prefill_plan(2, 1024, 4864, 896, 32, P16), "QMM_ERR_DTYPE"),
    (lambda: lib.qmm_prefill_plan(0, 1024, 4864, 896, 16, P16), "QMM_ERR_BLOCK"),
    (lambda: lib.qmm_prefill_plan(0, 1024, 4864, 900, 32, P16), "QMM_ERR_SHAPE"),
    (lambda: lib.qmm_prefill_plan(0, 0, 4864, 896, 32, P16), "QMM_ERR_SHAPE"),
    (lambda: lib.qmm_prefill_plan(1, 8, 8, 0, 32, P16), "QMM_ERR_SHAPE"),
])
def test_argument_errors_before_any_cuda_call(call, expect):
    st = call()
    assert st_name(st) == expect, lib.qmm_last_error_string()
    assert lib.qmm_last_error_string()  # a message is recorded


def test_empty_calls_are_ok_without_touching_cuda():
    assert lib.qmm_q8_gemv(0, 8, 64, 32, 0, 0, 0, 0) == 0
    assert lib.qmm_q8_gemv(1, 0, 64, 32, 0, 0, 0, 0) == 0
    assert lib.qmm_quantize_act_q8(0, 64, 32, 0, 0, 0, 0) == 0
    assert lib.qmm_quantize_act_q8(3, 0, 32, 0, 0, 0, 0) == 0
    assert lib.qmm_q4_swiglu_gateup(0, 5, 64, 32, 0, 0, 0, 0, 0) == 0
    assert lib.qmm_q8q8_gemv_fused(0, 5, 64, 32, 0, 0, 0, 0, 0, 0, 0) == 0
    assert lib.qmm_quant_matmul_prefill(1, 5, 0, 64, 32, 0, 0, 0, 0) == 0


def test_python_binding_raises_with_status():
    import torch
    with pytest.raises(qmm.QmmError) as e:
        qmm.qmm_q8_gemv(torch.zeros(10, dtype=torch.uint8), torch.zeros(1, 33), 4, torch.zeros(1, 4), stream=0)
    assert e.value.status == qmm.QMM_ERR_SHAPE


def test_multi_argument_errors_before_any_cuda_call():
    i64, vp = ctypes.c_int64, ctypes.c_void_p
    N = (i64 * 2)(8, 8)
    W = (vp * 2)(P16, P16)
    Y = (vp * 2)(P16, P16)
    W_odd = (vp * 2)(P16, P_ODD)
    Y_null = (vp * 2)(P16, 0)
    cases = [
        (lambda: lib.qmm_q8_gemv_multi(1, 64, 32, 0, N, W, P16, Y, 0, 0), "QMM_ERR_SHAPE"),
        (lambda: lib.qmm_q8_gemv_multi(1, 64, 32, 5, N, W, P16, Y, 0, 0), "QMM_ERR_SHAPE"),
        (lambda: lib.qmm_q8_gemv_multi(1, 64, 32, 2, None, W, P16, Y, 0, 0), "QMM_ERR_NULL"),
        (lambda: lib.qmm_q8_gemv_multi(1, 64, 32, 2, N, W_odd, P16, Y, 0, 0), "QMM_ERR_ALIGN"),
        (lambda: lib.qmm_q8_gemv_multi(1, 64, 32, 2, N, W, P16, Y_null, 0, 0), "QMM_ERR_NULL"),
        (lambda: lib.qmm_q8_gemv_multi(1, 64, 32, 2, N, W, 0, Y, 0, 0), "QMM_ERR_NULL"),
        (lambda: lib.qmm_q8_gemv_multi(9, 64, 32, 2, N, W, P16, Y, 0, 0), "QMM_ERR_SHAPE"),
        (lambda: lib.qmm_q8_gemv_multi(1, 64, 16, 2, N, W, P16, Y, 0, 0), "QMM_ERR_BLOCK"),
        (lambda: lib.qmm_q8_gemv_multi(1, 64, 32, 2, N, W, P16, Y, 4, 0), "QMM_ERR_SHAPE"),
    ]
    for call, expect in cases:
        assert st_name(call()) == expect, lib.qmm_last_error_string()
    zero = (i64 * 2)(0, 0)
    assert lib.qmm_q8_gemv_multi(1, 64, 32, 2, zero, W, 0, Y, 0, 0) == 0  # nothing to do
    assert lib.qmm_q8_gemv_multi(0, 64, 32, 2, N, W, 0, Y, 0, 0) == 0     # M = 0
