"""Python binding of libqmm.so: block-quantized weight matmul on B200 (sm_100a).

Argument marshalling only -- every step of every operation runs in the CUDA
kernels of libqmm.so. Functions carry the names of the C entry points
(include/qmm.h) and take torch tensors for device buffers; PyTorch supplies
device memory and streams, nothing else. Importing this package fails loudly
if the library has not been built (``python decode_gemv_qmm_b200/build.py``);
there is no fallback of any kind.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqmm.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python decode_gemv_qmm_b200/build.py`")

lib = ctypes.CDLL(LIB_PATH)

QMM_OK, QMM_ERR_NULL, QMM_ERR_SHAPE, QMM_ERR_BLOCK, QMM_ERR_ALIGN = 0, 1, 2, 3, 4
QMM_ERR_DTYPE, QMM_ERR_DEVICE, QMM_ERR_CUDA, QMM_ERR_DEVICE_CHECK = 5, 6, 7, 8
STATUS_NAMES = {0: "QMM_OK", 1: "QMM_ERR_NULL", 2: "QMM_ERR_SHAPE", 3: "QMM_ERR_BLOCK", 4: "QMM_ERR_ALIGN",
                5: "QMM_ERR_DTYPE", 6: "QMM_ERR_DEVICE", 7: "QMM_ERR_CUDA", 8: "QMM_ERR_DEVICE_CHECK"}
QMM_Q8_0, QMM_Q4_0 = 0, 1
QMM_FLAG_EARLY_WEIGHTS = 1
BLOCK = 32
MAX_DECODE_M = 8
MAX_K = 32768
MAX_PROJ = 4

_i64, _int, _u32, _p = ctypes.c_int64, ctypes.c_int, ctypes.c_uint32, ctypes.c_void_p
_SIGS = {
    "qmm_q8_gemv": [_i64, _i64, _i64, _int, _p, _p, _p, _p],
    "qmm_q8_gemv_ex": [_i64, _i64, _i64, _int, _p, _p, _p, _u32, _p],
    "qmm_quantize_act_q8": [_i64, _i64, _int, _p, _p, _p, _p],
    "qmm_q8q8_gemv": [_i64, _i64, _i64, _int, _p, _p, _p, _p, _p],
    "qmm_q8q8_gemv_ex": [_i64, _i64, _i64, _int, _p, _p, _p, _p, _u32, _p],
    "qmm_quantize_act_q8_0": [_i64, _i64, _int, _p, _p, _p],
    "qmm_q8q8_gemv_q8_0": [_i64, _i64, _i64, _int, _p, _p, _p, _u32, _p],
    "qmm_q8_gemv_auto": [_i64, _i64, _i64, _int, _p, _p, _p, _p, _p, _u32, _p],
    "qmm_q4_gemv": [_i64, _i64, _i64, _int, _p, _p, _p, _u32, _p],
    "qmm_q8_gemv_multi": [_i64, _i64, _int, _int, _p, _p, _p, _p, _u32, _p],
    "qmm_q8q8_gemv_fused": [_i64, _i64, _i64, _int, _p, _p, _p, _p, _p, _u32, _p],
    "qmm_q4_swiglu_gateup": [_i64, _i64, _i64, _int, _p, _p, _p, _p, _p],
    "qmm_q4_swiglu_gateup_ex": [_i64, _i64, _i64, _int, _p, _p, _p, _p, _u32, _p],
    "qmm_quant_matmul_prefill": [_int, _i64, _i64, _i64, _int, _p, _p, _p, _p],
    "qmm_quant_matmul_prefill_ex": [_int, _i64, _i64, _i64, _int, _p, _p, _p, _u32, _p],
    "qmm_q8q8_block_dots": [_i64, _i64, _i64, _int, _p, _p, _p, _p],
    "qmm_q4_gateup_unfused": [_i64, _i64, _i64, _int, _p, _p, _p, _p, _p, _p, _p],
    "qmm_prefill_plan": [_int, _i64, _i64, _i64, _int, _p],
    "qmm_q8q8_gemv_fused_dots": [_i64, _i64, _i64, _int, _p, _p, _p, _p, _p, _p, _p],
    "qmm_q8q8_block_dots_q8_0": [_i64, _i64, _i64, _int, _p, _p, _p, _p],
    "qmm_test_withheld_copy": [_int, _i64, _i64, _i64, _int, _p, _p, _p, ctypes.c_uint64, _p],
}
for _name, _args in _SIGS.items():
    _f = getattr(lib, _name, None)
    if _f is not None:
        _f.argtypes = _args
        _f.restype = ctypes.c_int
lib.qmm_last_error_string.restype = ctypes.c_char_p
lib.qmm_last_error_string.argtypes = []
lib.qmm_version.restype = ctypes.c_char_p
lib.qmm_version.argtypes = []
lib.qmm_device_status.restype = ctypes.c_int
lib.qmm_device_status.argtypes = [ctypes.POINTER(ctypes.c_uint32)]


class QmmError(RuntimeError):
    def __init__(self, status: int, fn: str):
        self.status = status
        msg = lib.qmm_last_error_string().decode(errors="replace")
        super().__init__(f"{fn}: {STATUS_NAMES.get(status, status)}: {msg}")


def _check(status: int, fn: str):
    if status != QMM_OK:
        raise QmmError(status, fn)


def _ptr(t) -> int:
    if t is None:
        return 0
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def version() -> str:
    return lib.qmm_version().decode()


def device_status() -> int:
    """Synchronise and read-and-clear the kernels' device status words (0 = clean;
    the library reports recorded bits as QMM_ERR_DEVICE_CHECK, returned here as
    the bits themselves)."""
    bits = ctypes.c_uint32(0)
    st = lib.qmm_device_status(ctypes.byref(bits))
    if st != QMM_ERR_DEVICE_CHECK:
        _check(st, "qmm_device_status")
    return bits.value


def _out(Y, shape, device, dtype=torch.float32):
    if Y is None:
        return torch.empty(shape, dtype=dtype, device=device)
    return Y


def qmm_q8_gemv(W: torch.Tensor, X: torch.Tensor, N: int, Y: torch.Tensor | None = None, *,
                block: int = BLOCK, flags: int = 0, stream=None) -> torch.Tensor:
    """Y[M, N] = X[M, K] . dequant(W)^T for Q8_0 blocks W (uint8, N*K/32*34 bytes)."""
    M, K = X.shape
    Y = _out(Y, (M, N), X.device)
    if flags:
        st = lib.qmm_q8_gemv_ex(M, N, K, block, _ptr(W), _ptr(X), _ptr(Y), flags, _stream(stream))
    else:
        st = lib.qmm_q8_gemv(M, N, K, block, _ptr(W), _ptr(X), _ptr(Y), _stream(stream))
    _check(st, "qmm_q8_gemv")
    return Y


def qmm_quantize_act_q8_0(X: torch.Tensor, XB: torch.Tensor | None = None, *, block: int = BLOCK, stream=None):
    """XB uint8[M, K/32*34]: X quantised into ggml Q8_0 blocks (fp16 scale, ggml rule)."""
    M, K = X.shape
    XB = _out(XB, (M, (K // BLOCK) * 34), X.device, torch.uint8)
    _check(lib.qmm_quantize_act_q8_0(M, K, block, _ptr(X), _ptr(XB), _stream(stream)), "qmm_quantize_act_q8_0")
    return XB


def qmm_q8q8_gemv_q8_0(W: torch.Tensor, XB: torch.Tensor, K: int, N: int, Y: torch.Tensor | None = None, *,
                       block: int = BLOCK, flags: int = 0, stream=None) -> torch.Tensor:
    """Y[M, N] from Q8_0 weights W and Q8_0 activation blocks XB (M rows of K/32 blocks)."""
    M = XB.shape[0]
    Y = _out(Y, (M, N), XB.device)
    _check(lib.qmm_q8q8_gemv_q8_0(M, N, K, block, _ptr(W), _ptr(XB), _ptr(Y), flags, _stream(stream)),
           "qmm_q8q8_gemv_q8_0")
    return Y


def qmm_q8_gemv_auto(W: torch.Tensor, X: torch.Tensor, N: int, Y: torch.Tensor | None = None,
                     QX: torch.Tensor | None = None, DX: torch.Tensor | None = None, *, block: int = BLOCK,
                     flags: int = 0, stream=None):
    """(Y, QX, DX): the Q8xQ8 GEMV for short K (activations quantised), else the fp32 GEMV."""
    M, K = X.shape
    Y = _out(Y, (M, N), X.device)
    QX = _out(QX, (M, K), X.device, torch.int8)
    DX = _out(DX, (M, K // BLOCK), X.device)
    _check(lib.qmm_q8_gemv_auto(M, N, K, block, _ptr(W), _ptr(X), _ptr(Y), _ptr(QX), _ptr(DX), flags,
                                _stream(stream)), "qmm_q8_gemv_auto")
    return Y, QX, DX


def qmm_q8_gemv_multi(Ws, X: torch.Tensor, Ns, Ys=None, *, block: int = BLOCK, flags: int = 0, stream=None):
    """[Y_i] = [X . dequant(W_i)^T]: several Q8_0 projections of the same X in one launch."""
    M, K = X.shape
    k = len(Ws)
    if Ys is None:
        Ys = [torch.empty((M, n), dtype=torch.float32, device=X.device) for n in Ns]
    n_arr = (ctypes.c_int64 * k)(*[int(n) for n in Ns])
    w_arr = (ctypes.c_void_p * k)(*[_ptr(w) for w in Ws])
    y_arr = (ctypes.c_void_p * k)(*[_ptr(y) for y in Ys])
    _check(lib.qmm_q8_gemv_multi(M, K, block, k, n_arr, w_arr, _ptr(X), y_arr, flags, _stream(stream)),
           "qmm_q8_gemv_multi")
    return Ys


def qmm_quantize_act_q8(X: torch.Tensor, QX: torch.Tensor | None = None, DX: torch.Tensor | None = None, *,
                        block: int = BLOCK, stream=None):
    """(QX int8[M, K], DX fp32[M, K/32]) = per-32-block Q8 quantisation of X."""
    M, K = X.shape
    QX = _out(QX, (M, K), X.device, torch.int8)
    DX = _out(DX, (M, K // BLOCK), X.device)
    _check(lib.qmm_quantize_act_q8(M, K, block, _ptr(X), _ptr(QX), _ptr(DX), _stream(stream)),
           "qmm_quantize_act_q8")
    return QX, DX


def qmm_q8q8_gemv(W: torch.Tensor, QX: torch.Tensor, DX: torch.Tensor, N: int, Y: torch.Tensor | None = None, *,
                  block: int = BLOCK, flags: int = 0, stream=None) -> torch.Tensor:
    """Y[M, N] from Q8_0 blocks W and Q8 activation codes QX with block scales DX."""
    M, K = QX.shape
    Y = _out(Y, (M, N), QX.device)
    if flags:
        st = lib.qmm_q8q8_gemv_ex(M, N, K, block, _ptr(W), _ptr(QX), _ptr(DX), _ptr(Y), flags, _stream(stream))
    else:
        st = lib.qmm_q8q8_gemv(M, N, K, block, _ptr(W), _ptr(QX), _ptr(DX), _ptr(Y), _stream(stream))
    _check(st, "qmm_q8q8_gemv")
    return Y


def qmm_q8q8_gemv_fused(W: torch.Tensor, X: torch.Tensor, N: int, Y: torch.Tensor | None = None,
                        QX: torch.Tensor | None = None, DX: torch.Tensor | None = None, *, block: int = BLOCK,
                        flags: int = 0, stream=None):
    """(Y, QX, DX): the Q8xQ8 GEMV of X with its own activation quantisation in the same call."""
    M, K = X.shape
    Y = _out(Y, (M, N), X.device)
    QX = _out(QX, (M, K), X.device, torch.int8)
    DX = _out(DX, (M, K // BLOCK), X.device)
    _check(lib.qmm_q8q8_gemv_fused(M, N, K, block, _ptr(W), _ptr(X), _ptr(QX), _ptr(DX), _ptr(Y), flags,
                                   _stream(stream)), "qmm_q8q8_gemv_fused")
    return Y, QX, DX


def qmm_q8q8_block_dots(W: torch.Tensor, QX: torch.Tensor, N: int, isum: torch.Tensor | None = None, *,
                        block: int = BLOCK, stream=None) -> torch.Tensor:
    M, K = QX.shape
    isum = _out(isum, (M, N, K // BLOCK), QX.device, torch.int32)
    _check(lib.qmm_q8q8_block_dots(M, N, K, block, _ptr(W), _ptr(QX), _ptr(isum), _stream(stream)),
           "qmm_q8q8_block_dots")
    return isum


def qmm_q8q8_gemv_fused_dots(W: torch.Tensor, X: torch.Tensor, N: int, *, block: int = BLOCK, stream=None):
    """(Y, QX, DX, isum): qmm_q8q8_gemv_fused plus its exact int32 block dots isum[M, N, K/32]."""
    M, K = X.shape
    Y = torch.empty((M, N), dtype=torch.float32, device=X.device)
    QX = torch.empty((M, K), dtype=torch.int8, device=X.device)
    DX = torch.empty((M, K // BLOCK), dtype=torch.float32, device=X.device)
    isum = torch.empty((M, N, K // BLOCK), dtype=torch.int32, device=X.device)
    _check(lib.qmm_q8q8_gemv_fused_dots(M, N, K, block, _ptr(W), _ptr(X), _ptr(QX), _ptr(DX), _ptr(Y), _ptr(isum),
                                        _stream(stream)), "qmm_q8q8_gemv_fused_dots")
    return Y, QX, DX, isum


def qmm_q8q8_block_dots_q8_0(W: torch.Tensor, XB: torch.Tensor, K: int, N: int, *, block: int = BLOCK,
                             stream=None) -> torch.Tensor:
    """isum[M, N, K/32]: the exact block dots of qmm_q8q8_gemv_q8_0."""
    M = XB.shape[0]
    isum = torch.empty((M, N, K // BLOCK), dtype=torch.int32, device=XB.device)
    _check(lib.qmm_q8q8_block_dots_q8_0(M, N, K, block, _ptr(W), _ptr(XB), _ptr(isum), _stream(stream)),
           "qmm_q8q8_block_dots_q8_0")
    return isum


def qmm_test_withheld_copy(kernel: int, W: torch.Tensor, X: torch.Tensor, N: int, Y: torch.Tensor, wait_ns: int, *,
                           block: int = BLOCK, stream=None) -> None:
    """Failure-path test launch (kernel 0: streaming Q8_0 GEMV, 1: small-M prefill): one copy of
    CTA 0 is never issued, so its waits give up after wait_ns; read the result with device_status()."""
    M, K = X.shape
    _check(lib.qmm_test_withheld_copy(kernel, M, N, K, block, _ptr(W), _ptr(X), _ptr(Y), wait_ns, _stream(stream)),
           "qmm_test_withheld_copy")


def qmm_q4_gemv(W: torch.Tensor, X: torch.Tensor, N: int, Y: torch.Tensor | None = None, *,
                block: int = BLOCK, flags: int = 0, stream=None) -> torch.Tensor:
    """Y[M, N] = X[M, K] . dequant(W)^T for Q4_0 blocks W (uint8, N*K/32*18 bytes)."""
    M, K = X.shape
    Y = _out(Y, (M, N), X.device)
    _check(lib.qmm_q4_gemv(M, N, K, block, _ptr(W), _ptr(X), _ptr(Y), flags, _stream(stream)), "qmm_q4_gemv")
    return Y


def qmm_q4_swiglu_gateup(Wg: torch.Tensor, Wu: torch.Tensor, X: torch.Tensor, N: int,
                         Y: torch.Tensor | None = None, *, block: int = BLOCK, flags: int = 0,
                         stream=None) -> torch.Tensor:
    """Y[M, N] = silu(X . Wg^T) * (X . Wu^T) for Q4_0 blocks Wg, Wu in one launch."""
    M, K = X.shape
    Y = _out(Y, (M, N), X.device)
    if flags:
        st = lib.qmm_q4_swiglu_gateup_ex(M, N, K, block, _ptr(Wg), _ptr(Wu), _ptr(X), _ptr(Y), flags,
                                         _stream(stream))
    else:
        st = lib.qmm_q4_swiglu_gateup(M, N, K, block, _ptr(Wg), _ptr(Wu), _ptr(X), _ptr(Y), _stream(stream))
    _check(st, "qmm_q4_swiglu_gateup")
    return Y


def qmm_q4_gateup_unfused(Wg, Wu, X, N, G=None, U=None, Y=None, *, block: int = BLOCK, stream=None):
    M, K = X.shape
    G, U, Y = (_out(t, (M, N), X.device) for t in (G, U, Y))
    _check(lib.qmm_q4_gateup_unfused(M, N, K, block, _ptr(Wg), _ptr(Wu), _ptr(X), _ptr(G), _ptr(U), _ptr(Y),
                                     _stream(stream)), "qmm_q4_gateup_unfused")
    return G, U, Y


def qmm_quant_matmul_prefill(wtype: int, W: torch.Tensor, X: torch.Tensor, N: int, Y: torch.Tensor | None = None,
                             *, block: int = BLOCK, flags: int = 0, stream=None) -> torch.Tensor:
    """Y[M, N] = bf16 X[M, K] . bf16(dequant(W))^T with fp32 accumulation (tensor cores)."""
    M, K = X.shape
    Y = _out(Y, (M, N), X.device)
    if flags:
        st = lib.qmm_quant_matmul_prefill_ex(wtype, M, N, K, block, _ptr(W), _ptr(X), _ptr(Y), flags,
                                             _stream(stream))
    else:
        st = lib.qmm_quant_matmul_prefill(wtype, M, N, K, block, _ptr(W), _ptr(X), _ptr(Y), _stream(stream))
    _check(st, "qmm_quant_matmul_prefill")
    return Y


def qmm_prefill_plan(wtype: int, M: int, N: int, K: int, *, block: int = BLOCK) -> dict:
    """The tiling qmm_quant_matmul_prefill launches for this problem on the current device."""
    out = (ctypes.c_int32 * 5)()
    _check(lib.qmm_prefill_plan(wtype, M, N, K, block, ctypes.addressof(out)), "qmm_prefill_plan")
    return {"mt": out[0], "split": out[1], "stages": out[2], "ctas": out[3],
            "kernel": "small_m" if out[4] == 1 else "tcgen05"}
