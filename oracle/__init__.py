"""CPU oracle for block-quantized weight matmul (ctypes wrapper over qmm_oracle.c).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg are the only code allowed to import this module.
The CUDA library never imports, links or calls it.

All functions take numpy arrays (block bytes as uint8, activations as float32,
bf16 activations as uint16 bit patterns) and return float64 results together
with the absolute norm ``S = sum |w*x|`` per output that the tolerances use.
Windows ``(m0, m1, n0, n1)`` select a rectangle of outputs so that full-size
workloads can be checked on sampled outputs.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "qmm_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_CFLAGS = ["-O2", "-std=c11", "-fno-fast-math", "-ffp-contract=off", "-shared", "-fPIC"]
_lock = threading.Lock()
_lib = None

Q8_0, Q4_0 = 0, 1
BLOCK = 32


def build(force: bool = False) -> str:
    """Compile qmm_oracle.c with gcc into liboracle.so next to it."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *_CFLAGS, _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _bind(lib):
    i64, p = ctypes.c_int64, ctypes.c_void_p
    lib.ora_half_to_double.restype = ctypes.c_double
    lib.ora_half_to_double.argtypes = [ctypes.c_uint16]
    lib.ora_bf16_to_double.restype = ctypes.c_double
    lib.ora_bf16_to_double.argtypes = [ctypes.c_uint16]
    lib.ora_decode_block.argtypes = [ctypes.c_int, p, p]
    lib.ora_dequantize.argtypes = [ctypes.c_int, i64, i64, p, p]
    lib.ora_gemv.argtypes = [ctypes.c_int, i64, i64, i64, p, p, i64, i64, i64, i64, p, p]
    lib.ora_quantize_act_q8.argtypes = [i64, i64, p, p, p]
    lib.ora_quantize_act_q8_0.argtypes = [i64, i64, p, p]
    lib.ora_float_to_half_rne.argtypes = [ctypes.c_float]
    lib.ora_float_to_half_rne.restype = ctypes.c_uint16
    lib.ora_q8q8_block_dots.restype = i64
    lib.ora_q8q8_block_dots.argtypes = [i64, i64, i64, p, p, i64, i64, i64, i64, p]
    lib.ora_q8q8_gemv.argtypes = [i64, i64, i64, p, p, p, i64, i64, i64, i64, p, p]
    lib.ora_swiglu.argtypes = [ctypes.c_int, i64, i64, i64, p, p, p, i64, i64, i64, i64,
                               p, p, p, p, p]
    lib.ora_prefill.argtypes = [ctypes.c_int, i64, i64, i64, p, p, i64, i64, i64, i64, p, p]
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            _lib = _bind(ctypes.CDLL(_LIB_PATH))
    return _lib


def _swap_library(path):
    """Use another build of qmm_oracle.c (``path``) until called again with None.

    Only the tests that plant a mistake in a copy of the oracle use this, to
    check that some pin catches the mistake."""
    global _lib
    with _lock:
        _lib = None if path is None else _bind(ctypes.CDLL(path))


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data


def _u8(w) -> np.ndarray:
    return np.ascontiguousarray(w, dtype=np.uint8)


def _window(M, N, window):
    if window is None:
        return 0, M, 0, N
    m0, m1, n0, n1 = window
    assert 0 <= m0 <= m1 <= M and 0 <= n0 <= n1 <= N
    return m0, m1, n0, n1


def half_to_double(bits: int) -> float:
    return _load().ora_half_to_double(int(bits))


def bf16_to_double(bits: int) -> float:
    return _load().ora_bf16_to_double(int(bits))


def decode_block(wtype: int, blk: np.ndarray) -> np.ndarray:
    blk = _u8(blk)
    assert blk.size == (34 if wtype == Q8_0 else 18)
    out = np.empty(BLOCK, dtype=np.float64)
    _load().ora_decode_block(wtype, _ptr(blk), _ptr(out))
    return out


def dequantize(wtype: int, W: np.ndarray, N: int, K: int) -> np.ndarray:
    W = _u8(W)
    out = np.empty((N, K), dtype=np.float64)
    _load().ora_dequantize(wtype, N, K, _ptr(W), _ptr(out))
    return out


def gemv(wtype: int, W: np.ndarray, X: np.ndarray, N: int, window=None):
    """Y[m][n] = sum_k X[m][k] W[n][k] in float64; returns (Y, S) over the window."""
    W, X = _u8(W), np.ascontiguousarray(X, dtype=np.float32)
    M, K = X.shape
    m0, m1, n0, n1 = _window(M, N, window)
    Y = np.empty((m1 - m0, n1 - n0), dtype=np.float64)
    S = np.empty_like(Y)
    _load().ora_gemv(wtype, M, N, K, _ptr(W), _ptr(X), m0, m1, n0, n1, _ptr(Y), _ptr(S))
    return Y, S


def quantize_act_q8(X: np.ndarray):
    """Per-32-block Q8 quantisation in binary32; returns (QX int8[M,K], DX float32[M,K/32])."""
    X = np.ascontiguousarray(X, dtype=np.float32)
    M, K = X.shape
    QX = np.empty((M, K), dtype=np.int8)
    DX = np.empty((M, K // BLOCK), dtype=np.float32)
    _load().ora_quantize_act_q8(M, K, _ptr(X), _ptr(QX), _ptr(DX))
    return QX, DX


def float_to_half_bits(f: float) -> int:
    """binary32 -> binary16 bits, round to nearest even."""
    return int(_load().ora_float_to_half_rne(float(np.float32(f))))


def quantize_act_q8_0(X: np.ndarray) -> np.ndarray:
    """Activations as Q8_0 blocks with an fp16 scale (ggml rule); uint8[M, K/32*34]."""
    X = np.ascontiguousarray(X, dtype=np.float32)
    M, K = X.shape
    XB = np.empty((M, (K // BLOCK) * 34), dtype=np.uint8)
    _load().ora_quantize_act_q8_0(M, K, _ptr(X), _ptr(XB))
    return XB


def split_q8_0_blocks(XB: np.ndarray, K: int):
    """Q8_0 activation blocks -> (codes int8[M, K], scales float32[M, K/32] = the fp16 scales)."""
    XB = np.ascontiguousarray(XB, dtype=np.uint8)
    M = XB.shape[0]
    kb = K // BLOCK
    blk = XB.reshape(M, kb, 34)
    codes = blk[:, :, 2:].copy().view(np.int8).reshape(M, K)
    dbits = blk[:, :, 0].astype(np.uint16) | (blk[:, :, 1].astype(np.uint16) << 8)
    scales = np.array([[half_to_double(int(b)) for b in row] for row in dbits], dtype=np.float32).reshape(M, kb)
    return codes, scales


def q8q8_block_dots(W: np.ndarray, QX: np.ndarray, N: int, window=None) -> np.ndarray:
    """Exact int32 block dots isum[m][n][b] over the window."""
    W, QX = _u8(W), np.ascontiguousarray(QX, dtype=np.int8)
    M, K = QX.shape
    m0, m1, n0, n1 = _window(M, N, window)
    out = np.empty((m1 - m0, n1 - n0, K // BLOCK), dtype=np.int32)
    bad = _load().ora_q8q8_block_dots(M, N, K, _ptr(W), _ptr(QX), m0, m1, n0, n1, _ptr(out))
    assert bad == 0, "block dot outside int32"
    return out


def q8q8_gemv(W: np.ndarray, QX: np.ndarray, DX: np.ndarray, N: int, window=None):
    W, QX = _u8(W), np.ascontiguousarray(QX, dtype=np.int8)
    DX = np.ascontiguousarray(DX, dtype=np.float32)
    M, K = QX.shape
    m0, m1, n0, n1 = _window(M, N, window)
    Y = np.empty((m1 - m0, n1 - n0), dtype=np.float64)
    S = np.empty_like(Y)
    _load().ora_q8q8_gemv(M, N, K, _ptr(W), _ptr(QX), _ptr(DX), m0, m1, n0, n1, _ptr(Y), _ptr(S))
    return Y, S


def swiglu(wtype: int, Wg: np.ndarray, Wu: np.ndarray, X: np.ndarray, N: int, window=None):
    """out = silu(x.Wg) * (x.Wu); returns dict with out, g, u, Sg, Su (float64)."""
    Wg, Wu = _u8(Wg), _u8(Wu)
    X = np.ascontiguousarray(X, dtype=np.float32)
    M, K = X.shape
    m0, m1, n0, n1 = _window(M, N, window)
    shape = (m1 - m0, n1 - n0)
    r = {k: np.empty(shape, dtype=np.float64) for k in ("out", "g", "u", "Sg", "Su")}
    _load().ora_swiglu(wtype, M, N, K, _ptr(Wg), _ptr(Wu), _ptr(X), m0, m1, n0, n1,
                       _ptr(r["out"]), _ptr(r["g"]), _ptr(r["u"]), _ptr(r["Sg"]), _ptr(r["Su"]))
    return r


def prefill(wtype: int, W: np.ndarray, Xbf16: np.ndarray, N: int, window=None):
    """Y[m][n] = sum_k bf16(X[m][k]) W[n][k] in float64; returns (Y, S)."""
    W = _u8(W)
    Xb = np.ascontiguousarray(Xbf16, dtype=np.uint16)
    M, K = Xb.shape
    m0, m1, n0, n1 = _window(M, N, window)
    Y = np.empty((m1 - m0, n1 - n0), dtype=np.float64)
    S = np.empty_like(Y)
    _load().ora_prefill(wtype, M, N, K, _ptr(W), _ptr(Xb), m0, m1, n0, n1, _ptr(Y), _ptr(S))
    return Y, S
