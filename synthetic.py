"""Seeded synthetic inputs for the block-quantized matmul library.

This module only draws random numbers and lays them out in the ggml-style block
byte format; it performs none of the matmul, quantisation or activation
arithmetic. Both the CPU oracle tests and the GPU tests/benchmark take their
inputs from here, so the two sides always see identical bytes.

Block formats (ggml style; the Lumen v0.2.0 release notes, "Phase 7.D --
Q8-native fused matmul", keep weights in this native block layout end to end):

* Q8_0: 34 bytes per 32 weights = fp16 scale ``d`` (little-endian) followed by
  32 signed int8 codes ``qs``; weight j of the block is ``qs[j] * d``.
* Q4_0: 18 bytes per 32 weights = fp16 scale ``d`` followed by 16 bytes ``qs``;
  weight j (j < 16) is the low nibble of ``qs[j]``, weight j + 16 the high
  nibble of ``qs[j]``; the value is ``(nibble - 8) * d``.

A weight matrix is N rows (output features) of K/32 blocks each, row-major,
blocks of one row contiguous (K is the contiguous direction).

Distributions (all from ``numpy.random.default_rng``):
* Q8_0 codes uniform in [-127, 127], scale ``fp16(|N(0,1)| * 0.02)``;
* Q4_0 nibbles uniform in [0, 15], scale ``fp16(|N(0,1)| * 0.01)``;
* fp32 activations N(0,1); bf16 activations ``bf16_rne(N(0,1))``.
"""
from __future__ import annotations

import numpy as np

BLOCK = 32
Q8_0_BYTES = 34
Q4_0_BYTES = 18
Q8_0, Q4_0 = 0, 1
BLOCK_BYTES = {Q8_0: Q8_0_BYTES, Q4_0: Q4_0_BYTES}

Q8_0_DTYPE = np.dtype([("d", "<u2"), ("qs", "i1", (32,))])
Q4_0_DTYPE = np.dtype([("d", "<u2"), ("qs", "u1", (16,))])
assert Q8_0_DTYPE.itemsize == Q8_0_BYTES and Q4_0_DTYPE.itemsize == Q4_0_BYTES


def rng(seed: int) -> np.random.Generator:
    return np.random.default_rng(seed)


def fp16_bits(values) -> np.ndarray:
    """fp16 bit patterns (uint16) of ``values`` rounded by numpy's float16 cast."""
    return np.asarray(values, dtype=np.float32).astype(np.float16).view(np.uint16)


def pack_q8_0(q: np.ndarray, d_bits: np.ndarray) -> np.ndarray:
    """Lay out int8 codes q[N, K] and fp16 scale bits d_bits[N, K/32] as Q8_0 bytes[N, K/32*34]."""
    n, k = q.shape
    kb = k // BLOCK
    assert k % BLOCK == 0 and d_bits.shape == (n, kb)
    blk = np.empty((n, kb), dtype=Q8_0_DTYPE)
    blk["d"] = d_bits
    blk["qs"] = q.astype(np.int8).reshape(n, kb, BLOCK)
    return blk.view(np.uint8).reshape(n, kb * Q8_0_BYTES)


def pack_q4_0(nib: np.ndarray, d_bits: np.ndarray) -> np.ndarray:
    """Lay out nibbles nib[N, K] (0..15) and fp16 scale bits as Q4_0 bytes[N, K/32*18]."""
    n, k = nib.shape
    kb = k // BLOCK
    assert k % BLOCK == 0 and d_bits.shape == (n, kb)
    nb = nib.astype(np.uint8).reshape(n, kb, BLOCK)
    assert int(nb.max(initial=0)) <= 15
    blk = np.empty((n, kb), dtype=Q4_0_DTYPE)
    blk["d"] = d_bits
    blk["qs"] = nb[:, :, :16] | (nb[:, :, 16:] << 4)
    return blk.view(np.uint8).reshape(n, kb * Q4_0_BYTES)


def q8_0_weights(g: np.random.Generator, n: int, k: int, dscale: float = 0.02,
                 qlo: int = -127, qhi: int = 127):
    """Random Q8_0 matrix. Returns (bytes[N, K/32*34], codes int8[N, K], d_bits uint16[N, K/32])."""
    q = g.integers(qlo, qhi + 1, size=(n, k), dtype=np.int16).astype(np.int8)
    d_bits = fp16_bits(np.abs(g.standard_normal((n, k // BLOCK))) * dscale)
    return pack_q8_0(q, d_bits), q, d_bits


def q4_0_weights(g: np.random.Generator, n: int, k: int, dscale: float = 0.01):
    """Random Q4_0 matrix. Returns (bytes[N, K/32*18], nibbles uint8[N, K], d_bits uint16[N, K/32])."""
    nib = g.integers(0, 16, size=(n, k), dtype=np.uint8)
    d_bits = fp16_bits(np.abs(g.standard_normal((n, k // BLOCK))) * dscale)
    return pack_q4_0(nib, d_bits), nib, d_bits


def weights(g: np.random.Generator, wtype: int, n: int, k: int):
    """Random weights of either type with the standard distributions; returns the packed bytes."""
    if wtype == Q8_0:
        return q8_0_weights(g, n, k)[0]
    return q4_0_weights(g, n, k)[0]


def act_f32(g: np.random.Generator, m: int, k: int, scale: float = 1.0) -> np.ndarray:
    return (g.standard_normal((m, k)) * scale).astype(np.float32)


def act_bf16_bits(g: np.random.Generator, m: int, k: int) -> np.ndarray:
    """bf16 bit patterns (uint16[M, K]) of N(0,1) samples rounded to nearest even."""
    import torch  # bf16 rounding of the generated samples only
    x = torch.from_numpy(g.standard_normal((m, k)).astype(np.float32))
    return x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()


# --- workload descriptions -------------------------------------------------

#: one transformer layer of a Qwen2.5-0.5B-shaped decoder: (name, N out, K in)
QWEN05B_LAYER = (("qkv", 1152, 896), ("wo", 896, 896), ("gate", 4864, 896),
                 ("up", 4864, 896), ("down", 896, 4864))
QWEN05B_LAYERS = 24
QWEN05B_LM_HEAD = ("lm_head", 151936, 896)


def decode_step_shapes():
    """The 121 weight matmuls of one M=1 decode step, in stream order."""
    out = []
    for layer in range(QWEN05B_LAYERS):
        for name, n, k in QWEN05B_LAYER:
            out.append((f"L{layer}.{name}", n, k))
    out.append(QWEN05B_LM_HEAD)
    return out


def sub_seed(seed: int, index: int) -> int:
    """Per-tensor seed of tensor ``index`` of a workload drawn with ``seed``."""
    return seed * 1000 + index


def decode_step_sources():
    """Data flow of the decode step's matmuls: for each of the 121, the index of
    the matmul whose output holds its input (-1: the step's input vector).
    qkv reads the previous layer's down output, wo reads (the first 896 values
    of) qkv, gate and up both read wo, down reads up, lm_head the last down."""
    shapes = decode_step_shapes()
    src = []
    last_down = -1
    for i, (name, _, _) in enumerate(shapes):
        kind = name.split(".")[-1]
        if kind == "qkv" or kind == "lm_head":
            src.append(last_down)
        elif kind == "wo":
            src.append(i - 1)
        elif kind in ("gate", "up"):
            src.append(i - 1 if kind == "gate" else i - 2)
        elif kind == "down":
            src.append(i - 1)
            last_down = i
        else:
            raise ValueError(name)
    return src


def chain_dscale(k: int) -> float:
    """Scale factor c of Q8_0 scales d = |N(0,1)| c for a chained decode step:
    with codes uniform in [-127, 127] (rms about 73.6) an output of a K-long
    row then has about the rms of its input, so 121 chained matmuls neither
    overflow nor vanish."""
    return 1.0 / (73.6 * float(np.sqrt(k)))
