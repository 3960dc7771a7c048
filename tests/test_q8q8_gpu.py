"""qmm_quantize_act_q8, qmm_q8q8_block_dots and qmm_q8q8_gemv against the CPU oracle.

Activation codes, scales and int32 block dots must match bit for bit; the
scaled fp32 output within 1e-5 * sum_b |d_w d_x| sum_j |q_w q_x| (the norm
against the quantised activations, which is what the method computes with).
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import synthetic as syn
from parity import TOL_FP32, assert_within, dev, host

pytestmark = pytest.mark.gpu

qmm = pytest.importorskip("decode_gemv_qmm_b200")
GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_blocks.json")


def quantize_gpu(x):
    QX, DX = qmm.qmm_quantize_act_q8(dev(x))
    torch.cuda.synchronize()
    return host(QX), host(DX)


@pytest.mark.parametrize("m,k,scale", [(1, 896, 1.0), (1, 4864, 1.0), (8, 5120, 1.0), (3, 96, 1e-30),
                                       (2, 64, 1e30), (64, 4864, 3.0), (1, 32, 1.0), (5, 32768, 1.0)])
def test_quantize_bit_exact(m, k, scale):
    g = syn.rng(m * 31 + k)
    x = syn.act_f32(g, m, k, scale=scale)
    x[0, :32] = 0.0                      # an all-zero block
    if k >= 64:
        x[0, 32:64] = np.arange(-16, 16, dtype=np.float32) + 0.5   # halfway cases
        x[0, 32] = 127.0
    q, d = quantize_gpu(x)
    qr, dr = oracle.quantize_act_q8(x)
    assert np.array_equal(d.view(np.uint32), dr.view(np.uint32)), "activation scales differ"
    assert np.array_equal(q, qr), f"{int((q != qr).sum())} activation codes differ"


def test_quantize_hand_cases():
    with open(GOLDEN) as f:
        cases = json.load(f)["quantize"]
    for c in cases:
        x = np.array(c["x"], dtype=np.float32)[None, :]
        q, d = quantize_gpu(x)
        assert d[0, 0] == np.float32(c["d"]) and q[0].tolist() == c["q"], c["name"]


@pytest.mark.parametrize("m,n,k", [(1, 4864, 896), (1, 896, 4864), (3, 37, 160), (8, 64, 1024), (1, 1, 32),
                                   (2, 300, 96), (7, 5, 32768)])
def test_block_dots_bit_exact(m, n, k):
    g = syn.rng(n + k + m)
    W, _, _ = syn.q8_0_weights(g, n, k, qlo=-128, qhi=127)
    qx = g.integers(-128, 128, size=(m, k)).astype(np.int8)
    isum = qmm.qmm_q8q8_block_dots(dev(W), dev(qx), n)
    torch.cuda.synchronize()
    ref = oracle.q8q8_block_dots(W, qx, n)
    assert np.array_equal(host(isum), ref)


def test_block_dots_extremes():
    with open(GOLDEN) as f:
        cases = json.load(f)["q8q8_dots"]
    for c in cases:
        W = syn.pack_q8_0(np.array([c["wq"]], np.int8), np.array([[0x3C00]], np.uint16))
        isum = qmm.qmm_q8q8_block_dots(dev(W), dev(np.array([c["xq"]], np.int8)), 1)
        torch.cuda.synchronize()
        assert int(host(isum)[0, 0, 0]) == c["isum"], c["name"]


@pytest.mark.parametrize("m,n,k", [(1, 4864, 896), (1, 896, 4864), (2, 77, 192), (8, 129, 2048),
                                   (1, 151936, 896), (4, 3, 32)])
def test_q8q8_gemv(m, n, k):
    g = syn.rng(7 * n + k)
    W, _, _ = syn.q8_0_weights(g, n, k)
    x = syn.act_f32(g, m, k)
    qx, dx = oracle.quantize_act_q8(x)
    Y = qmm.qmm_q8q8_gemv(dev(W), dev(qx), dev(dx), n)
    torch.cuda.synchronize()
    ref, S = oracle.q8q8_gemv(W, qx, dx, n)
    assert_within(host(Y), ref, S, TOL_FP32, f"q8q8 M={m} N={n} K={k}")


def test_quantize_then_q8q8_pipeline_and_flag():
    g = syn.rng(99)
    n, k = 4864, 896
    W, _, _ = syn.q8_0_weights(g, n, k)
    x = syn.act_f32(g, 1, k)
    Wd = dev(W)
    QX, DX = qmm.qmm_quantize_act_q8(dev(x))
    Y0 = qmm.qmm_q8q8_gemv(Wd, QX, DX, n)
    Y1 = qmm.qmm_q8q8_gemv(Wd, QX, DX, n, flags=qmm.QMM_FLAG_EARLY_WEIGHTS)
    torch.cuda.synchronize()
    qx, dx = oracle.quantize_act_q8(x)
    ref, S = oracle.q8q8_gemv(W, qx, dx, n)
    assert_within(host(Y0), ref, S, TOL_FP32, "quantize -> q8q8")
    assert np.array_equal(host(Y0).view(np.uint32), host(Y1).view(np.uint32))
    assert qmm.device_status() == 0
