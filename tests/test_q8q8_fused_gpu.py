"""qmm_q8q8_gemv_fused (activation quantisation inside the Q8xQ8 GEMV) against the CPU oracle.

The codes and scales it writes must equal the oracle's quantisation of X bit
for bit (and so those of qmm_quantize_act_q8); Y must lie within
1e-5 * sum_b |d_w d_x| sum_j |q_w q_x| of the oracle's Q8xQ8 GEMV on those
codes. Shapes cover the in-CTA resident form (M = 1, slices that fit), the
quantise-then-stream form (M > 1, large N), ragged row counts and the
degenerate blocks of the quantisation (all zero, halfway cases, extremes).
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic as syn
from parity import TOL_FP32, assert_within, dev, host

pytestmark = pytest.mark.gpu

qmm = pytest.importorskip("decode_gemv_qmm_b200")


def check(W, x, n, flags=0, label=""):
    Y, QX, DX = qmm.qmm_q8q8_gemv_fused(dev(W), dev(x), n, flags=flags)
    torch.cuda.synchronize()
    qr, dr = oracle.quantize_act_q8(x)
    assert np.array_equal(host(DX).view(np.uint32), dr.view(np.uint32)), f"{label}: activation scales differ"
    assert np.array_equal(host(QX), qr), f"{label}: {int((host(QX) != qr).sum())} activation codes differ"
    ref, S = oracle.q8q8_gemv(W, qr, dr, n)
    assert_within(host(Y), ref, S, TOL_FP32, label)
    assert qmm.device_status() == 0
    return host(Y)


@pytest.mark.parametrize("m,n,k", [
    (1, 4864, 896), (1, 896, 4864),          # the decode projections of the Q8xQ8 workload
    (1, 37, 256), (1, 5, 64), (1, 1, 32),     # fewer rows than CTAs
    (1, 2000, 2048), (1, 300, 8192),          # several 32-column windows per row
    (1, 1185, 896), (1, 4861, 896),           # ragged row splits
    (1, 151936, 896),                         # slice too large: quantise then stream
    (2, 77, 192), (8, 129, 2048), (4, 3, 32), # M > 1
])
def test_fused_matches_oracle(m, n, k):
    g = syn.rng(5 * n + 3 * k + m)
    W, _, _ = syn.q8_0_weights(g, n, k)
    x = syn.act_f32(g, m, k)
    check(W, x, n, label=f"fused M={m} N={n} K={k}")


@pytest.mark.parametrize("n,k", [(4864, 896), (896, 4864), (64, 1024)])
def test_fused_degenerate_blocks(n, k):
    g = syn.rng(n ^ k)
    W, _, _ = syn.q8_0_weights(g, n, k, qlo=-128, qhi=127)
    x = syn.act_f32(g, 1, k)
    x[0, :32] = 0.0                                                     # d = 0: all-zero codes
    x[0, 32:64] = np.arange(-16, 16, dtype=np.float32) + 0.5            # halfway cases
    x[0, 32] = 127.0
    x[0, 64:96] = np.float32(1e-30) * np.arange(1, 33, dtype=np.float32)  # tiny block
    x[0, 96:128] = -3.0e30                                              # large, equal magnitudes
    x[0, -32:] = np.float32(-1.0)
    x[0, -1] = np.float32(1.0)
    check(W, x, n, label=f"degenerate N={n} K={k}")


@pytest.mark.parametrize("n,k", [(4864, 896), (896, 4864)])
def test_fused_matches_two_step_codes_and_flag(n, k):
    """Same codes as qmm_quantize_act_q8; same Y with and without early weights."""
    g = syn.rng(n + 17 * k)
    W, _, _ = syn.q8_0_weights(g, n, k)
    x = dev(syn.act_f32(g, 1, k))
    Wd = dev(W)
    QX0, DX0 = qmm.qmm_quantize_act_q8(x)
    Y0 = qmm.qmm_q8q8_gemv(Wd, QX0, DX0, n)
    Y1, QX1, DX1 = qmm.qmm_q8q8_gemv_fused(Wd, x, n)
    Y2, _, _ = qmm.qmm_q8q8_gemv_fused(Wd, x, n, flags=qmm.QMM_FLAG_EARLY_WEIGHTS)
    torch.cuda.synchronize()
    assert torch.equal(QX0, QX1) and torch.equal(DX0.view(torch.int32), DX1.view(torch.int32))
    assert np.array_equal(host(Y1).view(np.uint32), host(Y2).view(np.uint32))
    qx, dx = host(QX0), host(DX0)
    ref, S = oracle.q8q8_gemv(W, qx, dx, n)
    assert_within(host(Y0), ref, S, TOL_FP32, "two-step")
    assert_within(host(Y1), ref, S, TOL_FP32, "fused")
    assert qmm.device_status() == 0


def test_fused_chained_calls():
    """Each call's X is the previous call's Y (dependent launches back to back)."""
    g = syn.rng(2024)
    k0, n0 = 896, 4864
    W0, _, _ = syn.q8_0_weights(g, n0, k0)
    W1, _, _ = syn.q8_0_weights(g, k0, n0)
    x = syn.act_f32(g, 1, k0)
    W0d, W1d = dev(W0), dev(W1)
    Xd = dev(x)
    outs = []
    for _ in range(3):
        H, QH0, DH0 = qmm.qmm_q8q8_gemv_fused(W0d, Xd, n0)
        Xd, QH1, DH1 = qmm.qmm_q8q8_gemv_fused(W1d, H, k0, flags=qmm.QMM_FLAG_EARLY_WEIGHTS)
        outs.append((H.clone(), QH0.clone(), DH0.clone(), Xd.clone(), QH1.clone(), DH1.clone()))
    torch.cuda.synchronize()
    xin = x
    for H, QH0, DH0, Xo, QH1, DH1 in outs:
        q0, d0 = oracle.quantize_act_q8(xin)
        assert np.array_equal(host(QH0), q0) and np.array_equal(host(DH0).view(np.uint32), d0.view(np.uint32))
        ref0, S0 = oracle.q8q8_gemv(W0, q0, d0, n0)
        assert_within(host(H), ref0, S0, TOL_FP32, "chain step 1")
        h = host(H)
        q1, d1 = oracle.quantize_act_q8(h)
        assert np.array_equal(host(QH1), q1) and np.array_equal(host(DH1).view(np.uint32), d1.view(np.uint32))
        ref1, S1 = oracle.q8q8_gemv(W1, q1, d1, k0)
        assert_within(host(Xo), ref1, S1, TOL_FP32, "chain step 2")
        xin = host(Xo)
    assert qmm.device_status() == 0


def test_fused_empty_and_zero_k():
    W = torch.zeros(0, dtype=torch.uint8, device="cuda")
    x = torch.zeros(1, 0, dtype=torch.float32, device="cuda")
    Y = torch.full((1, 7), 5.0, device="cuda")
    qx = torch.zeros(1, 0, dtype=torch.int8, device="cuda")
    dx = torch.zeros(1, 0, dtype=torch.float32, device="cuda")
    qmm.qmm_q8q8_gemv_fused(W, x, 7, Y=Y, QX=qx, DX=dx)
    torch.cuda.synchronize()
    assert torch.count_nonzero(Y).item() == 0
    g = syn.rng(1)
    W2, _, _ = syn.q8_0_weights(g, 4, 64)
    x2 = dev(syn.act_f32(g, 1, 64))
    Y0, _, _ = qmm.qmm_q8q8_gemv_fused(dev(W2), x2, 0)
    assert Y0.shape == (1, 0)
    assert qmm.device_status() == 0


@pytest.mark.parametrize("m,n,k", [
    (1, 4864, 896), (1, 896, 4864),           # the two Q8xQ8 decode shapes, resident kernel
    (1, 1185, 896), (1, 37, 256),              # ragged splits, fewer rows than CTAs
    (1, 151936, 896), (3, 129, 2048),          # quantise-then-stream forms
])
def test_fused_block_dots_bit_exact(m, n, k):
    """The int32 block dots of the fused Q8xQ8 path (the kernel qmm_q8q8_gemv_fused
    runs, in its dump instance) equal the oracle's exact dots on the oracle's
    codes; Y, QX and DX equal qmm_q8q8_gemv_fused's bit for bit."""
    g = syn.rng(11 * n + k + m)
    W, _, _ = syn.q8_0_weights(g, n, k, qlo=-128, qhi=127)
    x = syn.act_f32(g, m, k)
    x[0, :32] = np.float32(-2.5)                              # equal magnitudes: codes of +-127
    Y, QX, DX, isum = qmm.qmm_q8q8_gemv_fused_dots(dev(W), dev(x), n)
    Yf, QXf, DXf = qmm.qmm_q8q8_gemv_fused(dev(W), dev(x), n)
    torch.cuda.synchronize()
    qr, dr = oracle.quantize_act_q8(x)
    assert np.array_equal(host(QX), qr) and np.array_equal(host(DX).view(np.uint32), dr.view(np.uint32))
    win = (0, m, 0, min(n, 8192))
    ref = oracle.q8q8_block_dots(W, qr, n, window=win)
    got = host(isum)[:, :win[3], :]
    assert got.shape == ref.shape
    bad = int((got != ref).sum())
    assert bad == 0, f"{bad} of {ref.size} block dots differ"
    assert torch.equal(Y.view(torch.int32), Yf.view(torch.int32))
    assert torch.equal(QX, QXf) and torch.equal(DX.view(torch.int32), DXf.view(torch.int32))
    assert qmm.device_status() == 0
