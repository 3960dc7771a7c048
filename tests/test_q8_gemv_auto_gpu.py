"""qmm_q8_gemv_auto (per-K choice between the Q8xQ8 and the fp32-activation GEMV).

Short rows (K/32 <= 64) at M = 1 with a weight slice that fits on chip must
give exactly qmm_q8q8_gemv_fused's Y, codes and scales; every other shape
exactly qmm_q8_gemv_ex's Y with QX / DX left untouched. Both forms are also
checked against the oracle (the Q8xQ8 one on the oracle's own codes).
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic as syn
from parity import TOL_FP32, assert_within, dev, host

pytestmark = pytest.mark.gpu

qmm = pytest.importorskip("decode_gemv_qmm_b200")


def same(a, b):
    return torch.equal(a.view(torch.int32), b.view(torch.int32))


@pytest.mark.parametrize("n,k", [(4864, 896), (1152, 896), (896, 896), (64, 2048)])
def test_auto_short_k_is_fused_q8q8(n, k):
    g = syn.rng(n + k)
    W = syn.q8_0_weights(g, n, k)[0]
    x = syn.act_f32(g, 1, k)
    Wd, Xd = dev(W), dev(x)
    Y, QX, DX = qmm.qmm_q8_gemv_auto(Wd, Xd, n, flags=qmm.QMM_FLAG_EARLY_WEIGHTS)
    Yf, QXf, DXf = qmm.qmm_q8q8_gemv_fused(Wd, Xd, n, flags=qmm.QMM_FLAG_EARLY_WEIGHTS)
    torch.cuda.synchronize()
    assert same(Y, Yf) and torch.equal(QX, QXf) and same(DX, DXf)
    qr, dr = oracle.quantize_act_q8(x)
    ref, S = oracle.q8q8_gemv(W, qr, dr, n)
    assert_within(host(Y), ref, S, TOL_FP32, f"auto Q8xQ8 N={n} K={k}")


@pytest.mark.parametrize("m,n,k", [(1, 896, 4864), (1, 151936, 896), (2, 300, 896), (1, 64, 2080)])
def test_auto_otherwise_is_fp32_gemv(m, n, k):
    g = syn.rng(7 * n + k + m)
    W = syn.q8_0_weights(g, n, k)[0]
    x = syn.act_f32(g, m, k)
    Wd, Xd = dev(W), dev(x)
    QX = torch.full((m, k), 5, dtype=torch.int8, device="cuda")
    DX = torch.full((m, k // 32), 2.5, device="cuda")
    Y, _, _ = qmm.qmm_q8_gemv_auto(Wd, Xd, n, QX=QX, DX=DX)
    Yr = qmm.qmm_q8_gemv(Wd, Xd, n)
    torch.cuda.synchronize()
    assert same(Y, Yr)
    assert int((QX != 5).sum()) == 0 and bool((DX == 2.5).all())
    ref, S = oracle.gemv(syn.Q8_0, W, x, n, window=(0, m, 0, min(n, 2048)))
    assert_within(host(Y)[:, :min(n, 2048)], ref, S, TOL_FP32, f"auto fp32 M={m} N={n} K={k}")
    assert qmm.device_status() == 0
