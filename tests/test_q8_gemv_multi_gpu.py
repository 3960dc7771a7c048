"""qmm_q8_gemv_multi (several projections of one activation vector in one launch) against the CPU oracle.

Every projection must lie within 1e-5 * sum_k |w_k x_k| of the oracle's GEMV of
its own matrix. Cases cover the one-launch form (M = 1, K <= 2048: the row
chunks of all matrices in one work list, including chunks that end a matrix
mid-chunk and empty projections) and the per-projection fallback (M > 1, long K).
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic as syn
from parity import TOL_FP32, assert_within, dev, host

pytestmark = pytest.mark.gpu

qmm = pytest.importorskip("decode_gemv_qmm_b200")


def check(m, ns, k, seed, flags=0):
    g = syn.rng(seed)
    Ws = [syn.q8_0_weights(g, n, k)[0] if n > 0 else np.zeros(0, np.uint8) for n in ns]
    x = syn.act_f32(g, m, k)
    Ys = qmm.qmm_q8_gemv_multi([dev(w) if n > 0 else None for w, n in zip(Ws, ns)], dev(x), ns, flags=flags)
    torch.cuda.synchronize()
    for i, (W, n) in enumerate(zip(Ws, ns)):
        if n == 0:
            continue
        ref, S = oracle.gemv(syn.Q8_0, W, x, n)
        assert_within(host(Ys[i]), ref, S, TOL_FP32, f"multi M={m} K={k} projection {i} N={n}")
    assert qmm.device_status() == 0
    return Ws, x, Ys


@pytest.mark.parametrize("m,ns,k", [
    (1, [4864, 4864], 896),            # gate and up of the decode step
    (1, [1152, 896, 4864], 896),       # three projections of one x
    (1, [37, 1000, 5, 64], 256),       # ragged: projections end mid-chunk
    (1, [300, 0, 17], 96),             # an empty projection
    (1, [1, 1], 32),                   # fewer chunks than CTAs
    (1, [2000, 1500], 2048),           # 16-row chunks (K > 1024)
    (1, [300, 200], 4864),             # long K: one launch per projection
    (2, [77, 129], 192),               # M > 1: one launch per projection
    (8, [64, 33, 5], 1024),
])
def test_multi_matches_oracle(m, ns, k):
    check(m, ns, k, seed=sum(ns) + 3 * k + m)


def test_multi_early_weights_flag_same_bits():
    g = syn.rng(11)
    ns, k = [4864, 4864], 896
    Ws = [dev(syn.q8_0_weights(g, n, k)[0]) for n in ns]
    x = dev(syn.act_f32(g, 1, k))
    Y0 = qmm.qmm_q8_gemv_multi(Ws, x, ns)
    Y1 = qmm.qmm_q8_gemv_multi(Ws, x, ns, flags=qmm.QMM_FLAG_EARLY_WEIGHTS)
    torch.cuda.synchronize()
    for a, b in zip(Y0, Y1):
        assert torch.equal(a.view(torch.int32), b.view(torch.int32))


def test_multi_single_projection_equals_gemv_bitwise():
    """One large projection runs the same kernel, partition and arithmetic as qmm_q8_gemv."""
    g = syn.rng(12)
    n, k = 151936, 896
    W = dev(syn.q8_0_weights(g, n, k)[0])
    x = dev(syn.act_f32(g, 1, k))
    (Ym,) = qmm.qmm_q8_gemv_multi([W], x, [n])
    Ys = qmm.qmm_q8_gemv(W, x, n)
    torch.cuda.synchronize()
    assert torch.equal(Ym.view(torch.int32), Ys.view(torch.int32))


def test_multi_projection_outputs_independent_of_grouping():
    """A projection's outputs do not depend on which other projections share the launch."""
    g = syn.rng(13)
    k = 896
    Wa = dev(syn.q8_0_weights(g, 4864, k)[0])
    Wb = dev(syn.q8_0_weights(g, 4864, k)[0])
    Wc = dev(syn.q8_0_weights(g, 1152, k)[0])
    x = dev(syn.act_f32(g, 1, k))
    ya, yb = qmm.qmm_q8_gemv_multi([Wa, Wb], x, [4864, 4864])
    yc, ya2, yb2 = qmm.qmm_q8_gemv_multi([Wc, Wa, Wb], x, [1152, 4864, 4864])
    torch.cuda.synchronize()
    assert torch.equal(ya.view(torch.int32), ya2.view(torch.int32))
    assert torch.equal(yb.view(torch.int32), yb2.view(torch.int32))
