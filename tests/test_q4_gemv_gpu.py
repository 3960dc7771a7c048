"""qmm_q4_gemv (decode GEMV / small-M matmul on Q4_0 blocks) against the CPU oracle.

Outputs must lie within 1e-5 * sum_k |w_k x_k| of the oracle, and equal the
gate projection of qmm_q4_gateup_unfused bit for bit (same kernel, one matrix).
Shapes cover M = 1 and M = 8, the down projection of the gate/up workload
(K = 17408, N = 5120), ragged rows, and K that is not a multiple of 256 (the
kernel's direct-load path).
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic as syn
from parity import TOL_FP32, assert_within, dev, host, oracle_parallel

pytestmark = pytest.mark.gpu

qmm = pytest.importorskip("decode_gemv_qmm_b200")


def oracle_gemv(W, x, n):
    parts = oracle_parallel(lambda w, xx, N, window: oracle.gemv(syn.Q4_0, w, xx, N, window=window),
                            n, W, x, rows_per_job=512)
    return np.concatenate([p[0] for p in parts], axis=1), np.concatenate([p[1] for p in parts], axis=1)


def check(m, n, k, seed, flags=0):
    g = syn.rng(seed)
    W = syn.q4_0_weights(g, n, k)[0]
    x = syn.act_f32(g, m, k)
    Y = qmm.qmm_q4_gemv(dev(W), dev(x), n, flags=flags)
    torch.cuda.synchronize()
    ref, S = oracle_gemv(W, x, n)
    assert_within(host(Y), ref, S, TOL_FP32, f"q4_gemv M={m} N={n} K={k}")
    assert qmm.device_status() == 0
    return W, x, Y


@pytest.mark.parametrize("m,n,k", [
    (1, 17408, 5120),   # one projection of the gate/up workload, M = 1
    (8, 5120, 17408),   # its down projection at M = 8
    (1, 5120, 17408),
    (1, 16, 256), (3, 17, 512), (8, 33, 256), (5, 1000, 1024), (1, 4097, 2048),
    (1, 5, 32), (8, 40, 96), (4, 17, 288),   # K % 256 != 0: direct loads
])
def test_q4_gemv_matches_oracle(m, n, k):
    check(m, n, k, seed=m + 2 * n + 3 * k)


def test_q4_gemv_equals_unfused_projection_bitwise():
    g = syn.rng(21)
    m, n, k = 8, 4864, 2048
    Wg, Wu = syn.q4_0_weights(g, n, k)[0], syn.q4_0_weights(g, n, k)[0]
    x = dev(syn.act_f32(g, m, k))
    Wgd, Wud = dev(Wg), dev(Wu)
    G, U, _ = qmm.qmm_q4_gateup_unfused(Wgd, Wud, x, n)
    Yg = qmm.qmm_q4_gemv(Wgd, x, n)
    Yu = qmm.qmm_q4_gemv(Wud, x, n, flags=qmm.QMM_FLAG_EARLY_WEIGHTS)
    torch.cuda.synchronize()
    assert torch.equal(G.view(torch.int32), Yg.view(torch.int32))
    assert torch.equal(U.view(torch.int32), Yu.view(torch.int32))


def test_q4_gemv_empty_and_zero_k():
    Y = torch.full((2, 9), 3.0, device="cuda")
    qmm.qmm_q4_gemv(torch.zeros(0, dtype=torch.uint8, device="cuda"), torch.zeros(2, 0, device="cuda"), 9, Y=Y)
    torch.cuda.synchronize()
    assert torch.count_nonzero(Y).item() == 0
    assert qmm.qmm_q4_gemv(torch.zeros(16, dtype=torch.uint8, device="cuda"),
                           torch.zeros(1, 32, device="cuda"), 0).shape == (1, 0)
