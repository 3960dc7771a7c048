"""qmm_q4_gemv (decode GEMV / small-M matmul on Q4_0 blocks) against the CPU oracle.

Outputs must lie within 1e-5 * sum_k |w_k x_k| of the oracle. For M > 1 the
call is the gate/up kernel with one matrix and equals the gate projection of
qmm_q4_gateup_unfused bit for bit; M = 1 with K a multiple of 256 (up to the
shared-memory limit) runs the integer tensor-core GEMV instead (codes widened
to 16 (q - 8), activations as base-256 digits). Shapes cover M = 1 and M = 8,
the down projection of the gate/up workload (K = 17408, N = 5120), ragged
rows, and K that is not a multiple of 256 (the gate/up kernel's direct-load
path).
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
    (1, 3000, 768),     # M = 1 integer kernel: 32-row chunks, rows not padded (odd 16-byte count)
    (1, 2001, 4096),    # 16-row chunks, padded rows, ragged last chunk
    (1, 37, 7680),      # the longest K the integer kernel takes (one CTA per SM)
    (1, 1000, 8192),    # beyond it: the gate/up kernel with one matrix
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


def test_q4_gemv_m1_early_weights_same_bits_and_dynamic_range():
    g = syn.rng(22)
    n, k = 17408, 5120
    W = syn.q4_0_weights(g, n, k)[0]
    x = syn.act_f32(g, 1, k)
    Wd, xd = dev(W), dev(x)
    Y0 = qmm.qmm_q4_gemv(Wd, xd, n)
    Y1 = qmm.qmm_q4_gemv(Wd, xd, n, flags=qmm.QMM_FLAG_EARLY_WEIGHTS)
    torch.cuda.synchronize()
    assert torch.equal(Y0.view(torch.int32), Y1.view(torch.int32))
    n = 4096
    W = np.ascontiguousarray(W[:n])
    for name, scale in (("tiny", 1e-33), ("huge", 1e30), ("mixed", None)):
        xs = x * (10.0 ** g.uniform(-4, 4, size=x.shape)) if scale is None else x * scale
        xs = xs.astype(np.float32)
        Y = qmm.qmm_q4_gemv(dev(W), dev(xs), n)
        torch.cuda.synchronize()
        ref, S = oracle_gemv(W, xs, n)
        assert_within(host(Y), ref, S, TOL_FP32, f"q4_gemv M=1 x={name}")
    assert qmm.device_status() == 0
