"""Small-M prefill panels (M <= 32 tokens: the mma.sync kernel) against the CPU oracle.

This kernel multiplies the exact integer codes (bf16 holds every Q8 code and
every Q4 n - 8) by the bf16 activations and applies each block's scale in
fp32, so no decoded weight is rounded: its outputs must lie within the fp32
paths' bound 1e-5 * sum_k |w_k x_k| of the exact oracle, tighter than the
4e-3 that covers the tcgen05 path's bf16 weights. Shapes cover one to 32
tokens (partial token groups), ragged row groups, row pitches that are not a
multiple of 16 bytes, the last bytes of W (fetched without a 16-byte-wide
copy), split K over clusters, and the early-weights option.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic as syn
from parity import TOL_FP32, assert_within, dev, host, oracle_parallel

pytestmark = pytest.mark.gpu

qmm = pytest.importorskip("decode_gemv_qmm_b200")


def run(wtype, W, xb, n, flags=0):
    Y = qmm.qmm_quant_matmul_prefill(wtype, dev(W), dev(xb), n, flags=flags)
    torch.cuda.synchronize()
    assert qmm.device_status() == 0
    return host(Y)


def check(wtype, m, n, k, seed, W=None, xb=None):
    plan = qmm.qmm_prefill_plan(wtype, m, n, k)
    assert plan["kernel"] == "small_m", plan
    g = syn.rng(seed)
    W = syn.weights(g, wtype, n, k) if W is None else W
    xb = syn.act_bf16_bits(g, m, k) if xb is None else xb
    y = run(wtype, W, xb, n)
    parts = oracle_parallel(lambda a, b, N, window: oracle.prefill(wtype, a, b, N, window=window), n, W, xb,
                            rows_per_job=128)
    ref = np.concatenate([p[0] for p in parts], axis=1)
    S = np.concatenate([p[1] for p in parts], axis=1)
    assert_within(y, ref, S, TOL_FP32, f"small-M prefill wtype={wtype} M={m} N={n} K={k} plan={plan}")
    return plan


@pytest.mark.parametrize("wtype", [syn.Q8_0, syn.Q4_0])
@pytest.mark.parametrize("m,n,k", [
    (32, 4864, 896),   # the 32-token panel of the prefill workload (one K range per CTA)
    (32, 896, 4864),   # its long-K panel (K split over clusters)
    (1, 300, 256), (5, 77, 96), (8, 129, 512), (9, 64, 1024), (16, 1000, 288),
    (17, 5, 7200), (24, 2000, 160), (31, 3, 32), (32, 8191, 64),
])
def test_small_m_matches_oracle(wtype, m, n, k):
    check(wtype, m, n, k, seed=m * 131 + n + 7 * k)


@pytest.mark.parametrize("wtype", [syn.Q8_0, syn.Q4_0])
def test_small_m_extreme_codes_and_scales(wtype):
    """Codes at both ends of their range, zero and subnormal fp16 scales, and
    activations spanning many binades inside one block."""
    m, n, k = 12, 200, 512
    g = syn.rng(77 + wtype)
    if wtype == syn.Q8_0:
        W = syn.q8_0_weights(g, n, k, qlo=-128, qhi=127)[0]
        blocks = W.reshape(n, k // 32, 34)
        blocks[0, :, 2:] = np.uint8(0x80)                       # every code -128
        blocks[1, :, 0:2] = 0                                   # d = +0
        blocks[2, :, 0:2] = np.frombuffer(np.array([1], np.uint16).tobytes(), np.uint8)  # smallest subnormal d
    else:
        W = syn.q4_0_weights(g, n, k)[0]
        blocks = W.reshape(n, k // 32, 18)
        blocks[0, :, 2:] = np.uint8(0x00)                       # every nibble 0: value -8 d
        blocks[1, :, 0:2] = 0
        blocks[2, :, 2:] = np.uint8(0xFF)                       # every nibble 15: value 7 d
    xb = syn.act_bf16_bits(g, m, k)
    scales = (2.0 ** np.arange(-60, 60, 120 / 32)).astype(np.float32)[:32]
    xs = torch.from_numpy((np.tile(scales, k // 32)[None, :] * np.sign(g.standard_normal((m, k)))).astype(np.float32))
    xb[:4] = xs[:4].to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    check(wtype, m, n, k, seed=0, W=W, xb=xb)


@pytest.mark.parametrize("wtype,m,n,k", [(syn.Q8_0, 32, 4864, 896), (syn.Q8_0, 32, 896, 4864),
                                         (syn.Q4_0, 20, 333, 2048)])
def test_small_m_early_weights_and_repeat_same_bits(wtype, m, n, k):
    """Early weights only move the start of the weight copies; split K sums in
    rank order: every call gives the same bits."""
    g = syn.rng(m + n + k)
    W = dev(syn.weights(g, wtype, n, k))
    X = dev(syn.act_bf16_bits(g, m, k))
    Y0 = qmm.qmm_quant_matmul_prefill(wtype, W, X, n)
    Y1 = qmm.qmm_quant_matmul_prefill(wtype, W, X, n, flags=qmm.QMM_FLAG_EARLY_WEIGHTS)
    Y2 = qmm.qmm_quant_matmul_prefill(wtype, W, X, n)
    torch.cuda.synchronize()
    assert torch.equal(Y0.view(torch.int32), Y1.view(torch.int32))
    assert torch.equal(Y0.view(torch.int32), Y2.view(torch.int32))
    assert qmm.device_status() == 0


def test_small_m_chained_calls():
    """Dependent calls with early weights: each call's X is the previous call's
    Y rounded to bf16 (by torch on the device; the oracle side rounds the same
    values on the host), so a stale read of X or Y would show."""
    wtype, m, n, k = syn.Q8_0, 32, 896, 896
    g = syn.rng(4242)
    Ws = [syn.weights(g, wtype, n, k) for _ in range(3)]
    xb = syn.act_bf16_bits(g, m, k)
    Wd = [dev(w) for w in Ws]
    X = dev(xb)
    Ys = []
    for i in range(3):
        Y = qmm.qmm_quant_matmul_prefill(wtype, Wd[i], X, n, flags=qmm.QMM_FLAG_EARLY_WEIGHTS)
        Ys.append(Y)
        X = Y.to(torch.bfloat16).view(torch.int16)  # the next call's activations
    torch.cuda.synchronize()
    x = xb
    for i in range(3):
        ref, S = oracle.prefill(wtype, Ws[i], x, n)
        y = host(Ys[i])
        assert_within(y, ref, S, TOL_FP32, f"chain step {i}")
        x = torch.from_numpy(y.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert qmm.device_status() == 0
