"""qmm_quantize_act_q8_0 and qmm_q8q8_gemv_q8_0 (activations as ggml Q8_0 blocks) against the oracle.

The blocks written on the GPU (fp16 scale, 32 codes) must equal the oracle's
byte for byte; the GEMV on Q8_0 activation blocks must lie within
1e-5 * sum_b |d_w d_x| sum_j |q_w q_x| of the oracle's Q8xQ8 GEMV on the same
codes and scales, for blocks made on the GPU and for blocks made on the host.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic as syn
from parity import TOL_FP32, assert_within, dev, host

pytestmark = pytest.mark.gpu

qmm = pytest.importorskip("decode_gemv_qmm_b200")


@pytest.mark.parametrize("m,k,scale", [(1, 896, 1.0), (1, 4864, 1.0), (8, 5120, 1.0), (3, 96, 1e-3),
                                       (2, 64, 100.0), (5, 32768, 1.0), (1, 32, 1.0)])
def test_q8_0_blocks_bit_exact(m, k, scale):
    g = syn.rng(m * 13 + k)
    x = syn.act_f32(g, m, k, scale=scale)
    x[0, :32] = 0.0                                        # zero block: d = 0, codes 0
    if k >= 64:
        x[0, 32:64] = np.arange(-16, 16, dtype=np.float32) + 0.5
        x[0, 32] = 127.0                                   # d = 1: halfway codes round away from zero
    if k >= 128:
        x[0, 64:96] = np.float32(127.0 * 2.0 ** -20)       # fp16 subnormal scale
        x[0, 96:128] = np.float32(127.0 * (1 + 3 * 2.0 ** -11))  # scale rounds to even in fp16
    XB = qmm.qmm_quantize_act_q8_0(dev(x))
    torch.cuda.synchronize()
    ref = oracle.quantize_act_q8_0(x)
    got = host(XB)
    assert np.array_equal(got, ref), f"{int((got != ref).sum())} bytes differ"


@pytest.mark.parametrize("m,n,k", [(1, 4864, 896), (1, 896, 4864), (3, 37, 160), (8, 129, 2048), (4, 3, 32),
                                   (1, 151936, 896)])
def test_q8q8_gemv_on_q8_0_blocks(m, n, k):
    g = syn.rng(3 * n + k + m)
    W = syn.q8_0_weights(g, n, k)[0]
    x = syn.act_f32(g, m, k)
    xb = oracle.quantize_act_q8_0(x)                     # host-made blocks, e.g. from another library
    Y = qmm.qmm_q8q8_gemv_q8_0(dev(W), dev(xb), k, n)
    torch.cuda.synchronize()
    codes, scales = oracle.split_q8_0_blocks(xb, k)
    win = (0, m, 0, min(n, 4096))
    ref, S = oracle.q8q8_gemv(W, codes, scales, n, window=win)
    assert_within(host(Y)[:, :win[3]], ref, S, TOL_FP32, f"q8q8 on Q8_0 blocks M={m} N={n} K={k}")
    assert qmm.device_status() == 0


def test_quantize_then_gemv_chain_and_flag():
    g = syn.rng(77)
    n, k = 4864, 896
    W = dev(syn.q8_0_weights(g, n, k)[0])
    x = syn.act_f32(g, 1, k)
    XB = qmm.qmm_quantize_act_q8_0(dev(x))
    Y0 = qmm.qmm_q8q8_gemv_q8_0(W, XB, k, n)
    Y1 = qmm.qmm_q8q8_gemv_q8_0(W, XB, k, n, flags=qmm.QMM_FLAG_EARLY_WEIGHTS)
    torch.cuda.synchronize()
    assert torch.equal(Y0.view(torch.int32), Y1.view(torch.int32))
    codes, scales = oracle.split_q8_0_blocks(oracle.quantize_act_q8_0(x), k)
    ref, S = oracle.q8q8_gemv(host(W), codes, scales, n)
    assert_within(host(Y0), ref, S, TOL_FP32, "quantize_act_q8_0 -> q8q8_gemv_q8_0")


@pytest.mark.parametrize("m,n,k", [(1, 4864, 896), (1, 896, 4864), (3, 37, 160), (8, 129, 2048)])
def test_q8_0_block_dots_bit_exact(m, n, k):
    """The int32 block dots of the GEMV on Q8_0 activation blocks equal the
    oracle's exact dots on the blocks' codes."""
    g = syn.rng(7 * n + k + m)
    W = syn.q8_0_weights(g, n, k, qlo=-128, qhi=127)[0]
    x = syn.act_f32(g, m, k)
    xb = oracle.quantize_act_q8_0(x)
    isum = qmm.qmm_q8q8_block_dots_q8_0(dev(W), dev(xb), k, n)
    torch.cuda.synchronize()
    codes, _ = oracle.split_q8_0_blocks(xb, k)
    ref = oracle.q8q8_block_dots(W, codes, n)
    got = host(isum)
    bad = int((got != ref).sum())
    assert bad == 0, f"{bad} of {ref.size} block dots differ"
    assert qmm.device_status() == 0
