"""qmm_q8_gemv (decode GEMV on Q8_0 blocks) against the CPU oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
import synthetic as syn
from parity import TOL_FP32, assert_within, dev, host

pytestmark = pytest.mark.gpu

qmm = pytest.importorskip("decode_gemv_qmm_b200")


def run(W, x, n, flags=0):
    Wd, Xd = dev(W), dev(x)
    Y = qmm.qmm_q8_gemv(Wd, Xd, n, flags=flags)
    torch.cuda.synchronize()
    return host(Y)


def check(m, n, k, seed, flags=0, wkw=None):
    g = syn.rng(seed)
    W, _, _ = syn.q8_0_weights(g, n, k, **(wkw or {}))
    x = syn.act_f32(g, m, k)
    y = run(W, x, n, flags)
    ref, S = oracle.gemv(syn.Q8_0, W, x, n)
    assert_within(y, ref, S, TOL_FP32, f"q8_gemv M={m} N={n} K={k}")
    return W, x, y


def test_single_gemv_qkv_shape_seed0():
    # M=1, K=896, N=1152 with the standard distributions, seed 0
    check(1, 1152, 896, seed=0)


@pytest.mark.parametrize("m,n,k", [
    (1, 1, 32), (1, 7, 64), (1, 33, 96), (2, 17, 96), (3, 5, 160), (4, 64, 1024), (5, 3, 2048),
    (8, 29, 896), (7, 40, 4864), (1, 300, 4864), (1, 149, 32), (2, 1, 32768), (1, 3, 32768),
    (1, 1000, 928), (6, 257, 1056), (8, 1, 32), (1, 4097, 64),
])
def test_shapes(m, n, k):
    check(m, n, k, seed=100 + m * 7 + n + k)


@pytest.mark.parametrize("name,n,k", [("qkv", 1152, 896), ("wo", 896, 896), ("gate_up", 4864, 896),
                                      ("down", 896, 4864), ("lm_head", 151936, 896)])
def test_decode_step_shapes_full(name, n, k):
    check(1, n, k, seed=7)


def test_extreme_codes_and_scales():
    g = syn.rng(3)
    n, k = 37, 256
    q = g.integers(-128, 128, size=(n, k)).astype(np.int8)
    q[0, :] = -128
    q[1, :] = 127
    d = syn.fp16_bits(np.abs(g.standard_normal((n, k // 32))) * 0.02)
    d[2, :] = 0x0000            # +0 scale
    d[3, :] = 0x8000            # -0 scale
    d[4, :] = 0x0001            # smallest subnormal
    d[5, :] = 0x03FF            # largest subnormal
    d[6, :] = 0x7BFF            # largest normal
    d[7, :] = 0xBC00            # -1.0
    W = syn.pack_q8_0(q, d)
    x = syn.act_f32(g, 3, k)
    y = run(W, x, n)
    ref, S = oracle.gemv(syn.Q8_0, W, x, n)
    assert_within(y, ref, S, TOL_FP32, "extreme codes/scales")
    assert np.all(y[:, 2] == 0) and np.all(y[:, 3] == 0)


def test_early_weights_flag_identical_and_deterministic():
    g = syn.rng(4)
    n, k = 4864, 896
    W, _, _ = syn.q8_0_weights(g, n, k)
    x = syn.act_f32(g, 1, k)
    y0 = run(W, x, n, flags=0)
    y1 = run(W, x, n, flags=qmm.QMM_FLAG_EARLY_WEIGHTS)
    y2 = run(W, x, n, flags=0)
    assert np.array_equal(y0.view(np.uint32), y1.view(np.uint32))
    assert np.array_equal(y0.view(np.uint32), y2.view(np.uint32))


def test_unaligned_row_starts_and_offset_buffers():
    # W and X placed at a 16-byte (not 256-byte) offset inside larger allocations
    g = syn.rng(5)
    n, k = 45, 896  # 952-byte rows: every other row starts 8 bytes off a 16-byte boundary
    W, _, _ = syn.q8_0_weights(g, n, k)
    x = syn.act_f32(g, 2, k)
    Wbuf = torch.zeros(W.size + 64, dtype=torch.uint8, device="cuda")
    Wbuf[16:16 + W.size] = dev(W.reshape(-1))
    Xbuf = torch.zeros(x.size + 8, dtype=torch.float32, device="cuda")
    Xbuf[4:4 + x.size] = dev(x.reshape(-1))
    Y = torch.full((2, n), float("nan"), device="cuda")
    st = qmm.lib.qmm_q8_gemv(2, n, k, 32, Wbuf.data_ptr() + 16, Xbuf.data_ptr() + 16, Y.data_ptr(),
                             torch.cuda.current_stream().cuda_stream)
    assert st == 0
    ref, S = oracle.gemv(syn.Q8_0, W, x, n)
    assert_within(host(Y), ref, S, TOL_FP32, "offset buffers")


def test_empty_and_k0():
    x = torch.zeros((1, 0), device="cuda")
    Y = torch.full((1, 5), 7.0, device="cuda")
    st = qmm.lib.qmm_q8_gemv(1, 5, 0, 32, 0, 0, Y.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == 0
    torch.cuda.synchronize()
    assert torch.all(Y == 0)
    assert qmm.lib.qmm_q8_gemv(0, 5, 64, 32, 0, 0, 0, 0) == 0
    assert qmm.lib.qmm_q8_gemv(1, 0, 64, 32, 0, 0, 0, 0) == 0
    assert qmm.device_status() == 0
