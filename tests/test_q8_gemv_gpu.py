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


@pytest.mark.parametrize("n,k", [(37, 256), (2000, 2048), (10000, 896)])
def test_extreme_codes_and_scales_single_row(n, k):
    # the M = 1 kernels on the same extremes: (37, 256) takes the fp32 register-resident
    # kernel, (2000, 2048) the tensor-core resident one, (10000, 896) the integer
    # tensor-core streaming one
    g = syn.rng(13)
    q = g.integers(-128, 128, size=(n, k)).astype(np.int8)
    q[0, :] = -128
    q[1, :] = 127
    d = syn.fp16_bits(np.abs(g.standard_normal((n, k // 32))) * 0.02)
    d[2, :] = 0x0000
    d[3, :] = 0x8000
    d[4, :] = 0x0001
    d[5, :] = 0x03FF
    d[6, :] = 0x7BFF
    d[7, :] = 0xBC00
    W = syn.pack_q8_0(q, d)
    x = syn.act_f32(g, 1, k)
    y = run(W, x, n)
    ref, S = oracle.gemv(syn.Q8_0, W, x, n)
    assert_within(y, ref, S, TOL_FP32, "extreme codes/scales, M=1")
    assert y[0, 2] == 0 and y[0, 3] == 0


def _dynamic_range_inputs(g, k):
    x = syn.act_f32(g, 1, k)
    mixed = (x * 10.0 ** g.uniform(-4, 4, size=x.shape)).astype(np.float32)
    blocks = x.copy()
    blocks[0, 32:64] = 0.0                       # an all-zero block
    blocks[0, 64] = 2.0 ** 12                    # one element far above the rest of its block
    blocks[0, 96:128] = 2.0 ** np.arange(-15, 17, dtype=np.float64)  # exact powers of two
    blocks[0, 128] = -1.0                        # block max exactly a power of two
    blocks[0, 129:160] = 0.5
    return {
        "mixed_1e-4_1e4": mixed,
        "tiny_1e-33": (x * 1e-33).astype(np.float32),
        "subnormal": (x * 1e-40).astype(np.float32),
        "huge_1e30": (x * 1e30).astype(np.float32),
        "structured_blocks": blocks.astype(np.float32),
    }


@pytest.mark.parametrize("n,k", [(1152, 896), (896, 4864), (45, 160), (12000, 896), (9472, 2048)])
def test_single_row_activation_dynamic_range(n, k):
    g = syn.rng(21 + n + k)
    W, _, _ = syn.q8_0_weights(g, n, k)
    for name, x in _dynamic_range_inputs(g, k).items():
        y = run(W, x, n)
        ref, S = oracle.gemv(syn.Q8_0, W, x, n)
        assert_within(y, ref, S, TOL_FP32, f"M=1 N={n} K={k} x={name}")


def test_single_row_zero_activation_gives_exact_zero():
    g = syn.rng(22)
    n, k = 4864, 896
    W, _, _ = syn.q8_0_weights(g, n, k)
    y = run(W, np.zeros((1, k), np.float32), n)
    assert np.all(y == 0)


@pytest.mark.parametrize("n,k", [
    (4869, 896),   # ragged last row group, five groups per CTA
    (4864, 864),   # odd block count (a zero padding block), five groups per CTA
    (2000, 2048),  # two groups per CTA
    (1200, 2048),  # one or two groups per CTA, seven warps of five block pairs
    (3000, 1024),  # three groups per CTA
    (9000, 512),   # eight groups per CTA
    (600, 5120),   # long rows: register-resident kernel, two rows a warp (fp32 codes)
    (893, 4864),   # long rows, ragged N: four rows a warp (fp16 codes)
])
def test_single_row_large_slices(n, k):
    # M = 1 slices large enough for the tensor-core resident kernel (short rows)
    check(1, n, k, seed=31 + n + k)


def test_single_row_tensor_core_chained_calls():
    # consecutive launches in one stream (programmatic dependent launch, early weights):
    # each call reads the previous call's output as its activation vector
    g = syn.rng(41)
    k = 896
    Ws = [syn.q8_0_weights(g, k, k)[0] for _ in range(3)] + [syn.q8_0_weights(g, 4864, k)[0]]
    x = syn.act_f32(g, 1, k)
    Wd = [dev(w) for w in Ws]
    bufs = [dev(x)] + [torch.empty((1, k), dtype=torch.float32, device="cuda") for _ in range(3)]
    out = torch.empty((1, 4864), dtype=torch.float32, device="cuda")
    ys = bufs[1:] + [out]
    for i, w in enumerate(Wd):
        n = ys[i].shape[1]
        st = qmm.lib.qmm_q8_gemv_ex(1, n, k, 32, w.data_ptr(), bufs[i].data_ptr(), ys[i].data_ptr(),
                                    qmm.QMM_FLAG_EARLY_WEIGHTS, 0)
        assert st == 0
    torch.cuda.synchronize()
    assert qmm.device_status() == 0
    xin = x
    for i, w in enumerate(Ws):
        n = ys[i].shape[1]
        ref, S = oracle.gemv(syn.Q8_0, w, xin, n)
        got = host(ys[i])
        assert_within(got, ref, S, TOL_FP32, f"chained call {i}")
        xin = got.astype(np.float32)


@pytest.mark.parametrize("n,k", [
    (10000, 896),   # two 16-row tiles per stage, ragged rows per CTA
    (9472, 2048),   # one tile per stage (K > 1024)
    (20011, 32),    # one block per row: most K slices empty
    (30000, 864),   # odd block count
    (40000, 1024),
])
def test_single_row_integer_streaming_shapes(n, k):
    # M = 1 with many rows per CTA and K <= 2048: raw codes x 8-digit activations on the
    # integer tensor cores
    check(1, n, k, seed=61 + n + k)


def _slice_scaled_inputs(g, n, k, big_first):
    """Weights whose codes are zero over the first quarter of K, and activations of
    ~1e30 there and ~1e-30 elsewhere (or the reverse scales with the zero codes
    over the last three quarters): the output then comes from the tiny-magnitude
    part alone while the vector's largest block exponent sits in the other part."""
    W, _, _ = syn.q8_0_weights(g, n, k)
    kb = k // 32
    rows = W.reshape(n, kb, 34)
    x = syn.act_f32(g, 1, k).astype(np.float64)
    q = k // 4
    if big_first:
        rows[:, :kb // 4, 2:] = 0           # codes of the huge quarter
        x[0, :q] *= 1e30
        x[0, q:] *= 1e-30
    else:
        rows[:, kb // 4:, 2:] = 0           # codes of the huge three quarters
        x[0, :q] *= 1e-30
        x[0, q:] *= 1e30
    return rows.reshape(-1).copy(), x.astype(np.float32)


@pytest.mark.parametrize("big_first", [True, False], ids=["huge_first_quarter", "huge_last_quarters"])
@pytest.mark.parametrize("n,k", [(12000, 896), (9472, 2048)])
def test_integer_kernel_exponent_range_across_k(n, k, big_first):
    # The integer tensor-core kernel scales each K slice by its own largest block
    # exponent: a slice of ~1e30 activations times zero codes must not wipe out the
    # ~1e-30 contributions of the other slices (2^-200 below the vector's maximum).
    g = syn.rng(71 + n + k + big_first)
    W, x = _slice_scaled_inputs(g, n, k, big_first)
    y = run(W, x, n)
    ref, S = oracle.gemv(syn.Q8_0, W, x, n)
    assert np.all(np.abs(ref) > 0)
    assert_within(y, ref, S, TOL_FP32, f"N={n} K={k} big_first={big_first}")


def test_projection_table_exponent_range_across_k():
    g = syn.rng(75)
    k, ns = 896, [4864, 4864]
    W0, x = _slice_scaled_inputs(g, ns[0], k, True)
    W1 = W0.reshape(ns[0], -1)[::-1].reshape(-1).copy()   # same zeroed codes, other rows order
    Ys = qmm.qmm_q8_gemv_multi([dev(W0), dev(W1)], dev(x), ns)
    torch.cuda.synchronize()
    for W, Y, n in zip((W0, W1), Ys, ns):
        ref, S = oracle.gemv(syn.Q8_0, W, x, n)
        assert_within(host(Y), ref, S, TOL_FP32, "projection table, huge first quarter")
