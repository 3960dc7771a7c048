"""qmm_quant_matmul_prefill (tcgen05 tensor-core prefill panels) against the CPU oracle.

The weights are decoded to bf16 on the GPU, so outputs must be within
4e-3 * sum_k |w_k x_k| of the exact (fp64, undecoded) oracle.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic as syn
from parity import TOL_BF16, assert_within, dev, host, oracle_parallel

pytestmark = pytest.mark.gpu

qmm = pytest.importorskip("decode_gemv_qmm_b200")


def run(wtype, m, n, k, seed, window_rows=None):
    g = syn.rng(seed)
    W = syn.weights(g, wtype, n, k)
    xb = syn.act_bf16_bits(g, m, k)
    Y = qmm.qmm_quant_matmul_prefill(wtype, dev(W), dev(xb), n)
    torch.cuda.synchronize()
    assert qmm.device_status() == 0
    y = host(Y)
    return W, xb, y


def check_full(wtype, m, n, k, seed):
    W, xb, y = run(wtype, m, n, k, seed)
    parts = oracle_parallel(lambda a, b, N, window: oracle.prefill(wtype, a, b, N, window=window), n, W, xb,
                            rows_per_job=128)
    ref = np.concatenate([p[0] for p in parts], axis=1)
    S = np.concatenate([p[1] for p in parts], axis=1)
    assert_within(y, ref, S, TOL_BF16, f"prefill wtype={wtype} M={m} N={n} K={k}")


@pytest.mark.parametrize("wtype", [syn.Q8_0, syn.Q4_0])
@pytest.mark.parametrize("m,n,k", [(16, 128, 256), (32, 256, 512), (7, 130, 256), (100, 200, 1024), (1, 1, 256),
                                   (300, 129, 768)])
def test_prefill_rows_16_byte_multiple(wtype, m, n, k):
    # row pitch a multiple of 16 bytes (K % 256 == 0); small shapes split K over a cluster
    check_full(wtype, m, n, k, seed=m + n + k)


@pytest.mark.parametrize("wtype", [syn.Q8_0, syn.Q4_0])
@pytest.mark.parametrize("m,n,k", [(32, 128, 896), (16, 77, 96), (5, 3, 32), (64, 257, 160)])
def test_prefill_rows_not_16_byte_multiple(wtype, m, n, k):
    # widened per-row bulk copies; (64, 257, 160) splits three stages over three ranks
    check_full(wtype, m, n, k, seed=3 * m + n + k)


def check_sampled(wtype, m, n, k, seed, n_samples=96):
    """Full-size launch; compare every token of a spread of sampled weight rows
    (covering several 128-row tiles, the last tile included)."""
    W, xb, y = run(wtype, m, n, k, seed)
    g = np.random.default_rng(seed + 1)
    rows = np.unique(np.concatenate([g.choice(n, size=n_samples, replace=False), [0, 127, 128, n - 1]]))
    import concurrent.futures as cf
    import os
    with cf.ThreadPoolExecutor(max_workers=os.cpu_count() or 1) as ex:
        res = list(ex.map(lambda r: oracle.prefill(wtype, W, xb, n, window=(0, m, int(r), int(r) + 1)), rows))
    ref = np.concatenate([r[0] for r in res], axis=1)
    S = np.concatenate([r[1] for r in res], axis=1)
    assert_within(y[:, rows], ref, S, TOL_BF16, f"prefill wtype={wtype} M={m} N={n} K={k} (sampled rows)")


@pytest.mark.parametrize("m", [32, 1024])
@pytest.mark.parametrize("n,k", [(4864, 896), (896, 4864)])
def test_prefill_q8_panels_full_size(m, n, k):
    if m == 32:
        check_full(syn.Q8_0, m, n, k, seed=m + n)
    else:
        check_sampled(syn.Q8_0, m, n, k, seed=m + n)


def test_prefill_q4_m1024_k5120_n17408():
    check_sampled(syn.Q4_0, 1024, 17408, 5120, seed=11, n_samples=64)


@pytest.mark.parametrize("wtype", [syn.Q8_0, syn.Q4_0])
@pytest.mark.parametrize("m,n,k", [(48, 300, 4864), (40, 1000, 2048), (200, 129, 1312), (17, 5, 7200)])
def test_prefill_split_k(wtype, m, n, k):
    # few output tiles, long K: the K range is split across a thread-block cluster
    check_full(wtype, m, n, k, seed=5 * m + n + k)


def test_prefill_split_k_deterministic():
    g = syn.rng(9)
    n, k, m = 896, 4864, 32
    W = dev(syn.weights(g, syn.Q8_0, n, k))
    xb = dev(syn.act_bf16_bits(g, m, k))
    a = qmm.qmm_quant_matmul_prefill(syn.Q8_0, W, xb, n)
    b = qmm.qmm_quant_matmul_prefill(syn.Q8_0, W, xb, n)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    assert qmm.device_status() == 0


@pytest.mark.parametrize("wtype,m,n,k", [(syn.Q8_0, 1024, 4864, 896), (syn.Q8_0, 32, 896, 4864),
                                         (syn.Q4_0, 300, 129, 768), (syn.Q8_0, 64, 257, 160)])
def test_prefill_early_weights_same_bits(wtype, m, n, k):
    """With early weights the result is bit-identical (only the start of the weight stream moves)."""
    g = syn.rng(m + n + k + 5)
    W = dev(syn.weights(g, wtype, n, k))
    X = dev(syn.act_bf16_bits(g, m, k))
    Y0 = qmm.qmm_quant_matmul_prefill(wtype, W, X, n)
    Y1 = qmm.qmm_quant_matmul_prefill(wtype, W, X, n, flags=qmm.QMM_FLAG_EARLY_WEIGHTS)
    torch.cuda.synchronize()
    assert torch.equal(Y0.view(torch.int32), Y1.view(torch.int32))
    assert qmm.device_status() == 0


def test_prefill_plan_wide_tiles_for_a_nearly_empty_last_wave():
    """1024 tokens x 4864 rows: 152 tiles of 256 tokens are two waves on 148 SMs, the second
    nearly empty; 114 tiles of 352 tokens (two MMAs per k step) are one."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    p = qmm.qmm_prefill_plan(syn.Q8_0, 1024, 4864, 896)
    if 114 <= sms < 152:
        assert (p["mt"], p["split"], p["ctas"]) == (352, 1, 114), p
        assert p["stages"] >= 3, p
    # 544 tiles of 256 tokens against 408 of 352: four waves against three, no gain
    assert qmm.qmm_prefill_plan(syn.Q4_0, 1024, 17408, 5120)["mt"] == 256
    assert qmm.qmm_prefill_plan(syn.Q8_0, 1024, 4864, 896)["kernel"] == "tcgen05"
    # 32 tokens: the small-M kernel, K split over a cluster where rows are few
    p = qmm.qmm_prefill_plan(syn.Q8_0, 32, 4864, 896)
    assert p["kernel"] == "small_m" and p["split"] == 1 and p["ctas"] <= sms, p
    p = qmm.qmm_prefill_plan(syn.Q8_0, 32, 896, 4864)
    assert p["kernel"] == "small_m" and p["split"] > 1, p
    assert qmm.qmm_prefill_plan(syn.Q8_0, 33, 896, 4864)["kernel"] == "tcgen05"


@pytest.mark.parametrize("wtype", [syn.Q8_0, syn.Q4_0])
@pytest.mark.parametrize("m,n,k", [(520, 6390, 128),    # tiles of 288 tokens, the second one ragged
                                   (600, 6400, 96),     # odd block count, super-row TMA of the weights
                                   (1000, 4864, 256)])  # tiles of 352 tokens: 352 + 352 + 296
def test_prefill_wide_token_tiles(wtype, m, n, k):
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    plan = qmm.qmm_prefill_plan(wtype, m, n, k)
    if sms == 148:
        assert plan["mt"] > 256 and plan["split"] == 1, plan
    check_full(wtype, m, n, k, seed=7 * m + n + k)


@pytest.mark.parametrize("wtype", [syn.Q8_0, syn.Q4_0])
@pytest.mark.parametrize("m,n,k", [(16, 12000, 256), (32, 9600, 288)])
def test_prefill_few_tokens_many_rows_on_tcgen05_tiles(wtype, m, n, k):
    """At most 32 tokens but more rows than one wave of 64-row groups: the small-M kernel
    does not apply and the tcgen05 tiles (16 / 32 tokens wide) take the panel."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    plan = qmm.qmm_prefill_plan(wtype, m, n, k)
    if (n + 63) // 64 > sms:
        assert plan["kernel"] == "tcgen05" and plan["mt"] == m, plan
    check_full(wtype, m, n, k, seed=11 * m + n + k)
