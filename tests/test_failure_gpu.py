"""Failure detection without a fault: a bounded wait that runs out.

Every pipeline wait in the kernels is bounded; when one gives up, the kernel
records a bit in its device status word, stops waiting on that barrier,
finishes without touching the buffer the missing copy would have filled and
returns, so the context stays usable ("LSE v0.4.15", section "Qualification
and measurements": guarded execution). Here the wait is made to run out the
allowed way: a test launch (qmm_test_withheld_copy) in which CTA 0 never issues
one of its copies, with a wait limit of a few milliseconds. No copy is left in
flight, nothing faults, traps or hangs.

Checked: the call returns, qmm_device_status() reports the bits (as
QMM_ERR_DEVICE_CHECK) and clears them, the outputs of the other CTAs are still
correct, and the next ordinary call on the same device is correct with a clean
status.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic as syn
from parity import TOL_FP32, assert_within, dev, host

pytestmark = pytest.mark.gpu

qmm = pytest.importorskip("decode_gemv_qmm_b200")

WAIT_NS = 2_000_000  # 2 ms
FULL, DRAIN = 1, 2


def test_streaming_gemv_wait_runs_out():
    m, n, k = 2, 4096, 2048                     # the streaming kernel (M > 1), 148 CTAs of 27-28 rows
    g = syn.rng(404)
    W = syn.q8_0_weights(g, n, k)[0]
    x = syn.act_f32(g, m, k)
    Wd, xd = dev(W), dev(x)
    assert qmm.device_status() == 0
    Y = torch.full((m, n), float("nan"), device="cuda")
    qmm.qmm_test_withheld_copy(0, Wd, xd, n, Y, WAIT_NS)
    bits = qmm.device_status()
    assert bits & FULL, f"status bits {bits:#x}: the starved wait was not recorded"
    assert qmm.device_status() == 0, "the status word was not cleared"
    # rows past CTA 0's range are computed as usual
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    first = -(-n // min(n, sms))                 # CTA 0 owns at most this many rows
    ref, S = oracle.gemv(syn.Q8_0, W, x, n)
    assert_within(host(Y)[:, first:], ref[:, first:], S[:, first:], TOL_FP32, "rows of the other CTAs")
    # the next ordinary call is correct and clean
    Y2 = qmm.qmm_q8_gemv(Wd, xd, n)
    torch.cuda.synchronize()
    assert_within(host(Y2), ref, S, TOL_FP32, "ordinary call after the failure")
    assert qmm.device_status() == 0


def test_small_m_prefill_split_k_wait_runs_out():
    m, n, k = 32, 896, 4864                      # small-M kernel with split K (clusters of CTAs)
    plan = qmm.qmm_prefill_plan(syn.Q8_0, m, n, k)
    assert plan["kernel"] == "small_m" and plan["split"] > 1, plan
    groups = plan["ctas"] // plan["split"]
    g = syn.rng(405)
    W = syn.q8_0_weights(g, n, k)[0]
    xb = syn.act_bf16_bits(g, m, k)
    Wd, xd = dev(W), dev(xb.view(np.int16))
    assert qmm.device_status() == 0
    Y = torch.full((m, n), float("nan"), device="cuda")
    qmm.qmm_test_withheld_copy(1, Wd, xd, n, Y, WAIT_NS)
    bits = qmm.device_status()
    # rank 0 of the first cluster times out on W, cannot drain it (it was never
    # issued), skips its partial sums and output, and still meets the cluster barrier
    assert bits & FULL and bits & DRAIN, f"status bits {bits:#x}"
    assert qmm.device_status() == 0
    first = -(-n // groups)                      # rows of the first cluster (at most)
    ref, S = oracle.prefill(syn.Q8_0, W, xb, n)
    assert_within(host(Y)[:, first:], ref[:, first:], S[:, first:], TOL_FP32, "rows of the other clusters")
    Y2 = qmm.qmm_quant_matmul_prefill(syn.Q8_0, Wd, xd, n)
    torch.cuda.synchronize()
    assert_within(host(Y2), ref, S, TOL_FP32, "ordinary call after the failure")
    assert qmm.device_status() == 0
