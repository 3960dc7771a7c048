"""The decode step as the benchmark times it, checked against the CPU oracle.

The benchmark's step is a CUDA graph of stream-ordered calls (programmatic
dependent launch, weights streamed before the preceding kernel has finished)
that mixes every M = 1 kernel form of the library: the fp32 and tensor-core
resident kernels, the integer streaming kernel and (multi schedule) the
projection table. This test builds that graph with the benchmark's own code
(bench.DecodeStep, bench.step_graph), replays it several times and compares
every output of all 121 matmuls -- lm_head's 151,936 included -- with the
oracle element by element at 1e-5 * sum |w x|.

Two workloads:
* the benchmark's own (each matmul has its own input vector);
* a chained step where each matmul reads its predecessor's output along the
  model's data flow (qkv <- down, wo <- qkv, gate/up <- wo, down <- up,
  lm_head <- last down). There a kernel that read its input before the
  preceding kernel had finished writing it would see the poisoned (NaN) or an
  older value and fail the comparison, which is checked against the oracle on
  the final value of that input.

The whole decode is what the pages check against a plain reference ("Lumen
v0.2.0", section "Correctness"; "Lumen v0.4.0", section "Phase 7.P": the
per-step matmul set).
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic as syn
from parity import TOL_FP32, assert_within

pytestmark = pytest.mark.gpu

qmm = pytest.importorskip("decode_gemv_qmm_b200")
bench = pytest.importorskip("bench")

_REFS = {}


def oracle_outputs(step, Y_host):
    """(ref, S) of every matmul of the step on the inputs the GPU used."""
    out = []
    for i, (_, n, k) in enumerate(step.shapes):
        x = step.x_of(i, Y_host)
        if n > 8192:
            parts = [oracle.gemv(syn.Q8_0, step.host_w[i], x, n, window=(0, 1, n0, min(n, n0 + 16384)))
                     for n0 in range(0, n, 16384)]
            ref = np.concatenate([p[0] for p in parts], axis=1)
            S = np.concatenate([p[1] for p in parts], axis=1)
        else:
            ref, S = oracle.gemv(syn.Q8_0, step.host_w[i], x, n)
        out.append((ref[0], S[0]))
    return out


def check_step(step, Y_host, refs, label):
    assert np.all(np.isfinite(Y_host)), f"{label}: non-finite outputs (a poisoned value was read or not overwritten)"
    for i, (name, n, _) in enumerate(step.shapes):
        got = Y_host[int(step.y_offsets[i]):int(step.y_offsets[i + 1])]
        ref, S = refs[i]
        assert_within(got, ref, S, TOL_FP32, f"{label} {name}")


def run_graph(step, graph, stream, replays):
    with torch.cuda.stream(stream):
        for _ in range(replays):
            graph.replay()
    torch.cuda.synchronize()
    return step.Y.cpu().numpy().copy()


@pytest.mark.parametrize("chain", [False, True], ids=["own_inputs", "chained"])
@pytest.mark.parametrize("schedule", ["gemv", "multi"])
def test_decode_step_graph_matches_oracle(schedule, chain):
    step = bench.DecodeStep(0, torch.device("cuda", 0), keep_host=True, chain=chain)
    stream = torch.cuda.Stream()
    graph = bench.step_graph(qmm, step, stream, schedule, qmm.QMM_FLAG_EARLY_WEIGHTS)
    step.Y.fill_(float("nan"))
    torch.cuda.synchronize()
    first = run_graph(step, graph, stream, 1)
    key = chain
    if schedule == "multi" and not chain:
        # without the chain the multi schedule gives up its own input to the gate's
        key = "multi_own"
    if key not in _REFS:
        if key == "multi_own":
            xs = list(step.host_x)
            for i, (name, _, _) in enumerate(step.shapes):
                if name.endswith(".up"):
                    step.host_x[i] = xs[i - 1]
            refs = oracle_outputs(step, first)
            step.host_x[:] = xs
        else:
            refs = oracle_outputs(step, first)
        # chained inputs are the step's own outputs: cache only the unchained references
        if not chain:
            _REFS[key] = refs
    else:
        refs = _REFS[key]
    check_step(step, first, refs, f"{schedule} chain={chain} first replay")
    later = run_graph(step, graph, stream, 4)
    assert np.array_equal(later.view(np.uint32), first.view(np.uint32)), "replays of the step graph differ"
    assert qmm.device_status() == 0
    del graph


def test_chained_step_magnitudes_stay_bounded():
    """The chained workload's scales keep every output O(1) over all 121 matmuls,
    so the comparison above exercises ordinary numbers, not overflow or zeros."""
    step = bench.DecodeStep(0, torch.device("cuda", 0), keep_host=False, chain=True)
    stream = torch.cuda.Stream()
    graph = bench.step_graph(qmm, step, stream, "gemv", qmm.QMM_FLAG_EARLY_WEIGHTS)
    Y = run_graph(step, graph, stream, 1)
    for i, (name, _, _) in enumerate(step.shapes):
        y = Y[int(step.y_offsets[i]):int(step.y_offsets[i + 1])]
        rms = float(np.sqrt(np.mean(np.square(y.astype(np.float64)))))
        assert 0.05 < rms < 20.0, f"{name}: rms {rms}"
    del graph


def test_decode_step_auto_schedule_matches_oracle():
    """The per-K schedule the benchmark also times (qmm_q8_gemv_auto on every
    matmul, one code/scale buffer for the whole step): qkv, wo, gate and up
    (K = 896, slices on chip) are the Q8xQ8 product of the activations
    quantised per block, down (K = 4864) and lm_head (slice too large) the
    fp32 GEMV. Each output is compared with the oracle of the form it took,
    on a chained step, after replays of the graph."""
    step = bench.DecodeStep(0, torch.device("cuda", 0), keep_host=True, chain=True)
    stream = torch.cuda.Stream()
    graph = bench.step_graph(qmm, step, stream, "auto", qmm.QMM_FLAG_EARLY_WEIGHTS)
    step.Y.fill_(float("nan"))
    torch.cuda.synchronize()
    Y = run_graph(step, graph, stream, 2)
    assert np.all(np.isfinite(Y))
    for i, (name, n, k) in enumerate(step.shapes):
        got = Y[int(step.y_offsets[i]):int(step.y_offsets[i + 1])]
        x = step.x_of(i, Y)
        kind = name.split(".")[-1]
        if kind in ("qkv", "wo", "gate", "up"):
            qx, dx = oracle.quantize_act_q8(x)
            ref, S = oracle.q8q8_gemv(step.host_w[i], qx, dx, n)
        elif n > 8192:
            parts = [oracle.gemv(syn.Q8_0, step.host_w[i], x, n, window=(0, 1, n0, min(n, n0 + 16384)))
                     for n0 in range(0, n, 16384)]
            ref = np.concatenate([p[0] for p in parts], axis=1)
            S = np.concatenate([p[1] for p in parts], axis=1)
        else:
            ref, S = oracle.gemv(syn.Q8_0, step.host_w[i], x, n)
        assert_within(got, ref[0], S[0], TOL_FP32, f"auto {name}")
    assert qmm.device_status() == 0
    del graph
