"""qmm_q4_swiglu_gateup (fused gate/up SwiGLU on Q4_0 blocks) against the CPU oracle.

out = silu(x.Wg) * (x.Wu) must be within the propagated fp32 bound
1e-5 (1.1 |u| S_g + |silu(g)| S_u) + 8 ulp(out), and the fused launch must equal
the unfused path (two projection launches + a silu*mul launch) bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic as syn
from parity import dev, host, oracle_parallel, swiglu_tolerance

pytestmark = pytest.mark.gpu

qmm = pytest.importorskip("decode_gemv_qmm_b200")


def oracle_swiglu(Wg, Wu, x, n):
    parts = oracle_parallel(lambda a, b, c, N, window: oracle.swiglu(syn.Q4_0, a, b, c, N, window=window),
                            n, Wg, Wu, x, rows_per_job=512)
    return {k: np.concatenate([p[k] for p in parts], axis=1) for k in parts[0]}


def check(m, n, k, seed, xscale=1.0):
    g = syn.rng(seed)
    Wg, Wu = syn.q4_0_weights(g, n, k)[0], syn.q4_0_weights(g, n, k)[0]
    x = syn.act_f32(g, m, k, scale=xscale)
    Wgd, Wud, xd = dev(Wg), dev(Wu), dev(x)
    Y = qmm.qmm_q4_swiglu_gateup(Wgd, Wud, xd, n)
    G, U, Yu = qmm.qmm_q4_gateup_unfused(Wgd, Wud, xd, n)
    torch.cuda.synchronize()
    y = host(Y)
    r = oracle_swiglu(Wg, Wu, x, n)
    err = np.abs(y.astype(np.float64) - r["out"])
    bound = swiglu_tolerance(r)
    assert np.all(np.isfinite(y))
    assert np.all(err <= bound), f"M={m} N={n} K={k}: {int((err > bound).sum())} outputs outside tolerance, " \
                                 f"worst ratio {np.max(err / bound):.3g}"
    # the projections themselves (unfused path) against the oracle's g and u
    assert np.all(np.abs(host(G) - r["g"]) <= 1e-5 * r["Sg"])
    assert np.all(np.abs(host(U) - r["u"]) <= 1e-5 * r["Su"])
    assert np.array_equal(y.view(np.uint32), host(Yu).view(np.uint32)), "fused != unfused"
    return y


def test_gateup_m8_k5120_n17408_full():
    # the measured LSE shape: M=8, N=17408, K=5120 -> 139,264 outputs, fused == unfused bit for bit
    y = check(8, 17408, 5120, seed=0)
    assert y.size == 139264


@pytest.mark.parametrize("m,n,k", [(1, 16, 256), (3, 17, 512), (8, 33, 256), (5, 1000, 1024), (2, 129, 4096),
                                   (8, 16, 32768), (7, 260, 2048)])
def test_shapes_tma_path(m, n, k):
    check(m, n, k, seed=m + n + k)


@pytest.mark.parametrize("m,n,k", [(1, 5, 32), (8, 40, 96), (4, 17, 288), (2, 300, 5120 + 32)])
def test_shapes_direct_path(m, n, k):
    check(m, n, k, seed=m * n + k)


def test_activation_scales():
    # tiny and large activations exercise the per-block power-of-two scaling of the
    # fp16 split (scales chosen so silu(g) * u stays inside the fp32 range)
    check(8, 48, 512, seed=3, xscale=1e-15)
    check(8, 48, 512, seed=4, xscale=1e12)


def test_early_weights_flag_and_determinism():
    g = syn.rng(5)
    n, k = 2048, 5120
    Wg, Wu = dev(syn.q4_0_weights(g, n, k)[0]), dev(syn.q4_0_weights(g, n, k)[0])
    x = dev(syn.act_f32(g, 8, k))
    a = qmm.qmm_q4_swiglu_gateup(Wg, Wu, x, n)
    b = qmm.qmm_q4_swiglu_gateup(Wg, Wu, x, n, flags=qmm.QMM_FLAG_EARLY_WEIGHTS)
    c = qmm.qmm_q4_swiglu_gateup(Wg, Wu, x, n)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int32), b.view(torch.int32)) and torch.equal(a.view(torch.int32), c.view(torch.int32))
    assert qmm.device_status() == 0
