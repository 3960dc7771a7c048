"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each pin raises AssertionError when the oracle disagrees with:
  * hand-derived single-block cases (tests/golden/hand_blocks.json),
  * library decoders (numpy float16, torch bfloat16) over all 65,536 patterns,
  * independent dense numpy computations on tiny shapes (brute force),
  * invariants of the definitions (linearity in d, row independence, windows),
  * a second, independently written quantiser (numpy binary32 arithmetic).

The same pins are run against deliberately broken builds of the oracle in
test_oracle_mutants.py, which checks that every planted mistake is caught.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

import oracle
import synthetic as syn

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_blocks.json")


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


def _np_dequant(wtype: int, W: np.ndarray, n: int, k: int) -> np.ndarray:
    """Dense float64 weights via numpy's own float16 decoder (independent of the oracle)."""
    kb = k // 32
    if wtype == syn.Q8_0:
        blk = np.ascontiguousarray(W).view(syn.Q8_0_DTYPE).reshape(n, kb)
        d = blk["d"].view(np.float16).astype(np.float64)
        q = blk["qs"].astype(np.float64)
    else:
        blk = np.ascontiguousarray(W).view(syn.Q4_0_DTYPE).reshape(n, kb)
        d = blk["d"].view(np.float16).astype(np.float64)
        qs = blk["qs"].astype(np.int64)
        q = np.concatenate([(qs & 15) - 8, (qs >> 4) - 8], axis=-1).astype(np.float64)
    return (q * d[..., None]).reshape(n, k)


def _np_quantize(X: np.ndarray):
    """Independent binary32 quantiser: numpy float32 division, round half away
    from zero done in float64 (exact for float32 inputs), clamp to +-127."""
    X = np.asarray(X, dtype=np.float32)
    m, k = X.shape
    xb = X.reshape(m, k // 32, 32)
    amax = np.max(np.abs(xb), axis=-1)
    d = (amax / np.float32(127.0)).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        v = (xb / d[..., None]).astype(np.float32)
    v64 = v.astype(np.float64)
    r = np.sign(v64) * np.floor(np.abs(v64) + 0.5)
    r = np.clip(r, -127, 127)
    r[np.broadcast_to(d[..., None] == 0, r.shape)] = 0
    return r.astype(np.int8).reshape(m, k), d


# --------------------------------------------------------------------------- decoders

def pin_half_decoder_exhaustive():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle.half_to_double(b) for b in bits.tolist()])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))


def pin_bf16_decoder_exhaustive():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([oracle.bf16_to_double(b) for b in bits.tolist()])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))


# --------------------------------------------------------------------------- hand cases

def pin_hand_gemv_blocks():
    for c in _golden()["gemv"]:
        blk = np.frombuffer(bytes.fromhex(c["block"]), dtype=np.uint8).copy()
        x = np.array(c["x"], dtype=np.float32)[None, :]
        y, s = oracle.gemv(c["wtype"], blk, x, 1)
        assert y[0, 0] == c["expected"], (c["name"], y[0, 0], c["expected"])
        assert s[0, 0] >= abs(y[0, 0])
        # the prefill oracle decodes bf16 activations; these x are bf16-exact
        xb = torch.tensor(c["x"], dtype=torch.float32).to(torch.bfloat16)
        assert torch.equal(xb.float(), torch.tensor(c["x"], dtype=torch.float32))
        xbits = xb.view(torch.int16).numpy().view(np.uint16)[None, :]
        yp, _ = oracle.prefill(c["wtype"], blk, xbits, 1)
        assert yp[0, 0] == c["expected"], (c["name"], "prefill", yp[0, 0])


def pin_hand_quantizer():
    for c in _golden()["quantize"]:
        x = np.array(c["x"], dtype=np.float32)[None, :]
        q, d = oracle.quantize_act_q8(x)
        assert d[0, 0] == np.float32(c["d"]), (c["name"], d[0, 0])
        assert q[0].tolist() == c["q"], (c["name"], q[0].tolist())


def pin_hand_q8q8_dots():
    for c in _golden()["q8q8_dots"]:
        blk = syn.pack_q8_0(np.array([c["wq"]], dtype=np.int8), np.array([[0x3C00]], dtype=np.uint16))
        xq = np.array([c["xq"]], dtype=np.int8)
        isum = oracle.q8q8_block_dots(blk, xq, 1)
        assert int(isum[0, 0, 0]) == c["isum"], (c["name"], int(isum[0, 0, 0]))
        # with d_w = 1 and d_x = 1 the scaled output equals the dot
        y, _ = oracle.q8q8_gemv(blk, xq, np.ones((1, 1), np.float32), 1)
        assert y[0, 0] == c["isum"]


def pin_hand_swiglu():
    for c in _golden()["swiglu"]:
        wg = np.frombuffer(bytes.fromhex(c["wg"]), dtype=np.uint8).copy()
        wu = np.frombuffer(bytes.fromhex(c["wu"]), dtype=np.uint8).copy()
        x = np.array(c["x"], dtype=np.float32)[None, :]
        r = oracle.swiglu(syn.Q8_0, wg, wu, x, 1)
        assert r["g"][0, 0] == c["g"] and r["u"][0, 0] == c["u"], c["name"]
        assert r["out"][0, 0] == c["out"], (c["name"], r["out"][0, 0])
    # silu(1) * 1 in closed form: g = 1 from d = 1/32... use d=1, q_0=1, x_0=1
    wg = syn.pack_q8_0(np.array([[1] + [0] * 31], np.int8), np.array([[0x3C00]], np.uint16))
    x = np.array([[1.0] + [0.0] * 31], np.float32)
    r = oracle.swiglu(syn.Q8_0, wg, wg, x, 1)
    assert abs(r["out"][0, 0] - 1.0 / (1.0 + math.exp(-1.0))) < 1e-15


# --------------------------------------------------------------------------- properties

def pin_zero_scale():
    g = syn.rng(11)
    for wtype in (syn.Q8_0, syn.Q4_0):
        n, k = 5, 96
        if wtype == syn.Q8_0:
            W = syn.pack_q8_0(g.integers(-128, 128, (n, k)).astype(np.int8), np.zeros((n, 3), np.uint16))
        else:
            W = syn.pack_q4_0(g.integers(0, 16, (n, k)).astype(np.uint8), np.zeros((n, 3), np.uint16))
        x = syn.act_f32(g, 2, k)
        y, s = oracle.gemv(wtype, W, x, n)
        assert np.all(y == 0) and np.all(s == 0)


def pin_linearity_in_d():
    g = syn.rng(12)
    for wtype in (syn.Q8_0, syn.Q4_0):
        n, k = 6, 128
        if wtype == syn.Q8_0:
            _, q, d = syn.q8_0_weights(g, n, k)
            d2 = (d.view(np.float16) * np.float16(2)).view(np.uint16)
            W1, W2 = syn.pack_q8_0(q, d), syn.pack_q8_0(q, d2)
        else:
            _, q, d = syn.q4_0_weights(g, n, k)
            d2 = (d.view(np.float16) * np.float16(2)).view(np.uint16)
            W1, W2 = syn.pack_q4_0(q, d), syn.pack_q4_0(q, d2)
        x = syn.act_f32(g, 3, k)
        y1, _ = oracle.gemv(wtype, W1, x, n)
        y2, _ = oracle.gemv(wtype, W2, x, n)
        assert np.array_equal(y2, 2.0 * y1)


def pin_block_roundtrip():
    g = syn.rng(13)
    for wtype in (syn.Q8_0, syn.Q4_0):
        n, k = 4, 64
        if wtype == syn.Q8_0:
            W, q, d = syn.q8_0_weights(g, n, k, qlo=-128, qhi=127)
            qv = q.astype(np.float64)
        else:
            W, q, d = syn.q4_0_weights(g, n, k)
            qv = q.astype(np.float64) - 8.0
        dv = d.view(np.float16).astype(np.float64)
        expect = (qv.reshape(n, k // 32, 32) * dv[..., None]).reshape(n, k)
        got = oracle.dequantize(wtype, W, n, k)
        assert np.array_equal(got, expect)
        bb = syn.BLOCK_BYTES[wtype]
        blk = W.reshape(-1)[bb:2 * bb]
        assert np.array_equal(oracle.decode_block(wtype, blk), expect[0, 32:64])


def pin_bruteforce_gemv():
    g = syn.rng(14)
    for wtype in (syn.Q8_0, syn.Q4_0):
        for (m, n, k) in [(1, 1, 32), (2, 3, 64), (3, 7, 128), (1, 5, 96)]:
            W = syn.weights(g, wtype, n, k)
            x = syn.act_f32(g, m, k)
            y, s = oracle.gemv(wtype, W, x, n)
            wd = _np_dequant(wtype, W, n, k)
            ref = x.astype(np.float64) @ wd.T
            sref = np.abs(x.astype(np.float64)) @ np.abs(wd).T
            assert np.all(np.abs(y - ref) <= 1e-12 * sref + 1e-300), (wtype, m, n, k)
            assert np.allclose(s, sref, rtol=1e-12, atol=0)


def pin_row_independence_and_window():
    g = syn.rng(15)
    n, k = 9, 160
    W = syn.weights(g, syn.Q8_0, n, k)
    x = syn.act_f32(g, 4, k)
    y, s = oracle.gemv(syn.Q8_0, W, x, n)
    for m in range(4):
        ym, sm = oracle.gemv(syn.Q8_0, W, x[m:m + 1], n)
        assert np.array_equal(ym[0], y[m]) and np.array_equal(sm[0], s[m])
    yw, sw = oracle.gemv(syn.Q8_0, W, x, n, window=(1, 3, 2, 7))
    assert np.array_equal(yw, y[1:3, 2:7]) and np.array_equal(sw, s[1:3, 2:7])


def pin_quantizer_independent():
    g = syn.rng(16)
    cases = [syn.act_f32(g, 3, 256), syn.act_f32(g, 2, 128, scale=1e-30),
             syn.act_f32(g, 2, 128, scale=1e30), syn.act_f32(g, 1, 4864)]
    # crafted ties: multiples of d/2 with d = 1/127-rounded and power-of-two amax
    t = np.zeros((1, 64), np.float32)
    t[0, :32] = np.arange(-15.5, 16.5, 1.0, dtype=np.float32)
    t[0, 0] = 127.0
    t[0, 32:] = (np.arange(32, dtype=np.float32) - 16) * np.float32(0.5) + np.float32(0.25)
    t[0, 32] = 8.0
    cases.append(t)
    zero = np.zeros((1, 64), np.float32)
    zero[0, 40] = -3.0
    cases.append(zero)
    for x in cases:
        q, d = oracle.quantize_act_q8(x)
        qr, dr = _np_quantize(x)
        assert np.array_equal(d.view(np.uint32), dr.view(np.uint32))
        assert np.array_equal(q, qr)


def pin_quantizer_properties():
    g = syn.rng(17)
    x = syn.act_f32(g, 4, 512)
    q, d = oracle.quantize_act_q8(x)
    xb = x.reshape(4, 16, 32).astype(np.float64)
    qb = q.reshape(4, 16, 32).astype(np.float64)
    d64 = d.astype(np.float64)[..., None]
    assert np.all(np.abs(xb - d64 * qb) <= d64 / 2 * (1 + 2.0 ** -20))
    amax_idx = np.argmax(np.abs(xb), axis=-1)
    picked = np.take_along_axis(qb, amax_idx[..., None], -1)[..., 0]
    assert np.all(np.abs(picked) == 127)
    assert np.all(np.sign(picked) == np.sign(np.take_along_axis(xb, amax_idx[..., None], -1)[..., 0]))


def pin_q8q8_against_numpy():
    g = syn.rng(18)
    m, n, k = 3, 7, 256
    W, qw, dw = syn.q8_0_weights(g, n, k, qlo=-128, qhi=127)
    x = syn.act_f32(g, m, k)
    qx, dx = oracle.quantize_act_q8(x)
    isum = oracle.q8q8_block_dots(W, qx, n)
    ref = np.einsum("nbj,mbj->mnb", qw.reshape(n, k // 32, 32).astype(np.int64),
                    qx.reshape(m, k // 32, 32).astype(np.int64))
    assert np.array_equal(isum.astype(np.int64), ref)
    y, s = oracle.q8q8_gemv(W, qx, dx, n)
    dwf = dw.view(np.float16).astype(np.float64)
    scale = dwf[None, :, :] * dx.astype(np.float64)[:, None, :]
    yref = np.sum(scale * ref, axis=-1)
    sabs = np.einsum("nbj,mbj->mnb", np.abs(qw.reshape(n, k // 32, 32).astype(np.int64)),
                     np.abs(qx.reshape(m, k // 32, 32).astype(np.int64)))
    sref = np.sum(np.abs(scale) * sabs, axis=-1)
    assert np.all(np.abs(y - yref) <= 1e-12 * sref)
    assert np.allclose(s, sref, rtol=1e-12, atol=0)
    # the Q8xQ8 result approximates the fp32-activation result within the
    # quantisation error sum_b |d_w| * d_x/2 * sum_j |q_w|
    yf, _ = oracle.gemv(syn.Q8_0, W, x, n)
    qerr = np.einsum("nb,mb->mn", np.abs(dwf) * np.sum(np.abs(qw.reshape(n, k // 32, 32)), -1),
                     dx.astype(np.float64) / 2)
    assert np.all(np.abs(y - yf) <= qerr * (1 + 1e-6) + 1e-12)


def pin_swiglu_against_numpy():
    g = syn.rng(19)
    for wtype in (syn.Q4_0, syn.Q8_0):
        m, n, k = 3, 5, 128
        Wg, Wu = syn.weights(g, wtype, n, k), syn.weights(g, wtype, n, k)
        x = syn.act_f32(g, m, k, scale=4.0)
        r = oracle.swiglu(wtype, Wg, Wu, x, n)
        x64 = x.astype(np.float64)
        gd = x64 @ _np_dequant(wtype, Wg, n, k).T
        ud = x64 @ _np_dequant(wtype, Wu, n, k).T
        out = gd / (1.0 + np.exp(-gd)) * ud
        sg = np.abs(x64) @ np.abs(_np_dequant(wtype, Wg, n, k)).T
        su = np.abs(x64) @ np.abs(_np_dequant(wtype, Wu, n, k)).T
        assert np.all(np.abs(r["g"] - gd) <= 1e-12 * sg)
        assert np.all(np.abs(r["u"] - ud) <= 1e-12 * su)
        assert np.all(np.abs(r["out"] - out) <= 1e-12 * (np.abs(ud) * sg + np.abs(gd) * su) + 1e-300)
        assert np.allclose(r["Sg"], sg, rtol=1e-12) and np.allclose(r["Su"], su, rtol=1e-12)


def pin_prefill_against_numpy():
    g = syn.rng(20)
    for wtype in (syn.Q8_0, syn.Q4_0):
        m, n, k = 5, 6, 96
        W = syn.weights(g, wtype, n, k)
        xb = syn.act_bf16_bits(g, m, k)
        y, s = oracle.prefill(wtype, W, xb, n)
        x64 = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
        wd = _np_dequant(wtype, W, n, k)
        ref = x64 @ wd.T
        sref = np.abs(x64) @ np.abs(wd).T
        assert np.all(np.abs(y - ref) <= 1e-12 * sref)
        assert np.allclose(s, sref, rtol=1e-12)
        # bf16 -> fp32 is exact, so the prefill oracle equals the fp32 GEMV oracle
        yg, _ = oracle.gemv(wtype, W, x64.astype(np.float32), n)
        assert np.array_equal(y, yg)


def pin_half_encoder_against_numpy():
    """The oracle's binary32 -> binary16 (round to nearest even) against numpy's float16 cast."""
    g = syn.rng(31)
    edge = [0.0, -0.0, 1.0, 1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11, 2.0 ** -14, 2.0 ** -24, 2.0 ** -25,
            3 * 2.0 ** -26, 2.0 ** -20, 65504.0, 65519.0, 65519.99, 65520.0, 1e30, -2.5, 0.1, 1 / 3]
    vals = np.concatenate([np.array(edge, np.float32),
                           (g.standard_normal(20000) * np.exp2(g.integers(-26, 17, 20000))).astype(np.float32)])
    with np.errstate(over="ignore"):
        ref = vals.astype(np.float16).view(np.uint16)
    got = np.array([oracle.float_to_half_bits(v) for v in vals], np.uint16)
    assert np.array_equal(got, ref), vals[got != ref][:5]


def pin_hand_q8_0_activation_blocks():
    """Q8_0 activation blocks (ggml rule) worked out by hand."""
    x = np.zeros((1, 160), np.float32)
    # block 0: amax 127 -> d = 1 (fp16 0x3C00), id = 1, codes = round half away from zero
    x[0, :7] = [127.0, -127.0, 2.5, -2.5, 0.5, -0.5, np.float32(1.5) - np.float32(2.0 ** -23)]
    # block 1: amax = 127 (1 + 2^-11): d = 1 + 2^-11 exactly, halfway between two binary16 values -> even 0x3C00
    x[0, 32] = 127.0 * (1 + 2.0 ** -11)
    # block 2: amax = 127 (1 + 3 2^-11): d halfway between 1 + 2^-10 (odd) and 1 + 2^-9 (even) -> 0x3C02
    x[0, 64] = -127.0 * (1 + 3 * 2.0 ** -11)
    # block 3: amax = 127 2^-20: d = 2^-20 = 16 2^-24, a binary16 subnormal -> 0x0010
    x[0, 96] = 127.0 * 2.0 ** -20
    # block 4: all zero -> d = 0, codes 0
    xb = oracle.quantize_act_q8_0(x).reshape(5, 34)
    dbits = [int(b[0]) | int(b[1]) << 8 for b in xb]
    assert dbits == [0x3C00, 0x3C00, 0x3C02, 0x0010, 0x0000], [hex(v) for v in dbits]
    codes = xb[:, 2:].view(np.int8)
    assert codes[0, :8].tolist() == [127, -127, 3, -3, 1, -1, 1, 0]
    assert codes[1, 0] == 127 and codes[2, 0] == -127 and codes[3, 0] == 127
    assert not codes[4].any() and not codes[0, 8:].any()


def pin_q8_0_activation_properties():
    """Codes within one of the fp32-scale quantiser's, |x - q d| <= d/2, scale = binary16(d)."""
    g = syn.rng(32)
    x = syn.act_f32(g, 3, 1024)
    xb = oracle.quantize_act_q8_0(x)
    codes, scales = oracle.split_q8_0_blocks(xb, 1024)
    q, d = oracle.quantize_act_q8(x)
    assert np.all(np.abs(codes.astype(np.int32) - q.astype(np.int32)) <= 1)
    assert np.mean(codes == q) > 0.99
    d64 = d.astype(np.float64)[..., None]
    err = np.abs(x.reshape(3, 32, 32).astype(np.float64) - d64 * codes.reshape(3, 32, 32))
    assert np.all(err <= d64 / 2 * (1 + 2.0 ** -20))
    assert np.array_equal(scales.astype(np.float16).view(np.uint16),
                          np.array([[oracle.float_to_half_bits(v) for v in row] for row in d], np.uint16))


PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_") and callable(v)]
