"""Pins for the oracle's routed MoE FFN (CPU)."""
import numpy as np
import pytest

import synth
from oracle import formats as F
from oracle import mx, moe


def test_route_matches_bruteforce_with_ties():
    g = np.random.default_rng(3)
    logits = g.integers(-3, 4, (40, 12)).astype(np.float32)     # many ties
    r = moe.route(logits, 4)
    for t in range(40):
        want = sorted(range(12), key=lambda e: (-float(logits[t, e]), e))[:4]
        assert r["ids"][t].tolist() == want
    assert r["counts"].sum() == 40 * 4 and r["offsets"][-1] == 160
    np.testing.assert_allclose(r["gates"].sum(1), 1.0, rtol=1e-15)
    # entries: expert-major, ascending flat index inside an expert, each entry once
    flat = r["ids"].reshape(-1)
    assert sorted(r["entries"].tolist()) == list(range(160))
    for e in range(12):
        seg = r["entries"][r["offsets"][e]:r["offsets"][e + 1]]
        assert np.all(flat[seg] == e) and np.all(np.diff(seg) > 0)


def test_gate_weights_are_softmax_of_selected_logits():
    logits = np.array([[0.0, 1.0, 2.0, -1.0]], np.float32)
    r = moe.route(logits, 2)
    assert r["ids"][0].tolist() == [2, 1]
    e = np.exp([2.0, 1.0])
    np.testing.assert_allclose(r["gates"][0], e / e.sum(), rtol=1e-15)


def test_swiglu_special_values():
    assert moe.swiglu(np.array([0.0]), np.array([5.0]))[0] == 0.0
    np.testing.assert_allclose(moe.swiglu(np.array([40.0]), np.array([2.0])), [80.0], rtol=1e-15)
    np.testing.assert_allclose(moe.swiglu(np.array([1.0]), np.array([1.0])), [1 / (1 + np.exp(-1))])


def _model(seed, E, H, I, T):
    Wgu, Wd = [], []
    for e in range(E):
        cb, ix = synth.cluster_rows(seed * 100 + e, 2 * I, H)
        Wgu.append(moe.cluster_weight(cb, ix))
        cb, ix = synth.cluster_rows(seed * 100 + 50 + e, H, I)
        Wd.append(moe.cluster_weight(cb, ix))
    xb, _ = synth.activations_bf16(seed, T, H, 0.0, 1.0)
    return Wgu, Wd, F.bf16_decode(xb)


def test_single_expert_top1_is_the_dense_gated_ffn():
    Wgu, Wd, x = _model(5, 1, 64, 32, 6)
    logits = np.zeros((6, 1), np.float32)
    res = moe.forward(x, logits, Wgu, Wd, 1)
    xc, xs = mx.quantize_e8m0_b32(x)
    xq = mx.dequant_e8m0_b32(xc, xs)
    gu = xq @ Wgu[0].T
    h = gu[:, :32] / (1 + np.exp(-gu[:, :32])) * gu[:, 32:]
    hc, hs = mx.quantize_e8m0_b32(h)
    want = mx.dequant_e8m0_b32(hc, hs) @ Wd[0].T
    np.testing.assert_allclose(res["out"], want, rtol=1e-12, atol=1e-12 * np.abs(want).max())


def test_gate_rows_come_first():
    """PRQuant Eq. (1) gives the gated FFN h = act(g) * u; the fused gate/up weight holds the gate
    rows first (reading: rows 0..I-1 gate, I..2I-1 up).  With a one-hot input the two GEMMs pick
    out one centroid each: every gate row is -40 and every up row +40, so g = -40 and u = 40
    exactly and h = SiLU(-40) * 40 = -1600 / (1 + e^40), about -6.8e-15.  The other row order
    would give SiLU(40) * (-40), about -1600."""
    H, I = 64, 32
    bits = lambda v: synth.to_bf16_bits(np.full((1, 16), v))
    cent = np.concatenate([np.repeat(bits(-40.0), I, 0), np.repeat(bits(40.0), I, 0)])
    idx = np.zeros((2 * I, H), np.uint8)
    Wgu = [moe.cluster_weight(cent, idx)]
    Wd = [moe.cluster_weight(np.repeat(bits(1.0), H, 0), np.zeros((H, I), np.uint8))]
    x = np.zeros((1, H))
    x[0, 0] = 1.0                                        # MXFP4: amax 1, code 4 * 2^-2 = 1 exactly
    res = moe.forward(x, np.zeros((1, 1), np.float32), Wgu, Wd, 1)
    assert np.all(res["g"] == -40.0) and np.all(res["u"] == 40.0)
    want = -1600.0 / (1.0 + np.exp(40.0))
    np.testing.assert_allclose(res["h"], want, rtol=1e-12)
    assert np.all(np.abs(res["h"]) < 1e-13)


def test_expert_relabeling_invariance():
    E, H, I, T, k = 4, 64, 32, 10, 2
    Wgu, Wd, x = _model(6, E, H, I, T)
    logits = synth.zipf_router_logits(6, T, E)
    a = moe.forward(x, logits, Wgu, Wd, k)["out"]
    p = np.array([2, 0, 3, 1])
    b = moe.forward(x, logits[:, p], [Wgu[i] for i in p], [Wd[i] for i in p], k)["out"]
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-12 * np.abs(a).max())


def test_combine_is_the_gate_weighted_sum_of_slots():
    E, H, I, T, k = 3, 32, 32, 4, 3
    Wgu, Wd, x = _model(7, E, H, I, T)
    logits = synth.zipf_router_logits(7, T, E)
    res = moe.forward(x, logits, Wgu, Wd, k)
    r, hq = res["route"], mx.dequant_e8m0_b32(res["h_codes"], res["h_scales"])
    pos = np.empty(T * k, int)
    pos[r["entries"]] = np.arange(T * k)
    for t in range(T):
        acc = np.zeros(H)
        for s in range(k):
            e = r["ids"][t, s]
            acc += r["gates"][t, s] * (Wd[e] @ hq[pos[t * k + s]])
        np.testing.assert_allclose(res["out"][t], acc, rtol=1e-12, atol=1e-12)


def test_zipf_router_is_skewed():
    logits = synth.zipf_router_logits(4, 2048, 128)
    r = moe.route(logits, 8)
    c = np.sort(r["counts"])[::-1]
    assert c.sum() == 16384 and c[0] > 1000 and c[-1] < 64
