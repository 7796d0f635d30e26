"""Pins for the oracle's PRQuant tail-residual path (CPU)."""
import json
import os

import numpy as np

import synth
from oracle import mx, prquant
from tests.conftest import GOLDEN


def _case(seed=3, N=64, C=512, k=64, M=8):
    w = synth.bf16_bits_to_f64(synth.to_bf16_bits(synth.student_t(seed, (N, C), 3.0)))
    xb, _ = synth.activations_bf16(seed, M, C, 0.005 * 4, 50.0)
    return w, synth.bf16_bits_to_f64(xb), k


def test_permutation_invariance_eq1():
    """X W^T = (X P)(W P)^T for the unquantized operands (Eq. 1)."""
    w, x, k = _case()
    prep = prquant.prepare(w, k)
    p = prep["perm"]
    assert sorted(p.tolist()) == list(range(w.shape[1]))
    np.testing.assert_allclose(x @ w.T, x[:, p] @ w[:, p].T, rtol=1e-12, atol=1e-9)


def test_tail_holds_the_k_largest_errors():
    w, _, k = _case()
    err = prquant.column_errors(w)
    tail = prquant.select_tail(err, k)
    kept = np.setdiff1d(np.arange(w.shape[1]), tail)
    assert len(tail) == k and err[tail].min() >= err[kept].max()
    p = prquant.permutation(w.shape[1], tail)
    assert np.array_equal(p[-k:], np.sort(tail)) and np.all(np.diff(p[:-k]) > 0)


def test_online_copy_equals_quantizing_the_augmented_activation():
    """Copying the quantized tail with its scales equals quantizing [Z~, Z~_tail] when the
    tail is block aligned ("Kernel design for efficient inference")."""
    w, x, k = _case()
    xp = x[:, prquant.prepare(w, k)["perm"]]
    c1, s1 = prquant.quantize_activation_augmented(xp, k)
    c2, s2 = mx.quantize_e8m0_b32(np.concatenate([xp, xp[:, -k:]], axis=1))
    assert np.array_equal(c1, c2) and np.array_equal(s1, s2)


def test_augmented_gemm_is_base_plus_residual_product():
    w, x, k = _case()
    prep = prquant.prepare(w, k)
    C = w.shape[1]
    xp = x[:, prep["perm"]]
    y, _ = prquant.forward(xp, prep, k)
    xc, xs = mx.quantize_e8m0_b32(xp)
    xd = mx.dequant_e8m0_b32(xc, xs)
    wd = mx.dequant_e8m0_b32(prep["w_codes"][:, :C], prep["w_sb"][:, :C // 32])
    rd = mx.dequant_e8m0_b32(prep["w_codes"][:, C:], prep["w_sb"][:, C // 32:])
    two = xd @ wd.T + xd[:, C - k:] @ rd.T
    np.testing.assert_allclose(y, two, rtol=1e-12, atol=1e-12 * np.abs(two).max())


def test_residual_is_exact_weight_error():
    w, _, k = _case()
    prep = prquant.prepare(w, k)
    C = w.shape[1]
    wp = w[:, prep["perm"]]
    base = mx.dequant_e8m0_b32(prep["w_codes"][:, :C], prep["w_sb"][:, :C // 32])
    assert np.array_equal(prep["residual"], wp[:, C - k:] - base[:, C - k:])
    # compensation shrinks the tail's weight error
    rd = mx.dequant_e8m0_b32(prep["w_codes"][:, C:], prep["w_sb"][:, C // 32:])
    assert np.abs(wp[:, C - k:] - base[:, C - k:] - rd).sum() < np.abs(prep["residual"]).sum()


def test_tail_ratio_printed():
    with open(os.path.join(GOLDEN, "table1_formats.json")) as f:
        cases = json.load(f)["prquant_tail_ratio"]["cases"]
    for C, k, pct in cases:
        assert round(100.0 * k / C, 1) == pct


def test_e8m0_scale_search_hand_worked():
    """PRQuant (E8M0-W), §5.3: block [7.9, 1, 0, ...]: the OCP exponent is 0 (7.9 saturates to 6,
    squared error 1.9^2 + 0 = 3.61); e = 1 gives 7.9/2 = 3.95 -> 4 -> 8 (error 0.01) and 1/2 = 0.5
    -> 0.5 -> 1 (error 0): e = 1 wins, byte 128.  Block [6, 1.25, ...]: e0 = 0 is exact for 6
    (code 7) and 1.25 ties to 1.0 (error 0.0625); e = 1 gives 3 -> 6, 0.625 -> 0.5 -> 1.0 (same
    error 0.0625, not strictly better) and e = -1 saturates 6 -> 3 (worse): e0 stays, byte 127."""
    x = np.zeros((1, 64))
    x[0, :2] = [7.9, 1.0]
    x[0, 32:34] = [6.0, 1.25]
    codes, sb = mx.quantize_e8m0_b32_searched(x)
    assert sb[0].tolist() == [128, 127]
    assert codes[0, :2].tolist() == [6, 1] and codes[0, 32:34].tolist() == [7, 2]


def test_e8m0_scale_search_never_worse_and_includes_default():
    g = np.random.default_rng(31)
    x = g.standard_t(3, (64, 256)) * np.exp(g.uniform(-3, 3, (64, 1)))
    c0, s0 = mx.quantize_e8m0_b32(x)
    c1, s1 = mx.quantize_e8m0_b32_searched(x)
    e0 = ((x - mx.dequant_e8m0_b32(c0, s0)) ** 2).reshape(64, 8, 32).sum(-1)
    e1 = ((x - mx.dequant_e8m0_b32(c1, s1)) ** 2).reshape(64, 8, 32).sum(-1)
    assert np.all(e1 <= e0 + 1e-12 * np.abs(e0))
    same = s1 == s0
    assert np.array_equal(c1.reshape(64, 8, 32)[same], c0.reshape(64, 8, 32)[same])
    assert (~same).any() and same.any()
    assert np.all(np.abs(s1.astype(int) - s0.astype(int)) <= 1)


def test_prquant_with_scale_search_keeps_the_identities():
    """With the searched scales the tail residual is still W~_tail - deq Q(W~_tail) and the
    augmented GEMM still equals base plus residual products."""
    w = synth.bf16_bits_to_f64(synth.to_bf16_bits(synth.student_t(33, (32, 256), 3.0)))
    k = 64
    p = prquant.prepare(w, k, search=True)
    C = w.shape[1]
    wp = w[:, p["perm"]]
    base = mx.dequant_e8m0_b32(p["w_codes"][:, :C], p["w_sb"][:, :C // 32])
    assert np.allclose(p["residual"], wp[:, C - k:] - base[:, C - k:], rtol=0, atol=0)
    qc, qs = mx.quantize_e8m0_b32_searched(wp)
    assert np.array_equal(qc, p["w_codes"][:, :C]) and np.array_equal(qs, p["w_sb"][:, :C // 32])
