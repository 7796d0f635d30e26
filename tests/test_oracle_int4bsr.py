"""Pins for the oracle's INT4 dense + block-sparse residual path (CPU)."""
import numpy as np

import synth
from oracle import int4bsr, mx


def _case(N=64, K=512, T=32, seed=5):
    w = synth.bf16_bits_to_f64(synth.to_bf16_bits(synth.student_t(seed, (N, K), 4.0)))
    xb, _ = synth.activations_bf16(seed, T, K, 0.01 * 8, 30.0)
    return w, synth.bf16_bits_to_f64(xb)


def test_int4_row_quant_golden():
    """amax 7 -> scale exactly 1 in fp16: codes are the rounded values (ties to even)."""
    w = np.zeros((1, 128), np.float32)
    w[0, :5] = [7.0, -3.5, 2.5, 0.49, -7.0]
    q, s = int4bsr.quant_rows_g128(w)
    assert s[0, 0] == np.float16(1.0)
    assert q[0, :5].tolist() == [7, -4, 2, 0, -7]


def test_fp16_scale_rounding_is_rne():
    w = np.zeros((1, 128), np.float32)
    w[0, 0] = 7.0 * 1.0009765625                   # amax / 7 = 1 + 2^-10: exactly an fp16 value
    w[0, 1] = 1.0
    q, s = int4bsr.quant_rows_g128(w)
    assert float(s[0, 0]) == 1.0009765625


def test_density_count_printed_reading():
    """2 % of 512 x 64 blocks (the 8192 x 8192 layer with 16 x 128 blocks) rounds to 655."""
    assert int(round(0.02 * (8192 // 16) * (8192 // 128))) == 655


def test_selection_takes_top_scores_with_ties_to_lower_id():
    w, x = _case()
    prep = int4bsr.prepare(w, x, density=0.05)
    flat = prep["scores"].reshape(-1)
    sel = set(prep["sel"].tolist())
    assert len(sel) == int(round(0.05 * flat.size))
    kept_min = min(flat[i] for i in sel)
    assert all(flat[i] <= kept_min for i in range(flat.size) if i not in sel)
    assert np.all(np.diff(prep["rowptr"]) >= 0) and prep["rowptr"][-1] == len(sel)


def test_score_is_the_plain_double_sum():
    w, x = _case(N=32, K=256, T=8)
    prep = int4bsr.prepare(w, x)
    a = np.abs(x).mean(0)
    nb, g = 1, 1
    direct = sum(a[k] * abs(prep["dw"][n, k]) for n in range(16 * nb, 16 * nb + 16)
                 for k in range(128 * g, 128 * g + 128))
    assert abs(prep["scores"][nb, g] - direct) <= 1e-12 * abs(direct)


def test_forward_equals_grouped_integer_form():
    w, x = _case()
    prep = int4bsr.prepare(w, x, density=0.1)
    y, t = int4bsr.forward(x[:5], prep)
    yg = int4bsr.forward_grouped(x[:5], prep)
    np.testing.assert_allclose(y, yg, rtol=1e-12, atol=1e-12 * np.abs(y).max())


def test_residual_reduces_weight_error_on_selected_blocks():
    w, x = _case()
    prep = int4bsr.prepare(w, x, density=0.1)
    base, res = int4bsr.weight_dense(prep)
    assert np.abs(w - base - res).sum() < np.abs(w - base).sum()


def test_activation_quant_matches_int4_rule():
    x = np.zeros((1, 128), np.float32)
    x[0, :3] = [14.0, -1.0, 3.0]                    # s = 2: 7, -0.5 -> -0 -> 0, 1.5 -> 2
    q, s = int4bsr.quant_act(x)
    assert s[0, 0] == 2.0 and q[0, :3].tolist() == [7, 0, 2]
