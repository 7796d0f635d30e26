"""Pins for the oracle's online block-Hadamard rotation (CodeQuant "had" variants, CPU)."""
import numpy as np

from oracle import hadamard as Hd
from oracle import gemm as G


def test_sylvester_is_hadamard():
    for n in (1, 2, 4, 8, 16, 32):
        h = Hd.sylvester(n)
        assert np.array_equal(h @ h.T, n * np.eye(n, dtype=np.int64))
        assert set(np.unique(h).tolist()) <= {-1, 1}


def test_hand_worked_4():
    """H_4 rows: [1 1 1 1], [1 -1 1 -1], [1 1 -1 -1], [1 -1 -1 1]; x = [1, 2, 3, 4] gives
    x H_4 = [10, -2, -4, 0]."""
    assert Hd.sylvester(4).tolist() == [[1, 1, 1, 1], [1, -1, 1, -1], [1, 1, -1, -1], [1, -1, -1, 1]]
    out = Hd.rotate_activation_f32(np.array([[1, 2, 3, 4]], np.float32), b=4)
    assert out.tolist() == [[10.0, -2.0, -4.0, 0.0]]


def test_butterfly_equals_the_matrix_on_exact_inputs():
    """On small integers every butterfly step is exact, so the float32 butterfly is x . H."""
    g = np.random.default_rng(1)
    x = g.integers(-1000, 1000, (7, 96)).astype(np.float32)
    want = (x.astype(np.int64).reshape(7, 3, 32) @ Hd.sylvester(32)).reshape(7, 96)
    assert np.array_equal(Hd.rotate_activation_f32(x), want.astype(np.float32))


def test_butterfly_step_order_is_fixed():
    """Inputs whose float32 sums round: the result is the butterfly in the stated order (checked
    against an explicit scalar loop of the same steps), which differs from a plain x . H rounded
    once."""
    g = np.random.default_rng(2)
    x = (g.standard_normal((4, 32)) * np.exp(g.uniform(-20, 20, (4, 32)))).astype(np.float32)
    out = Hd.rotate_activation_f32(x)
    for r in range(4):
        v = [np.float32(t) for t in x[r]]
        h = 1
        while h < 32:
            for i in range(0, 32, 2 * h):
                for j in range(i, i + h):
                    a, b = v[j], v[j + h]
                    v[j], v[j + h] = np.float32(a + b), np.float32(a - b)
            h *= 2
        assert np.array_equal(np.array(v, np.float32), out[r])
    exact = (x.astype(np.float64) @ Hd.sylvester(32).astype(np.float64)).astype(np.float32)
    assert not np.array_equal(exact, out)


def test_rotation_leaves_the_layer_unchanged():
    """x' W'^T = x W^T: the weight rotation undoes the activation rotation (float64 sums)."""
    g = np.random.default_rng(3)
    x = g.integers(-8, 8, (5, 64)).astype(np.float32)
    w = g.standard_normal((6, 64))
    y0 = G.gemm_ref(x.astype(np.float64), w)
    y1 = G.gemm_ref(Hd.rotate_activation_f32(x).astype(np.float64), Hd.rotate_weight(w))
    np.testing.assert_allclose(y1, y0, rtol=1e-12, atol=1e-12)
