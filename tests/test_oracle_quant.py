"""Pins for the oracle's block quantizers and GEMM reference (CPU)."""
import json
import os

import numpy as np

from oracle import formats as F
from oracle import gemm as G
from oracle import mx
from tests.conftest import GOLDEN


def _num(s):
    return float.fromhex(s) if "0x" in s else float(s)


def test_mx_e8m0_golden_blocks():
    with open(os.path.join(GOLDEN, "mx_e8m0_blocks.json")) as f:
        g = json.load(f)
    for blk in g["blocks"]:
        x = np.zeros((1, 32))
        vals = [_num(s) for s in blk["x"]]
        x[0, :len(vals)] = vals
        codes, sb = mx.quantize_e8m0_b32(x)
        assert int(sb[0, 0]) == blk["byte"], blk["note"]
        assert codes[0, :len(vals)].tolist() == blk["codes"], blk["note"]
        assert np.all(codes[0, len(vals):] == 0)


def test_mx_exponent_invariant():
    """For an unclamped non-zero block, amax / 2^e lies in [4, 8): the largest element lands on
    the top binade of E2M1 (4 or 6, or saturates at 6)."""
    g = np.random.default_rng(1)
    x = g.standard_normal((64, 32 * 16)) * np.exp(g.uniform(-20, 20, (64, 1)))
    codes, sb = mx.quantize_e8m0_b32(x)
    e = sb.astype(np.int64) - 127
    amax = np.abs(x.reshape(64, 16, 32)).max(-1)
    r = amax / np.ldexp(1.0, e)
    assert np.all((r >= 4) & (r < 8))


def test_mx_dequant_error_bound():
    """|x - deq| <= half the E2M1 step at the element's magnitude (0.5 / 1 / 2 on [0,2] / [2,4] /
    [4,6]) times the block scale, except in the saturated range (6, 8) * 2^e where it is below
    2 * 2^e."""
    g = np.random.default_rng(2)
    x = g.standard_normal((8, 256))
    codes, sb = mx.quantize_e8m0_b32(x)
    d = mx.dequant_e8m0_b32(codes, sb)
    scale = np.repeat(F.e8m0_decode(sb), 32, axis=1)
    err = np.abs(x - d) / scale
    assert np.all(err < 2.0)
    a = np.abs(x) / scale
    half_step = np.where(a <= 2, 0.25, np.where(a <= 4, 0.5, 1.0))
    assert np.all(err[a <= 6] <= half_step[a <= 6] + 1e-12)


def test_e4m3_b16_golden_blocks():
    """Hand-worked E4M3-B16 blocks (MXCode Table 1, row E4M3-B16-FP4) that tell the binary32 step
    order apart from the plausible alternatives (6*ts formed first, one rounding of
    amax/(6*ts), division by ts before 6, the block scale or the quotient taken in float64) and
    drive x/S onto every E2M1 tie, a subnormal block scale and a scale that underflows."""
    with open(os.path.join(GOLDEN, "e4m3_b16_blocks.json")) as f:
        g = json.load(f)["tensor"]
    x = np.array([[_num(v) for blk in g["blocks"] for v in blk["x"]]], dtype=np.float32)
    codes, sb, ts = mx.quantize_e4m3_b16(x)
    assert ts == np.float32(_num(g["ts"]))
    for i, blk in enumerate(g["blocks"]):
        assert int(sb[0, i]) == blk["byte"], blk["note"]
        assert codes[0, 16 * i:16 * i + 16].tolist() == blk["codes"], blk["note"]


def test_e4m3_b16_invariants():
    g = np.random.default_rng(3)
    x = (g.standard_normal((16, 256)) * 3).astype(np.float32)
    codes, sb, ts = mx.quantize_e4m3_b16(x)
    amax_t = np.abs(x).max()
    assert ts == np.float32(np.float32(amax_t) / np.float32(2688.0))
    S = F.e4m3_decode(sb) * float(ts)
    amax_b = np.abs(x.reshape(16, 16, 16)).max(-1)
    # the decoded block scale is amax_b / 6 up to E4M3 relative rounding (2^-4) and the
    # two fp32 roundings
    rel = np.abs(S - amax_b / 6) / (amax_b / 6)
    assert np.all(rel <= 2.0 ** -4 + 1e-6)
    d = mx.dequant_e4m3_b16(codes, sb, ts)
    assert np.all(np.abs(d - x) <= np.repeat(S, 16, axis=1) * 1.0 + 1e-9)


def test_e4m3_b16_zero_tensor_and_underflow():
    x = np.zeros((2, 32), np.float32)
    codes, sb, ts = mx.quantize_e4m3_b16(x)
    assert ts == 1.0 and np.all(sb == 0) and np.all(codes == 0)
    # one huge block and one tiny block: the tiny block's scale underflows to 0 -> codes 0
    x = np.zeros((1, 32), np.float32)
    x[0, 0] = 1e6
    x[0, 16] = 1e-6
    codes, sb, ts = mx.quantize_e4m3_b16(x)
    assert sb[0, 1] == 0 and np.all(codes[0, 16:] == 0)


def test_int4_g128_golden():
    """amax 7 -> s = 1: 7 -> 7, -3.5 -> -4 (tie to even), 0.5 -> 0 (tie to even), 2.5 -> 2."""
    x = np.zeros((1, 128), np.float32)
    x[0, :4] = [7, -3.5, 0.5, 2.5]
    q, s = mx.quantize_int4_g128(x)
    assert s[0, 0] == 1.0
    assert q[0, :4].tolist() == [7, -4, 0, 2]
    q, s = mx.quantize_int4_g128(np.zeros((1, 128), np.float32))
    assert s[0, 0] == 0 and np.all(q == 0)


def test_gemm_bruteforce_32cubed():
    g = np.random.default_rng(4)
    xc = g.integers(0, 16, (32, 32)).astype(np.uint8)
    wc = g.integers(0, 16, (32, 32)).astype(np.uint8)
    xs = g.integers(120, 131, (32, 1)).astype(np.uint8)
    ws = g.integers(120, 131, (32, 1)).astype(np.uint8)
    xd, wd = mx.dequant_e8m0_b32(xc, xs), mx.dequant_e8m0_b32(wc, ws)
    assert np.array_equal(G.gemm_ref(xd, wd), G.naive_gemm(xd, wd))


def test_gemm_integer_special_case():
    """Scale byte 127 (x1) and codes whose magnitudes are integers: the layer reduces to a
    textbook integer matmul."""
    g = np.random.default_rng(6)
    int_codes = np.array([0, 2, 4, 5, 6, 7, 8, 10, 12, 13, 14, 15], dtype=np.uint8)
    xc = int_codes[g.integers(0, len(int_codes), (16, 64))]
    wc = int_codes[g.integers(0, len(int_codes), (24, 64))]
    one = np.full((16, 2), 127, np.uint8)
    xd = mx.dequant_e8m0_b32(xc, one)
    wd = mx.dequant_e8m0_b32(wc, np.full((24, 2), 127, np.uint8))
    xi, wi = xd.astype(np.int64), wd.astype(np.int64)
    assert np.array_equal(xi, xd) and np.array_equal(wi, wd)
    assert np.array_equal(G.gemm_ref(xd, wd), (xi @ wi.T).astype(np.float64))


def test_bf16_rne_matches_torch():
    import torch
    g = np.random.default_rng(7)
    v = np.concatenate([g.standard_normal(50000) * 10.0 ** g.uniform(-30, 30, 50000),
                        np.ldexp(g.integers(1, 1 << 20, 2000).astype(np.float64), -150)])
    v32 = v.astype(np.float32).astype(np.float64)          # fp32-representable inputs
    ref = torch.from_numpy(v32.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(G.bf16_rne(v32), ref)
    ulp = G.bf16_ulp(np.array([1.0, 1.5, 2.0 ** -130]))
    assert ulp.tolist() == [2.0 ** -7, 2.0 ** -7, 2.0 ** -133]
