"""Pins for the oracle's number-format codecs (CPU).

Each test ties a codec to something other than itself: values printed in MXCode Table 1,
hand-worked rounding pairs, or an independent library decoder (torch's float8_e4m3fn).
"""
import json
import os

import numpy as np
import pytest
import torch

from oracle import formats as F
from oracle import mx
from tests.conftest import GOLDEN


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _num(s):
    return float.fromhex(s) if "0x" in s else float(s)


def test_e2m1_value_set():
    vals = F.e2m1_decode(np.arange(16))
    assert sorted(set(np.abs(vals).tolist())) == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert np.all(vals[8:] == -vals[:8])
    assert np.signbit(vals[8])                     # code 0x8 is -0


def test_e2m1_rounding_golden():
    g = _golden("e2m1_rounding.json")
    for s, code in g["pairs"]:
        got = int(F.e2m1_encode(np.array([_num(s)]))[0])
        assert got == code, (s, got, code)


def test_e2m1_roundtrip_all_codes():
    codes = np.arange(16, dtype=np.uint8)
    assert np.array_equal(F.e2m1_encode(F.e2m1_decode(codes)), codes)


def test_e2m1_nearest_over_all_bf16():
    """Every finite bf16 value in [-8, 8] maps to a grid value no farther than any other."""
    bits = np.arange(0, 1 << 16, dtype=np.uint32)
    v = (bits << 16).view(np.float32)
    v = v[np.isfinite(v)].astype(np.float64)
    v = v[np.isfinite(v) & (np.abs(v) <= 8)]
    dec = np.abs(F.e2m1_decode(F.e2m1_encode(v)))
    grid = F.E2M1_MAGNITUDES
    best = np.abs(np.abs(v)[:, None] - grid).min(axis=1)
    assert np.all(np.abs(np.abs(v) - dec) == best)


def test_e8m0_range_table1():
    t = _golden("table1_formats.json")["formats"]["E8M0-B32-FP4"]
    assert F.e8m0_decode(np.array([0]))[0] == _num(t["min_scale"])
    top = F.e8m0_decode(np.array([254]))[0]
    assert abs(top - t["max_scale_printed"]) / t["max_scale_printed"] < 0.005   # "1.70x10^38"
    with pytest.raises(ValueError):
        F.e8m0_decode(np.array([255]))


def test_e4m3_decode_matches_torch():
    b = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn)
    ref = b.to(torch.float64).numpy()
    ours = F.e4m3_decode(np.arange(256))
    both_nan = np.isnan(ref) & np.isnan(ours)
    assert np.all(both_nan | (ref == ours))


def test_e4m3_range_table1():
    t = _golden("table1_formats.json")["formats"]["E4M3-B16-FP4"]
    finite = F.E4M3_TABLE[np.isfinite(F.E4M3_TABLE)]
    assert finite.max() == t["max_scale_printed"]
    assert finite[finite > 0].min() == _num(t["min_scale"])


def test_e4m3_encode_matches_torch_rne():
    g = np.random.default_rng(5)
    v = np.concatenate([g.uniform(0, 448, 20000), np.exp(g.uniform(np.log(2.0**-12), np.log(448), 20000)),
                        F.E4M3_TABLE[:127], (F.E4M3_TABLE[:126] + F.E4M3_TABLE[1:127]) / 2])
    v32 = v.astype(np.float32)
    ref = torch.from_numpy(v32).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = F.e4m3_encode_nonneg(v32.astype(np.float64))
    assert np.array_equal(ours, ref)


def test_e4m3_satfinite():
    assert F.e4m3_encode_nonneg(np.array([448.0, 460.0, 1e9]))[0] == 0x7E
    assert np.all(F.e4m3_encode_nonneg(np.array([460.0, 1e9])) == 0x7E)


def test_ue5m3_range_table1():
    t = _golden("table1_formats.json")["formats"]["E5M3-B16-FP4"]
    v = F.ue5m3_decode(np.arange(256))
    finite = v[np.isfinite(v)]
    assert finite.max() == t["max_scale_printed"]
    assert finite[finite > 0].min() == _num(t["min_scale"])


def test_bpe_from_packed_sizes():
    """Bits per element measured from the packed buffers the quantizers produce."""
    t = _golden("table1_formats.json")["formats"]
    x = np.random.default_rng(0).standard_normal((4, 1024))
    codes, sb = mx.quantize_e8m0_b32(x)
    packed = F.pack_nibbles(codes)
    assert (packed.nbytes + sb.nbytes) * 8 / x.size == t["E8M0-B32-FP4"]["bpe"]
    codes, sb, ts = mx.quantize_e4m3_b16(x.astype(np.float32))
    packed = F.pack_nibbles(codes)
    assert (packed.nbytes + sb.nbytes) * 8 / x.size == t["E4M3-B16-FP4"]["bpe"]


def test_nibble_pack_order():
    codes = np.array([[1, 2, 3, 4]], dtype=np.uint8)
    assert F.pack_nibbles(codes).tolist() == [[0x21, 0x43]]
    assert np.array_equal(F.unpack_nibbles(F.pack_nibbles(codes)), codes)


def test_int4_codec():
    q = np.arange(-7, 8)
    assert np.array_equal(F.int4_decode(F.int4_encode(q)), q)
