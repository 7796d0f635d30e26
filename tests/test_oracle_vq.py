"""Pins for the oracle's MXCode PreScale VQ path (CPU)."""
import itertools
import json
import os

import numpy as np

import synth
from oracle import formats as F
from oracle import mx, vq
from tests.conftest import GOLDEN


def _table():
    with open(os.path.join(GOLDEN, "table1_formats.json")) as f:
        return json.load(f)


def _weight(N=128, K=256, seed=2):
    return synth.bf16_bits_to_f64(synth.to_bf16_bits(synth.student_t(seed, (N, K), 4.0)))


def test_index_bpe_and_lut_size_printed():
    """VQ index BPE = log2(K)/d = 2.0 for K = 256, d = 4; an FP4 codebook of 256 x 4 E2M1 entries
    is 512 B, within the 1 KB LUT budget."""
    t = _table()["vq"]
    w = _weight()
    cb = synth.vq_codebooks(2, w)
    prep = vq.prepare(w, cb)
    assert prep["idx"].nbytes * 8 / w.size == t["index_bpe"] == np.log2(t["K"]) / t["d"]
    packed = vq.pack_codebooks(cb)
    per_lut = packed[0, 0].nbytes
    assert per_lut == t["K"] * t["d"] * 4 // 8 == 512 and per_lut <= t["lut_max_bytes"]


def test_prescale_scales_equal_the_e4m3_b16_rule():
    w = _weight()
    ts, sb = vq.prescale(w)
    _, sb2, ts2 = mx.quantize_e4m3_b16(w.astype(np.float32))
    assert ts == ts2 and np.array_equal(sb, sb2)
    assert ts == np.float32(np.float32(np.abs(w).max()) / np.float32(2688.0))


def test_normalized_golden():
    """Hand-worked PreScale normalisation v = w / RN(dec(s) * ts) (MXCode abstract, Table 1):
    values chosen so that dividing by the two scales one after the other, multiplying by the
    reciprocal, or dividing in float64 would each give a different binary32 result; an all-zero
    block (scale byte 0) gives v = 0."""
    with open(os.path.join(GOLDEN, "vq_normalized.json")) as f:
        g = json.load(f)
    num = lambda s: float.fromhex(s) if "0x" in s else float(s)
    w = np.array([[num(v) for v in g["w"]]], dtype=np.float32)
    ts, sb = vq.prescale(w)
    assert ts == np.float32(num(g["ts"])) and sb[0].tolist() == g["bytes"]
    v = vq.normalized(w, sb, ts)
    assert v.dtype == np.float32
    for k, want in g["v"].items():
        assert v[0, int(k)] == np.float32(num(want)), k
    assert np.all(v[0, 16:32] == 0) and np.all(v[0, 35:] == 0) and np.all(v[0, 1:16] == 0)


def test_assignment_bruteforce_tiny():
    """Nearest entry by explicit loops over every entry, first minimum wins."""
    g = np.random.default_rng(9)
    cb = g.integers(0, 16, (1, 1, 256, 4)).astype(np.uint8)
    cb[0, 0, 7] = cb[0, 0, 3]                      # a duplicated entry: index 3 must win
    v = g.uniform(-6, 6, (64, 64)).astype(np.float32)
    v[0, :4] = F.e2m1_decode(cb[0, 0, 3])           # exactly an entry
    idx = vq.assign(v, cb)
    vals = F.e2m1_decode(cb[0, 0])
    for r, j in itertools.product(range(0, 64, 7), range(16)):
        p = v[r, 4 * j:4 * j + 4].astype(np.float64)
        best, bd = 0, None
        for e in range(256):
            d = sum((float(p[i]) - float(vals[e, i])) ** 2 for i in range(4))
            if bd is None or d < bd:
                best, bd = e, d
        assert idx[r, j] == best
    assert idx[0, 0] == 3


def test_decode_selects_codebook_entries():
    w = _weight()
    cb = synth.vq_codebooks(2, w)
    prep = vq.prepare(w, cb)
    codes = vq.decode_codes(prep["idx"], cb)
    for n, j in [(0, 0), (5, 17), (127, 63), (64, 40)]:
        e = prep["idx"][n, j]
        assert np.array_equal(codes[n, 4 * j:4 * j + 4], cb[n // 64, (4 * j) // 64, e])


def test_synthetic_codebook_sqnr_plausible():
    """MXCode Figure 2 sets SQNR >= 10 dB as a design constraint; the seeded k-means synthesis of
    this workload lands above it (a plausibility check on the synthetic data, not a parity pin)."""
    w = _weight(N=128, K=512)
    cb = synth.vq_codebooks(2, w)
    prep = vq.prepare(w, cb)
    wd = vq.dequant_weight(prep["idx"], cb, prep["sb"], prep["ts"])
    sqnr = 10 * np.log10((w ** 2).sum() / ((w - wd) ** 2).sum())
    assert sqnr >= 10.0
