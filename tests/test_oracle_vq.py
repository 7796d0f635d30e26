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


# ------------------------------------------------------------------ PostScale / PreScale+
def test_postscale_codebook_quantization_hand_worked():
    """Two QBlock codebooks; the tensor maximum 2688 makes ts = 1 exactly.  Codebook 0 has amax
    2688: s = E4M3(448) = 0x7e, S = 448; 2688 -> 6 (code 7), -896 -> -2 (code 12), 672 -> 1.5
    (code 3).  Codebook 1 has amax 3: s = E4M3(0.5) = 0x30, S = 0.5; 3 -> 6 (7), 0.75 -> 1.5 (3),
    -0.375 -> -0.75 -> tie between 0.5 and 1.0 -> 1.0 (code 10), 0.125 -> 0.25 -> tie -> 0."""
    cent = np.zeros((1, 2, 256, 4), np.float32)
    cent[0, 0, 0, :3] = [2688.0, -896.0, 672.0]
    cent[0, 1, 0, :4] = [3.0, 0.75, -0.375, 0.125]
    codes, sb, ts = vq.postscale_quantize_codebooks(cent)
    assert ts == np.float32(1.0)
    assert sb.tolist() == [[0x7E, 0x30]]
    assert codes[0, 0, 0, :3].tolist() == [7, 12, 3]
    assert codes[0, 1, 0].tolist() == [7, 3, 10, 0]
    assert np.all(codes[0, 0, 1:] == 0) and np.all(codes[0, 1, 1:] == 0)


def test_postscale_assignment_bruteforce_tiny():
    """Nearest quantized entry in value space, explicit loops, first minimum wins."""
    g = np.random.default_rng(21)
    cent = (g.standard_normal((1, 1, 256, 4)) * 0.05).astype(np.float32)
    codes, sb, ts = vq.postscale_quantize_codebooks(cent)
    codes[0, 0, 9] = codes[0, 0, 4]                       # duplicate entry: index 4 must win
    w = synth.bf16_bits_to_f64(synth.to_bf16_bits(g.standard_normal((64, 64)) * 0.05))
    S = float(F.e4m3_decode(sb)[0, 0] * np.float64(ts))     # the operand's exact scale
    w[0, :4] = F.e2m1_decode(codes[0, 0, 4]) * S           # exactly entry 4
    idx = vq.postscale_assign(w, codes, sb, ts)
    vals = F.e2m1_decode(codes[0, 0]) * S
    for r, j in itertools.product(range(0, 64, 9), range(16)):
        p = w[r, 4 * j:4 * j + 4]
        best, bd = 0, None
        for e in range(256):
            d = sum((float(p[i]) - float(vals[e, i])) ** 2 for i in range(4))
            if bd is None or d < bd:
                best, bd = e, d
        assert idx[r, j] == best
    assert idx[0, 0] == 4


def test_postscale_operand_is_mx_native_and_bpe():
    """The decoded weight of a QBlock is E2M1 codes times ONE scale (so every 16-block of the
    operand shares it: MX-native), and the stored bits per weight are 2.0 (indices) plus 512 B of
    codebook and one scale byte per 64 x 64 QBlock."""
    g = np.random.default_rng(22)
    w = synth.bf16_bits_to_f64(synth.to_bf16_bits(g.standard_t(4, (128, 128)) * 0.02))
    cent = synth.vq_raw_codebooks(22, w)
    p = vq.postscale_prepare(w, cent)
    sb16 = vq.postscale_block_scales(p["sbq"], 128, 128)
    assert sb16.shape == (128, 8)
    for qr in range(2):
        for qc in range(2):
            assert np.all(sb16[qr * 64:(qr + 1) * 64, qc * 4:(qc + 1) * 4] == p["sbq"][qr, qc])
    wd = mx.dequant_e4m3_b16(vq.decode_codes(p["idx"], p["codes"]), sb16, p["ts"])
    scale = F.e4m3_decode(p["sbq"][0, 0]) * np.float64(p["ts"])       # one real scale per QBlock
    assert np.array_equal(wd[:64, :64],
                          F.e2m1_decode(vq.decode_codes(p["idx"], p["codes"]))[:64, :64] * scale)
    bits = p["idx"].nbytes * 8 + vq.pack_codebooks(p["codes"]).nbytes * 8 + p["sbq"].nbytes * 8
    assert bits / w.size == 2.0 + (512 * 8 + 8) / (64 * 64)


def test_prescale_plus_scale_assignment_bruteforce_with_ties():
    g = np.random.default_rng(23)
    sb = g.integers(0x20, 0x50, (6, 32), dtype=np.uint8)
    scb = g.integers(0x20, 0x50, (256, 8), dtype=np.uint8)
    scb[17] = scb[5]                                       # a duplicate: index 5 must win
    sb[0, :8] = scb[5]
    sidx = vq.prescale_plus_assign_scales(sb, scb)
    vals = F.e4m3_decode(scb)
    for n in range(6):
        for gi in range(4):
            v = F.e4m3_decode(sb[n, 8 * gi:8 * gi + 8])
            d = [sum((float(v[i]) - float(vals[e, i])) ** 2 for i in range(8)) for e in range(256)]
            assert sidx[n, gi] == int(np.argmin(d))
    assert sidx[0, 0] == 5
    comp = vq.prescale_plus_scales(sidx, scb)
    assert comp.shape == sb.shape and np.array_equal(comp[0, :8], scb[5])


def test_prescale_plus_with_exact_scale_codebook_is_prescale():
    """When every group of 8 PreScale scales is itself an entry of the scale codebook, the
    compressed scales are the original ones and PreScale+ prepares exactly what PreScale does."""
    w = _weight(N=64, K=256)
    cb = synth.vq_codebooks(24, w)
    ts, sb = vq.prescale(w)
    groups = np.unique(sb.reshape(-1, 8), axis=0)
    assert len(groups) <= 256
    scb = np.zeros((256, 8), np.uint8)
    scb[:len(groups)] = groups
    p_plus = vq.prescale_plus_prepare(w, cb, scb)
    p = vq.prepare(w, cb)
    assert np.array_equal(p_plus["sb"], p["sb"]) and np.array_equal(p_plus["idx"], p["idx"])
    assert p_plus["ts"] == p["ts"]
    # scale storage: 8-bit indices per 8 x 16 weights = 0.0625 bits per weight
    assert p_plus["sidx"].nbytes * 8 / w.size == 8 / 128
