"""The C-ABI library loads on a machine without a GPU, exports every entry point that
include/qlinear.h declares, rejects bad arguments before touching the device, and its host-side
offline preparation matches the oracle bit for bit (CPU)."""
import ctypes
import os
import re

import numpy as np
import pytest

import synth
from tests.conftest import ROOT


def _declared_functions():
    with open(os.path.join(ROOT, "include", "qlinear.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*([A-Za-z_][A-Za-z0-9_]*)\s*\(",
                       text, flags=re.M)
    return sorted(set(n for n in names if n not in ("if", "defined")))


def test_library_loads_and_exports_every_declared_symbol():
    import bit_quantized_moe_tcgen05_b200 as ql
    declared = _declared_functions()
    assert len(declared) >= 9
    for name in declared:
        assert hasattr(ql.lib, name), f"{name} declared in qlinear.h but not exported"
    assert set(declared) == set(ql.EXPORTED_SYMBOLS)
    assert b"sm_100a" in ql.lib.ql_version()


def test_bad_arguments_rejected_without_device():
    import bit_quantized_moe_tcgen05_b200 as ql
    h = ctypes.c_void_p()
    assert ql.lib.qlinear_create(None, None, ctypes.byref(h)) == 1
    codes = np.zeros((16, 64), np.uint8)
    scales = np.zeros((16, 4), np.uint8)
    d = ql.WeightDesc(wfmt=1, N=16, K=100, k_tail=0, codes=codes.ctypes.data, scales=scales.ctypes.data)
    assert ql.lib.qlinear_create(ctypes.byref(d), None, ctypes.byref(h)) == 2      # K % 128
    d = ql.WeightDesc(wfmt=1, N=16, K=128, k_tail=128, codes=codes.ctypes.data, scales=scales.ctypes.data)
    assert ql.lib.qlinear_create(ctypes.byref(d), None, ctypes.byref(h)) == 1      # k_tail >= K
    d = ql.WeightDesc(wfmt=1, N=16, K=128, k_tail=0, codes=None, scales=None)
    assert ql.lib.qlinear_create(ctypes.byref(d), None, ctypes.byref(h)) == 1
    assert b"codes" in ql.lib.ql_last_error()
    assert ql.lib.quantize_act(1, None, 4, 32, None, None, None, None) == 1
    assert ql.lib.quantize_act(1, None, 0, 32, None, None, None, None) == 0        # empty is a no-op


@pytest.mark.parametrize("N,C,k,search", [(32, 512, 128, False), (64, 1024, 256, False),
                                          (32, 512, 128, True), (64, 1024, 256, True)])
def test_prquant_host_preparation_matches_oracle(N, C, k, search):
    import bit_quantized_moe_tcgen05_b200 as ql
    from oracle import formats as F, prquant
    wb = synth.to_bf16_bits(synth.student_t(11 + N, (N, C), 3.0))
    perm, codes, scales = ql.prepare_prquant(wb, k, scale_search=search)
    ref = prquant.prepare(synth.bf16_bits_to_f64(wb), k, search=search)
    assert np.array_equal(perm, ref["perm"])
    assert np.array_equal(codes, F.pack_nibbles(ref["w_codes"]))
    assert np.array_equal(scales, ref["w_sb"])


@pytest.mark.parametrize("N,K", [(64, 256), (128, 512)])
def test_vq_prescale_host_preparation_matches_oracle(N, K):
    import bit_quantized_moe_tcgen05_b200 as ql
    from oracle import vq
    wb = synth.to_bf16_bits(synth.student_t(17 + K, (N, K), 4.0))
    w = synth.bf16_bits_to_f64(wb)
    cb = synth.vq_codebooks(17, w)
    ts, sb, idx = ql.prepare_vq_prescale(wb, vq.pack_codebooks(cb))
    ref = vq.prepare(w, cb)
    assert ts == ref["ts"]
    assert np.array_equal(sb, ref["sb"])
    assert np.array_equal(idx, ref["idx"])


@pytest.mark.parametrize("N,K", [(64, 256), (128, 512)])
def test_vq_postscale_host_preparation_matches_oracle(N, K):
    import bit_quantized_moe_tcgen05_b200 as ql
    from oracle import vq
    wb = synth.to_bf16_bits(synth.student_t(19 + K, (N, K), 4.0) * 0.02)
    w = synth.bf16_bits_to_f64(wb)
    cent = synth.vq_raw_codebooks(19, w)
    ts, cbp, qs, idx = ql.prepare_vq_postscale(wb, cent)
    ref = vq.postscale_prepare(w, cent)
    assert ts == ref["ts"]
    assert np.array_equal(qs, ref["sbq"])
    assert np.array_equal(cbp, vq.pack_codebooks(ref["codes"]))
    assert np.array_equal(idx, ref["idx"])


@pytest.mark.parametrize("N,K", [(64, 256), (128, 512)])
def test_vq_prescale_plus_host_preparation_matches_oracle(N, K):
    import bit_quantized_moe_tcgen05_b200 as ql
    from oracle import vq
    wb = synth.to_bf16_bits(synth.student_t(23 + K, (N, K), 4.0))
    w = synth.bf16_bits_to_f64(wb)
    cb = synth.vq_codebooks(23, w)
    _, sb0 = vq.prescale(w)
    scb = synth.scale_codebook(23, sb0, entries=256)
    scb[:40] = synth.scale_codebook(24, sb0, entries=40)       # fewer distinct vectors than groups
    ts, sb, sidx, idx = ql.prepare_vq_prescale_plus(wb, vq.pack_codebooks(cb), scb)
    ref = vq.prescale_plus_prepare(w, cb, scb)
    assert ts == ref["ts"]
    assert np.array_equal(sidx, ref["sidx"])
    assert np.array_equal(sb, ref["sb"])
    assert np.array_equal(idx, ref["idx"])


@pytest.mark.parametrize("N,K,T", [(64, 512, 32), (128, 1024, 16)])
def test_int4_bsr_host_preparation_matches_oracle(N, K, T):
    import bit_quantized_moe_tcgen05_b200 as ql
    from oracle import formats as F, int4bsr
    wb = synth.to_bf16_bits(synth.student_t(23 + K, (N, K), 4.0))
    xb, _ = synth.activations_bf16(23, T, K, 0.01 * 8, 30.0)
    got = ql.prepare_int4_bsr(wb, xb, density=0.05)
    ref = int4bsr.prepare(synth.bf16_bits_to_f64(wb), synth.bf16_bits_to_f64(xb), density=0.05)
    assert np.array_equal(got["codes"], F.pack_nibbles(F.int4_encode(ref["q"])))
    assert np.array_equal(got["scales"], ref["sw"].view(np.uint16))
    assert np.array_equal(got["rowptr"], ref["rowptr"])
    assert np.array_equal(got["col"], ref["col"])
    assert np.array_equal(got["rcodes"].reshape(len(ref["sel"]), 16, 64),
                          F.pack_nibbles(F.int4_encode(ref["rq"])))
    assert np.array_equal(got["rscales"], ref["rs"].view(np.uint16))


def test_decode_mode_and_augmented_quantizer_checks_without_device():
    """Host-side checks of two entry points: the decode organisation switch accepts -1..3 only,
    and the augmented (offline tail copy) quantizer refuses bad formats and shapes before any
    launch; an empty tensor is a no-op."""
    import bit_quantized_moe_tcgen05_b200 as ql
    for bad in (-2, 4, 100):
        assert ql.lib.ql_decode_fuse_mode(bad) == 1
    for good in (0, 1, 2, 3, -1):
        assert ql.lib.ql_decode_fuse_mode(good) == 0   # ends on -1, the measured choice
    assert ql.lib.quantize_act_augmented(1, None, -1, 64, 32, None, None, None) == 1    # negative M
    assert ql.lib.quantize_act_augmented(2, None, 4, 64, 32, None, None, None) == 2     # not MXFP4
    assert ql.lib.quantize_act_augmented(1, None, 4, 64, 16, None, None, None) == 2     # k_tail % 32
    assert ql.lib.quantize_act_augmented(1, None, 4, 64, 96, None, None, None) == 2     # k_tail > C
    assert ql.lib.quantize_act_augmented(1, None, 4, 64, 32, None, None, None) == 1     # null pointers
    assert ql.lib.quantize_act_augmented(1, None, 0, 64, 32, None, None, None) == 0     # empty


def test_moe_arguments_rejected_without_device():
    """moe_create and the MoE workspace / forward calls check their arguments on the host, before
    any device allocation or launch."""
    import bit_quantized_moe_tcgen05_b200 as ql
    h = ctypes.c_void_p()
    codes = np.zeros((256, 64), np.uint8)
    cb = np.zeros((256, 16), np.uint16)
    good = dict(wfmt=4, N=256, K=128, codes=codes.ctypes.data, codebooks=cb.ctypes.data)
    gu, dn = ql.WeightDesc(**good), ql.WeightDesc(**good)
    assert ql.lib.moe_create(None, ctypes.byref(dn), 2, 1, None, ctypes.byref(h)) == 1
    bad_fmt = ql.WeightDesc(**dict(good, wfmt=1))
    assert ql.lib.moe_create(ctypes.byref(bad_fmt), ctypes.byref(dn), 2, 1, None, ctypes.byref(h)) == 2
    for E, k in ((0, 1), (300, 8), (8, 0), (8, 17), (4, 8)):          # 0 < k <= 16, k <= E <= 256
        assert ql.lib.moe_create(ctypes.byref(gu), ctypes.byref(dn), E, k, None, ctypes.byref(h)) == 2
    no_cb = ql.WeightDesc(**dict(good, codebooks=None))
    assert ql.lib.moe_create(ctypes.byref(no_cb), ctypes.byref(dn), 2, 1, None, ctypes.byref(h)) == 1
    uneven = ql.WeightDesc(**dict(good, N=250))
    assert ql.lib.moe_create(ctypes.byref(uneven), ctypes.byref(dn), 4, 1, None, ctypes.byref(h)) == 1
    nbytes = ctypes.c_size_t()
    assert ql.lib.moe_workspace_bytes(None, 16, ctypes.byref(nbytes)) == 1
    assert ql.lib.moe_grouped_forward(None, None, 16, None, None, None, None, None, None, 0, None) == 1


def test_offline_preparation_rejects_bad_arguments():
    """The host preparation entries refuse null buffers and unsupported shapes (CPU only)."""
    import bit_quantized_moe_tcgen05_b200 as ql
    w = np.zeros((128, 256), np.uint16)
    perm = np.zeros(256, np.int32)
    codes = np.zeros((128, 256), np.uint8)
    sc = np.zeros((128, 16), np.uint8)
    P = lambda a: a.ctypes.data
    f = ql.lib.qlinear_prepare_prquant_ex
    assert f(None, 128, 256, 128, 0, P(perm), P(codes), P(sc)) == 1          # null weight
    assert f(P(w), 128, 256, 0, 0, P(perm), P(codes), P(sc)) == 1            # k = 0
    assert f(P(w), 128, 256, 384, 0, P(perm), P(codes), P(sc)) == 1          # k > C
    assert f(P(w), 128, 256, 64, 0, P(perm), P(codes), P(sc)) == 2           # k % 128
    assert f(P(w), 128, 200, 128, 0, P(perm), P(codes), P(sc)) == 2          # C % 128
    ts = np.zeros(1, np.float32)
    cbk = np.zeros(4096, np.uint8)
    idx = np.zeros((128, 64), np.uint8)
    g = ql.lib.qlinear_prepare_vq_prescale
    assert g(P(w), 128, 256, None, 64, 64, P(ts), P(sc), P(idx)) == 1          # null codebooks
    assert g(P(w), 128, 256, P(cbk), 32, 64, P(ts), P(sc), P(idx)) == 2        # QBlock not 64 x 64
    assert g(P(w), 100, 256, P(cbk), 64, 64, P(ts), P(sc), P(idx)) == 2        # N % 64
