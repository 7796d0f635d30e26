"""GPU parity of the MosaicQuant-style INT4 path: the INT4 activation quantizer (bit-exact) and
the fused INT4 dense + block-sparse residual tcgen05 kind::i8 GEMM (float tolerance)."""
import numpy as np
import pytest
import torch

import synth
from oracle import formats as F
from oracle import gemm as G
from oracle import int4bsr
from tests._parity import check_bf16, check_fp32

pytestmark = pytest.mark.gpu


def _ql():
    import bit_quantized_moe_tcgen05_b200 as ql
    return ql


def dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


@pytest.mark.parametrize("M,K", [(1, 128), (16, 8192), (37, 512)])
def test_quant_int4_bitexact(M, K):
    ql = _ql()
    xb, _ = synth.activations_bf16(300 + M, M, K, 0.01, 30.0)
    codes, sc = ql.quantize_act(dev_bf16(xb), fmt=ql.QL_A_INT4_TOK_G128)
    ql.check()
    q, s = int4bsr.quant_act(synth.bf16_bits_to_f64(xb))
    assert np.array_equal(sc.cpu().numpy(), s)
    assert np.array_equal(codes.cpu().numpy(), F.pack_nibbles(F.int4_encode(q)))


def _layer(prep):
    ql = _ql()
    bsr = dict(rowptr=prep["rowptr"], col=prep["col"],
               rcodes=F.pack_nibbles(F.int4_encode(prep["rq"])) if len(prep["sel"]) else np.zeros((0, 16, 64)),
               rscales=prep["rs"].view(np.uint16))
    return ql.QLinear(F.pack_nibbles(F.int4_encode(prep["q"])), prep["sw"].view(np.uint16),
                      wfmt=ql.QL_W_INT4_G128_BSR, bsr=bsr)


def _run_check(prep, xb, what):
    ql = _ql()
    lin = _layer(prep)
    x = dev_bf16(xb)
    y32 = torch.empty((x.shape[0], lin.N), dtype=torch.float32, device="cuda")
    y = lin(x, out_f32=y32)
    ql.check()
    lin.close()
    ref, t = int4bsr.forward(synth.bf16_bits_to_f64(xb), prep)
    check_fp32(y32.cpu().numpy(), ref, t, what)
    check_bf16(y.float().cpu().numpy(), ref, t, what)


@pytest.mark.parametrize("N,K,M,density", [(256, 512, 1, 0.1), (128, 1024, 16, 0.05),
                                           (384, 512, 100, 0.2), (256, 256, 64, 0.0)])
def test_int4_bsr_linear_small(N, K, M, density):
    w = synth.bf16_bits_to_f64(synth.to_bf16_bits(synth.student_t(40 + K, (N, K), 4.0)))
    xc, _ = synth.activations_bf16(41, 64, K, 0.01 * 8, 30.0)
    prep = int4bsr.prepare(w, synth.bf16_bits_to_f64(xc), density=density)
    xb, _ = synth.activations_bf16(42, M, K, 0.01 * 8, 30.0)
    _run_check(prep, xb, f"int4 N={N} K={K} M={M}")


_C5 = {}


def _c5():
    if not _C5:
        wb = synth.to_bf16_bits(synth.student_t(5, (8192, 8192), 4.0))
        xb, _ = synth.activations_bf16(5, 4096, 8192, 0.01, 30.0)
        _C5.update(prep=int4bsr.prepare(synth.bf16_bits_to_f64(wb), synth.bf16_bits_to_f64(xb)), x=xb)
    return _C5


@pytest.mark.parametrize("M", [1, 16, 256, 4096])
def test_int4_bsr_workload_full_size(M):
    """The dense + block-sparse prefill workload: W [8192, 8192] Student-t(4), INT4 per 128-group
    plus 655 residual blocks of 16 x 128 (2 %) chosen by the activation-aware score over the
    4096-token calibration X (1 % outlier channels x30); every output compared."""
    c = _c5()
    assert len(c["prep"]["sel"]) == 655
    xb = np.ascontiguousarray(c["x"][:M])
    _run_check(c["prep"], xb, f"C5 M={M}")
