"""qlinear_forward_fixed_scratch: the forward for callers that may not allocate device memory
(an engine that pre-plans all device memory, a plugin without an allocator, a latency-critical
loop).  It must give the same result as qlinear_forward, call after call, using only the
library's fixed scratch array.  This file is collected last on purpose."""
import numpy as np
import pytest
import torch

import synth
from oracle import formats as F
from oracle import gemm as G
from oracle import mx

pytestmark = pytest.mark.gpu


def _layer_inputs(seed, N, K):
    codes = synth.uniform_nibble_bytes(seed, N, K)
    sb = synth.uniform_bytes(seed + 1, (N, K // 32), 120, 130)
    return codes, sb


@pytest.mark.parametrize("M", [16, 100])
def test_fixed_scratch_forward_matches_forward_two_calls(M):
    import bit_quantized_moe_tcgen05_b200 as ql
    N, K = 1024, 2048
    codes, sb = _layer_inputs(31, N, K)
    lin = ql.QLinear(codes, sb)
    wq = mx.dequant_e8m0_b32(F.unpack_nibbles(codes), sb)
    for call in range(2):                       # two calls in a row, different inputs
        xb, _ = synth.activations_bf16(40 + call, M, K, 0.01, 20.0)
        x = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).cuda()
        ref32 = torch.empty((M, N), dtype=torch.float32, device="cuda")
        ref = lin.forward(x, out_f32=ref32)
        got32 = torch.empty((M, N), dtype=torch.float32, device="cuda")
        got = lin.forward_fixed_scratch(x, out_f32=got32)
        ql.check()
        xc, xs = mx.quantize_e8m0_b32(synth.bf16_bits_to_f64(xb))
        t = G.abs_scale(mx.dequant_e8m0_b32(xc, xs), wq)
        a, b = got32.cpu().numpy().astype(np.float64), ref32.cpu().numpy().astype(np.float64)
        assert np.all(np.abs(a - b) <= 1e-5 * t), f"call {call}: fp32 outputs differ"
        ya, yb = got.float().cpu().numpy().astype(np.float64), ref.float().cpu().numpy().astype(np.float64)
        assert np.all(np.abs(ya - yb) <= G.bf16_ulp(yb) + 1e-5 * t), f"call {call}: bf16 outputs differ"
    lin.close()


def test_fixed_scratch_rejects_m_beyond_its_size():
    import bit_quantized_moe_tcgen05_b200 as ql
    codes, sb = _layer_inputs(33, 1024, 2048)
    lin = ql.QLinear(codes, sb)
    M = 8192                                    # needs far more than the fixed scratch holds
    assert lin.workspace_bytes(M) > (8 << 20)
    x = torch.zeros((M, 2048), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ql.QLError) as e:
        lin.forward_fixed_scratch(x)
    assert e.value.status == 6 and "8 MiB" in str(e.value)
    lin.close()


def test_fixed_scratch_layers_of_different_formats_take_turns():
    """Three layers of different formats share the one fixed scratch array, call after call: a VQ
    layer at 64 x 9728 (one-launch decode forward, whose grid-wide agreement keeps a launch
    counter and tagged words in the scratch), an INT4 + block-sparse layer (whose activation
    codes start right after those words) and an MXFP4 layer.  Every call must reproduce, bit for
    bit, the same layer's forward on a private workspace."""
    import bit_quantized_moe_tcgen05_b200 as ql
    from oracle import int4bsr
    g = np.random.default_rng(77)
    N, K = 256, 9728
    cb = g.integers(0, 16, (N // 64, K // 64, 256, 4), dtype=np.uint8)
    vql = ql.QLinear(None, g.integers(0x28, 0x48, (N, K // 16), dtype=np.uint8),
                     wfmt=ql.QL_W_VQ_PRESCALE_E4M3_B16, w_tensor_scale=0.0071,
                     indices=g.integers(0, 256, (N, K // 4), dtype=np.uint8),
                     codebooks=F.pack_nibbles(cb))
    w4 = synth.bf16_bits_to_f64(synth.to_bf16_bits(synth.student_t(78, (256, 1024), 4.0)))
    xc, _ = synth.activations_bf16(79, 64, 1024, 0.08, 30.0)
    p4 = int4bsr.prepare(w4, synth.bf16_bits_to_f64(xc), density=0.1)
    i4l = ql.QLinear(F.pack_nibbles(F.int4_encode(p4["q"])), p4["sw"].view(np.uint16),
                     wfmt=ql.QL_W_INT4_G128_BSR,
                     bsr=dict(rowptr=p4["rowptr"], col=p4["col"],
                              rcodes=F.pack_nibbles(F.int4_encode(p4["rq"])),
                              rscales=p4["rs"].view(np.uint16)))
    codes, sb = _layer_inputs(80, 1024, 2048)
    mxl = ql.QLinear(codes, sb)
    cases = [(vql, 64, K), (i4l, 16, 1024), (mxl, 16, 2048)]
    for rnd in range(3):
        for i, (lin, M, KK) in enumerate(cases):
            xb, _ = synth.activations_bf16(90 + 7 * rnd + i, M, KK, 0.01, 20.0)
            x = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).cuda()
            ws = torch.empty(lin.workspace_bytes(M), dtype=torch.uint8, device="cuda")
            ref32 = torch.empty((M, lin.N), dtype=torch.float32, device="cuda")
            ref = lin.forward(x, out_f32=ref32, ws=ws).clone()
            got32 = torch.empty((M, lin.N), dtype=torch.float32, device="cuda")
            got = lin.forward_fixed_scratch(x, out_f32=got32)
            ql.check()
            assert torch.equal(got, ref), f"round {rnd} layer {i}: bf16 outputs differ"
            assert torch.equal(got32, ref32), f"round {rnd} layer {i}: fp32 outputs differ"
    for lin, _, _ in cases:
        lin.close()
