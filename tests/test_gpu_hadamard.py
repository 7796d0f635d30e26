"""GPU parity of the online block-32 Hadamard in front of MXFP4 activation quantization
(CodeQuant "had" variants): the standalone quantizer (bit-exact codes and scales), linear layers
whose activations pass it (decode kernel, separate quantizer + GEMM, prefill), and the MoE FFN
with x and h rotated."""
import numpy as np
import pytest
import torch

import synth
from oracle import formats as F
from oracle import gemm as G
from oracle import hadamard as Hd
from oracle import mx
from tests._parity import check_bf16, check_fp32

pytestmark = pytest.mark.gpu


def _ql():
    import bit_quantized_moe_tcgen05_b200 as ql
    return ql


def dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _oracle_codes(xb):
    xr = Hd.rotate_activation_f32(synth.bf16_bits_to_f64(xb).astype(np.float32))
    return mx.quantize_e8m0_b32(xr.astype(np.float64))


@pytest.mark.parametrize("M,K", [(1, 32), (16, 2048), (37, 9728), (300, 768)])
def test_quant_hadamard_bitexact(M, K):
    ql = _ql()
    xb, _ = synth.activations_bf16(120 + M, M, K, 0.01, 20.0)
    codes, sb = ql.quantize_act(dev_bf16(xb), had_block=32)
    ql.check()
    rc, rs = _oracle_codes(xb)
    assert np.array_equal(sb.cpu().numpy(), rs)
    assert np.array_equal(codes.cpu().numpy(), F.pack_nibbles(rc))


def test_quant_hadamard_edge_values():
    """Zero blocks, signed zeros, bf16 subnormals, one spike (spread evenly by the rotation),
    a constant block (rotated onto a single element) and rounding-heavy magnitudes."""
    ql = _ql()
    rows = [[0.0] * 32, [-0.0] * 32, [2.0 ** -133 * i for i in range(32)],
            [5.0] + [0.0] * 31, [1.5] * 32, [(-1.0) ** i * 2.0 ** (i % 7) * 1.375 for i in range(32)]]
    g = np.random.default_rng(5)
    rows.append(list(g.standard_normal(32) * 1e-30))
    rows.append(list(g.standard_normal(32) * 3e36))
    xb = synth.to_bf16_bits(np.array(rows, dtype=np.float64))
    codes, sb = ql.quantize_act(dev_bf16(xb), had_block=32)
    ql.check()
    rc, rs = _oracle_codes(xb)
    assert np.array_equal(sb.cpu().numpy(), rs)
    assert np.array_equal(codes.cpu().numpy(), F.pack_nibbles(rc))


@pytest.mark.parametrize("N,K,M", [(1280, 4096, 1), (1280, 4096, 16), (1280, 4096, 64),
                                   (512, 1024, 300)])
def test_hadamard_linear(N, K, M):
    """A layer with the rotation: the weight is W . blockdiag(H_32) / 32 quantized to MXFP4
    (offline, by the oracle); y is compared with the oracle's Q(x H) against the same codes, in
    every decode quantization mode where M <= 64."""
    ql = _ql()
    w = synth.bf16_bits_to_f64(synth.to_bf16_bits(synth.student_t(130 + M, (N, K), 4.0)))
    wc, ws = mx.quantize_e8m0_b32(Hd.rotate_weight(w))
    codes = F.pack_nibbles(wc)
    lin = ql.QLinear(codes, ws, had_block=32)
    xb, _ = synth.activations_bf16(131 + M, M, K, 0.01, 20.0)
    x = dev_bf16(xb)
    xc, xs = _oracle_codes(xb)
    xq = mx.dequant_e8m0_b32(xc, xs)
    wq = mx.dequant_e8m0_b32(wc, ws)
    ref, t = G.gemm_ref(xq, wq), G.abs_scale(xq, wq)
    outs = {}
    try:
        for mode in ((-1, 1, 2, 3) if M <= 64 else (-1,)):
            ql.decode_fuse_mode(mode)
            y32 = torch.empty((M, N), dtype=torch.float32, device="cuda")
            y = lin(x, out_f32=y32)
            ql.check()
            check_fp32(y32.cpu().numpy(), ref, t, f"had M={M} mode {mode}")
            check_bf16(y.float().cpu().numpy(), ref, t, f"had M={M} mode {mode}")
            outs[mode] = y32.cpu().numpy()
    finally:
        ql.decode_fuse_mode(-1)
    if M <= 64:   # the two modes that split K alike sum in the same order
        assert np.array_equal(outs[1], outs[2])
    # the two-call path (separate quantizer, then the GEMM) gives the same bits
    wsp = torch.empty(lin.workspace_bytes(M), dtype=torch.uint8, device="cuda")
    lin.quantize_input(x, wsp)
    y2 = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    y2_32 = torch.empty((M, N), dtype=torch.float32, device="cuda")
    lin.gemm(M, y2, wsp, out_f32=y2_32)
    ql.check()
    assert np.array_equal(y2_32.cpu().numpy(), outs[-1])
    lin.close()


def test_hadamard_layer_matches_unrotated_product():
    """The rotation changes only the quantization: with x and W already exact on the FP4 grid of
    their rotated blocks' scales the product equals x W^T; here checked loosely on Student-t
    weights, relative to the unrotated quantized layer's own error."""
    ql = _ql()
    N, K, M = 256, 1024, 8
    w = synth.bf16_bits_to_f64(synth.to_bf16_bits(synth.student_t(140, (N, K), 4.0)))
    xb, _ = synth.activations_bf16(141, M, K, 0.01, 20.0)
    xd = synth.bf16_bits_to_f64(xb)
    exact = G.gemm_ref(xd, w)
    wc, ws = mx.quantize_e8m0_b32(Hd.rotate_weight(w))
    lin = ql.QLinear(F.pack_nibbles(wc), ws, had_block=32)
    y32 = torch.empty((M, N), dtype=torch.float32, device="cuda")
    lin(dev_bf16(xb), out_f32=y32)
    ql.check()
    lin.close()
    err = np.abs(y32.cpu().numpy() - exact)
    scale = np.abs(xd) @ np.abs(w).T
    assert float((err / scale).max()) < 0.25   # 4-bit operands: the product, not noise


def test_moe_hadamard_small():
    """MoE with x rotated before gate/up and h rotated before down: codes of x and h exact, the
    output within the derived tolerances (the same checks as the unrotated MoE)."""
    from tests.test_gpu_moe import build_model, check_all, _view
    from oracle import moe
    import bit_quantized_moe_tcgen05_b200 as ql
    E, H, I, T, k = 8, 256, 128, 64, 2
    gi, gc, di, dc = build_model(150, E, H, I)
    layer = ql.MoE(gi, gc, di, dc, E, k, had_x=True, had_h=True)
    layer.capture_intermediate(True)
    xb, _ = synth.activations_bf16(150, T, H, 0.0, 1.0)
    logits = synth.zipf_router_logits(150, T, E)
    x = dev_bf16(xb)
    lg = torch.from_numpy(np.ascontiguousarray(logits)).cuda()
    y32 = torch.empty((T, H), dtype=torch.float32, device="cuda")
    ws = layer.workspace(T, x.device)
    y = layer(x, lg, out_f32=y32, ws=ws)
    ql.check()
    lay = layer.layout(T)
    P = T * k
    got = dict(
        y=y.float().cpu().numpy(), y32=y32.cpu().numpy(),
        ids=_view(ws, lay["ids"], P, torch.int32).cpu().numpy().reshape(T, k),
        gates=_view(ws, lay["gates"], P, torch.float32).cpu().numpy().reshape(T, k),
        counts=_view(ws, lay["counts"], E, torch.int32).cpu().numpy(),
        offsets=_view(ws, lay["offsets"], E + 1, torch.int32).cpu().numpy(),
        entries=_view(ws, lay["entries"], P, torch.int32).cpu().numpy(),
        x_codes=_view(ws, lay["x_codes"], T * H // 2, torch.uint8).cpu().numpy().reshape(T, H // 2),
        x_scales=_view(ws, lay["x_scales"], T * H // 32, torch.uint8).cpu().numpy().reshape(T, H // 32),
        h32=_view(ws, lay["h32"], P * I, torch.float32).cpu().numpy().reshape(P, I),
        h_codes=_view(ws, lay["h_codes"], P * I // 2, torch.uint8).cpu().numpy().reshape(P, I // 2),
        h_scales=_view(ws, lay["h_scales"], P * I // 32, torch.uint8).cpu().numpy().reshape(P, I // 32))
    layer.close()
    Wgu = [moe.cluster_weight(gc[e * 2 * I:(e + 1) * 2 * I], gi[e * 2 * I:(e + 1) * 2 * I]) for e in range(E)]
    Wd = [moe.cluster_weight(dc[e * H:(e + 1) * H], di[e * H:(e + 1) * H]) for e in range(E)]
    check_all(got, xb, logits, Wgu, Wd, k, had_x=True, had_h=True)
