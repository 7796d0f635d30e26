"""GPU parity: MX activation quantizer (bit-exact) and the tcgen05 block-scaled FP4 GEMM with the
PRQuant K-extension (float tolerance), through the C ABI, against the CPU oracle."""
import numpy as np
import pytest
import torch

import synth
from oracle import formats as F
from oracle import gemm as G
from oracle import mx, prquant
from tests._parity import check_bf16, check_fp32

pytestmark = pytest.mark.gpu


def _ql():
    import bit_quantized_moe_tcgen05_b200 as ql
    return ql


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


# ----------------------------------------------------------------------------- quantizer
@pytest.mark.parametrize("M,K", [(1, 32), (16, 2048), (5, 96), (37, 9728), (300, 768)])
def test_quant_mx_bitexact(M, K):
    ql = _ql()
    xb, _ = synth.activations_bf16(100 + M, M, K, 0.01, 20.0)
    codes, sb = ql.quantize_act(dev_bf16(xb))
    ql.check()
    rc, rs = mx.quantize_e8m0_b32(synth.bf16_bits_to_f64(xb))
    assert np.array_equal(sb.cpu().numpy(), rs)
    assert np.array_equal(codes.cpu().numpy(), F.pack_nibbles(rc))


def test_quant_mx_edge_values():
    """Zero blocks, signed zeros, bf16 subnormals, the largest bf16, every E2M1 rounding
    midpoint, and blocks whose amax saturates (amax / 2^e in (6, 8))."""
    ql = _ql()
    rows = []
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.5, 7.0, 7.5]
    rows.append(mids + [-v for v in mids] + [0.0, -0.0] + [0.1] * 10)
    rows.append([0.0] * 32)
    rows.append([-0.0] * 32)
    rows.append([2.0 ** -133 * i for i in range(32)])                 # bf16 subnormals
    rows.append([3.3895313892515355e38] + [1e37] * 31)                 # bf16 max
    rows.append([2.0 ** -125, 2.0 ** -126, 1.5 * 2.0 ** -127, 2.0 ** -130] + [0.0] * 28)
    rows.append([7.0 * 2.0 ** 20] + [-5.0 * 2.0 ** 20] * 31)
    g = np.random.default_rng(0)
    rows.append(list(g.standard_normal(32) * 1e-30))
    x = np.array(rows, dtype=np.float64)
    xb = synth.to_bf16_bits(x)
    codes, sb = ql.quantize_act(dev_bf16(xb))
    ql.check()
    rc, rs = mx.quantize_e8m0_b32(synth.bf16_bits_to_f64(xb))
    assert np.array_equal(sb.cpu().numpy(), rs)
    assert np.array_equal(codes.cpu().numpy(), F.pack_nibbles(rc))


# ----------------------------------------------------------------------------- GEMM
def random_mx_weight(seed, N, K):
    """Uniform random E2M1 codes and E8M0 bytes in [120, 130] (the MXFP4 linear workload)."""
    codes = synth.uniform_nibble_bytes(seed, N, K)
    sb = synth.uniform_bytes(seed + 1, (N, K // 32), 120, 130)
    return codes, sb


def run_gpu(codes, sb, k_tail, xb):
    ql = _ql()
    lin = ql.QLinear(codes, sb, k_tail=k_tail)
    x = dev_bf16(xb)
    y32 = torch.empty((x.shape[0], lin.N), dtype=torch.float32, device="cuda")
    y = lin(x, out_f32=y32)
    ql.check()
    out = y.float().cpu().numpy(), y32.cpu().numpy()
    lin.close()
    return out


def run_oracle(codes, sb, k_tail, xb):
    xd = synth.bf16_bits_to_f64(xb)
    if k_tail:
        xc, xs = prquant.quantize_activation_augmented(xd, k_tail)
    else:
        xc, xs = mx.quantize_e8m0_b32(xd)
    xq = mx.dequant_e8m0_b32(xc, xs)
    wq = mx.dequant_e8m0_b32(F.unpack_nibbles(codes), sb)
    return G.gemm_ref(xq, wq), G.abs_scale(xq, wq)


def check_linear(codes, sb, k_tail, xb, what):
    y, y32 = run_gpu(codes, sb, k_tail, xb)
    ref, t = run_oracle(codes, sb, k_tail, xb)
    check_fp32(y32, ref, t, what)
    check_bf16(y, ref, t, what)


def test_mxfp4_linear_workload_m16():
    """The single MXFP4 linear layer: X [16, 2048] with 1% outlier channels x20, W [2048, 2048]."""
    codes, sb = random_mx_weight(1, 2048, 2048)
    xb, _ = synth.activations_bf16(1, 16, 2048, 0.01, 20.0)
    check_linear(codes, sb, 0, xb, "C1")


@pytest.mark.parametrize("M", [1, 7, 16, 33, 64, 100, 129, 256, 300])
def test_fp4_gemm_token_counts(M):
    """Every token-tile width (8..256), split-K for small M, a ragged last token tile."""
    codes, sb = random_mx_weight(7, 256, 1024)
    xb, _ = synth.activations_bf16(7, M, 1024, 0.01, 20.0)
    check_linear(codes, sb, 0, xb, f"M={M}")


@pytest.mark.parametrize("N,K", [(272, 512), (128, 384), (16, 128), (2560, 2048)])
def test_fp4_gemm_ragged_shapes(N, K):
    """N not a multiple of the 128-row weight tile; K ending in a half stage; tiny problem."""
    codes, sb = random_mx_weight(9, N, K)
    xb, _ = synth.activations_bf16(9, 40, K, 0.01, 20.0)
    check_linear(codes, sb, 0, xb, f"N={N} K={K}")


def test_fp4_gemm_bruteforce_tiny():
    """32 tokens x 32 outputs x 128 channels against a pure-Python triple loop."""
    codes, sb = random_mx_weight(13, 32, 128)
    xb, _ = synth.activations_bf16(13, 32, 128, 0.0, 1.0)
    y, y32 = run_gpu(codes, sb, 0, xb)
    xc, xs = mx.quantize_e8m0_b32(synth.bf16_bits_to_f64(xb))
    xq = mx.dequant_e8m0_b32(xc, xs)
    wq = mx.dequant_e8m0_b32(F.unpack_nibbles(codes), sb)
    check_fp32(y32, G.naive_gemm(xq, wq), G.abs_scale(xq, wq), "tiny")


@pytest.mark.parametrize("N,C,k,M,search", [(256, 512, 128, 8, False), (256, 640, 256, 100, False),
                                            (128, 384, 128, 300, False), (384, 1024, 384, 1, False),
                                            (256, 1024, 256, 16, True), (256, 1024, 128, 300, True)])
def test_prquant_tail_gemm_small(N, C, k, M, search):
    """PRQuant augmented GEMM, with the OCP block scales or the E8M0-W block-scale search (§5.3)."""
    w = synth.bf16_bits_to_f64(synth.to_bf16_bits(synth.student_t(21 + C, (N, C), 3.0)))
    prep = prquant.prepare(w, k, search=search)
    xb, _ = synth.activations_bf16(21, M, C, 0.005 * 8, 50.0)
    xpb = np.ascontiguousarray(xb[:, prep["perm"]])
    check_linear(F.pack_nibbles(prep["w_codes"]), prep["w_sb"], k, xpb, f"tail N={N} C={C} k={k} M={M}")


_C3 = {}


def _c3_prep():
    if not _C3:
        wb = synth.to_bf16_bits(synth.student_t(3, (2560, 9728), 3.0))
        prep = prquant.prepare(synth.bf16_bits_to_f64(wb), 128)
        _C3.update(prep=prep, codes=F.pack_nibbles(prep["w_codes"]))
    return _C3


@pytest.mark.parametrize("M", [16, 512, 2048])
def test_prquant_workload_full_size(M):
    """The PRQuant tail-residual workload at its full size: W [2560, 9728] Student-t(3), k = 128
    (K' = 9856), X with 0.5% outlier channels x50, every output element compared."""
    c3 = _c3_prep()
    xb, _ = synth.activations_bf16(3, M, 9728, 0.005, 50.0)
    xpb = np.ascontiguousarray(xb[:, c3["prep"]["perm"]])
    check_linear(c3["codes"], c3["prep"]["w_sb"], 128, xpb, f"C3 M={M}")


def test_forward_is_deterministic_and_reentrant():
    """Repeated calls (split-K tickets reset in between) give bit-identical outputs."""
    ql = _ql()
    codes, sb = random_mx_weight(5, 1024, 2048)
    xb, _ = synth.activations_bf16(5, 4, 2048, 0.01, 20.0)
    lin = ql.QLinear(codes, sb)
    x = dev_bf16(xb)
    outs = [lin(x).clone() for _ in range(3)]
    ql.check()
    for o in outs[1:]:
        assert torch.equal(o, outs[0])
    lin.close()


@pytest.mark.parametrize("M", [1, 16, 64])
def test_gemm_repeat_without_requantize(M):
    """The GEMM run again and again on one quantized input (qlinear_quantize_input once) reproduces
    the forward's output bit for bit: the split-K hand-off needs nothing re-armed between launches,
    and the one-launch forward (quantizer fused in) computes the same bits as the two calls."""
    ql = _ql()
    codes, sb = random_mx_weight(17, 2560, 2048)
    xb, _ = synth.activations_bf16(17, M, 2048, 0.01, 20.0)
    lin = ql.QLinear(codes, sb)
    x = dev_bf16(xb)
    ws = torch.empty(lin.workspace_bytes(M), dtype=torch.uint8, device="cuda")
    ref = lin.forward(x, ws=ws).clone()
    lin.quantize_input(x, ws)
    outs = []
    for _ in range(3):
        y = torch.empty_like(ref)
        lin.gemm(M, y, ws)
        outs.append(y)
    ql.check()
    for o in outs:
        assert torch.equal(o, ref)
    lin.close()


@pytest.mark.parametrize("N,K,M", [(2560, 2048, 300), (1280, 4096, 520), (2048, 1024, 2048),
                                   (2560, 1024, 2000)])
def test_fp4_gemm_prefill_shapes(N, K, M):
    """Prefill shapes: 256-token tiles, split-K across a few CTAs where the tiles alone do not fill
    the SMs, ragged token tiles; 2560 x 2000 runs ragged 160-token tiles."""
    codes, sb = random_mx_weight(23, N, K)
    xb, _ = synth.activations_bf16(23, M, K, 0.01, 20.0)
    check_linear(codes, sb, 0, xb, f"prefill N={N} K={K} M={M}")


@pytest.mark.parametrize("M,C,k", [(1, 1024, 128), (37, 640, 64), (300, 9728, 128), (5, 96, 32)])
def test_quant_augmented_bitexact(M, C, k):
    """quantize_act with k_tail (PRQuant's offline tail copy): Q(x) followed by a copy of the codes
    and scales of its last k channels, against the oracle's augmented activation."""
    ql = _ql()
    xb, _ = synth.activations_bf16(170 + M, M, C, 0.005, 50.0)
    codes, sb = ql.quantize_act(dev_bf16(xb), k_tail=k)
    ql.check()
    rc, rs = prquant.quantize_activation_augmented(synth.bf16_bits_to_f64(xb), k)
    assert np.array_equal(sb.cpu().numpy(), rs)
    assert np.array_equal(codes.cpu().numpy(), F.pack_nibbles(rc))


@pytest.mark.parametrize("M", [1, 16, 64, 300])
def test_prquant_offline_tail_copy_layer(M):
    """A PRQuant layer whose quantizer writes the augmented activation (tail_copy) computes the
    same bits as the online layer (the GEMM reading the tail twice), in the one-launch forward and
    through quantize_input + gemm, in every decode organisation, and matches the oracle."""
    ql = _ql()
    N, C, k = 512, 2048, 256
    w = synth.bf16_bits_to_f64(synth.to_bf16_bits(synth.student_t(180, (N, C), 3.0)))
    prep = prquant.prepare(w, k)
    codes = F.pack_nibbles(prep["w_codes"])
    online = ql.QLinear(codes, prep["w_sb"], k_tail=k)
    offline = ql.QLinear(codes, prep["w_sb"], k_tail=k, tail_copy=True)
    xb, _ = synth.activations_bf16(181 + M, M, C, 0.005, 50.0)
    x = dev_bf16(np.ascontiguousarray(xb[:, prep["perm"]]))
    xq = mx.dequant_e8m0_b32(*prquant.quantize_activation_augmented(synth.bf16_bits_to_f64(
        np.ascontiguousarray(xb[:, prep["perm"]])), k))
    wq = mx.dequant_e8m0_b32(prep["w_codes"], prep["w_sb"])
    ref, t = G.gemm_ref(xq, wq), G.abs_scale(xq, wq)
    try:
        for mode in ((-1, 0, 1, 2, 3) if M <= 64 else (-1,)):
            ql.decode_fuse_mode(mode)
            outs = []
            for lin in (online, offline):
                y32 = torch.empty((M, N), dtype=torch.float32, device="cuda")
                lin(x, out_f32=y32)
                ws = torch.empty(lin.workspace_bytes(M), dtype=torch.uint8, device="cuda")
                lin.quantize_input(x, ws)
                y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
                y2_32 = torch.empty((M, N), dtype=torch.float32, device="cuda")
                lin.gemm(M, y, ws, out_f32=y2_32)
                ql.check()
                outs += [y32.cpu().numpy(), y2_32.cpu().numpy()]
            check_fp32(outs[0], ref, t, f"online M={M} mode {mode}")
            for o in outs[1:]:
                assert np.array_equal(o, outs[0]), f"M={M} mode {mode}: offline / two-call differ"
    finally:
        ql.decode_fuse_mode(-1)
    online.close()
    offline.close()
