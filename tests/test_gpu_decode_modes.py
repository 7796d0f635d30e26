"""GPU parity of the decode kernel's organisations (M <= 64): the cooperative mode (activation
units shared out over the grid, stage tiles exchanged through the workspace), the local mode
(every CTA quantizes its own K stages into shared memory; the E4M3 tensor amax read from all of
x, or gathered over the grid for larger x) and the cluster mode (the local mode with each weight
tile's K-splits in one thread-block cluster: amax shares and split-K partials meet in distributed
shared memory).  Each mode against the CPU oracle, and the two modes that split K alike
against each other bit for bit."""
import numpy as np
import pytest
import torch

import synth
from oracle import formats as F
from oracle import gemm as G
from oracle import mx, prquant, vq
from tests._parity import check_bf16, check_fp32

pytestmark = pytest.mark.gpu

MODES = (-1, 0, 1, 2, 3)


def _ql():
    import bit_quantized_moe_tcgen05_b200 as ql
    return ql


def dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _run_modes(lin, xb):
    """y (bf16 as float) and y32 per mode; the mode is restored to -1 afterwards."""
    ql = _ql()
    x = dev_bf16(xb)
    out = {}
    try:
        for mode in MODES:
            ql.decode_fuse_mode(mode)
            y32 = torch.empty((x.shape[0], lin.N), dtype=torch.float32, device="cuda")
            y = lin(x, out_f32=y32)
            ql.check()
            out[mode] = (y.float().cpu().numpy(), y32.cpu().numpy())
    finally:
        ql.decode_fuse_mode(-1)
    return out


def _check(out, ref, t, what):
    """Every mode within the oracle's tolerance.  Modes 1 and 2 split K alike, so their split-K
    sums run in the same order and agree bit for bit; the cluster mode may pick another split
    count (the clusters must fit the device at once), which changes the fp32 summation order."""
    for mode, (y, y32) in out.items():
        check_fp32(y32, ref, t, f"{what} mode {mode}")
        check_bf16(y, ref, t, f"{what} mode {mode}")
    assert np.array_equal(out[1][1], out[2][1]), f"{what}: modes 1 and 2 differ"
    assert np.array_equal(out[1][0], out[2][0]), f"{what}: modes 1 and 2 differ (bf16)"


@pytest.mark.parametrize("N,K,M", [(1280, 9728, 1), (1280, 9728, 8), (1280, 9728, 64),
                                   (384, 640, 37)])
def test_mx_decode_modes(N, K, M):
    ql = _ql()
    codes = synth.uniform_nibble_bytes(80 + M, N, K)
    sb = synth.uniform_bytes(81 + M, (N, K // 32), 120, 130)
    lin = ql.QLinear(codes, sb)
    xb, _ = synth.activations_bf16(82 + M, M, K, 0.01, 20.0)
    out = _run_modes(lin, xb)
    lin.close()
    xc, xs = mx.quantize_e8m0_b32(synth.bf16_bits_to_f64(xb))
    xq = mx.dequant_e8m0_b32(xc, xs)
    wq = mx.dequant_e8m0_b32(F.unpack_nibbles(codes), sb)
    _check(out, G.gemm_ref(xq, wq), G.abs_scale(xq, wq), f"mx N={N} K={K} M={M}")


@pytest.mark.parametrize("M", [1, 16, 64])
def test_prquant_tail_decode_modes(M):
    """PRQuant K-extension: the tail stages read the activation's last k channels again."""
    ql = _ql()
    N, C, k = 512, 2048, 256
    w = synth.bf16_bits_to_f64(synth.to_bf16_bits(synth.student_t(90, (N, C), 3.0)))
    prep = prquant.prepare(w, k)
    codes = F.pack_nibbles(prep["w_codes"])
    lin = ql.QLinear(codes, prep["w_sb"], k_tail=k)
    xb, _ = synth.activations_bf16(91 + M, M, C, 0.005, 50.0)
    xpb = np.ascontiguousarray(xb[:, prep["perm"]])
    out = _run_modes(lin, xpb)
    lin.close()
    xc, xs = prquant.quantize_activation_augmented(synth.bf16_bits_to_f64(xpb), k)
    xq = mx.dequant_e8m0_b32(xc, xs)
    wq = mx.dequant_e8m0_b32(prep["w_codes"], prep["w_sb"])
    _check(out, G.gemm_ref(xq, wq), G.abs_scale(xq, wq), f"tail M={M}")


@pytest.mark.parametrize("N,K,M", [(1280, 9728, 1), (1280, 9728, 8), (1280, 9728, 64),
                                   (256, 512, 13)])
def test_nvfp4_decode_modes(N, K, M):
    """E4M3-B16: at K = 9728 the local mode reads all of x for the amax at M = 1 and 8 and
    gathers it over the grid at M = 64."""
    ql = _ql()
    codes = synth.uniform_nibble_bytes(100 + M, N, K)
    sb = synth.uniform_bytes(101 + M, (N, K // 16), 0x28, 0x48)
    ts_w = np.float32(0.0123)
    lin = ql.QLinear(codes, sb, wfmt=ql.QL_W_NVFP4_E4M3_B16, w_tensor_scale=float(ts_w))
    xb, _ = synth.activations_bf16(102 + M, M, K, 0.01, 30.0)
    out = _run_modes(lin, xb)
    lin.close()
    xc, xs, xts = mx.quantize_e4m3_b16(synth.bf16_bits_to_f64(xb).astype(np.float32))
    xd = mx.dequant_e4m3_b16(xc, xs, xts)
    wd = mx.dequant_e4m3_b16(F.unpack_nibbles(codes), sb, ts_w)
    _check(out, G.gemm_ref(xd, wd), G.abs_scale(xd, wd), f"nvfp4 N={N} K={K} M={M}")


@pytest.mark.parametrize("M", [1, 8, 64])
def test_vq_decode_modes(M):
    """VQ PreScale weights with random indices, codebooks and scales, N = 1280, K = 9728."""
    ql = _ql()
    g = np.random.default_rng(110 + M)
    N, K = 1280, 9728
    cb = g.integers(0, 16, (N // 64, K // 64, 256, 4), dtype=np.uint8)
    prep = dict(ts=np.float32(0.0071), sb=g.integers(0x28, 0x48, (N, K // 16), dtype=np.uint8),
                idx=g.integers(0, 256, (N, K // 4), dtype=np.uint8))
    lin = ql.QLinear(None, prep["sb"], wfmt=ql.QL_W_VQ_PRESCALE_E4M3_B16,
                     w_tensor_scale=float(prep["ts"]), indices=prep["idx"],
                     codebooks=vq.pack_codebooks(cb))
    xb, _ = synth.activations_bf16(111 + M, M, K, 0.01, 30.0)
    out = _run_modes(lin, xb)
    lin.close()
    ref, t = vq.forward(synth.bf16_bits_to_f64(xb), prep, cb)
    _check(out, ref, t, f"vq M={M}")


def test_bad_mode_rejected():
    ql = _ql()
    for bad in (4, -2):
        with pytest.raises(ql.QLError):
            ql.decode_fuse_mode(bad)


@pytest.mark.parametrize("M", [1, 16, 64])
def test_cluster_gemm_only_path(M):
    """qlinear_quantize_input + qlinear_gemm (the decode kernel reading the plain layout) under the
    cluster mode reproduces the one-launch forward bit for bit, repeatedly."""
    ql = _ql()
    codes = synth.uniform_nibble_bytes(160 + M, 1280, 4096)
    sb = synth.uniform_bytes(161 + M, (1280, 4096 // 32), 120, 130)
    lin = ql.QLinear(codes, sb)
    xb, _ = synth.activations_bf16(162 + M, M, 4096, 0.01, 20.0)
    x = dev_bf16(xb)
    try:
        ql.decode_fuse_mode(3)
        ws = torch.empty(lin.workspace_bytes(M), dtype=torch.uint8, device="cuda")
        ref = lin.forward(x, ws=ws).clone()
        lin.quantize_input(x, ws)
        for _ in range(3):
            y = torch.empty_like(ref)
            lin.gemm(M, y, ws)
            ql.check()
            assert torch.equal(y, ref)
    finally:
        ql.decode_fuse_mode(-1)
    lin.close()
