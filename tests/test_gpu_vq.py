"""GPU parity: E4M3-B16 activation quantizer (bit-exact, with its FP32 tensor scale), E4M3-B16
weights on the kind::mxf4nvf4 MMA, and MXCode PreScale VQ weights decoded inside the GEMM."""
import numpy as np
import pytest
import torch

import synth
from oracle import formats as F
from oracle import gemm as G
from oracle import mx, vq
from tests._parity import check_bf16, check_fp32

pytestmark = pytest.mark.gpu


def _ql():
    import bit_quantized_moe_tcgen05_b200 as ql
    return ql


def dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _check_quant(xb):
    ql = _ql()
    codes, sb, ts = ql.quantize_act(dev_bf16(xb), fmt=ql.QL_A_FP4_E4M3_B16_TS)
    ql.check()
    rc, rs, rts = mx.quantize_e4m3_b16(synth.bf16_bits_to_f64(xb).astype(np.float32))
    assert ts.cpu().numpy()[0] == rts
    assert np.array_equal(sb.cpu().numpy(), rs)
    assert np.array_equal(codes.cpu().numpy(), F.pack_nibbles(rc))


@pytest.mark.parametrize("M,K", [(1, 16), (7, 9728), (64, 512), (300, 160)])
def test_quant_e4m3_b16_bitexact(M, K):
    xb, _ = synth.activations_bf16(200 + M, M, K, 0.01, 30.0)
    _check_quant(xb)


def test_quant_e4m3_b16_edge_values():
    _check_quant(synth.to_bf16_bits(np.zeros((3, 64))))                  # ts = 1, codes 0
    x = np.zeros((2, 64))
    x[0, 0] = 1e6
    x[0, 16:32] = 1e-6                                                    # scale underflows
    x[1, 32:48] = -1e-30
    x[1, 48] = -0.0
    _check_quant(synth.to_bf16_bits(x))
    g = np.random.default_rng(1)
    _check_quant(synth.to_bf16_bits(g.standard_normal((4, 256)) * 10.0 ** g.uniform(-30, 30, (4, 1))))


def test_quant_e4m3_b16_golden_blocks():
    """The hand-worked E4M3-B16 blocks (MXCode Table 1, row E4M3-B16-FP4; every value bf16) through
    the GPU quantizer: tensor scale, block bytes and codes equal the worked values."""
    import json
    import os
    from tests.conftest import GOLDEN
    with open(os.path.join(GOLDEN, "e4m3_b16_blocks.json")) as f:
        g = json.load(f)["tensor"]
    num = lambda s: float.fromhex(s) if "0x" in s else float(s)
    x = np.array([[num(v) for blk in g["blocks"] for v in blk["x"]]])
    xb = synth.to_bf16_bits(x)
    assert np.array_equal(synth.bf16_bits_to_f64(xb), x)            # every input is a bf16 value
    ql = _ql()
    codes, sb, ts = ql.quantize_act(dev_bf16(xb), fmt=ql.QL_A_FP4_E4M3_B16_TS)
    ql.check()
    assert ts.cpu().numpy()[0] == np.float32(num(g["ts"]))
    want_codes = np.array([[c for blk in g["blocks"] for c in blk["codes"]]], np.uint8)
    assert sb.cpu().numpy()[0].tolist() == [blk["byte"] for blk in g["blocks"]]
    assert np.array_equal(codes.cpu().numpy(), F.pack_nibbles(want_codes))


def _run(lin, xb):
    x = dev_bf16(xb)
    y32 = torch.empty((x.shape[0], lin.N), dtype=torch.float32, device="cuda")
    y = lin(x, out_f32=y32)
    _ql().check()
    return y.float().cpu().numpy(), y32.cpu().numpy()


def _x_deq(xb):
    xc, xs, xts = mx.quantize_e4m3_b16(synth.bf16_bits_to_f64(xb).astype(np.float32))
    return mx.dequant_e4m3_b16(xc, xs, xts)


@pytest.mark.parametrize("N,K,M", [(256, 512, 1), (128, 1024, 64), (272, 320, 100), (512, 9728, 8)])
def test_nvfp4_weight_linear(N, K, M):
    """E4M3-B16 weights (random codes, block scales and a tensor scale) on the block16 MMA."""
    ql = _ql()
    codes = synth.uniform_nibble_bytes(50 + N, N, K)
    sb = synth.uniform_bytes(51 + N, (N, K // 16), 0x28, 0x48)
    ts_w = np.float32(0.0123)
    lin = ql.QLinear(codes, sb, wfmt=ql.QL_W_NVFP4_E4M3_B16, w_tensor_scale=float(ts_w))
    xb, _ = synth.activations_bf16(52, M, K, 0.01, 30.0)
    y, y32 = _run(lin, xb)
    lin.close()
    xd = _x_deq(xb)
    wd = mx.dequant_e4m3_b16(F.unpack_nibbles(codes), sb, ts_w)
    ref, t = G.gemm_ref(xd, wd), G.abs_scale(xd, wd)
    check_fp32(y32, ref, t, "nvfp4")
    check_bf16(y, ref, t, "nvfp4")


def _vq_layer(w, cb, prep):
    ql = _ql()
    return ql.QLinear(None, prep["sb"], wfmt=ql.QL_W_VQ_PRESCALE_E4M3_B16,
                      w_tensor_scale=float(prep["ts"]), indices=prep["idx"],
                      codebooks=vq.pack_codebooks(cb))


@pytest.mark.parametrize("N,K,M", [(128, 256, 1), (256, 512, 8), (128, 768, 64), (256, 512, 200)])
def test_vq_linear_small(N, K, M):
    w = synth.bf16_bits_to_f64(synth.to_bf16_bits(synth.student_t(60 + K, (N, K), 4.0)))
    cb = synth.vq_codebooks(60, w)
    prep = vq.prepare(w, cb)
    lin = _vq_layer(w, cb, prep)
    xb, _ = synth.activations_bf16(61, M, K, 0.0, 1.0)
    y, y32 = _run(lin, xb)
    lin.close()
    ref, t = vq.forward(synth.bf16_bits_to_f64(xb), prep, cb)
    check_fp32(y32, ref, t, f"vq N={N} K={K} M={M}")
    check_bf16(y, ref, t, f"vq N={N} K={K} M={M}")


_C2 = {}


def _c2():
    if not _C2:
        w = synth.bf16_bits_to_f64(synth.to_bf16_bits(synth.student_t(2, (2560, 9728), 4.0)))
        cb = synth.vq_codebooks(2, w)
        _C2.update(w=w, cb=cb, prep=vq.prepare(w, cb))
    return _C2


@pytest.mark.parametrize("M", [1, 8, 64])
def test_vq_workload_full_size(M):
    """MXCode-style VQ layer at its full size: W [2560, 9728] Student-t(4), 64 x 64 QBlocks,
    K = 256 entries of d = 4; X N(0,1); every output compared."""
    c = _c2()
    lin = _vq_layer(c["w"], c["cb"], c["prep"])
    xb, _ = synth.activations_bf16(2, M, 9728, 0.0, 1.0)
    y, y32 = _run(lin, xb)
    lin.close()
    ref, t = vq.forward(synth.bf16_bits_to_f64(xb), c["prep"], c["cb"])
    check_fp32(y32, ref, t, f"C2 M={M}")
    check_bf16(y, ref, t, f"C2 M={M}")


@pytest.mark.parametrize("M", [300, 2048])
def test_nvfp4_weight_linear_prefill(M):
    """E4M3-B16 weights at prefill shapes: M = 300 runs 256-token tiles split along K; M = 2048
    runs 160-token tiles (260 tiles, two full waves), whose activation scales are grouped per
    160-row tile."""
    ql = _ql()
    N, K = 2560, 2048
    codes = synth.uniform_nibble_bytes(60, N, K)
    sb = synth.uniform_bytes(61, (N, K // 16), 0x28, 0x48)
    ts_w = np.float32(0.0123)
    lin = ql.QLinear(codes, sb, wfmt=ql.QL_W_NVFP4_E4M3_B16, w_tensor_scale=float(ts_w))
    xb, _ = synth.activations_bf16(62, M, K, 0.01, 30.0)
    y, y32 = _run(lin, xb)
    lin.close()
    xd = _x_deq(xb)
    wd = mx.dequant_e4m3_b16(F.unpack_nibbles(codes), sb, ts_w)
    ref, t = G.gemm_ref(xd, wd), G.abs_scale(xd, wd)
    check_fp32(y32, ref, t, "nvfp4 prefill")
    check_bf16(y, ref, t, "nvfp4 prefill")


@pytest.mark.parametrize("M", [300, 16, 2048])
def test_vq_linear_random_codebooks(M):
    """VQ weights with random indices, codebooks and scales at N = 2560, K = 2048: M = 300 as a
    prefill tile, M = 16 as split-K with the decode running ahead of the activation quantizer,
    M = 2048 as 160-token tiles."""
    g = np.random.default_rng(70 + M)
    N, K = 2560, 2048
    cb = g.integers(0, 16, (N // 64, K // 64, 256, 4), dtype=np.uint8)
    prep = dict(ts=np.float32(0.0071), sb=g.integers(0x28, 0x48, (N, K // 16), dtype=np.uint8),
                idx=g.integers(0, 256, (N, K // 4), dtype=np.uint8))
    lin = _vq_layer(None, cb, prep)
    xb, _ = synth.activations_bf16(71, M, K, 0.01, 30.0)
    y, y32 = _run(lin, xb)
    lin.close()
    ref, t = vq.forward(synth.bf16_bits_to_f64(xb), prep, cb)
    check_fp32(y32, ref, t, f"vq random M={M}")
    check_bf16(y, ref, t, f"vq random M={M}")


def test_quant_e4m3_b16_rounding_thresholds():
    """Quotients x/S at and next to every E2M1 rounding threshold (ties included), which the
    quantizer must resolve exactly as the fp32 division does; plus blocks whose scale product S
    is an fp32 subnormal."""
    thr = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    rows = []
    for j in range(-3, 4):                        # S = 2^j: ts = 1 (amax 2688), s = 2^j
        row = [2688.0] + [0.0] * 15               # block 0 fixes the tensor scale
        for t in thr:
            blk = [6.0 * 2.0 ** j]                # block amax -> E4M3 scale 2^j exactly
            v = t * 2.0 ** j
            up, dn = np.nextafter(np.float32(v), np.float32(np.inf)), np.nextafter(np.float32(v), np.float32(0))
            blk += [v, -v, float(up), float(dn), v * (1 + 2 ** -8), v * (1 - 2 ** -8), -v * (1 + 2 ** -8)]
            blk += [0.0] * (16 - len(blk))
            row += blk
        rows.append(row)
    width = max(len(r) for r in rows)
    x = np.array([r + [0.0] * (width - len(r)) for r in rows])
    _check_quant(synth.to_bf16_bits(x))
    g = np.random.default_rng(5)
    tiny = g.standard_normal((2, 128)) * 1e-39    # subnormal block scales
    tiny[:, 0] = 3e-36
    _check_quant(synth.to_bf16_bits(tiny))


def test_e4m3_grid_quantizer_shared_workspace():
    """The grid-wide E4M3-B16 quantizer (more 16-element blocks than a cluster has threads)
    agrees on the tensor amax through tagged words in the caller's workspace: it must work on a
    workspace full of random bytes, when two layers of different shapes take turns on one
    workspace, and give identical results when repeated."""
    ql = _ql()
    g = np.random.default_rng(90)
    layers, refs, xs = [], [], []
    for N, K, M in ((256, 8192, 64), (384, 4096, 80)):   # 32768 and 20480 blocks of 16
        codes = synth.uniform_nibble_bytes(91 + N, N, K)
        sb = synth.uniform_bytes(92 + N, (N, K // 16), 0x28, 0x48)
        ts_w = np.float32(0.0123)
        lin = ql.QLinear(codes, sb, wfmt=ql.QL_W_NVFP4_E4M3_B16, w_tensor_scale=float(ts_w))
        xb, _ = synth.activations_bf16(93 + N, M, K, 0.01, 30.0)
        xd = _x_deq(xb)
        wd = mx.dequant_e4m3_b16(F.unpack_nibbles(codes), sb, ts_w)
        layers.append(lin)
        xs.append(dev_bf16(xb))
        refs.append((G.gemm_ref(xd, wd), G.abs_scale(xd, wd)))
    need = max(l.workspace_bytes(x.shape[0]) for l, x in zip(layers, xs))
    ws = torch.from_numpy(g.integers(0, 256, need, dtype=np.uint8)).cuda()
    first = {}
    for rnd in range(3):
        for i, (lin, x) in enumerate(zip(layers, xs)):
            y32 = torch.empty((x.shape[0], lin.N), dtype=torch.float32, device="cuda")
            y = lin(x, out_f32=y32, ws=ws)
            ql.check()
            yb, y32h = y.float().cpu().numpy(), y32.cpu().numpy()
            ref, t = refs[i]
            check_fp32(y32h, ref, t, f"shared ws layer {i} round {rnd}")
            check_bf16(yb, ref, t, f"shared ws layer {i} round {rnd}")
            if rnd == 0:
                first[i] = y32h
            else:
                assert np.array_equal(first[i], y32h), f"layer {i} round {rnd} not repeatable"
    for lin in layers:
        lin.close()


# ------------------------------------------------------------------ PostScale / PreScale+
def _postscale_layer(prep, ql):
    return ql.QLinear(None, prep["sbq"], wfmt=ql.QL_W_VQ_POSTSCALE_E4M3_B16,
                      w_tensor_scale=float(prep["ts"]), indices=prep["idx"],
                      codebooks=vq.pack_codebooks(prep["codes"]))


@pytest.mark.parametrize("N,K,M", [(256, 512, 1), (256, 1024, 8), (128, 768, 64), (256, 512, 200),
                                   (512, 2048, 300)])
def test_vq_postscale_linear(N, K, M):
    """MXCode PostScale weights (one E4M3 scale per 64 x 64 QBlock codebook, no per-weight
    scales): decode launches build the scale factors in TMEM, prefill launches in shared memory."""
    ql = _ql()
    w = synth.bf16_bits_to_f64(synth.to_bf16_bits(synth.student_t(80 + K, (N, K), 4.0) * 0.02))
    cent = synth.vq_raw_codebooks(80, w)
    prep = vq.postscale_prepare(w, cent)
    lin = _postscale_layer(prep, ql)
    xb, _ = synth.activations_bf16(81, M, K, 0.01, 30.0)
    y, y32 = _run(lin, xb)
    lin.close()
    ref, t = vq.postscale_forward(synth.bf16_bits_to_f64(xb), prep)
    check_fp32(y32, ref, t, f"postscale N={N} K={K} M={M}")
    check_bf16(y, ref, t, f"postscale N={N} K={K} M={M}")


@pytest.mark.parametrize("N,K,M", [(256, 512, 1), (256, 1024, 8), (128, 768, 64), (256, 512, 200),
                                   (512, 2048, 300)])
def test_vq_prescale_plus_linear(N, K, M):
    """MXCode PreScale+ weights (block scales replaced by 8-scale vectors of a 256-entry scale
    codebook): the decoders look the scales up per row and per 128-column group."""
    ql = _ql()
    w = synth.bf16_bits_to_f64(synth.to_bf16_bits(synth.student_t(82 + K, (N, K), 4.0)))
    cb = synth.vq_codebooks(82, w)
    _, sb0 = vq.prescale(w)
    scb = synth.scale_codebook(82, sb0)
    prep = vq.prescale_plus_prepare(w, cb, scb)
    lin = ql.QLinear(None, prep["sidx"], wfmt=ql.QL_W_VQ_PRESCALE_PLUS_E4M3_B16,
                     w_tensor_scale=float(prep["ts"]), indices=prep["idx"],
                     codebooks=vq.pack_codebooks(cb), scale_codebook=scb)
    xb, _ = synth.activations_bf16(83, M, K, 0.01, 30.0)
    y, y32 = _run(lin, xb)
    lin.close()
    ref, t = vq.forward(synth.bf16_bits_to_f64(xb), prep, cb)
    check_fp32(y32, ref, t, f"prescale+ N={N} K={K} M={M}")
    check_bf16(y, ref, t, f"prescale+ N={N} K={K} M={M}")
