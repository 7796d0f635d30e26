"""GPU parity of the routed MoE FFN (CodeQuant-style cluster-codebook experts): routing (exact),
x quantization (exact), gate/up + SwiGLU (float tolerance), the MXFP4 requantization of h
(exact, stage-wise on the GPU's own h), down + slot-ordered combine (float tolerance)."""
import numpy as np
import pytest
import torch

import synth
from oracle import formats as F
from oracle import gemm as G
from oracle import mx, moe

pytestmark = pytest.mark.gpu


def build_model(seed, E, H, I):
    gi, gc, di, dc = [], [], [], []
    for e in range(E):
        c, i = synth.cluster_rows(seed * 1000 + e, 2 * I, H)
        gc.append(c); gi.append(i)
        c, i = synth.cluster_rows(seed * 1000 + 500 + e, H, I)
        dc.append(c); di.append(i)
    return (np.concatenate(gi), np.concatenate(gc), np.concatenate(di), np.concatenate(dc))


def _view(ws, off, n, dtype):
    nbytes = n * torch.empty((), dtype=dtype).element_size()
    return ws[off:off + nbytes].view(dtype)


def run_case(seed, E, H, I, T, k, logits=None):
    import bit_quantized_moe_tcgen05_b200 as ql
    gi, gc, di, dc = build_model(seed, E, H, I)
    layer = ql.MoE(gi, gc, di, dc, E, k)
    layer.capture_intermediate(True)
    xb, _ = synth.activations_bf16(seed, T, H, 0.0, 1.0)
    if logits is None:
        logits = synth.zipf_router_logits(seed, T, E)
    x = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).cuda()
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
    return got, xb, logits, Wgu, Wd


def check_all(got, xb, logits, Wgu, Wd, k, had_x=False, had_h=False):
    T, H = got["y"].shape
    I = Wd[0].shape[1]
    xd = F.bf16_decode(xb)
    ref = moe.forward(xd, logits, Wgu, Wd, k, h_given=got["h32"].astype(np.float64), had_x=had_x,
                      had_h=had_h)
    r = ref["route"]
    # routing: exact
    assert np.array_equal(got["ids"], r["ids"])
    assert np.array_equal(got["counts"], r["counts"])
    assert np.array_equal(got["offsets"], r["offsets"])
    assert np.array_equal(got["entries"], r["entries"])
    # gate weights: an fp32 softmax of the selected logits on the GPU (the largest logit
    # subtracted in fp32, expf within 2 ulp, k - 1 additions in slot order, one division) against
    # float64.  First-order relative bound per gate: the argument rounding 2^-24 |d| and expf's
    # 2^-22 in the numerator and (at most) in the denominator, plus the k - 1 additions and the
    # division at 2^-24 each.
    sel = np.take_along_axis(logits.astype(np.float64), r["ids"], axis=1)
    dmax = np.abs(sel - sel[:, :1]).max(axis=1, keepdims=True)
    eps_g = 2 * (2.0 ** -22 + 2.0 ** -24 * dmax) + k * 2.0 ** -24
    gerr = np.abs(got["gates"].astype(np.float64) - r["gates"])
    assert np.all(gerr <= eps_g * r["gates"]), f"gates: worst ratio {float((gerr / (eps_g * r['gates'])).max()):.3g}"
    # x quantization: exact
    assert np.array_equal(got["x_codes"], F.pack_nibbles(ref["x_codes"]))
    assert np.array_equal(got["x_scales"], ref["x_scales"])
    # h (fp32, before requant) against the fp64 chain: GEMM bound propagated through SwiGLU
    g, u = ref["g"], ref["u"]
    sg = g / (1 + np.exp(-g))
    dsg = 1.1 * np.abs(u)
    # plus the fp32 evaluation of silu(g) * u itself: expf (2 ulp = 2^-22) and three correctly
    # rounded operations (1 + e, the division, the product with u); 2^-149 covers an h that
    # underflows to zero
    eps_h = 2.0 ** -22 + 3 * 2.0 ** -24
    bound = dsg * 1e-5 * ref["tg"] + np.abs(sg) * 1e-5 * ref["tu"] + eps_h * np.abs(ref["h"]) + 2.0 ** -149
    err = np.abs(got["h32"].astype(np.float64) - ref["h"])
    assert np.all(err <= bound), f"h: worst ratio {float((err / bound).max()):.3g}"
    # requantization of the GPU's own h: exact
    assert np.array_equal(got["h_codes"], F.pack_nibbles(ref["h_codes"]))
    assert np.array_equal(got["h_scales"], ref["h_scales"])
    # output: the down GEMM's 1e-5 * sum|h_q w| bound, weighted by the gates (t_out), plus what
    # the fp32 combine adds on top: each gate's own relative error eps_g, the product gate * y and
    # the k - 1 slot additions at 2^-24 each, all relative to sum_s |g_s y_s| <= t_out
    t_out = ref["t_out"]
    err = np.abs(got["y32"].astype(np.float64) - ref["out"])
    allow = (1e-5 + eps_g.max(axis=1, keepdims=True) + k * 2.0 ** -24) * t_out
    assert np.all(err <= allow), f"out: worst ratio {float((err / np.maximum(allow, 1e-300)).max()):.3g}"
    refb = G.bf16_rne(ref["out"])
    errb = np.abs(got["y"].astype(np.float64) - refb)
    assert np.all(errb <= G.bf16_ulp(refb) + allow)


@pytest.mark.parametrize("E,H,I,T,k", [(8, 256, 128, 100, 2), (16, 512, 192, 300, 4),
                                       (4, 128, 64, 1, 1)])
def test_moe_small(E, H, I, T, k):
    got, xb, logits, Wgu, Wd = run_case(7 + E, E, H, I, T, k)
    check_all(got, xb, logits, Wgu, Wd, k)


def test_moe_routing_ties():
    """Integer logits with many ties: the lower expert id wins."""
    E, H, I, T, k = 8, 128, 64, 64, 3
    g = np.random.default_rng(11)
    logits = g.integers(-2, 3, (T, E)).astype(np.float32)
    got, xb, logits, Wgu, Wd = run_case(11, E, H, I, T, k, logits=logits)
    check_all(got, xb, logits, Wgu, Wd, k)


def test_moe_workload_full_size():
    """The MoE grouped FFN workload: 128 experts, top-8, hidden 2048, intermediate 768, 2048 tokens,
    Zipf(1.1) router."""
    E, H, I, T, k = 128, 2048, 768, 2048, 8
    got, xb, logits, Wgu, Wd = run_case(4, E, H, I, T, k)
    check_all(got, xb, logits, Wgu, Wd, k)
