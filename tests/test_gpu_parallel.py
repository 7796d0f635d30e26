"""The N-sharded linear's per-rank layers on one GPU: every rank's slice of the weight (MXFP4
codes and scales; VQ indices, QBlock codebooks and scales) as its own layer, the slices'
outputs side by side against the oracle of the whole layer.  (The all-gather that joins them
across GPUs is tested on CPU over gloo; this run has one GPU.)"""
import numpy as np
import pytest
import torch

import synth
from oracle import formats as F
from oracle import gemm as G
from oracle import mx, vq
from tests._parity import check_bf16, check_fp32

pytestmark = pytest.mark.gpu


def dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _joined(make_rank_layer, world, N, M, x):
    from bit_quantized_moe_tcgen05_b200 import parallel as P
    outs = []
    for r in range(world):
        n0, n1 = P.shard_rows(N, world, r)
        lin = make_rank_layer(n0, n1)
        y32 = torch.empty((M, n1 - n0), dtype=torch.float32, device="cuda")
        y = lin(x, out_f32=y32)
        outs.append((y.float().cpu().numpy(), y32.cpu().numpy()))
        lin.close()
    return np.concatenate([o[0] for o in outs], 1), np.concatenate([o[1] for o in outs], 1)


@pytest.mark.parametrize("world,M", [(2, 1), (4, 16), (3, 300)])
def test_sharded_mxfp4(world, M):
    import bit_quantized_moe_tcgen05_b200 as ql
    from bit_quantized_moe_tcgen05_b200 import parallel as P
    N, K = 1536, 2048
    codes = synth.uniform_nibble_bytes(190, N, K)
    sb = synth.uniform_bytes(191, (N, K // 32), 120, 130)
    xb, _ = synth.activations_bf16(192 + M, M, K, 0.01, 20.0)
    x = dev_bf16(xb)

    def make(n0, n1):
        sl = P.slice_weight(n0, n1, codes=codes, scales=sb)
        return ql.QLinear(sl["codes"], sl["scales"])

    y, y32 = _joined(make, world, N, M, x)
    ql.check()
    xc, xs = mx.quantize_e8m0_b32(synth.bf16_bits_to_f64(xb))
    xq = mx.dequant_e8m0_b32(xc, xs)
    wq = mx.dequant_e8m0_b32(F.unpack_nibbles(codes), sb)
    ref, t = G.gemm_ref(xq, wq), G.abs_scale(xq, wq)
    check_fp32(y32, ref, t, f"sharded mx world={world} M={M}")
    check_bf16(y, ref, t, f"sharded mx world={world} M={M}")


@pytest.mark.parametrize("world,M", [(2, 8), (5, 64)])
def test_sharded_vq(world, M):
    import bit_quantized_moe_tcgen05_b200 as ql
    from bit_quantized_moe_tcgen05_b200 import parallel as P
    g = np.random.default_rng(193)
    N, K = 1280, 2048
    cb = g.integers(0, 16, (N // 64, K // 64, 256, 4), dtype=np.uint8)
    prep = dict(ts=np.float32(0.0071), sb=g.integers(0x28, 0x48, (N, K // 16), dtype=np.uint8),
                idx=g.integers(0, 256, (N, K // 4), dtype=np.uint8))
    packed = vq.pack_codebooks(cb)
    xb, _ = synth.activations_bf16(194 + M, M, K, 0.01, 30.0)
    x = dev_bf16(xb)

    def make(n0, n1):
        sl = P.slice_weight(n0, n1, scales=prep["sb"], indices=prep["idx"], codebooks=packed)
        return ql.QLinear(None, sl["scales"], wfmt=ql.QL_W_VQ_PRESCALE_E4M3_B16,
                          w_tensor_scale=float(prep["ts"]), indices=sl["indices"],
                          codebooks=sl["codebooks"])

    y, y32 = _joined(make, world, N, M, x)
    ql.check()
    ref, t = vq.forward(synth.bf16_bits_to_f64(xb), prep, cb)
    check_fp32(y32, ref, t, f"sharded vq world={world} M={M}")
    check_bf16(y, ref, t, f"sharded vq world={world} M={M}")
