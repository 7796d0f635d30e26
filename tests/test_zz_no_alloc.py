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
