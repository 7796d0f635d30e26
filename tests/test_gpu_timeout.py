"""The device-timeout path, made to happen without any fault: a test hook withholds one CTA's
publications to other CTAs (the E4M3-B16 amax slot, the decode flags, its arrivals on cluster
peers' barriers) and lowers the wait limit to 2 ms, so that the bounded waits on them run out.
The kernels record QL_ERR_TIMEOUT and return; ql_check reports it; after the hook is lifted the
same workspace gives the same bits as a fresh one (the launch counters moved past every tag the
failed launch left behind)."""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


def _ql():
    import bit_quantized_moe_tcgen05_b200 as ql
    return ql


def _nvfp4_layer(N, K, seed):
    ql = _ql()
    codes = synth.uniform_nibble_bytes(seed, N, K)
    sb = synth.uniform_bytes(seed + 1, (N, K // 16), 0x28, 0x48)
    return ql.QLinear(codes, sb, wfmt=ql.QL_W_NVFP4_E4M3_B16, w_tensor_scale=0.0123)


def _x(M, K, seed):
    xb, _ = synth.activations_bf16(seed, M, K, 0.01, 30.0)
    return torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).cuda()


def _expect_timeout(fn):
    ql = _ql()
    ql.debug_inject(withhold_cta=1, wait_limit_ns=2_000_000)
    try:
        fn()
        with pytest.raises(ql.QLError) as e:
            ql.check()
        assert e.value.status == 5 and "expired" in str(e.value)
    finally:
        ql.debug_inject()
    ql.check()                                     # the error word was cleared


@pytest.mark.parametrize("mode", [1, 2, 3])
def test_decode_forward_timeout_then_recovers(mode):
    """One-launch decode forward (E4M3-B16 activations quantized inside the GEMM), in each of the
    decode kernel's organisations: CTA 1 withholds what it publishes to the others (mode 1: its
    amax slot and its quantized and split-K flags in the workspace; mode 2: its slot and split-K
    flag; mode 3: its arrivals on its cluster peers' split-K barriers), and the waits on them run
    out."""
    ql = _ql()
    lin = _nvfp4_layer(512, 2048, 61)
    M = 8
    x = _x(M, 2048, 62)
    try:
        ql.decode_fuse_mode(mode)
        ws = torch.empty(lin.workspace_bytes(M), dtype=torch.uint8, device="cuda")
        y = torch.empty((M, 512), dtype=torch.bfloat16, device="cuda")
        _expect_timeout(lambda: lin.forward(x, out=y, ws=ws))
        for _ in range(2):                         # the same workspace, twice, after the failure
            got = lin.forward(x, ws=ws).clone()
            fresh = lin.forward(x, ws=torch.zeros_like(ws)).clone()
            ql.check()
            assert torch.equal(got, fresh)
    finally:
        ql.decode_fuse_mode(-1)
    lin.close()


def test_grid_quantizer_timeout_then_recovers():
    """The E4M3-B16 grid quantizer (64 x 9728 activations, quantize_input of the two-call API):
    CTA 1 withholds its slot, CTA 0's gather and every other CTA's wait for the result run out."""
    ql = _ql()
    lin = _nvfp4_layer(256, 9728, 63)
    M = 64
    x = _x(M, 9728, 64)
    ws = torch.empty(lin.workspace_bytes(M), dtype=torch.uint8, device="cuda")
    y = torch.empty((M, 256), dtype=torch.bfloat16, device="cuda")

    def two_calls(w):
        lin.quantize_input(x, w)
        lin.gemm(M, y, w)

    _expect_timeout(lambda: two_calls(ws))
    for _ in range(2):
        two_calls(ws)
        got = y.clone()
        two_calls(torch.zeros_like(ws))
        ql.check()
        assert torch.equal(got, y)
    lin.close()
