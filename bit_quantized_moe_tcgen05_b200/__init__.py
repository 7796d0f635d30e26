"""W4A4 quantized linear layer for NVIDIA B200 (sm_100a): Python binding over libqlinear.

Argument marshalling only.  Every step of the forward path runs in the CUDA kernels of
``libqlinear.so`` (built in-tree by ``bit_quantized_moe_tcgen05_b200.build``); torch supplies
device memory and the current stream.  Importing this package fails if the library is missing:
there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

__all__ = [
    "lib", "LIB_PATH", "QLError", "WeightDesc", "QLinear", "quantize_act", "prepare_prquant",
    "check", "debug_inject", "decode_fuse_mode", "QL_W_MXFP4_E8M0_B32", "QL_A_MXFP4_E8M0_B32", "EXPORTED_SYMBOLS",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libqlinear.so")

QL_OK = 0
QL_W_MXFP4_E8M0_B32, QL_W_NVFP4_E4M3_B16, QL_W_VQ_PRESCALE_E4M3_B16 = 1, 2, 3
QL_W_CLUSTER4_ROW16_BF16, QL_W_INT4_G128_BSR = 4, 5
QL_W_VQ_POSTSCALE_E4M3_B16, QL_W_VQ_PRESCALE_PLUS_E4M3_B16 = 6, 7
QL_A_MXFP4_E8M0_B32, QL_A_FP4_E4M3_B16_TS, QL_A_INT4_TOK_G128 = 1, 2, 3

_STATUS = {0: "QL_OK", 1: "QL_ERR_INVALID_ARG", 2: "QL_ERR_UNSUPPORTED", 3: "QL_ERR_CUDA",
           4: "QL_ERR_OOM", 5: "QL_ERR_TIMEOUT", 6: "QL_ERR_WORKSPACE"}

# Every entry point declared in include/qlinear.h.
EXPORTED_SYMBOLS = (
    "ql_version", "ql_last_error", "qlinear_create", "qlinear_destroy", "qlinear_workspace_bytes",
    "qlinear_forward", "quantize_act", "ql_check", "qlinear_prepare_prquant",
    "qlinear_quantize_input", "qlinear_gemm", "qlinear_forward_fixed_scratch",
    "qlinear_prepare_vq_prescale", "moe_create", "moe_destroy", "moe_capture_intermediate",
    "moe_workspace_bytes", "moe_workspace_layout", "moe_grouped_forward",
    "qlinear_prepare_int4_bsr", "ql_tensor_peak", "ql_debug_inject",
    "qlinear_prepare_vq_postscale", "qlinear_prepare_vq_prescale_plus",
    "qlinear_prepare_prquant_ex", "quantize_act_hadamard", "ql_decode_fuse_mode",
    "quantize_act_augmented",
)


class QLError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = lib.ql_last_error().decode(errors="replace")
        super().__init__(f"{where}: {_STATUS.get(status, status)}: {msg}")
        self.status = status


class WeightDesc(ctypes.Structure):
    _fields_ = [
        ("wfmt", ctypes.c_int), ("N", ctypes.c_int64), ("K", ctypes.c_int64),
        ("k_tail", ctypes.c_int32), ("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p),
        ("w_tensor_scale", ctypes.c_float), ("indices", ctypes.c_void_p),
        ("codebooks", ctypes.c_void_p), ("qblock_n", ctypes.c_int32), ("qblock_k", ctypes.c_int32),
        ("bsr_rowptr", ctypes.c_void_p), ("bsr_col", ctypes.c_void_p),
        ("bsr_codes", ctypes.c_void_p), ("bsr_scales", ctypes.c_void_p),
        ("bsr_block_n", ctypes.c_int32), ("bsr_block_k", ctypes.c_int32),
        ("bsr_nnzb", ctypes.c_int32), ("scale_codebook", ctypes.c_void_p),
        ("scale_codebook_entries", ctypes.c_int32), ("scale_group", ctypes.c_int32),
        ("had_block", ctypes.c_int32), ("tail_copy", ctypes.c_int32),
    ]


class MoeWsLayout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in (
        "counts", "offsets", "entries", "ids", "gates", "x_codes", "x_scales", "x_dq", "h_codes",
        "h_scales", "h_dq", "h32", "yslot", "total")]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing; build it with "
                          "`python -m bit_quantized_moe_tcgen05_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
    L.ql_version.restype = ctypes.c_char_p
    L.ql_last_error.restype = ctypes.c_char_p
    sig = {
        "qlinear_create": [ctypes.POINTER(WeightDesc), vp, ctypes.POINTER(vp)],
        "qlinear_destroy": [vp],
        "qlinear_workspace_bytes": [vp, i64, ctypes.POINTER(sz)],
        "qlinear_forward": [vp, vp, i64, vp, vp, vp, sz, vp],
        "qlinear_quantize_input": [vp, vp, i64, vp, sz, vp],
        "qlinear_gemm": [vp, i64, vp, vp, vp, sz, vp],
        "qlinear_forward_fixed_scratch": [vp, vp, i64, vp, vp, vp],
        "quantize_act": [ctypes.c_int, vp, i64, i64, vp, vp, vp, vp],
        "ql_check": [vp],
        "qlinear_prepare_prquant": [vp, i64, i64, i32, vp, vp, vp],
        "qlinear_prepare_prquant_ex": [vp, i64, i64, i32, i32, vp, vp, vp],
        "quantize_act_hadamard": [ctypes.c_int, i32, vp, i64, i64, vp, vp, vp],
        "quantize_act_augmented": [ctypes.c_int, vp, i64, i64, i32, vp, vp, vp],
        "qlinear_prepare_vq_prescale": [vp, i64, i64, vp, i32, i32, vp, vp, vp],
        "moe_create": [ctypes.POINTER(WeightDesc), ctypes.POINTER(WeightDesc), i32, i32, vp,
                       ctypes.POINTER(vp)],
        "moe_destroy": [vp],
        "moe_capture_intermediate": [vp, i32],
        "moe_workspace_bytes": [vp, i64, ctypes.POINTER(sz)],
        "moe_workspace_layout": [vp, i64, ctypes.POINTER(MoeWsLayout)],
        "moe_grouped_forward": [vp, vp, i64, vp, vp, vp, vp, vp, vp, sz, vp],
        "qlinear_prepare_int4_bsr": [vp, i64, i64, vp, i64, ctypes.c_float, vp, vp, vp, vp, vp, vp,
                                     i32, vp],
        "ql_tensor_peak": [i32, i32, i32, i32, ctypes.POINTER(ctypes.c_double), vp],
        "ql_debug_inject": [i32, ctypes.c_uint64],
        "ql_decode_fuse_mode": [i32],
        "qlinear_prepare_vq_postscale": [vp, i64, i64, vp, i32, i32, vp, vp, vp, vp],
        "qlinear_prepare_vq_prescale_plus": [vp, i64, i64, vp, vp, i32, i32, vp, vp, vp, vp],
    }
    for name, args in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = ctypes.c_int
    return L


lib = _load()


def _ok(status: int, where: str) -> None:
    if status != QL_OK:
        raise QLError(status, where)


def _stream(stream=None) -> int:
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def check(stream=None) -> None:
    """Synchronise and raise if any kernel recorded a device-side timeout."""
    _ok(lib.ql_check(_stream(stream)), "ql_check")


def debug_inject(withhold_cta: int = -1, wait_limit_ns: int = 0) -> None:
    """Test hook for the timeout path: lower the kernels' wait limit and withhold one CTA's
    grid-wide publications so that the waits on them run out (see ql_debug_inject).
    debug_inject() restores the defaults."""
    _ok(lib.ql_debug_inject(int(withhold_cta), int(wait_limit_ns)), "ql_debug_inject")


def decode_fuse_mode(mode: int = -1) -> None:
    """How the decode kernel is organised: 1 activations quantized cooperatively over the grid,
    2 each CTA its own stages, 3 as 2 with each weight tile's K-splits in one cluster, -1 chosen
    per launch (see ql_decode_fuse_mode).  Every mode matches the oracle; modes 1 and 2 give
    identical bits, mode 3 may split K differently."""
    _ok(lib.ql_decode_fuse_mode(int(mode)), "ql_decode_fuse_mode")


def quantize_act(x, fmt: int = QL_A_MXFP4_E8M0_B32, stream=None, had_block: int = 0,
                 k_tail: int = 0):
    """Quantize bf16 activations [M, K] on the GPU.
    MXFP4 E8M0-B32 -> (codes uint8 [M, K/2], E8M0 scales uint8 [M, K/32]), optionally after an
    online block-32 Hadamard (had_block = 32), or (k_tail > 0) the PRQuant augmented activation
    (codes [M, (K + k_tail)/2], scales [M, (K + k_tail)/32]: the last k_tail channels appended);
    E4M3-B16 + tensor scale -> (codes, E4M3 scales uint8 [M, K/16], ts float32 [1])."""
    import torch
    assert x.is_cuda and x.dtype == torch.bfloat16 and x.dim() == 2 and x.is_contiguous()
    M, K = x.shape
    if k_tail:
        assert fmt == QL_A_MXFP4_E8M0_B32 and not had_block
        codes = torch.empty((M, (K + k_tail) // 2), dtype=torch.uint8, device=x.device)
        scales = torch.empty((M, (K + k_tail) // 32), dtype=torch.uint8, device=x.device)
        _ok(lib.quantize_act_augmented(fmt, x.data_ptr(), M, K, int(k_tail), codes.data_ptr(),
                                       scales.data_ptr(), _stream(stream)), "quantize_act_augmented")
        return codes, scales
    codes = torch.empty((M, K // 2), dtype=torch.uint8, device=x.device)
    if fmt == QL_A_MXFP4_E8M0_B32:
        scales = torch.empty((M, K // 32), dtype=torch.uint8, device=x.device)
        if had_block:
            _ok(lib.quantize_act_hadamard(fmt, had_block, x.data_ptr(), M, K, codes.data_ptr(),
                                          scales.data_ptr(), _stream(stream)), "quantize_act_hadamard")
        else:
            _ok(lib.quantize_act(fmt, x.data_ptr(), M, K, codes.data_ptr(), scales.data_ptr(), None,
                                 _stream(stream)), "quantize_act")
        return codes, scales
    if fmt == QL_A_INT4_TOK_G128:
        scales = torch.empty((M, K // 128), dtype=torch.float32, device=x.device)
        _ok(lib.quantize_act(fmt, x.data_ptr(), M, K, codes.data_ptr(), scales.data_ptr(), None,
                             _stream(stream)), "quantize_act")
        return codes, scales
    if fmt == QL_A_FP4_E4M3_B16_TS:
        scales = torch.empty((M, K // 16), dtype=torch.uint8, device=x.device)
        ts = torch.empty(1, dtype=torch.float32, device=x.device)
        _ok(lib.quantize_act(fmt, x.data_ptr(), M, K, codes.data_ptr(), scales.data_ptr(),
                             ts.data_ptr(), _stream(stream)), "quantize_act")
        return codes, scales, ts
    raise ValueError(f"activation format {fmt} not exposed")


class QLinear:
    """A quantized linear layer y = x W^T whose weight lives in library-owned device memory.

    MXFP4 (E8M0-B32) weights: ``codes`` uint8 [N, K/2] (low nibble = even k) and ``scales``
    uint8 [N, K/32] E8M0 bytes, host numpy arrays.  ``k_tail`` > 0 makes it a PRQuant
    augmented weight whose last ``k_tail`` columns are the tail residual; the activation then
    has K - k_tail channels.
    """

    def __init__(self, codes: np.ndarray | None, scales: np.ndarray, k_tail: int = 0,
                 wfmt: int = QL_W_MXFP4_E8M0_B32, w_tensor_scale: float = 1.0,
                 indices: np.ndarray | None = None, codebooks: np.ndarray | None = None,
                 bsr: dict | None = None, scale_codebook: np.ndarray | None = None,
                 had_block: int = 0, tail_copy: bool = False, stream=None):
        """MXFP4: codes [N, K/2] + E8M0 scales [N, K/32] (+ k_tail).  NVFP4 (E4M3-B16): codes +
        E4M3 scales [N, K/16] + w_tensor_scale.  VQ PreScale: indices [N, K/4] + packed codebooks
        [N/64, K/64, 256, 2] + E4M3 scales [N, K/16] + w_tensor_scale (codes = None).
        INT4 + block-sparse residual: codes [N, K/2], fp16 scale bits [N, K/128] and
        bsr = {rowptr, col, rcodes, rscales} as returned by prepare_int4_bsr."""
        scales = np.ascontiguousarray(scales, dtype=np.uint8 if wfmt != QL_W_INT4_G128_BSR else np.uint16)
        keep = [scales]
        if wfmt == QL_W_INT4_G128_BSR:
            codes = np.ascontiguousarray(codes, dtype=np.uint8)
            N, K = codes.shape[0], 2 * codes.shape[1]
            b = bsr or {}
            rowptr = np.ascontiguousarray(b.get("rowptr", np.zeros(N // 16 + 1)), dtype=np.int32)
            col = np.ascontiguousarray(b.get("col", np.zeros(0)), dtype=np.int16)
            rcodes = np.ascontiguousarray(b.get("rcodes", np.zeros((0, 16, 64))), dtype=np.uint8)
            rscales = np.ascontiguousarray(b.get("rscales", np.zeros((0, 16))), dtype=np.uint16)
            keep += [codes, rowptr, col, rcodes, rscales]
            self.N, self.K, self.k_tail, self.C, self.wfmt = N, K, 0, K, wfmt
            d = WeightDesc(wfmt=wfmt, N=N, K=K, codes=codes.ctypes.data, scales=scales.ctypes.data,
                           bsr_rowptr=rowptr.ctypes.data, bsr_col=col.ctypes.data,
                           bsr_codes=rcodes.ctypes.data, bsr_scales=rscales.ctypes.data,
                           bsr_block_n=16, bsr_block_k=128, bsr_nnzb=len(col))
            h = ctypes.c_void_p()
            _ok(lib.qlinear_create(ctypes.byref(d), _stream(stream), ctypes.byref(h)), "qlinear_create")
            self._h = h
            self._ws = None
            return
        scb_ptr = None
        if wfmt in (QL_W_VQ_PRESCALE_E4M3_B16, QL_W_VQ_POSTSCALE_E4M3_B16,
                    QL_W_VQ_PRESCALE_PLUS_E4M3_B16):
            indices = np.ascontiguousarray(indices, dtype=np.uint8)
            codebooks = np.ascontiguousarray(codebooks, dtype=np.uint8)
            N, K = indices.shape[0], 4 * indices.shape[1]
            keep += [indices, codebooks]
            cptr, iptr, cbptr = None, indices.ctypes.data, codebooks.ctypes.data
            if wfmt == QL_W_VQ_PRESCALE_PLUS_E4M3_B16:
                scb = np.ascontiguousarray(scale_codebook, dtype=np.uint8)
                keep.append(scb)
                scb_ptr = scb.ctypes.data
        else:
            codes = np.ascontiguousarray(codes, dtype=np.uint8)
            N, K = codes.shape[0], 2 * codes.shape[1]
            keep.append(codes)
            cptr, iptr, cbptr = codes.ctypes.data, None, None
        self.N, self.K, self.k_tail = N, K, int(k_tail)
        self.C = self.K - self.k_tail
        self.wfmt = wfmt
        d = WeightDesc(wfmt=wfmt, N=N, K=self.K, k_tail=self.k_tail, codes=cptr,
                       scales=scales.ctypes.data, w_tensor_scale=float(w_tensor_scale),
                       indices=iptr, codebooks=cbptr, qblock_n=64, qblock_k=64,
                       scale_codebook=scb_ptr, scale_codebook_entries=256 if scb_ptr else 0,
                       scale_group=8 if scb_ptr else 0, had_block=int(had_block),
                       tail_copy=1 if tail_copy else 0)
        h = ctypes.c_void_p()
        _ok(lib.qlinear_create(ctypes.byref(d), _stream(stream), ctypes.byref(h)), "qlinear_create")
        self._h = h
        self._ws = None

    def workspace_bytes(self, M: int) -> int:
        n = ctypes.c_size_t()
        _ok(lib.qlinear_workspace_bytes(self._h, M, ctypes.byref(n)), "qlinear_workspace_bytes")
        return n.value

    def _workspace(self, M: int, device):
        import torch
        need = self.workspace_bytes(M)
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(need, dtype=torch.uint8, device=device)
        return self._ws

    def forward(self, x, out=None, out_f32=None, ws=None, stream=None):
        """x: bf16 [M, K - k_tail] on the GPU.  Returns y bf16 [M, N] (and fills out_f32)."""
        import torch
        assert x.is_cuda and x.dtype == torch.bfloat16 and x.dim() == 2 and x.is_contiguous()
        M, C = x.shape
        if C != self.C:
            raise ValueError(f"x has {C} channels, layer expects {self.C}")
        if out is None:
            out = torch.empty((M, self.N), dtype=torch.bfloat16, device=x.device)
        if ws is None:
            ws = self._workspace(M, x.device)
        _ok(lib.qlinear_forward(self._h, x.data_ptr(), M, out.data_ptr(), _ptr(out_f32),
                                ws.data_ptr(), ws.numel(), _stream(stream)), "qlinear_forward")
        return out

    __call__ = forward

    def forward_fixed_scratch(self, x, out=None, out_f32=None, stream=None):
        """forward() without a workspace: the library's own fixed 8 MiB scratch is used, so
        nothing is allocated on the device (for callers that may not allocate).  Calls that can
        overlap on the GPU share that scratch and must be serialised by the caller."""
        import torch
        assert x.is_cuda and x.dtype == torch.bfloat16 and x.dim() == 2 and x.is_contiguous()
        M, C = x.shape
        if C != self.C:
            raise ValueError(f"x has {C} channels, layer expects {self.C}")
        if out is None:
            out = torch.empty((M, self.N), dtype=torch.bfloat16, device=x.device)
        _ok(lib.qlinear_forward_fixed_scratch(self._h, x.data_ptr(), M, out.data_ptr(),
                                              _ptr(out_f32), _stream(stream)),
            "qlinear_forward_fixed_scratch")
        return out

    def quantize_input(self, x, ws, stream=None) -> None:
        """First half of forward: quantize x into the workspace ``ws``."""
        M = x.shape[0]
        _ok(lib.qlinear_quantize_input(self._h, x.data_ptr(), M, ws.data_ptr(), ws.numel(),
                                       _stream(stream)), "qlinear_quantize_input")

    def gemm(self, M: int, out, ws, out_f32=None, stream=None) -> None:
        """Second half of forward: the FP4 GEMM from the quantized input in ``ws``."""
        _ok(lib.qlinear_gemm(self._h, M, out.data_ptr(), _ptr(out_f32), ws.data_ptr(), ws.numel(),
                             _stream(stream)), "qlinear_gemm")

    def close(self) -> None:
        if getattr(self, "_h", None):
            lib.qlinear_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def prepare_prquant(w_bf16_bits: np.ndarray, k: int, scale_search: bool = False):
    """Offline PRQuant preparation on the host (library C++ code, not the oracle); scale_search
    selects the E8M0-W block-scale search.
    Returns (perm int32 [C], codes uint8 [N, (C+k)/2], scales uint8 [N, (C+k)/32])."""
    w = np.ascontiguousarray(w_bf16_bits, dtype=np.uint16)
    N, C = w.shape
    perm = np.empty(C, np.int32)
    codes = np.empty((N, (C + k) // 2), np.uint8)
    scales = np.empty((N, (C + k) // 32), np.uint8)
    _ok(lib.qlinear_prepare_prquant_ex(w.ctypes.data, N, C, k, int(bool(scale_search)),
                                       perm.ctypes.data, codes.ctypes.data, scales.ctypes.data),
        "qlinear_prepare_prquant_ex")
    return perm, codes, scales


def prepare_vq_prescale(w_bf16_bits: np.ndarray, codebooks_packed: np.ndarray, qn: int = 64,
                        qk: int = 64):
    """Offline MXCode PreScale preparation on the host (library C++ code).  codebooks_packed:
    uint8 [N/qn, K/qk, 256, 2].  Returns (ts float, E4M3 scales uint8 [N, K/16], idx uint8 [N, K/4])."""
    w = np.ascontiguousarray(w_bf16_bits, dtype=np.uint16)
    cb = np.ascontiguousarray(codebooks_packed, dtype=np.uint8)
    N, K = w.shape
    ts = np.zeros(1, np.float32)
    scales = np.empty((N, K // 16), np.uint8)
    idx = np.empty((N, K // 4), np.uint8)
    _ok(lib.qlinear_prepare_vq_prescale(w.ctypes.data, N, K, cb.ctypes.data, qn, qk, ts.ctypes.data,
                                        scales.ctypes.data, idx.ctypes.data),
        "qlinear_prepare_vq_prescale")
    return np.float32(ts[0]), scales, idx


def prepare_vq_postscale(w_bf16_bits: np.ndarray, centroids: np.ndarray):
    """Offline MXCode PostScale preparation on the host (library C++ code).  centroids: learned
    codebooks float32 [N/64, K/64, 256, 4].  Returns (ts, packed E2M1 codebooks uint8
    [N/64, K/64, 256, 2], QBlock E4M3 scale bytes [N/64, K/64], indices uint8 [N, K/4])."""
    w = np.ascontiguousarray(w_bf16_bits, dtype=np.uint16)
    c = np.ascontiguousarray(centroids, dtype=np.float32)
    N, K = w.shape
    ts = ctypes.c_float()
    cb = np.empty((N // 64, K // 64, 256, 2), np.uint8)
    qs = np.empty((N // 64, K // 64), np.uint8)
    idx = np.empty((N, K // 4), np.uint8)
    _ok(lib.qlinear_prepare_vq_postscale(w.ctypes.data, N, K, c.ctypes.data, 64, 64,
                                         ctypes.addressof(ts), cb.ctypes.data, qs.ctypes.data,
                                         idx.ctypes.data), "qlinear_prepare_vq_postscale")
    return np.float32(ts.value), cb, qs, idx


def prepare_vq_prescale_plus(w_bf16_bits: np.ndarray, codebooks_packed: np.ndarray,
                             scale_codebook: np.ndarray):
    """Offline MXCode PreScale+ preparation on the host (library C++ code).  Returns (ts,
    compressed E4M3 scales [N, K/16], scale indices [N, K/128], weight indices [N, K/4])."""
    w = np.ascontiguousarray(w_bf16_bits, dtype=np.uint16)
    cb = np.ascontiguousarray(codebooks_packed, dtype=np.uint8)
    scb = np.ascontiguousarray(scale_codebook, dtype=np.uint8)
    N, K = w.shape
    ts = ctypes.c_float()
    sb = np.empty((N, K // 16), np.uint8)
    sidx = np.empty((N, K // 128), np.uint8)
    idx = np.empty((N, K // 4), np.uint8)
    _ok(lib.qlinear_prepare_vq_prescale_plus(w.ctypes.data, N, K, cb.ctypes.data, scb.ctypes.data,
                                             64, 64, ctypes.addressof(ts), sb.ctypes.data,
                                             sidx.ctypes.data, idx.ctypes.data),
        "qlinear_prepare_vq_prescale_plus")
    return np.float32(ts.value), sb, sidx, idx


def _pack4(idx: np.ndarray) -> np.ndarray:
    idx = np.ascontiguousarray(idx, dtype=np.uint8)
    return ((idx[..., 0::2] & 0xF) | ((idx[..., 1::2] & 0xF) << 4)).astype(np.uint8)


class MoE:
    """Routed MoE FFN with CodeQuant-style cluster-codebook experts (see moe_create in qlinear.h).

    gu_idx uint8 [E*2I, H] 4-bit indices (values 0..15), gu_cent bf16 bit patterns [E*2I, 16];
    dn_idx [E*H, I], dn_cent [E*H, 16]; per expert the gate rows come first, then the up rows."""

    def __init__(self, gu_idx, gu_cent, dn_idx, dn_cent, E: int, top_k: int, had_x: bool = False,
                 had_h: bool = False, stream=None):
        """had_x / had_h: x (before gate/up), resp. h (before down), passes the online block-32
        Hadamard before its MXFP4 quantization; the expert weights given are the rotated ones."""
        gi, di = _pack4(gu_idx), _pack4(dn_idx)
        gc = np.ascontiguousarray(gu_cent, dtype=np.uint16)
        dc = np.ascontiguousarray(dn_cent, dtype=np.uint16)
        self.E, self.k = E, top_k
        self.H = gu_idx.shape[1]
        self.I = dn_idx.shape[1]
        g = WeightDesc(wfmt=QL_W_CLUSTER4_ROW16_BF16, N=gu_idx.shape[0], K=self.H,
                       codes=gi.ctypes.data, codebooks=gc.ctypes.data, had_block=32 if had_x else 0)
        d = WeightDesc(wfmt=QL_W_CLUSTER4_ROW16_BF16, N=dn_idx.shape[0], K=self.I,
                       codes=di.ctypes.data, codebooks=dc.ctypes.data, had_block=32 if had_h else 0)
        h = ctypes.c_void_p()
        _ok(lib.moe_create(ctypes.byref(g), ctypes.byref(d), E, top_k, _stream(stream),
                           ctypes.byref(h)), "moe_create")
        self._h = h
        self._ws = None

    def capture_intermediate(self, enable: bool = True) -> None:
        _ok(lib.moe_capture_intermediate(self._h, 1 if enable else 0), "moe_capture_intermediate")

    def workspace_bytes(self, T: int) -> int:
        n = ctypes.c_size_t()
        _ok(lib.moe_workspace_bytes(self._h, T, ctypes.byref(n)), "moe_workspace_bytes")
        return n.value

    def layout(self, T: int) -> dict:
        lay = MoeWsLayout()
        _ok(lib.moe_workspace_layout(self._h, T, ctypes.byref(lay)), "moe_workspace_layout")
        return {n: getattr(lay, n) for n, _ in MoeWsLayout._fields_}

    def workspace(self, T: int, device):
        import torch
        need = self.workspace_bytes(T)
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(need, dtype=torch.uint8, device=device)
        return self._ws

    def forward(self, x, logits, out=None, out_f32=None, ids_out=None, gates_out=None, ws=None,
                stream=None):
        import torch
        assert x.is_cuda and x.dtype == torch.bfloat16 and x.is_contiguous()
        assert logits.is_cuda and logits.dtype == torch.float32 and logits.is_contiguous()
        T = x.shape[0]
        if out is None:
            out = torch.empty((T, self.H), dtype=torch.bfloat16, device=x.device)
        if ws is None:
            ws = self.workspace(T, x.device)
        _ok(lib.moe_grouped_forward(self._h, x.data_ptr(), T, logits.data_ptr(), out.data_ptr(),
                                    _ptr(out_f32), _ptr(ids_out), _ptr(gates_out), ws.data_ptr(),
                                    ws.numel(), _stream(stream)), "moe_grouped_forward")
        return out

    __call__ = forward

    def close(self) -> None:
        if getattr(self, "_h", None):
            lib.moe_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def prepare_int4_bsr(w_bf16_bits: np.ndarray, x_calib_bf16_bits: np.ndarray,
                     density: float = 0.02) -> dict:
    """Offline INT4 dense + block-sparse residual preparation on the host (library C++ code).
    Returns codes [N,K/2], fp16 scale bits [N,K/128], rowptr, col, residual codes/scale bits."""
    w = np.ascontiguousarray(w_bf16_bits, dtype=np.uint16)
    x = np.ascontiguousarray(x_calib_bf16_bits, dtype=np.uint16)
    N, K = w.shape
    cap = int(round(density * (N // 16) * (K // 128))) + 1
    codes = np.empty((N, K // 2), np.uint8)
    scales = np.empty((N, K // 128), np.uint16)
    rowptr = np.empty(N // 16 + 1, np.int32)
    col = np.empty(cap, np.int16)
    rcodes = np.empty((cap, 16, 64), np.uint8)
    rscales = np.empty((cap, 16), np.uint16)
    nnzb = np.zeros(1, np.int32)
    _ok(lib.qlinear_prepare_int4_bsr(w.ctypes.data, N, K, x.ctypes.data, x.shape[0], density,
                                     codes.ctypes.data, scales.ctypes.data, rowptr.ctypes.data,
                                     col.ctypes.data, rcodes.ctypes.data, rscales.ctypes.data, cap,
                                     nnzb.ctypes.data), "qlinear_prepare_int4_bsr")
    n = int(nnzb[0])
    return dict(codes=codes, scales=scales, rowptr=rowptr, col=col[:n], rcodes=rcodes[:n],
                rscales=rscales[:n])
