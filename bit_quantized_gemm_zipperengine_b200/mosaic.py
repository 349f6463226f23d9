"""ctypes binding of libmosaic (include/mosaic.h).

Argument marshalling only: every step of the path runs in the CUDA library. PyTorch
provides device memory and the current stream. There is no CPU fallback: a missing
library or a non-CUDA tensor raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmosaic.so")
_lib = None

MQ_OK = 0
MQ_GEMM_AUTO = 0
MQ_GEMM_DECODE = 1
MQ_GEMM_PREFILL = 2
MQ_GEMM_BASE_ONLY = 4
MQ_GEMM_RESIDUAL_ONLY = 8
MQ_LAYER_PREPARED = 16
MQ_GEMM_WEIGHTS_READY = 32

EXPORTED = (
    "mq_sf_swz_bytes", "mq_budget_blocks", "mq_quantize_weight_workspace_bytes", "mq_delta_topk_workspace_bytes",
    "mq_gemm_workspace_bytes", "mq_quantize_weight", "mq_hessian_diag", "mq_delta_score_topk", "mq_pack_residual",
    "mq_quantize_act", "mq_gemm", "mq_run_layer", "mq_get_error", "mq_status_string", "mq_launch_count",
    "mq_gemm_noalloc", "mq_gemm_noalloc_scratch_limit", "mq_quantize_weight_delta", "mq_topk_blocks",
    "mq_pack_residual_weight", "mq_gemm_act", "mq_weight_bytes", "mq_fp4_mma_loop", "mq_fp4_mma_loop_flops",
    "mq_test_arm_wait_fault", "mq_smooth_scales", "mq_smooth_apply", "mq_timeline_read",
)


class MosaicError(RuntimeError):
    pass


class NVFP4Mat(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_int), ("cols", ctypes.c_int), ("codes", ctypes.c_void_p), ("sf", ctypes.c_void_p),
                ("sf_swz", ctypes.c_void_p), ("gscale", ctypes.c_void_p)]


class ResidualPacked(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int), ("K", ctypes.c_int), ("nblk", ctypes.c_int), ("blk_codes", ctypes.c_void_p),
                ("blk_sf", ctypes.c_void_p), ("blk_kt", ctypes.c_void_p), ("tile_ptr", ctypes.c_void_p),
                ("bitmap", ctypes.c_void_p)]


class LayerBuffers(ctypes.Structure):
    _fields_ = [("base", NVFP4Mat), ("resid_full", NVFP4Mat), ("xq", NVFP4Mat), ("H", ctypes.c_void_p),
                ("delta", ctypes.c_void_p), ("rank", ctypes.c_void_p), ("sel", ctypes.c_void_p),
                ("packed", ResidualPacked), ("ws_quant", ctypes.c_void_p), ("ws_quant_bytes", ctypes.c_size_t),
                ("ws_gemm", ctypes.c_void_p), ("ws_gemm_bytes", ctypes.c_size_t), ("W_dev", ctypes.c_void_p),
                ("X_dev", ctypes.c_void_p), ("Xcal_dev", ctypes.c_void_p), ("Y_dev", ctypes.c_void_p)]


def lib():
    """Load libmosaic.so (built by ``__graft_entry__.build()`` or ``build.py``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise MosaicError(f"libmosaic.so is not built ({LIB_PATH}); run __graft_entry__.build()")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    P = ctypes.POINTER
    L.mq_sf_swz_bytes.argtypes = [i32, i32]
    L.mq_sf_swz_bytes.restype = sz
    L.mq_weight_bytes.argtypes = [i32, i32]
    L.mq_weight_bytes.restype = sz
    L.mq_fp4_mma_loop.argtypes = [i32, i32, vp]
    L.mq_fp4_mma_loop.restype = i32
    L.mq_fp4_mma_loop_flops.argtypes = [i32, i32]
    L.mq_fp4_mma_loop_flops.restype = ctypes.c_double
    L.mq_timeline_read.argtypes = [vp, ctypes.c_size_t]
    L.mq_timeline_read.restype = i32
    L.mq_test_arm_wait_fault.argtypes = [i32, ctypes.c_double]
    L.mq_test_arm_wait_fault.restype = i32
    L.mq_smooth_scales.argtypes = [vp, i32, vp, i32, i32, vp, vp]
    L.mq_smooth_scales.restype = i32
    L.mq_smooth_apply.argtypes = [vp, i32, i32, vp, i32, vp, vp]
    L.mq_smooth_apply.restype = i32
    L.mq_budget_blocks.argtypes = [i32, i32, ctypes.c_double]
    L.mq_budget_blocks.restype = i32
    L.mq_quantize_weight_workspace_bytes.argtypes = [i32, i32]
    L.mq_quantize_weight_workspace_bytes.restype = sz
    L.mq_delta_topk_workspace_bytes.argtypes = [i32, i32, i32]
    L.mq_delta_topk_workspace_bytes.restype = sz
    L.mq_gemm_workspace_bytes.argtypes = [i32, i32, i32, ctypes.c_uint]
    L.mq_gemm_workspace_bytes.restype = sz
    L.mq_quantize_weight.argtypes = [vp, i32, i32, P(NVFP4Mat), P(NVFP4Mat), vp, sz, vp]
    L.mq_hessian_diag.argtypes = [vp, i32, i32, vp, vp]
    L.mq_delta_score_topk.argtypes = [vp, vp, P(NVFP4Mat), P(NVFP4Mat), i32, vp, vp, vp, vp, sz, vp]
    L.mq_pack_residual.argtypes = [P(NVFP4Mat), vp, i32, P(ResidualPacked), vp]
    L.mq_quantize_act.argtypes = [vp, i32, i32, P(NVFP4Mat), vp]
    L.mq_gemm.argtypes = [P(NVFP4Mat), P(NVFP4Mat), P(ResidualPacked), vp, i32, i32, i32, ctypes.c_uint, vp, sz, vp]
    for f in ("mq_quantize_weight", "mq_hessian_diag", "mq_delta_score_topk", "mq_pack_residual", "mq_quantize_act",
              "mq_gemm", "mq_get_error"):
        getattr(L, f).restype = i32
    L.mq_run_layer.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, ctypes.c_uint, i32, P(LayerBuffers), vp]
    L.mq_run_layer.restype = i32
    L.mq_gemm_noalloc.argtypes = [P(NVFP4Mat), P(NVFP4Mat), P(ResidualPacked), vp, i32, i32, i32, ctypes.c_uint, vp]
    L.mq_gemm_noalloc.restype = i32
    L.mq_gemm_noalloc_scratch_limit.argtypes = []
    L.mq_gemm_noalloc_scratch_limit.restype = sz
    L.mq_quantize_weight_delta.argtypes = [vp, i32, i32, vp, P(NVFP4Mat), P(NVFP4Mat), vp, vp, sz, vp]
    L.mq_quantize_weight_delta.restype = i32
    L.mq_topk_blocks.argtypes = [vp, i32, i32, vp, vp, vp]
    L.mq_topk_blocks.restype = i32
    L.mq_pack_residual_weight.argtypes = [vp, P(NVFP4Mat), vp, i32, P(ResidualPacked), vp]
    L.mq_pack_residual_weight.restype = i32
    L.mq_gemm_act.argtypes = [vp, P(NVFP4Mat), P(ResidualPacked), vp, i32, i32, i32, ctypes.c_uint, vp, sz, vp, vp]
    L.mq_gemm_act.restype = i32
    L.mq_get_error.argtypes = [vp]
    L.mq_status_string.argtypes = [i32]
    L.mq_status_string.restype = ctypes.c_char_p
    L.mq_launch_count.argtypes = []
    L.mq_launch_count.restype = ctypes.c_uint64
    _lib = L
    return L


def _check(status: int, what: str):
    if status != MQ_OK:
        raise MosaicError(f"{what}: {lib().mq_status_string(status).decode()} (status {status})")


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise MosaicError("libmosaic takes CUDA tensors only")
    return t.data_ptr()


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _u8(*shape, device):
    return torch.empty(shape, dtype=torch.uint8, device=device)


def mat(d: dict) -> NVFP4Mat:
    return NVFP4Mat(d["rows"], d["cols"], _ptr(d.get("codes")), _ptr(d.get("sf")), _ptr(d.get("sf_swz")),
                    _ptr(d.get("gscale")))


def packed_struct(p: dict | None) -> ResidualPacked | None:
    if p is None:
        return None
    return ResidualPacked(p["N"], p["K"], p["nblk"], _ptr(p.get("blk_codes")), _ptr(p.get("blk_sf")),
                          _ptr(p.get("blk_kt")), _ptr(p.get("tile_ptr")), _ptr(p.get("bitmap")))


# ------------------------------------------------------------------ allocation helpers
def alloc_weight(N: int, K: int, device, with_sf: bool = True) -> tuple[dict, dict]:
    """Base (GEMM-ready NVFP4 weight) and full-residual buffers of an N x K weight.

    The base's codes, tiled scales and tensor scale are views of ONE allocation of
    mq_weight_bytes(N, K) bytes at the offsets include/mosaic.h states; its optional
    linear scales and the residual are separate tensors."""
    L = lib()
    nbytes = L.mq_weight_bytes(N, K)
    if nbytes == 0:
        raise MosaicError(f"bad weight shape {N} x {K}")
    blob = _u8(nbytes, device=device)
    nc, ns = N * (K // 2), L.mq_sf_swz_bytes(N, K)
    base = {"rows": N, "cols": K, "codes": blob[:nc].view(N, K // 2),
            "sf": _u8(N, K // 16, device=device) if with_sf else None,
            "sf_swz": blob[nc:nc + ns],
            "gscale": blob[nc + ns:nc + ns + 4].view(torch.float32), "blob": blob}
    resid = {"rows": N, "cols": K, "codes": _u8(N, K // 2, device=device), "sf": _u8(N, K // 16, device=device),
             "sf_swz": None, "gscale": None}
    return base, resid


def alloc_act(M: int, K: int, device, with_sf: bool = False) -> dict:
    L = lib()
    return {"rows": M, "cols": K, "codes": _u8(M, K // 2, device=device),
            "sf": _u8(M, K // 16, device=device) if with_sf else None,
            "sf_swz": _u8(L.mq_sf_swz_bytes(M, K), device=device),
            "gscale": torch.empty(M, dtype=torch.float32, device=device)}


def alloc_packed(N: int, K: int, budget: int, device) -> dict:
    KB = K // 64
    KW = (KB + 31) // 32
    nb = max(budget, 1)
    return {"N": N, "K": K, "nblk": budget, "blk_codes": _u8(nb, 2048, device=device),
            "blk_sf": _u8(nb, 512, device=device), "blk_kt": torch.empty(nb, dtype=torch.int32, device=device),
            "tile_ptr": torch.empty(N // 64 + 1, dtype=torch.int32, device=device),
            "bitmap": torch.empty((N // 64, KW), dtype=torch.int32, device=device)}


# ------------------------------------------------------------------ the path (C names)
def mq_smooth_scales(Xcal: torch.Tensor, W: torch.Tensor, s: torch.Tensor, stream=None):
    T, K = Xcal.shape
    N = W.shape[0]
    _check(lib().mq_smooth_scales(_ptr(Xcal), T, _ptr(W), N, K, _ptr(s), _stream(stream)), "mq_smooth_scales")


def mq_smooth_apply(A: torch.Tensor, s: torch.Tensor, invert: bool, out: torch.Tensor, stream=None):
    rows, K = A.shape
    _check(lib().mq_smooth_apply(_ptr(A), rows, K, _ptr(s), 1 if invert else 0, _ptr(out), _stream(stream)),
           "mq_smooth_apply")


def mq_quantize_weight(W: torch.Tensor, base: dict, resid: dict, ws: torch.Tensor, stream=None):
    N, K = W.shape
    _check(lib().mq_quantize_weight(_ptr(W), N, K, ctypes.byref(mat(base)), ctypes.byref(mat(resid)), _ptr(ws),
                                    ws.numel() * ws.element_size(), _stream(stream)), "mq_quantize_weight")


def mq_quantize_weight_delta(W: torch.Tensor, H: torch.Tensor, base: dict, resid: dict | None, delta: torch.Tensor,
                             ws: torch.Tensor, stream=None):
    """resid None: the full residual is not stored (see mq_pack_residual_weight)."""
    N, K = W.shape
    r = None if resid is None else ctypes.byref(mat(resid))
    _check(lib().mq_quantize_weight_delta(_ptr(W), N, K, _ptr(H), ctypes.byref(mat(base)), r,
                                          _ptr(delta), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "mq_quantize_weight_delta")


def mq_topk_blocks(delta: torch.Tensor, budget: int, rank, sel, stream=None):
    _check(lib().mq_topk_blocks(_ptr(delta), delta.numel(), budget, _ptr(rank), _ptr(sel), _stream(stream)),
           "mq_topk_blocks")


def mq_hessian_diag(Xcal: torch.Tensor, H: torch.Tensor, stream=None):
    T, K = Xcal.shape
    _check(lib().mq_hessian_diag(_ptr(Xcal), T, K, _ptr(H), _stream(stream)), "mq_hessian_diag")


def mq_delta_score_topk(W, H, base: dict, resid: dict | None, budget: int, delta, rank, sel, ws=None, stream=None):
    wsb = 0 if ws is None else ws.numel() * ws.element_size()
    rs = None if resid is None else ctypes.byref(mat(resid))
    _check(lib().mq_delta_score_topk(_ptr(W), _ptr(H), ctypes.byref(mat(base)), rs, budget, _ptr(delta), _ptr(rank),
                                     _ptr(sel), _ptr(ws), wsb, _stream(stream)), "mq_delta_score_topk")


def mq_pack_residual(resid: dict, sel, budget: int, packed: dict, stream=None):
    _check(lib().mq_pack_residual(ctypes.byref(mat(resid)), _ptr(sel), budget, ctypes.byref(packed_struct(packed)),
                                  _stream(stream)), "mq_pack_residual")


def mq_pack_residual_weight(W: torch.Tensor, base: dict, sel, budget: int, packed: dict, stream=None):
    _check(lib().mq_pack_residual_weight(_ptr(W), ctypes.byref(mat(base)), _ptr(sel), budget,
                                         ctypes.byref(packed_struct(packed)), _stream(stream)),
           "mq_pack_residual_weight")


def mq_quantize_act(X: torch.Tensor, xq: dict, stream=None):
    M, K = X.shape
    _check(lib().mq_quantize_act(_ptr(X), M, K, ctypes.byref(mat(xq)), _stream(stream)), "mq_quantize_act")


def mq_gemm(xq: dict, wq: dict, packed: dict | None, Y: torch.Tensor, M: int, N: int, K: int, flags: int = 0,
            ws: torch.Tensor | None = None, stream=None):
    ps = packed_struct(packed)
    wsb = 0 if ws is None else ws.numel() * ws.element_size()
    _check(lib().mq_gemm(ctypes.byref(mat(xq)), ctypes.byref(mat(wq)), None if ps is None else ctypes.byref(ps),
                         _ptr(Y), M, N, K, flags, _ptr(ws), wsb, _stream(stream)), "mq_gemm")


def mq_run_layer(W, X, Xcal, Y, M: int, N: int, K: int, T: int, budget: int, flags: int, host: bool,
                 buf: LayerBuffers, stream=None):
    """Whole path in one call. With host=True, W/X/Xcal/Y are pinned CPU tensors."""
    def p(t):
        if t is None:
            return None
        if host:
            if t.is_cuda:
                raise MosaicError("host=True expects CPU tensors")
            return t.data_ptr()
        return _ptr(t)
    _check(lib().mq_run_layer(p(W), p(X), p(Xcal), p(Y), M, N, K, T, budget, flags, 1 if host else 0,
                              ctypes.byref(buf), _stream(stream)), "mq_run_layer")


def mq_gemm_act(X: torch.Tensor, wq: dict, packed: dict | None, Y: torch.Tensor, M: int, N: int, K: int,
                flags: int = 0, ws: torch.Tensor | None = None, gx: torch.Tensor | None = None, stream=None):
    """Decode-kernel GEMM that quantizes the bf16 activations itself (gx receives g_x)."""
    ps = packed_struct(packed)
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(lib().mq_gemm_act(_ptr(X), ctypes.byref(mat(wq)), None if ps is None else ctypes.byref(ps), _ptr(Y), M, N,
                             K, flags, _ptr(ws), nbytes, _ptr(gx), _stream(stream)), "mq_gemm_act")


def mq_gemm_noalloc(xq: dict, wq: dict, packed: dict | None, Y: torch.Tensor, M: int, N: int, K: int,
                    flags: int = 0, stream=None):
    """mq_gemm for callers that cannot allocate device memory: no workspace argument,
    the split-K scratch is a static buffer inside the library (see include/mosaic.h)."""
    ps = packed_struct(packed)
    _check(lib().mq_gemm_noalloc(ctypes.byref(mat(xq)), ctypes.byref(mat(wq)), None if ps is None else ctypes.byref(ps),
                                 _ptr(Y), M, N, K, flags, _stream(stream)), "mq_gemm_noalloc")


def mq_fp4_mma_loop(ctas: int, iters: int, stream=None) -> float:
    """Launch the FP4 MMA-loop probe (include/mosaic_probe.h); returns its flop count."""
    _check(lib().mq_fp4_mma_loop(ctas, iters, _stream(stream)), "mq_fp4_mma_loop")
    return float(lib().mq_fp4_mma_loop_flops(ctas, iters))


def mq_get_error(stream=None) -> int:
    return lib().mq_get_error(_stream(stream))


def mq_launch_count() -> int:
    return int(lib().mq_launch_count())


def gemm_workspace(M: int, N: int, K: int, flags: int, device) -> torch.Tensor | None:
    """Zero-initialised workspace for mq_gemm (the tile counters must start at zero)."""
    n = lib().mq_gemm_workspace_bytes(M, N, K, flags)
    return torch.zeros(max(n, 16), dtype=torch.uint8, device=device) if n else None


# ------------------------------------------------------------------ convenience
class Layer:
    """One linear layer through the whole path: quantize W, H from calibration tokens,
    Delta + top-K, pack, then per call quantize X and run the fused GEMM. Buffers are
    allocated once (torch) and reused."""

    def __init__(self, N: int, K: int, budget: int, device="cuda", with_sf: bool = True):
        self.N, self.K, self.budget, self.device = N, K, budget, device
        self.base, self.resid = alloc_weight(N, K, device, with_sf)
        self.qws = torch.empty(lib().mq_quantize_weight_workspace_bytes(N, K), dtype=torch.uint8, device=device)
        self.H = torch.empty(K, dtype=torch.float32, device=device)
        self.delta = torch.empty((N // 64) * (K // 64), dtype=torch.float64, device=device)
        self.rank = torch.empty(max(budget, 1), dtype=torch.int32, device=device)
        self.sel = torch.empty(max(budget, 1), dtype=torch.int32, device=device)
        self.packed = alloc_packed(N, K, budget, device)
        self._act = {}

    def prepare(self, W: torch.Tensor, Xcal: torch.Tensor, stream=None):
        """A1..A5 through the separate calls (quantize, H, Delta + top-K, pack)."""
        mq_quantize_weight(W, self.base, self.resid, self.qws, stream)
        mq_hessian_diag(Xcal, self.H, stream)
        mq_delta_score_topk(W, self.H, self.base, None, self.budget, self.delta, self.rank, self.sel, None, stream)
        mq_pack_residual(self.resid, self.sel, self.budget, self.packed, stream)

    def prepare_fused(self, W: torch.Tensor, Xcal: torch.Tensor, stream=None):
        """A1..A5 with quantization and Delta in one pass over W; the full residual is stored
        and the selected blocks packed from it."""
        mq_hessian_diag(Xcal, self.H, stream)
        mq_quantize_weight_delta(W, self.H, self.base, self.resid, self.delta, self.qws, stream)
        mq_topk_blocks(self.delta, self.budget, self.rank, self.sel, stream)
        mq_pack_residual(self.resid, self.sel, self.budget, self.packed, stream)

    def prepare_path(self, W: torch.Tensor, Xcal: torch.Tensor, stream=None):
        """A1..A5 as mq_run_layer: the full residual is not stored; the selected blocks are
        recomputed from W when packed."""
        mq_hessian_diag(Xcal, self.H, stream)
        mq_quantize_weight_delta(W, self.H, self.base, None, self.delta, self.qws, stream)
        mq_topk_blocks(self.delta, self.budget, self.rank, self.sel, stream)
        mq_pack_residual_weight(W, self.base, self.sel, self.budget, self.packed, stream)

    def act_buffers(self, M: int, flags: int = 0, slot: int = 0):
        """Quantized X, Y and the GEMM workspace for M tokens (cached per M, flags and slot:
        calls in flight together on different streams take different slots)."""
        key = (M, flags, slot)
        if key not in self._act:
            self._act[key] = (alloc_act(M, self.K, self.device),
                              torch.empty((M, self.N), dtype=torch.bfloat16, device=self.device),
                              gemm_workspace(M, self.N, self.K, flags, self.device))
        return self._act[key]

    def buffers(self, M: int, T: int, flags: int = 0, staging: bool = False, slot: int = 0) -> LayerBuffers:
        """The ctypes struct mq_run_layer takes (staging buffers for host inputs). Every slot
        has its own activation and staging buffers; the layer's weights are shared."""
        xq, Y, ws = self.act_buffers(M, flags, slot)
        b = LayerBuffers()
        b.base, b.resid_full, b.xq = mat(self.base), mat(self.resid), mat(xq)
        b.H, b.delta, b.rank, b.sel = _ptr(self.H), _ptr(self.delta), _ptr(self.rank), _ptr(self.sel)
        b.packed = packed_struct(self.packed)
        b.ws_quant, b.ws_quant_bytes = _ptr(self.qws), self.qws.numel()
        b.ws_gemm, b.ws_gemm_bytes = (_ptr(ws), ws.numel()) if ws is not None else (None, 0)
        if staging:
            key = ("staging", M, T, slot)
            if key not in self._act:
                bf = torch.bfloat16
                self._act[key] = (torch.empty((self.N, self.K), dtype=bf, device=self.device),
                                  torch.empty((M, self.K), dtype=bf, device=self.device),
                                  torch.empty((T, self.K), dtype=bf, device=self.device))
            w, x, xc = self._act[key]
            b.W_dev, b.X_dev, b.Xcal_dev, b.Y_dev = _ptr(w), _ptr(x), _ptr(xc), _ptr(Y)
        return b

    def forward(self, X: torch.Tensor, flags: int = 0, stream=None) -> torch.Tensor:
        """A6 + A7/A8 on bf16 X [M][K] (device). Returns the layer's output buffer for this M
        and flags: the next call with the same M and flags writes into the same tensor."""
        M = X.shape[0]
        xq, Y, ws = self.act_buffers(M, flags)
        mq_quantize_act(X, xq, stream)
        mq_gemm(xq, self.base, self.packed, Y, M, self.N, self.K, flags, ws, stream)
        return Y
