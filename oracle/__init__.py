"""CPU oracle for the MosaicQuant / ZipperEngine hot path (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
may import this package. The CUDA library never calls it; the two share no code.

Thin numpy wrappers around ``mq_oracle.c`` (plain C, fp32/fp64 IEEE, compiled with
``-ffp-contract=off``). Each function states the definition it follows; the C file's
header gives the method's sources on the MosaicQuant pages and the readings taken
where those pages are silent.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mq_oracle.c")
_LIB = os.path.join(_HERE, "libmq_oracle.so")
_lib = None

CFLAGS = ["-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC", "-Wall"]


def build(force: bool = False) -> str:
    """Compile ``libmq_oracle.so`` next to its source."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _p(a: np.ndarray | None):
    return None if a is None else a.ctypes.data


def lib():
    global _lib
    if _lib is not None:
        return _lib
    L = ctypes.CDLL(build())
    vp, i32, f32, u8 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_uint8
    L.orc_e2m1_value.argtypes = [u8]
    L.orc_e2m1_value.restype = ctypes.c_double
    L.orc_e2m1_encode.argtypes = [f32]
    L.orc_e2m1_encode.restype = u8
    L.orc_e4m3_value.argtypes = [u8]
    L.orc_e4m3_value.restype = ctypes.c_double
    L.orc_e4m3_encode.argtypes = [f32]
    L.orc_e4m3_encode.restype = u8
    L.orc_global_scale_f32.argtypes = [vp, ctypes.c_int64]
    L.orc_global_scale_f32.restype = f32
    L.orc_nvfp4_quantize.argtypes = [vp, i32, i32, vp, i32, vp, vp, vp]
    L.orc_nvfp4_dequantize.argtypes = [vp, vp, i32, i32, vp, i32, vp]
    L.orc_quantize_weight.argtypes = [vp, i32, i32, vp, vp, vp, vp, vp]
    L.orc_quantize_act.argtypes = [vp, i32, i32, vp, vp, vp]
    L.orc_hessian_diag.argtypes = [vp, i32, i32, vp]
    L.orc_delta_score.argtypes = [vp, i32, i32, vp, vp, vp, f32, vp, vp, vp]
    L.orc_topk.argtypes = [vp, i32, i32, vp, vp]
    L.orc_pack_residual.argtypes = [vp, vp, i32, i32, vp, i32, vp, vp, vp, vp, vp]
    L.orc_sf_tile.argtypes = [vp, i32, i32, vp]
    L.orc_gemm_rows.argtypes = [vp, vp, vp, vp, vp, f32, vp, vp, vp, i32, i32, i32, i32, vp, i32, vp, vp]
    L.orc_smooth_scales.argtypes = [vp, i32, vp, i32, i32, vp]
    L.orc_smooth_apply.argtypes = [vp, i32, i32, vp, i32, vp]
    for name in ("orc_nvfp4_quantize", "orc_nvfp4_dequantize", "orc_quantize_weight", "orc_quantize_act",
                 "orc_hessian_diag", "orc_delta_score", "orc_topk", "orc_pack_residual", "orc_sf_tile",
                 "orc_gemm_rows", "orc_smooth_scales", "orc_smooth_apply"):
        getattr(L, name).restype = None
    _lib = L
    return L


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ---------------------------------------------------------------- formats
def e2m1_value(code: int) -> float:
    return lib().orc_e2m1_value(code)


def e2m1_encode(v: float) -> int:
    return lib().orc_e2m1_encode(v)


def e4m3_value(code: int) -> float:
    return lib().orc_e4m3_value(code)


def e4m3_encode(v: float) -> int:
    return lib().orc_e4m3_encode(v)


# ---------------------------------------------------------------- NVFP4
def nvfp4_quantize(a: np.ndarray, g) -> dict:
    """NVFP4 of fp32 rows with scale g (scalar, or one per row)."""
    a = _c(a, np.float32)
    rows, cols = a.shape
    gs = np.atleast_1d(_c(g, np.float32))
    stride = 1 if gs.size == rows and gs.size > 1 else 0
    codes = np.zeros((rows, cols // 2), np.uint8)
    sf = np.zeros((rows, cols // 16), np.uint8)
    deq = np.zeros((rows, cols), np.float32)
    lib().orc_nvfp4_quantize(_p(a), rows, cols, _p(gs), stride, _p(codes), _p(sf), _p(deq))
    return {"codes": codes, "sf": sf, "deq": deq}


def nvfp4_dequantize(codes: np.ndarray, sf: np.ndarray, g) -> np.ndarray:
    codes, sf = _c(codes, np.uint8), _c(sf, np.uint8)
    rows, cols = codes.shape[0], codes.shape[1] * 2
    gs = np.atleast_1d(_c(g, np.float32))
    stride = 1 if gs.size == rows and gs.size > 1 else 0
    out = np.zeros((rows, cols), np.float32)
    lib().orc_nvfp4_dequantize(_p(codes), _p(sf), rows, cols, _p(gs), stride, _p(out))
    return out


def global_scale(a: np.ndarray) -> float:
    a = _c(a, np.float32)
    return lib().orc_global_scale_f32(_p(a), a.size)


def quantize_weight(W: np.ndarray) -> dict:
    """A1: base NVFP4(W, g_w) and the full residual NVFP4(W - deq Q(W), g_w)."""
    W = _c(W, np.uint16)
    N, K = W.shape
    out = {k: np.zeros((N, K // 2), np.uint8) for k in ("codes", "r_codes")}
    out.update({k: np.zeros((N, K // 16), np.uint8) for k in ("sf", "r_sf")})
    g = np.zeros(1, np.float32)
    lib().orc_quantize_weight(_p(W), N, K, _p(out["codes"]), _p(out["sf"]), _p(g), _p(out["r_codes"]),
                              _p(out["r_sf"]))
    out["g"] = np.float32(g[0])
    return out


def quantize_act(X: np.ndarray) -> dict:
    """A6: per-token g_x[m] = amax(X[m]) / 2688, then NVFP4 of each row."""
    X = _c(X, np.uint16)
    M, K = X.shape
    codes = np.zeros((M, K // 2), np.uint8)
    sf = np.zeros((M, K // 16), np.uint8)
    g = np.zeros(M, np.float32)
    lib().orc_quantize_act(_p(X), M, K, _p(codes), _p(sf), _p(g))
    return {"codes": codes, "sf": sf, "g": g}


def hessian_diag(Xcal: np.ndarray) -> np.ndarray:
    """A2: H_k = fp32(sum_t x_tk^2 / T), fp64 sum by a pairwise tree over t."""
    Xcal = _c(Xcal, np.uint16)
    T, K = Xcal.shape
    H = np.zeros(K, np.float32)
    lib().orc_hessian_diag(_p(Xcal), T, K, _p(H))
    return H


def delta_score(W: np.ndarray, H: np.ndarray, wq: dict) -> np.ndarray:
    """A3: Delta [N/64, K/64] (fp64) with the fixed pairwise reduction tree."""
    W = _c(W, np.uint16)
    N, K = W.shape
    H = _c(H, np.float32)
    d = np.zeros((N // 64, K // 64), np.float64)
    lib().orc_delta_score(_p(W), N, K, _p(H), _p(_c(wq["codes"], np.uint8)), _p(_c(wq["sf"], np.uint8)),
                          float(wq["g"]), _p(_c(wq["r_codes"], np.uint8)), _p(_c(wq["r_sf"], np.uint8)), _p(d))
    return d


def topk(delta: np.ndarray, budget: int):
    """A4: rank (Delta desc, b asc) and sel (ascending b), int32 each."""
    d = _c(delta.reshape(-1), np.float64)
    rank = np.zeros(max(budget, 1), np.int32)
    sel = np.zeros(max(budget, 1), np.int32)
    lib().orc_topk(_p(d), d.size, budget, _p(rank), _p(sel))
    return rank[:budget], sel[:budget]


def pack_residual(wq: dict, sel: np.ndarray, N: int, K: int) -> dict:
    """A5: compact residual store, per-row-of-blocks CSR and bitmap."""
    sel = _c(sel, np.int32)
    nb = sel.size
    KB, NBr = K // 64, N // 64
    KW = (KB + 31) // 32
    out = {"blk_codes": np.zeros((max(nb, 1), 2048), np.uint8), "blk_sf": np.zeros((max(nb, 1), 512), np.uint8),
           "blk_kt": np.zeros(max(nb, 1), np.int32), "tile_ptr": np.zeros(NBr + 1, np.int32),
           "bitmap": np.zeros((NBr, KW), np.uint32)}
    lib().orc_pack_residual(_p(_c(wq["r_codes"], np.uint8)), _p(_c(wq["r_sf"], np.uint8)), N, K, _p(sel), nb,
                            _p(out["blk_codes"]), _p(out["blk_sf"]), _p(out["blk_kt"]), _p(out["tile_ptr"]),
                            _p(out["bitmap"]))
    for k in ("blk_codes", "blk_sf", "blk_kt"):
        out[k] = out[k][:nb]
    return out


def sf_tile(sf: np.ndarray, rows: int, cols: int) -> np.ndarray:
    """Tiled (GEMM) scale layout of a row-major [rows][cols/16] scale array."""
    sf = _c(sf, np.uint8)
    rt = (rows + 127) // 128
    out = np.zeros(rt * 128 * (cols // 16), np.uint8)
    lib().orc_sf_tile(_p(sf), rows, cols, _p(out))
    return out


def block_mask(sel: np.ndarray, N: int, K: int) -> np.ndarray:
    m = np.zeros((N // 64) * (K // 64), np.uint8)
    m[np.asarray(sel, dtype=np.int64)] = 1
    return m.reshape(N // 64, K // 64)


def gemm_rows(xq: dict, wq: dict, sel, M: int, N: int, K: int, mode: int = 0, rows=None):
    """A7-A8 fp64 reference for the given output rows: (y [r, N], yabs [r, N]).

    mode 0: base + selected residual; 1: base only; 2: residual only.
    """
    rows = np.arange(M, dtype=np.int32) if rows is None else _c(rows, np.int32)
    mask = None if sel is None else block_mask(sel, N, K)
    y = np.zeros((rows.size, N), np.float64)
    ya = np.zeros((rows.size, N), np.float64)
    gx = _c(xq["g"], np.float32)
    lib().orc_gemm_rows(_p(_c(xq["codes"], np.uint8)), _p(_c(xq["sf"], np.uint8)), _p(gx),
                        _p(_c(wq["codes"], np.uint8)), _p(_c(wq["sf"], np.uint8)), float(wq["g"]),
                        _p(_c(wq["r_codes"], np.uint8)), _p(_c(wq["r_sf"], np.uint8)), _p(mask), M, N, K, mode,
                        _p(rows), rows.size, _p(y), _p(ya))
    return y, ya


def smooth_scales(Xcal: np.ndarray, W: np.ndarray) -> np.ndarray:
    """Equivalent transform (SmoothQuant, alpha = 1/2): s_k = sqrt(max|Xcal_k| / max|W_k|)."""
    Xcal, W = _c(Xcal, np.uint16), _c(W, np.uint16)
    T, K = Xcal.shape
    N = W.shape[0]
    s = np.zeros(K, np.float32)
    lib().orc_smooth_scales(_p(Xcal), T, _p(W), N, K, _p(s))
    return s


def smooth_apply(A: np.ndarray, s: np.ndarray, invert: bool) -> np.ndarray:
    """bf16(A * s_k) (weights) or bf16(A / s_k) (activations), as bf16 bits."""
    A = _c(A, np.uint16)
    rows, K = A.shape
    out = np.zeros_like(A)
    lib().orc_smooth_apply(_p(A), rows, K, _p(_c(s, np.float32)), 1 if invert else 0, _p(out))
    return out


def run_path(W: np.ndarray, X: np.ndarray, Xcal: np.ndarray, budget: int, rows=None) -> dict:
    """The whole path in the method's order: quantize W, H, Delta, top-K, pack,
    quantize X, reference GEMM."""
    N, K = W.shape
    M = X.shape[0]
    wq = quantize_weight(W)
    H = hessian_diag(Xcal)
    delta = delta_score(W, H, wq)
    rank, sel = topk(delta, budget)
    packed = pack_residual(wq, sel, N, K)
    xq = quantize_act(X)
    y, ya = gemm_rows(xq, wq, sel, M, N, K, 0, rows)
    return {"wq": wq, "H": H, "delta": delta, "rank": rank, "sel": sel, "packed": packed, "xq": xq,
            "y": y, "yabs": ya}
