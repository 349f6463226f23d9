"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI and the
CPU oracle on the same seeded inputs, and compare."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import synth


def to_dev(bits: np.ndarray, dev) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)


def prepare(layer, W, Xc, fused):
    """fused: False = separate calls, True = one quantize+Delta pass with the full residual
    stored and packed from it, "path" = as mq_run_layer (residual packed from W)."""
    if fused == "path":
        layer.prepare_path(W, Xc)
    elif fused:
        layer.prepare_fused(W, Xc)
    else:
        layer.prepare(W, Xc)


def gpu_run(L: dict, budget: int, dev, flags: int = 0, X_bits=None, fused=False):
    """Whole path on the GPU for layer inputs L (bf16 bits); returns numpy copies.
    fused: see prepare()."""
    from bit_quantized_gemm_zipperengine_b200 import mosaic
    N, K = L["N"], L["K"]
    W = to_dev(L["W"], dev)
    Xc = to_dev(L["Xcal"], dev)
    X = to_dev(L["X"] if X_bits is None else X_bits, dev)
    layer = mosaic.Layer(N, K, budget, dev)
    prepare(layer, W, Xc, fused)
    Y = layer.forward(X, flags)
    xq = layer.act_buffers(X.shape[0], flags)[0]
    torch.cuda.synchronize()
    assert mosaic.mq_get_error() == 0
    out = {"layer": layer, "W": W, "X": X,
           "codes": layer.base["codes"].cpu().numpy(), "sf": layer.base["sf"].cpu().numpy(),
           "sf_swz": layer.base["sf_swz"].cpu().numpy(), "g": layer.base["gscale"].cpu().numpy()[0],
           "r_codes": layer.resid["codes"].cpu().numpy(), "r_sf": layer.resid["sf"].cpu().numpy(),
           "H": layer.H.cpu().numpy(), "delta": layer.delta.cpu().numpy().reshape(N // 64, K // 64),
           "rank": layer.rank[:budget].cpu().numpy(), "sel": layer.sel[:budget].cpu().numpy(),
           "packed": {k: (v[:budget] if k in ("blk_codes", "blk_sf", "blk_kt") else v).cpu().numpy()
                      for k, v in layer.packed.items() if isinstance(v, torch.Tensor)},
           "xq_codes": xq["codes"].cpu().numpy(), "xq_swz": xq["sf_swz"].cpu().numpy(),
           "xq_g": xq["gscale"].cpu().numpy(), "Y": Y.float().cpu().numpy().astype(np.float64)}
    return out


def check_gemm(y: np.ndarray, y_ref: np.ndarray, yabs: np.ndarray, what: str = ""):
    """Per element |y - y_ref| <= 1e-2 |y_ref| + 2e-3 yabs, and relative Frobenius <= 5e-3,
    where yabs = g_x g_w sum_k |xh (wh + rh)| (the GEMM's tolerance)."""
    err = np.abs(y - y_ref)
    bound = 1e-2 * np.abs(y_ref) + 2e-3 * yabs
    bad = np.argwhere(err > bound)
    assert bad.size == 0, (f"{what}: {len(bad)} elements outside tolerance, first {bad[:5].tolist()}, "
                           f"y={y[tuple(bad[0])]}, ref={y_ref[tuple(bad[0])]}")
    rel = np.linalg.norm(y - y_ref) / max(np.linalg.norm(y_ref), 1e-300)
    assert rel <= 5e-3, f"{what}: relative Frobenius error {rel}"
    return rel


def oracle_ref(L: dict, budget: int, rows=None):
    return oracle.run_path(L["W"], L["X"], L["Xcal"], budget, rows)
