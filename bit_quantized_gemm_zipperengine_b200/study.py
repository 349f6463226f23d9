"""Distortion-recovery study (MosaicQuant summary (pt), "Metodologia" section 2, and the
arXiv abstract: the Hessian-guided Delta-score stands in for an exact evaluation of each
block's reduction of the output distortion, and giving the residual to about 10% of the
blocks recovers more than half of the distortion).

For a layer W, calibration activations X (T x K) and a set S of blocks that carry the
residual, the output distortion is

    E(S) = || X D_S^T ||_F^2,   D_S = e outside S, e' inside S,

with e = fp32(W - deq Q(W)) and e' = fp32(e - deq R) exactly as the library computes them.
With G = X^T X and U = D G, adding block b (rows R_b, columns C_b, d = e' - e on it)
changes E by

    dE_b = 2 <d, U[R_b, C_b]> + <d G[C_b, C_b], d>,

and U[R_b, :] += d G[C_b, :]. The Delta-score is -dE_b / T with G replaced by its
diagonal, at S = {}; the exact greedy selection takes the most negative dE_b at every
step. Both curves are exact E(S) values (fp64), so they can be compared with each other
and with E({}) and E(all blocks).

The quantization, H, Delta and the Delta-order selection come from the library (the
CUDA path); this module only evaluates them. The evaluation is in fp64 on the device.

    python -m bit_quantized_gemm_zipperengine_b200.study --workload llama3_8b_qproj_decode
"""
from __future__ import annotations

import argparse
import json

import torch

E2M1_VALUES = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)


def dequant_nvfp4(codes: torch.Tensor, sf: torch.Tensor, g: torch.Tensor) -> torch.Tensor:
    """fp32 values of an NVFP4 matrix: codes u8 [rows][cols/2] (element 2j in the low
    nibble of byte j), linear E4M3 scales u8 [rows][cols/16], tensor scale g (fp32, [1]).
    value = fp32(val(code) * fp32(dec(sf) * g)), the quantizers' dequantization."""
    rows = codes.shape[0]
    c = codes.to(torch.int32)
    nib = torch.stack((c & 0xF, c >> 4), dim=-1).reshape(rows, -1)
    mag = torch.tensor(E2M1_VALUES, dtype=torch.float32, device=codes.device)[nib & 7]
    val = torch.where((nib & 8) != 0, -mag, mag)
    s = sf.to(torch.int32)
    e, m = (s >> 3) & 15, s & 7
    dec = torch.where(e == 0, m.to(torch.float32) * 2.0 ** -9,
                      torch.exp2((e - 7).to(torch.float32)) * (1.0 + m.to(torch.float32) / 8.0))
    d = dec * g.to(torch.float32).reshape(1, 1)                 # fp32(dec * g)
    return val * d.repeat_interleave(16, dim=1)                   # fp32(val * d)


class Distortion:
    """Exact E(S) for selections built one block at a time (fp64)."""

    def __init__(self, e: torch.Tensor, ep: torch.Tensor, X: torch.Tensor, block: int = 64):
        self.b = block
        self.N, self.K = e.shape
        self.NB, self.KB = self.N // block, self.K // block
        X = X.to(torch.float64)
        self.T = X.shape[0]
        self.G = X.T @ X
        self.D0 = e.to(torch.float64)
        self.delta = ep.to(torch.float64) - self.D0               # change of D on every block
        self.E_all = float(((ep.to(torch.float64) @ self.G) * ep.to(torch.float64)).sum())
        b, KB = block, self.KB
        quad = torch.empty(self.NB, KB, dtype=torch.float64, device=e.device)
        for kt in range(KB):
            cols = slice(kt * b, (kt + 1) * b)
            dk = self.delta[:, cols]
            quad[:, kt] = ((dk @ self.G[cols, cols]) * dk).sum(1).reshape(self.NB, b).sum(1)
        self.quad = quad
        self.reset()

    def reset(self):
        self.U = self.D0 @ self.G
        self.E = float((self.D0 * self.U).sum())
        self.E0 = self.E
        self.taken = torch.zeros(self.NB * self.KB, dtype=torch.bool, device=self.U.device)
        self.lin = self._lin_rows(0, self.NB)

    def _lin_rows(self, nt0: int, nt1: int) -> torch.Tensor:
        b = self.b
        r = slice(nt0 * b, nt1 * b)
        p = (self.delta[r] * self.U[r]).reshape(nt1 - nt0, b, self.KB, b)
        return 2.0 * p.sum(dim=(1, 3))

    def gains(self) -> torch.Tensor:
        """dE_b for every block at the current S (flattened b = nt*KB + kt)."""
        return (self.lin + self.quad).reshape(-1)

    def add(self, blk: int) -> float:
        """Add block blk to S; returns the new E(S)."""
        nt, kt = divmod(int(blk), self.KB)
        b = self.b
        rows, cols = slice(nt * b, (nt + 1) * b), slice(kt * b, (kt + 1) * b)
        self.E += float(self.lin[nt, kt] + self.quad[nt, kt])
        self.U[rows] += self.delta[rows, cols] @ self.G[cols]
        self.lin[nt] = self._lin_rows(nt, nt + 1)[0]
        self.taken[blk] = True
        return self.E

    def curve(self, order) -> list[float]:
        """E after each block of `order`, starting from S = {}."""
        self.reset()
        return [self.E0] + [self.add(b) for b in order]

    def greedy(self, k: int) -> tuple[list[int], list[float]]:
        """Exact greedy: k steps, each taking the block with the most negative dE."""
        self.reset()
        order, Es = [], [self.E0]
        for _ in range(k):
            g = self.gains().masked_fill(self.taken, float("inf"))
            blk = int(torch.argmin(g))
            order.append(blk)
            Es.append(self.add(blk))
        return order, Es

    def diagonal_gains(self) -> torch.Tensor:
        """dE_b at S = {} with G replaced by its diagonal (the surrogate the Delta-score
        scales by -1/T)."""
        g = torch.diagonal(self.G)
        b = self.b
        d2 = (self.D0 + self.delta) ** 2 - self.D0 ** 2
        return (d2 * g.reshape(1, -1)).reshape(self.NB, b, self.KB, b).sum(dim=(1, 3)).reshape(-1)

    def recovery(self, E: float) -> float:
        den = self.E0 - self.E_all
        return (self.E0 - E) / den if den != 0 else float("nan")


def run(workload: str, matrix: str | None = None, fracs=(0.01, 0.02, 0.05, 0.10, 0.20), device="cuda",
        with_greedy: bool = True) -> dict:
    """The study on one synthetic layer: the library's quantization, H, Delta and
    Delta-order selection, then exact E(S) for that order and for exact greedy."""
    import numpy as np

    import synth
    from . import mosaic

    dev = torch.device(device)
    L = synth.layer(workload, matrix=matrix, with_x=False)
    N, K = L["N"], L["K"]
    nblk = (N // 64) * (K // 64)
    kmax = synth.budget_blocks(N, K, max(fracs))
    W = torch.from_numpy(L["W"].view(np.int16)).view(torch.bfloat16).to(dev)
    Xc = torch.from_numpy(L["Xcal"].view(np.int16)).view(torch.bfloat16).to(dev)
    layer = mosaic.Layer(N, K, kmax, dev, with_sf=True)
    layer.prepare(W, Xc)
    torch.cuda.synchronize(dev)
    if mosaic.mq_get_error() != 0:
        raise RuntimeError("device error in the library path")
    base, resid = layer.base, layer.resid
    deqQ = dequant_nvfp4(base["codes"], base["sf"], base["gscale"])
    e = W.to(torch.float32) - deqQ                                  # fp32(w - deq Q)
    deqR = dequant_nvfp4(resid["codes"], resid["sf"], base["gscale"])
    ep = e - deqR                                                   # fp32(e - deq R)
    model = Distortion(e, ep, Xc.to(torch.float32))
    rank = layer.rank[:kmax].tolist()
    E_delta = model.curve(rank)
    # the Delta-score against its diagonal surrogate: Delta_b = -dE_b(diag) / T
    diag = model.diagonal_gains()
    dl = layer.delta.to(torch.float64)
    scale = torch.clamp(dl.abs().max(), min=1e-300)
    surrogate_err = float(((-diag / model.T) - dl).abs().max() / scale)
    out = {"workload": workload, "matrix": L["matrix"], "N": N, "K": K, "T": model.T, "blocks": nblk,
           "E_none": model.E0, "E_all": model.E_all, "delta_vs_diagonal_max_rel": surrogate_err, "budgets": []}
    if with_greedy:
        _, E_greedy = model.greedy(kmax)
    for f in fracs:
        k = synth.budget_blocks(N, K, f)
        row = {"frac": f, "blocks": k, "E_delta": E_delta[k], "recovery_delta": model.recovery(E_delta[k])}
        if with_greedy:
            row["E_greedy"] = E_greedy[k]
            row["recovery_greedy"] = model.recovery(E_greedy[k])
        out["budgets"].append(row)
    return out


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--workload", default="llama3_8b_qproj_decode")
    ap.add_argument("--matrix", default=None)
    ap.add_argument("--fracs", default="0.01,0.02,0.05,0.10,0.20")
    ap.add_argument("--no-greedy", action="store_true")
    args = ap.parse_args()
    fr = tuple(float(x) for x in args.fracs.split(","))
    print(json.dumps(run(args.workload, args.matrix, fr, with_greedy=not args.no_greedy)))


if __name__ == "__main__":
    main()
