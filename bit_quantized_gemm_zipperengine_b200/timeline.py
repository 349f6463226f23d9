"""Where a small decode GEMM call's time goes: per-CTA event times of the cluster-split
decode kernel (k_gemm_small), from the timeline build of the library.

The build with MQ_TIMELINE defined (libmosaic_timeline.so) records %globaltimer at fixed
points of every CTA of each launch (mq_timeline_read in include/mosaic_probe.h lists them).
This script prepares one layer, replays a graph of back-to-back mq_gemm calls over operand
copies larger than 2.5x the L2 (as the bench does), and prints, for the last call of the
graph, each event's time over the CTAs (min / median / max) from the earliest CTA's
set-up, and the call's own duration from CUDA events.

    python -m bit_quantized_gemm_zipperengine_b200.timeline --workload llama3_8b_qproj_decode
"""
from __future__ import annotations

import argparse
import ctypes
import math
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

EVENTS = ("set up", "first W issued", "preceding kernel done", "first X issued", "first stage landed",
          "last MMAs issued", "accumulator complete", "partial shared (cluster barrier 1)",
          "rows added and stored", "last cluster barrier")
CTAS, NEV = 160, 16
L2_BYTES = 126e6


def run(workload: str, weights_ready: bool, budget_frac: float = 0.10) -> dict:
    import numpy as np
    import torch

    import synth
    from bit_quantized_gemm_zipperengine_b200 import build, mosaic

    mosaic.LIB_PATH = build.build(timeline=True)
    lib = mosaic.lib()
    dev = torch.device("cuda", torch.cuda.current_device())
    wl = synth.WORKLOADS[workload]
    mat = wl.matrices[0]
    N, K, M = mat.N, mat.K, wl.Ms[0]
    budget = synth.budget_blocks(N, K, budget_frac)
    L = synth.layer(wl, M=M)
    W = torch.from_numpy(L["W"].view(np.int16)).view(torch.bfloat16).to(dev)
    C = torch.from_numpy(L["Xcal"].view(np.int16)).view(torch.bfloat16).to(dev)
    X = torch.from_numpy(L["X"].view(np.int16)).view(torch.bfloat16).to(dev)
    layer = mosaic.Layer(N, K, budget, dev, with_sf=False)
    layer.prepare_path(W, C)
    xq, Y, ws = layer.act_buffers(M)
    mosaic.mq_quantize_act(X, xq)
    per_call = 0.5625 * N * K + 2304 * budget + 0.5625 * M * K + 2 * M * N
    R = max(2, int(math.ceil(2.5 * L2_BYTES / per_call)))

    def cl(d):
        return {k: (v.clone() if isinstance(v, torch.Tensor) else v) for k, v in d.items() if k != "blob"}
    copies = [(cl(layer.base), cl(layer.packed), cl(xq), torch.empty_like(Y), None if ws is None else ws.clone())
              for _ in range(R)]
    flags = mosaic.MQ_GEMM_WEIGHTS_READY if weights_ready else 0
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for b, p, a, y, w in copies:
            mosaic.mq_gemm(a, b, p, y, M, N, K, flags, w)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    table = np.zeros((CTAS, NEV), np.uint64)
    lib.mq_timeline_read(table.ctypes.data, table.nbytes)  # clears it
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    g.replay()
    e1.record()
    torch.cuda.synchronize()
    st = lib.mq_timeline_read(table.ctypes.data, table.nbytes)
    if st != 0:
        raise RuntimeError(f"mq_timeline_read: status {st}")
    if mosaic.mq_get_error() != 0:
        raise RuntimeError("device error word set")
    t = table.astype(np.int64)
    live = t[:, 0] > 0
    t0 = t[live, 0].min()
    rows = []
    for ev, name in enumerate(EVENTS):
        v = t[live, ev]
        v = v[v > 0]
        if v.size == 0:
            continue
        d = (v - t0) / 1000.0
        rows.append((ev, name, int(v.size), float(d.min()), float(np.median(d)), float(d.max())))
    return {"workload": workload, "M": M, "N": N, "K": K, "budget_blocks": budget, "weights_ready": weights_ready,
            "copies": R, "us_per_call": e0.elapsed_time(e1) * 1e3 / R, "events": rows}


def main() -> None:
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--workload", default="llama3_8b_qproj_decode")
    ap.add_argument("--weights-ready", action="store_true", help="pass MQ_GEMM_WEIGHTS_READY")
    args = ap.parse_args()
    r = run(args.workload, args.weights_ready)
    print(f"{r['workload']} M={r['M']} N={r['N']} K={r['K']} budget={r['budget_blocks']} "
          f"weights_ready={r['weights_ready']}: {r['us_per_call']:.2f} us per call over {r['copies']} copies")
    print("event | CTAs | min us | median us | max us")
    for ev, name, n, lo, med, hi in r["events"]:
        print(f"{ev} {name} | {n} | {lo:.2f} | {med:.2f} | {hi:.2f}")


if __name__ == "__main__":
    main()
