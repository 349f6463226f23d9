#!/usr/bin/env python
"""Benchmark of the MosaicQuant / ZipperEngine path on B200.

One step = one pass of the whole path over one batch of synthetic inputs, the
sequence `mq_run_layer` runs, captured in a CUDA graph: H from the calibration tokens,
quantize W (base + full residual) and score every block in one pass, top-K, pack the
residual, quantize X, fused NVFP4 GEMM. Default workload: LLaMA3-8B q_proj at decode batch 16 (M=16, N=K=4096, 512
calibration tokens, 10% block budget = 409 blocks).

value  = algorithmic bytes of the step (what each call must read and write once)
         / device time per step, GB/s, summed over ranks (weak scaling, one replica
         per GPU; the path has no exchange step).
e2e    = same metric through mq_run_layer with pinned HOST buffers: the H2D copies of
         W, X, Xcal and the D2H copy of Y are inside the timed region.
Timing: CUDA events on the launching stream around K graph replays, barrier +
synchronize on both sides, max over ranks. Six input sets rotate so that the touched
footprint (~340 MB) is far above L2 (126 MB): every step starts L2-cold.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "fused NVFP4 base+residual GEMM TFLOPS, GB/s and % of FP4/HBM roofline vs M"
DEFAULT_WORKLOAD = "llama3_8b_qproj_decode"
FP4_PER_BF16 = 4.0  # nominal dense FP4 / bf16 tensor throughput ratio (9 / 2.25 PFLOP/s)


# ------------------------------------------------------------------ work accounting
def step_bytes(M: int, N: int, K: int, T: int, nblk: int) -> dict:
    """Algorithmic bytes per call: every input read once, every output written once."""
    KB, NBr = K // 64, N // 64
    KW = (KB + 31) // 32
    B = NBr * KB
    NK = N * K
    Mp = (M + 127) // 128 * 128
    idx = 4 * (NBr + 1) + 4 * NBr * KW
    return {
        "hessian_diag": 2 * T * K + 4 * K,
        # W, H in; base codes + tiled scales + g, Delta out (the full residual is not stored)
        "quantize_weight_delta": 2 * NK + 4 * K + NK // 2 + NK // 16 + 4 + 8 * B,
        # Delta in; rank + sel out
        "topk_blocks": 8 * B + 8 * nblk,
        # selected W blocks (bf16) + g + sel in; packed residual blocks + kt + index out
        "pack_residual": nblk * (8192 + 4) + 4 + nblk * (2048 + 512 + 4) + idx,
        "quantize_act": 2 * M * K + M * K // 2 + Mp * K // 16 + 4 * M,
        # NVFP4 W (codes + scales) + residual blocks (codes + scales) + index + X (codes + scales
        # + per-token scale) + bf16 Y
        "gemm": NK // 2 + NK // 16 + 4 + nblk * 2304 + idx + M * K // 2 + M * K // 16 + 4 * M + 2 * M * N,
    }


def gemm_flops(M: int, N: int, K: int, nblk: int) -> tuple[float, float]:
    """(executed = dense + residual, dense-equivalent) flops of the fused GEMM."""
    dense = 2.0 * M * N * K
    return dense + 2.0 * M * 4096 * nblk, dense


def load_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def source_hash() -> str:
    h = hashlib.sha256()
    d = os.path.join(ROOT, "bit_quantized_gemm_zipperengine_b200", "csrc")
    for name in sorted(os.listdir(d)):
        with open(os.path.join(d, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def dram_traffic(call: str):
    """Bytes per call from a committed ncu capture, if it was taken on the current sources."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(call)
    if not e or e.get("source_hash") != source_hash():
        return None
    return e.get("bytes_per_call")


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.samples = []
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        threading.Thread(target=self._read, daemon=True).start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 10:
                self.samples.append((time.time(), parts))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0: float, t1: float):
        rows = [p for (t, p) in self.samples if t0 - 0.25 <= t <= t1 + 0.25]
        if not rows:
            return None

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = sorted(v for v in (num(r[2]) for r in rows) if v is not None)
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({n for r in rows for n, v in zip(names, r[6:10]) if v.strip().lower() == "active"})
        return {"sm_mhz": sm[len(sm) // 2] if sm else None, "sm_max_mhz": num(rows[0][3]), "reasons": reasons,
                "samples": len(rows), "window_s": round(t1 - t0, 3)}


# ------------------------------------------------------------------ oracle CPU baseline
def oracle_band(wl, M: int, rows: int):
    import synth
    L = synth.layer(wl, M=M)
    band = L["W"][:rows]
    budget = synth.budget_blocks(rows, L["K"], 0.10)
    return band, L["X"], L["Xcal"], budget


def cpu_baseline(wl_name: str, M: int, min_seconds: float = 10.0, max_runs: int = 50):
    """The oracle (as it stands) on a row band of the workload until >= min_seconds of CPU
    work; GB/s of the band's algorithmic bytes."""
    import oracle
    import synth
    wl = synth.WORKLOADS[wl_name]
    K, T = wl.matrices[0].K, wl.T
    rows = min(wl.matrices[0].N, 1024)
    band, X, Xcal, budget = oracle_band(wl, M, rows)
    oracle.run_path(band, X, Xcal, budget)  # build + page in
    t0 = time.perf_counter()
    runs = 0
    while True:
        oracle.run_path(band, X, Xcal, budget)
        runs += 1
        el = time.perf_counter() - t0
        if el >= min_seconds or runs >= max_runs:
            break
    per = el / runs
    b = sum(step_bytes(M, rows, K, T, budget).values())
    return {"value": b / per / 1e9, "unit": "GB/s", "cores": os.cpu_count(), "kind": "oracle",
            "sample": f"whole path on a {rows}-row band of W ({rows}x{K}, M={M}, T={T}, {budget} blocks), "
                      f"{runs} runs, {per:.3f} s/run"}


def run_reference(args):
    """CPU oracle arm: rank 0 times the oracle's whole path on a bounded band sample."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    import synth
    wl = synth.WORKLOADS[args.workload]
    M, K, T = wl.Ms[0], wl.matrices[0].K, wl.T
    rows = min(wl.matrices[0].N, 512)
    band, X, Xcal, budget = oracle_band(wl, M, rows)
    for _ in range(args.warmup):
        oracle.run_path(band, X, Xcal, budget)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.run_path(band, X, Xcal, budget)
    el = time.perf_counter() - t0
    b = sum(step_bytes(M, rows, K, T, budget).values())
    value = b * args.steps / el / 1e9
    sample = f"whole path on a {rows}-row band of W ({rows}x{K}, M={M}, T={T}, {budget} blocks) per step"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32/f64 (CPU oracle)",
            "data": "synthetic", "config": {"workload": args.workload, "M": M, "N": wl.matrices[0].N, "K": K,
                                            "T": T, "budget_frac": 0.10},
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": os.cpu_count(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ GPU arm
def isolated_profile(sets, calls, M, N, K, budget, reps, stream):
    """Average device time of each call alone: a graph of len(sets) launches over the
    rotating input sets, replayed until `reps` launches were timed."""
    import torch
    from bit_quantized_gemm_zipperengine_b200 import mosaic

    def issue(c, s):
        layer = s["layer"]
        xq, Yb, ws = layer.act_buffers(M)
        if c == "quantize_weight_delta":
            mosaic.mq_quantize_weight_delta(s["W"], layer.H, layer.base, None, layer.delta, layer.qws)
        elif c == "hessian_diag":
            mosaic.mq_hessian_diag(s["Xcal"], layer.H)
        elif c == "topk_blocks":
            mosaic.mq_topk_blocks(layer.delta, budget, layer.rank, layer.sel)
        elif c == "pack_residual":
            mosaic.mq_pack_residual_weight(s["W"], layer.base, layer.sel, budget, layer.packed)
        elif c == "quantize_act":
            mosaic.mq_quantize_act(s["X"], xq)
        else:
            mosaic.mq_gemm(xq, layer.base, layer.packed, Yb, M, N, K, 0, ws)

    out = {}
    inner = 4  # passes over the sets per graph, so graph launch gaps are amortised
    for c in calls:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(inner):
                for s in sets:
                    issue(c, s)
        g.replay()
        torch.cuda.synchronize()
        n = max(1, reps // (inner * len(sets)))
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n):
            g.replay()
        b.record(stream)
        torch.cuda.synchronize()
        out[c] = a.elapsed_time(b) / (n * inner * len(sets)) * reps
    return out


# ------------------------------------------------------------------ GEMM vs M
SWEEP = (("qwen3_32b", "q", (1, 16, 128, 1024, 8192)), ("qwen3_32b", "up", (16, 1024, 8192)),
         ("llama3_8b_mlp_prefill", "up", (2048,)))


def gemm_sweep(peaks: dict, reps: int = 20) -> list:
    """The fused GEMM alone (and dense-only) across token counts: device time per call from
    CUDA events around graphs of back-to-back calls over enough rotating copies of the
    quantized weight, residual and activations that every call reads them from HBM."""
    import numpy as np
    import torch

    import synth
    from bit_quantized_gemm_zipperengine_b200 import mosaic

    dev = torch.device("cuda", torch.cuda.current_device())
    fp4_sus = peaks["bf16_tflops_sustained"] * FP4_PER_BF16
    fp4_burst = peaks["bf16_tflops"] * FP4_PER_BF16
    out = []
    for wl, mat, Ms in SWEEP:
        L = synth.layer(wl, matrix=mat, M=max(Ms))
        N, K = L["N"], L["K"]
        budget = synth.budget_blocks(N, K, 0.10)
        layer = mosaic.Layer(N, K, budget, dev, with_sf=False)
        W = torch.from_numpy(L["W"].view(np.int16)).view(torch.bfloat16).to(dev)
        C = torch.from_numpy(L["Xcal"].view(np.int16)).view(torch.bfloat16).to(dev)
        Xall = torch.from_numpy(L["X"].view(np.int16)).view(torch.bfloat16).to(dev)
        layer.prepare_path(W, C)
        del W, C
        for M in Ms:
            X = Xall[:M].contiguous()
            xq, Y, ws = layer.act_buffers(M)
            mosaic.mq_quantize_act(X, xq)
            per_call = N * K * 0.5625 + budget * 2304 + M * K * 0.5625 + 4 * M + 2 * M * N
            R = max(2, int(np.ceil(3 * 126e6 / per_call)))
            copies = []
            for _ in range(R):
                b = {k: (v.clone() if isinstance(v, torch.Tensor) else v) for k, v in layer.base.items()}
                p = {k: (v.clone() if isinstance(v, torch.Tensor) else v) for k, v in layer.packed.items()}
                a = {k: (v.clone() if isinstance(v, torch.Tensor) else v) for k, v in xq.items()}
                copies.append((b, p, a, torch.empty_like(Y), None if ws is None else ws.clone()))
            res = {}
            for flags, lab in ((0, "fused"), (mosaic.MQ_GEMM_BASE_ONLY, "base"),
                               (mosaic.MQ_GEMM_RESIDUAL_ONLY, "resid")):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    for b, p, a, y, w in copies:
                        mosaic.mq_gemm(a, b, p, y, M, N, K, flags, w)
                g.replay()
                torch.cuda.synchronize()
                n = max(1, reps * 4 // R)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                for _ in range(n):
                    g.replay()
                e1.record()
                torch.cuda.synchronize()
                res[lab] = e0.elapsed_time(e1) * 1e3 / (n * R)
            # the decode kernel quantizing the bf16 activations itself (mq_gemm_act)
            if M <= 128:
                ga = torch.cuda.CUDAGraph()
                with torch.cuda.graph(ga):
                    for b, p, a, y, w in copies:
                        mosaic.mq_gemm_act(X, b, p, y, M, N, K, 0, w)
                ga.replay()
                torch.cuda.synchronize()
                n = max(1, reps * 4 // R)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                for _ in range(n):
                    ga.replay()
                e1.record()
                torch.cuda.synchronize()
                res["act_fused"] = e0.elapsed_time(e1) * 1e3 / (n * R)
                del ga
                # the same with the separate activation quantizer in front
                gs = torch.cuda.CUDAGraph()
                with torch.cuda.graph(gs):
                    for b, p, a, y, w in copies:
                        mosaic.mq_quantize_act(X, a)
                        mosaic.mq_gemm(a, b, p, y, M, N, K, 0, w)
                gs.replay()
                torch.cuda.synchronize()
                e0.record()
                for _ in range(n):
                    gs.replay()
                e1.record()
                torch.cuda.synchronize()
                res["act_separate"] = e0.elapsed_time(e1) * 1e3 / (n * R)
                del gs
            # the unfused design the pages argue against: dense GEMM, a separate residual-block
            # GEMM (it reads X again), then an elementwise merge of the two outputs (a torch
            # add here: this ablation is not part of the path)
            g = torch.cuda.CUDAGraph()
            ys = [torch.empty_like(Y) for _ in range(2)]
            with torch.cuda.graph(g):
                for _ in range(R):
                    ys[0].add_(ys[1])
            g.replay()
            torch.cuda.synchronize()
            n = max(1, reps * 4 // R)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(n):
                g.replay()
            e1.record()
            torch.cuda.synchronize()
            res["merge"] = e0.elapsed_time(e1) * 1e3 / (n * R)
            del copies, ys
            fl = 2.0 * M * N * K + 2.0 * M * 4096 * budget
            us = res["fused"]
            tf = fl / (us * 1e-6) / 1e12
            gbs = per_call / (us * 1e-6) / 1e9
            out.append({"workload": wl, "matrix": mat, "M": M, "N": N, "K": K, "budget_blocks": budget,
                        "kernel": "prefill" if (M > 128 and N % 256 == 0) else "decode", "us": round(us, 3),
                        "us_dense_only": round(res["base"], 3),
                        "residual_overhead": round(us / res["base"] - 1.0, 4),
                        "us_residual_only": round(res["resid"], 3),
                        "us_unfused": round(res["base"] + res["resid"] + res["merge"], 3),
                        "us_quantize_act_then_gemm": round(res["act_separate"], 3) if "act_separate" in res else None,
                        "us_gemm_act": round(res["act_fused"], 3) if "act_fused" in res else None,
                        "tflops_executed": round(tf, 1), "gbs": round(gbs, 1),
                        "frac_fp4_sustained": round(tf / fp4_sus, 4), "frac_fp4_burst": round(tf / fp4_burst, 4),
                        "frac_hbm": round(gbs / peaks["hbm_gbs"], 4),
                        "bound": "hbm" if M <= 316 else "tensor", "rotating_copies": R})
        del layer, Xall
        torch.cuda.empty_cache()
    assert mosaic.mq_get_error() == 0
    return out


# ------------------------------------------------------------------ replicas
def max_over_ranks(ms: float, world: int, device) -> float:
    """The slowest rank's time (every rank calls this, in the same order on every rank)."""
    if world <= 1:
        return ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_gbs(bytes_per_step: float, world: int, ms_per_step: float) -> float:
    """Whole-job GB/s: every replica processes its own step of bytes_per_step in the
    slowest rank's ms_per_step."""
    return bytes_per_step * world / (ms_per_step * 1e-3) / 1e9


# the kernels of each call whose DRAM traffic a capture sums (in launch order per call)
TRAFFIC_KERNELS = {"quantize_weight_delta": ("k_amax_partial", "k_quant_delta")}


def write_traffic(csv_path: str, call: str = "quantize_weight_delta", skip: int = 0, out_path: str | None = None) -> dict:
    """Turn an ncu CSV (--csv --print-units base, metrics dram__bytes_read.sum and
    dram__bytes_write.sum, kernels of `call` only, caches not flushed) into
    profiles/traffic.json: DRAM bytes per call, averaged over the complete calls captured
    after the first `skip`, keyed to the current source hash."""
    import csv
    with open(csv_path) as f:
        lines = [ln for ln in f if not ln.startswith("==")]
    launches = {}
    for r in csv.DictReader(lines):
        if r.get("Metric Name") not in ("dram__bytes_read.sum", "dram__bytes_write.sum"):
            continue
        e = launches.setdefault(int(r["ID"]), {"kernel": r["Kernel Name"], "bytes": 0.0})
        e["bytes"] += float(r["Metric Value"].replace(",", ""))
    first, last = TRAFFIC_KERNELS[call]
    per_call, cur = [], None
    for i in sorted(launches):
        k = launches[i]
        if first in k["kernel"]:
            cur = k["bytes"]
        elif last in k["kernel"] and cur is not None:
            per_call.append(cur + k["bytes"])
            cur = None
    per_call = per_call[skip:]
    if not per_call:
        raise SystemExit(f"no complete {call} call in {csv_path} after the first {skip}")
    p = out_path or os.path.join(ROOT, "profiles", "traffic.json")
    d = {}
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
    d[call] = {"bytes_per_call": int(round(sum(per_call) / len(per_call))), "calls": len(per_call),
               "kernels": list(TRAFFIC_KERNELS[call]), "source_hash": source_hash()}
    with open(p, "w") as f:
        json.dump(d, f, indent=1)
        f.write("\n")
    return d[call]


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--sets", type=int, default=6, help="rotating input sets (L2 defeat)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-sweep", action="store_true", help="skip the GEMM-vs-M sweep")
    ap.add_argument("--traffic-from", metavar="CSV",
                    help="write profiles/traffic.json from an ncu DRAM-bytes capture and exit (no GPU)")
    ap.add_argument("--traffic-skip", type=int, default=0, metavar="N",
                    help="with --traffic-from: leave out the first N captured calls (warm-up)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.traffic_from:
        print(json.dumps(write_traffic(args.traffic_from, skip=args.traffic_skip)))
        return

    if args.impl == "reference":
        run_reference(args)
        return

    import numpy as np
    import torch
    import torch.distributed as dist

    import synth
    from bit_quantized_gemm_zipperengine_b200 import build as libbuild
    from bit_quantized_gemm_zipperengine_b200 import mosaic

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if not os.path.exists(mosaic.LIB_PATH):
        libbuild.build()

    wl = synth.WORKLOADS[args.workload]
    mat = wl.matrices[0]
    N, K, M, T = mat.N, mat.K, wl.Ms[0], wl.T
    budget = synth.budget_blocks(N, K, 0.10)
    L = synth.layer(wl, M=M)
    W0 = torch.from_numpy(L["W"].view(np.int16)).view(torch.bfloat16)
    X0 = torch.from_numpy(L["X"].view(np.int16)).view(torch.bfloat16)
    C0 = torch.from_numpy(L["Xcal"].view(np.int16)).view(torch.bfloat16)

    R = max(1, args.sets)
    sets = []
    for i in range(R):
        layer = mosaic.Layer(N, K, budget, dev, with_sf=False)
        Wd, Xd, Cd = W0.to(dev), X0.to(dev), C0.to(dev)
        Y = layer.act_buffers(M)[1]
        sets.append({"layer": layer, "W": Wd, "X": Xd, "Xcal": Cd, "Y": Y, "buf": layer.buffers(M, T)})
    stream = torch.cuda.current_stream(dev)

    def step(i):
        s = sets[i % R]
        mosaic.mq_run_layer(s["W"], s["X"], s["Xcal"], s["Y"], M, N, K, T, budget, 0, False, s["buf"])

    # eager warm-up (sets kernel attributes, pages everything in); count launches per step
    c0 = mosaic.mq_launch_count()
    step(0)
    launches_per_step = mosaic.mq_launch_count() - c0
    for i in range(R):
        step(i)
    torch.cuda.synchronize()
    assert mosaic.mq_get_error() == 0

    # per input set: the timed step graph is one mq_run_layer call (the whole path as a
    # user issues it; consecutive kernels overlap through programmatic dependent launch),
    # and a profiling graph issues the same steps as separate public calls with event
    # nodes between them (which serialise them) for the in-step per-call times
    calls = ["hessian_diag", "quantize_weight_delta", "quantize_act", "topk_blocks", "pack_residual", "gemm"]

    def issue_step(s, events=None, cs=None):
        layer = s["layer"]
        xq, Yb, ws = layer.act_buffers(M)
        ops = [lambda: mosaic.mq_hessian_diag(s["Xcal"], layer.H),
               lambda: mosaic.mq_quantize_weight_delta(s["W"], layer.H, layer.base, None, layer.delta, layer.qws),
               lambda: mosaic.mq_quantize_act(s["X"], xq),
               lambda: mosaic.mq_topk_blocks(layer.delta, budget, layer.rank, layer.sel),
               lambda: mosaic.mq_pack_residual_weight(s["W"], layer.base, layer.sel, budget, layer.packed),
               lambda: mosaic.mq_gemm(xq, layer.base, layer.packed, Yb, M, N, K, 0, ws)]
        for j, op in enumerate(ops):
            if events is not None:
                events[j].record(cs)
            op()
        if events is not None:
            events[len(ops)].record(cs)

    graphs, pgraphs, evs = [], [], []
    for i in range(R):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step(i)
        graphs.append(g)
        e = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(len(calls) + 1)]
        pg = torch.cuda.CUDAGraph()
        with torch.cuda.graph(pg):
            issue_step(sets[i], e, torch.cuda.current_stream())
        pgraphs.append(pg)
        evs.append(e)

    # the timed steps: a graph of R consecutive steps (input sets 0..R-1) replayed back to
    # back, as a layer runs inside a model's captured forward, and the single-step graphs
    # for the remainder; step k always uses input set k % R
    gall = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gall):
        for i in range(R):
            step(i)

    def run_steps(n):
        for _ in range(n // R):
            gall.replay()
        for k in range(n - n % R, n):
            graphs[k % R].replay()

    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    warmup_done = max(args.warmup, R)  # every graph replayed once before the timed region
    run_steps(warmup_done)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    run_steps(args.steps)
    ev1.record(stream)
    torch.cuda.synchronize()
    t_wall1 = time.time()
    if world > 1:
        dist.barrier()
    ms_total = max_over_ranks(ev0.elapsed_time(ev1), world, dev)
    time.sleep(0.3)
    sampler.stop()
    clocks = sampler.summary(t_wall0, t_wall1)
    err = mosaic.mq_get_error()
    if err != 0:
        raise RuntimeError(f"device error word {err}")

    ms_step = ms_total / args.steps
    per_call = step_bytes(M, N, K, T, budget)
    bytes_step = sum(per_call.values())
    value = replica_gbs(bytes_step, world, ms_step)

    # per-call device time: each call replayed back to back over the R rotating input sets
    # (CUDA events around graphs of R launches; programmatic dependent launch hides the
    # launch latency between them, so this is the kernel's own duration). The same calls
    # timed inside the step graph (event nodes between calls, which serialise them and
    # add the launch gap to every call) are reported beside it as in_step_us.
    prof_reps = min(args.steps, 300)
    profile_mode = f"isolated (each call replayed back to back, {R} rotating sets)"
    acc = isolated_profile(sets, calls, M, N, K, budget, prof_reps, stream)
    in_step = {c: 0.0 for c in calls}
    try:
        for r in range(prof_reps):
            i = r % R
            pgraphs[i].replay()
            torch.cuda.synchronize()
            e = evs[i]
            for j, c in enumerate(calls):
                in_step[c] += e[j].elapsed_time(e[j + 1])
    except RuntimeError:
        in_step = None
    peaks = load_peaks()
    kern = {}
    for c in calls:
        us = acc[c] / prof_reps * 1e3
        gbs = per_call[c] / (us * 1e-6) / 1e9
        kern[c] = {"us": round(us, 3), "alg_bytes": per_call[c], "gbs": round(gbs, 1),
                   "frac_hbm": round(gbs / peaks["hbm_gbs"], 4), "traffic": dram_traffic(c),
                   "in_step_us": None if in_step is None else round(in_step[c] / prof_reps * 1e3, 3)}
    dom = max(calls, key=lambda c: kern[c]["us"])
    roofline = {"bound": "hbm", "kernel": dom, "timing": profile_mode, "achieved": kern[dom]["gbs"], "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": kern[dom]["frac_hbm"], "traffic": kern[dom]["traffic"],
                "peak_source": f"{peaks['source']} (copy bandwidth)"}
    fl_exec, fl_dense = gemm_flops(M, N, K, budget)
    g_us = kern["gemm"]["us"]
    fp4_peak = peaks["bf16_tflops_sustained"] * FP4_PER_BF16
    gemm = {"us": g_us, "gbs": kern["gemm"]["gbs"], "frac_hbm": kern["gemm"]["frac_hbm"],
            "tflops_executed": round(fl_exec / (g_us * 1e-6) / 1e12, 2),
            "tflops_dense_equiv": round(fl_dense / (g_us * 1e-6) / 1e12, 2),
            "frac_fp4": round(fl_exec / (g_us * 1e-6) / 1e12 / fp4_peak, 5),
            "fp4_peak_tflops": fp4_peak, "bound": "hbm" if M <= 316 else "tensor"}

    # end to end: whole path through mq_run_layer with pinned host buffers
    e2e = None
    if not args.no_e2e:
        s = sets[0]
        hb = s["layer"].buffers(M, T, staging=True)
        Wh, Xh, Ch = W0.pin_memory(), X0.pin_memory(), C0.pin_memory()
        Yh = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
        for _ in range(3):
            mosaic.mq_run_layer(Wh, Xh, Ch, Yh, M, N, K, T, budget, 0, True, hb)
        torch.cuda.synchronize()
        ke = max(3, min(args.steps, 50))
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        a0 = torch.cuda.Event(enable_timing=True)
        a1 = torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for _ in range(ke):
            mosaic.mq_run_layer(Wh, Xh, Ch, Yh, M, N, K, T, budget, 0, True, hb)
        a1.record(stream)
        torch.cuda.synchronize()
        ms_e = max_over_ranks(a0.elapsed_time(a1) / ke, world, dev)
        e2e = {"value": replica_gbs(bytes_step, world, ms_e), "unit": "GB/s", "ms_per_step": ms_e,
               "h2d_bytes_per_step": 2 * N * K + 2 * M * K + 2 * T * K, "d2h_bytes_per_step": 2 * M * N,
               "steps": ke}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(args.workload, M)

    sweep = None
    if world == 1 and not args.no_sweep:
        for st in sets:
            st.clear()
        sets.clear()
        graphs.clear()
        pgraphs.clear()
        torch.cuda.empty_cache()
        sweep = gemm_sweep(load_peaks())

    if world > 1:
        graphs.clear()
        pgraphs.clear()
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {"metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": warmup_done, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "nvfp4 (e2m1 x e2m1, e4m3 scales, fp32 accumulate; fp32/fp64 prep)",
            "data": "synthetic",
            "config": {"workload": args.workload, "M": M, "N": N, "K": K, "T": T, "budget_frac": 0.10,
                       "budget_blocks": budget, "parallelism": f"replicas x{world}",
                       "l2": f"{R} rotating input sets (~{R * 57} MB touched) > 2x L2; no flush",
                       "graphs": f"{R} steps per graph replay (one per input set)"},
            "roofline": roofline, "gemm": gemm, "gemm_vs_M": sweep, "kernels": kern, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": int(launches_per_step * args.steps), "clocks": clocks}
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
