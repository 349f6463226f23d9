#!/usr/bin/env python
"""Benchmark of the MosaicQuant / ZipperEngine path on B200.

The metric is the fused NVFP4 base + sparse-residual GEMM's throughput (TFLOPS, GB/s and
fraction of the FP4 / HBM roofline) against the token count M.

One step = one call of the fused GEMM (mq_gemm, A7 + A8) on the LLaMA3-8B q_proj decode
layer (M=16 tokens, N=K=4096, 10% block budget = 409 residual blocks), with its
quantized weight, packed residual and quantized activations resident in HBM.

value  = the call's algorithmic bytes (W codes and scales, residual blocks and index,
         X codes and scales, bf16 Y) / device time per call, GB/s, summed over ranks
         (weak scaling, one replica per GPU; the path has no exchange step).
         Consecutive steps rotate over copies of the operands whose total exceeds 2x the
         L2, so every call reads its bytes from HBM.
e2e    = the same bytes per step through mq_run_layer with pinned HOST buffers and a
         prepared layer: the H2D copy of the step's bf16 X, the activation quantizer, the
         GEMM and the D2H copy of Y are all in the timed region. Two steps are in flight on
         two streams (own buffers each) and replayed from a CUDA graph; steps rotate over
         the weight copies; the one-stream, call-after-call time is reported beside it.
whole_path = one mq_run_layer step (A1..A8: H, quantize + Delta, top-K, pack, quantize X,
         GEMM) and each of its calls timed alone, for the same layer.
sweep  = the fused GEMM on every workload's layers and token counts (and the 70B MLP's
         budget sweep), beside its dense-only time (residual overhead), the unfused
         ablation, and for M <= 128 the in-kernel activation quantization.
fp4_peak = the measured dense FP4 tensor rate (tcgen05 mxf4nvf4 MMA loop, operands
         resident on chip), the denominator of the prefill fractions beside 4x the
         measured bf16 cuBLAS rate.
Timing: CUDA events on the launching stream, barrier + synchronize on both sides, max
over ranks.

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
L2_BYTES = 126e6


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


def dram_traffic(call: str, workload: str):
    """Bytes per call from a committed ncu capture, if it was taken on the current sources
    and on this workload."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(call)
    if not e or e.get("source_hash") != source_hash() or e.get("workload") != workload:
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
def gemm_bytes(M: int, N: int, K: int, nblk: int) -> int:
    """Algorithmic bytes of one fused GEMM call (step_bytes()["gemm"])."""
    return step_bytes(M, N, K, 512, nblk)["gemm"]


def oracle_gemm_sample(wl_name: str, target_s: float):
    """A bounded sample of the headline workload for the CPU oracle: its fp64 GEMM
    reference on a band of weight rows (every token), with the band sized so that one call
    takes about target_s seconds. Returns (run, bytes of the band's GEMM, description)."""
    import numpy as np

    import oracle
    import synth
    wl = synth.WORKLOADS[wl_name]
    M, N, K = wl.Ms[0], wl.matrices[0].N, wl.matrices[0].K
    L = synth.layer(wl_name, M=M)
    budget = synth.budget_blocks(N, K, 0.10)
    ref = oracle.run_path(L["W"], L["X"], L["Xcal"], budget, rows=np.arange(1, dtype=np.int32))
    xq, wq, sel = ref["xq"], ref["wq"], ref["sel"]

    def band(rows):
        # the first `rows` weight rows (a multiple of 64) and their selected blocks
        KB = K // 64
        s = sel[sel < (rows // 64) * KB]
        w = {k: (v[:rows] if isinstance(v, np.ndarray) and v.ndim == 2 else v) for k, v in wq.items()}
        return w, s, rows

    def run(b):
        w, s, rows = b
        oracle.gemm_rows(xq, w, s, M, rows, K)

    rows = 64
    t0 = time.perf_counter()
    run(band(rows))
    per_row = (time.perf_counter() - t0) / rows
    rows = int(max(64, min(N, target_s / max(per_row, 1e-9))) // 64 * 64)
    b = band(rows)
    nblk = len(b[1])
    return (lambda: run(b)), gemm_bytes(M, rows, K, nblk), \
        f"fp64 GEMM reference on a {rows}-row band of W ({rows}x{K}, all {M} tokens, {nblk} residual blocks)"


def cpu_baseline(wl_name: str, min_seconds: float = 10.0, max_runs: int = 200):
    """The oracle (as it stands) on a band of the headline GEMM until >= min_seconds of CPU
    work; GB/s of the band's algorithmic bytes."""
    run, nbytes, desc = oracle_gemm_sample(wl_name, 0.5)
    run()  # page in
    t0 = time.perf_counter()
    runs = 0
    while True:
        run()
        runs += 1
        el = time.perf_counter() - t0
        if el >= min_seconds or runs >= max_runs:
            break
    per = el / runs
    return {"value": nbytes / per / 1e9, "unit": "GB/s", "cores": os.cpu_count(), "kind": "oracle",
            "sample": f"{desc}, {runs} runs, {per:.3f} s/run"}


def run_reference(args):
    """CPU oracle arm: rank 0 times the oracle's GEMM reference on a band of the headline
    workload, one band per step, sized so the whole run ends within about two minutes."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import synth
    wl = synth.WORKLOADS[args.workload]
    M, N, K = wl.Ms[0], wl.matrices[0].N, wl.matrices[0].K
    per_step = min(0.5, 120.0 / max(1, args.steps + args.warmup))
    run, nbytes, desc = oracle_gemm_sample(args.workload, per_step)
    for _ in range(args.warmup):
        run()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run()
    el = time.perf_counter() - t0
    value = nbytes * args.steps / el / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64 (CPU oracle)",
            "data": "synthetic",
            "config": {"workload": args.workload + " fused GEMM", "M": M, "N": N, "K": K, "budget_frac": 0.10},
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": os.cpu_count(), "kind": "oracle",
                             "sample": desc + " per step"},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ GPU helpers
def graph_time_us(issue, n_calls: int, reps: int, stream=None, target_ms: float = 40.0) -> float:
    """Device time per call: `issue()` captured once as a CUDA graph of n_calls launches,
    replayed between CUDA events after one untimed replay. The replay count is `reps`, or
    fewer when one replay is long, so that each measurement takes about target_ms (at
    least one replay)."""
    import torch
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        issue()
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    one_ms = max(e0.elapsed_time(e1), 1e-3)
    reps = max(1, min(reps, int(target_ms / one_ms)))
    e0.record(stream)
    for _ in range(reps):
        g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    del g
    return e0.elapsed_time(e1) * 1e3 / (reps * n_calls)


def small_split(M: int, N: int, K: int, sms: int = 148) -> int:
    """The library's choice of the small-problem decode kernel (its cluster split S), or 0
    for the stream-K kernel (the rule of plan_small in the library's GEMM host code)."""
    tiles, KS = N // 128, K // 256
    if M > 32 or 2 * tiles > sms:
        return 0
    S = min(8, sms // tiles, KS)
    return 0 if (KS + S - 1) // S > 8 else S


def gemm_kernel(M: int, N: int, K: int, sms: int = 148) -> tuple[str, str]:
    """(kernel, description) that mq_gemm runs with flags 0 (the library's rule: the
    CTA-pair prefill kernel for M > 128 with N % 256 == 0, else a decode kernel)."""
    if M > 128 and N % 256 == 0:
        return "k_gemm_prefill2", "prefill (CTA pairs)"
    bn = 16 if M <= 16 else 32 if M <= 32 else 64 if M <= 64 else 128
    S = small_split(M, N, K, sms)
    if S:
        return f"k_gemm_small<{bn}>", f"decode, {S}-CTA cluster split"
    return f"k_gemm_streamk<{bn}>", "decode, stream-K"


def operand_copies(layer, xq, Y, ws, per_call: float, min_copies: int = 1):
    """Copies of the GEMM's operands (quantized weight, packed residual, quantized X, Y,
    workspace) whose total exceeds 2.5x the L2, so that back-to-back calls over them
    read every byte from HBM."""
    import torch
    R = max(min_copies, int(math.ceil(2.5 * L2_BYTES / per_call)))

    def cl(d):
        return {k: (v.clone() if isinstance(v, torch.Tensor) else v) for k, v in d.items() if k != "blob"}
    return [(cl(layer.base), cl(layer.packed), cl(xq), torch.empty_like(Y), None if ws is None else ws.clone())
            for _ in range(R)]


def fp4_peak(sampler, ctas: int = 148, iters: int = 40000) -> dict:
    """The FP4 MMA-loop probe on every SM: TFLOP/s from CUDA events, with the SM clock
    sampled meanwhile (repeated for about a second)."""
    import torch
    from bit_quantized_gemm_zipperengine_b200 import mosaic
    mosaic.mq_fp4_mma_loop(ctas, 1000)
    torch.cuda.synchronize()
    best, runs = None, 0
    t0 = time.time()
    while time.time() - t0 < 1.0 or runs < 3:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fl = mosaic.mq_fp4_mma_loop(ctas, iters)
        e1.record()
        torch.cuda.synchronize()
        tf = fl / (e0.elapsed_time(e1) * 1e-3) / 1e12
        best = tf if best is None else max(best, tf)
        runs += 1
    t1 = time.time()
    assert mosaic.mq_get_error() == 0
    return {"tflops": round(best, 1), "ctas": ctas, "iters_per_cta": iters, "runs": runs,
            "shape": "tcgen05.mma kind::mxf4nvf4 M=128 N=256 K=64, operands resident on chip",
            "clocks": sampler.summary(t0, t1) if sampler else None}


# ------------------------------------------------------------------ GEMM sweep over every workload
SWEEP = (("tiny", "w", (16,), (0.10,)),
         ("llama3_8b_qproj_decode", "q_proj", (16,), (0.10,)),
         ("llama3_8b_mlp_prefill", "up", (2048,), (0.10,)),      # gate has the same shape
         ("llama3_8b_mlp_prefill", "down", (2048,), (0.10,)),
         ("qwen3_32b", "q", (1, 16, 128, 1024, 8192), (0.10,)),
         ("qwen3_32b", "up", (1, 16, 128, 1024, 8192), (0.10,)),
         ("qwen3_32b", "down", (1, 16, 128, 1024, 8192), (0.10,)),
         ("llama3_70b_mlp", "up", (4096,), (0.0, 0.05, 0.10, 0.20)),
         ("llama3_70b_mlp", "down", (4096,), (0.0, 0.05, 0.10, 0.20)))


def gemm_sweep(peaks: dict, fp4_measured: float | None, reps: int = 20) -> tuple[list, list]:
    """The fused GEMM alone, dense-only and residual-only on every workload's layers and
    token counts: device time per call from CUDA events around graphs of back-to-back
    calls over copies of the operands that exceed 2.5x the L2. Also the Delta-score +
    top-K pass of the 70B MLP layers at every budget. Returns (gemm rows, delta rows)."""
    import numpy as np
    import torch

    import synth
    from bit_quantized_gemm_zipperengine_b200 import mosaic

    dev = torch.device("cuda", torch.cuda.current_device())
    fp4_burst = peaks["bf16_tflops"] * FP4_PER_BF16
    rows, drows = [], []
    for wl, mat, Ms, fracs in SWEEP:
        L = synth.layer(wl, matrix=mat, M=max(Ms))
        N, K = L["N"], L["K"]
        W = torch.from_numpy(L["W"].view(np.int16)).view(torch.bfloat16).to(dev)
        C = torch.from_numpy(L["Xcal"].view(np.int16)).view(torch.bfloat16).to(dev)
        Xall = torch.from_numpy(L["X"].view(np.int16)).view(torch.bfloat16).to(dev)
        del L
        for frac in fracs:
            budget = synth.budget_blocks(N, K, frac)
            layer = mosaic.Layer(N, K, budget, dev, with_sf=False)
            layer.prepare_path(W, C)
            torch.cuda.synchronize()
            if wl == "llama3_70b_mlp":
                # the Delta-score + top-K pass (A1 + A3 in one pass over W, then A4), two
                # copies of W (> 2x L2)
                Ws = [W, W.clone()]
                us_qd = graph_time_us(lambda: [mosaic.mq_quantize_weight_delta(w, layer.H, layer.base, None,
                                                                                layer.delta, layer.qws) for w in Ws],
                                      len(Ws), 5)
                # ten back-to-back calls per graph replay (a replay boundary costs
                # microseconds, as much as a call)
                us_tk = graph_time_us(lambda: [mosaic.mq_topk_blocks(layer.delta, budget, layer.rank, layer.sel)
                                               for _ in range(10)], 10, 20) if budget else 0.0
                qd_bytes = step_bytes(16, N, K, 512, budget)["quantize_weight_delta"]
                drows.append({"workload": wl, "matrix": mat, "N": N, "K": K, "blocks": (N // 64) * (K // 64),
                              "budget_blocks": budget, "us_quantize_delta": round(us_qd, 2),
                              "gbs_quantize_delta": round(qd_bytes / (us_qd * 1e-6) / 1e9, 1),
                              "frac_hbm_quantize_delta": round(qd_bytes / (us_qd * 1e-6) / 1e9 / peaks["hbm_gbs"], 4),
                              "us_topk": round(us_tk, 2)})
                del Ws
                layer.prepare_path(W, C)  # restore this budget's selection after the timing
            for M in Ms:
                X = Xall[:M].contiguous()
                xq, Y, ws = layer.act_buffers(M)
                mosaic.mq_quantize_act(X, xq)
                per_call = gemm_bytes(M, N, K, budget)
                copies = operand_copies(layer, xq, Y, ws, per_call)
                R = len(copies)
                n = max(2, reps * 4 // R)
                res = {}
                for flags, lab in ((0, "fused"), (mosaic.MQ_GEMM_BASE_ONLY, "base"),
                                   (mosaic.MQ_GEMM_RESIDUAL_ONLY, "resid")):
                    if lab != "fused" and budget == 0:
                        continue

                    def issue(flags=flags):
                        for b, p, a, y, w in copies:
                            mosaic.mq_gemm(a, b, p, y, M, N, K, flags, w)
                    res[lab] = graph_time_us(issue, R, n)
                if M <= 128 and budget:
                    def issue_act():
                        for b, p, a, y, w in copies:
                            mosaic.mq_gemm_act(X, b, p, y, M, N, K, 0, w)
                    res["act_fused"] = graph_time_us(issue_act, R, n)

                    def issue_sep():
                        for b, p, a, y, w in copies:
                            mosaic.mq_quantize_act(X, a)
                            mosaic.mq_gemm(a, b, p, y, M, N, K, 0, w)
                    res["act_separate"] = graph_time_us(issue_sep, R, n)
                if budget:
                    # the unfused design the pages argue against: dense GEMM, a separate
                    # residual-block GEMM (it reads X again), then an elementwise merge of
                    # the two outputs (a torch add: this ablation is not part of the path)
                    ys = [torch.empty_like(Y) for _ in range(2)]
                    res["merge"] = graph_time_us(lambda: [ys[0].add_(ys[1]) for _ in range(R)], R, n)
                    del ys
                del copies
                us = res["fused"]
                fl_exec, fl_dense = gemm_flops(M, N, K, budget)
                tf = fl_exec / (us * 1e-6) / 1e12
                gbs = per_call / (us * 1e-6) / 1e9
                kname = "%s (%s)" % gemm_kernel(M, N, K)
                rows.append({
                    "workload": wl, "matrix": mat, "M": M, "N": N, "K": K, "budget_frac": frac,
                    "budget_blocks": budget, "kernel": kname,
                    "us": round(us, 3), "tflops_executed": round(tf, 1),
                    "tflops_dense_equiv": round(fl_dense / (us * 1e-6) / 1e12, 1), "gbs": round(gbs, 1),
                    "frac_hbm": round(gbs / peaks["hbm_gbs"], 4), "frac_fp4_burst": round(tf / fp4_burst, 4),
                    "frac_fp4_measured": round(tf / fp4_measured, 4) if fp4_measured else None,
                    "bound": "hbm" if M <= 316 else "tensor",
                    "us_dense_only": round(res["base"], 3) if "base" in res else None,
                    "residual_overhead": round(us / res["base"] - 1.0, 4) if "base" in res else None,
                    "us_residual_only": round(res["resid"], 3) if "resid" in res else None,
                    "us_unfused": round(res["base"] + res["resid"] + res["merge"], 3) if "merge" in res else None,
                    "us_quantize_act_then_gemm": round(res["act_separate"], 3) if "act_separate" in res else None,
                    "us_gemm_act": round(res["act_fused"], 3) if "act_fused" in res else None,
                    "rotating_copies": R})
                print(json.dumps(rows[-1]), file=sys.stderr, flush=True)
            del layer
            torch.cuda.empty_cache()
        del W, C, Xall
        torch.cuda.empty_cache()
    assert mosaic.mq_get_error() == 0
    return rows, drows


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
TRAFFIC_KERNELS = {"quantize_weight_delta": ("k_amax_partial", "k_quant_delta"), "gemm": ("k_gemm_small",)}


def write_traffic(csv_path: str, call: str = "quantize_weight_delta", skip: int = 0, out_path: str | None = None,
                  workload: str = DEFAULT_WORKLOAD) -> dict:
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
    names = TRAFFIC_KERNELS[call]  # the call's kernels in launch order
    per_call, cur, nxt = [], 0.0, 0
    for i in sorted(launches):
        k = launches[i]
        if names[0] in k["kernel"]:
            cur, nxt = 0.0, 0
        if nxt < len(names) and names[nxt] in k["kernel"]:
            cur += k["bytes"]
            nxt += 1
            if nxt == len(names):
                per_call.append(cur)
                cur, nxt = 0.0, len(names)
    per_call = per_call[skip:]
    if not per_call:
        raise SystemExit(f"no complete {call} call in {csv_path} after the first {skip}")
    p = out_path or os.path.join(ROOT, "profiles", "traffic.json")
    d = {}
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
    d[call] = {"bytes_per_call": int(round(sum(per_call) / len(per_call))), "calls": len(per_call),
               "kernels": list(TRAFFIC_KERNELS[call]), "workload": workload, "source_hash": source_hash()}
    with open(p, "w") as f:
        json.dump(d, f, indent=1)
        f.write("\n")
    return d[call]


def whole_path(dev, wl_name: str, sets_n: int, steps: int, stream) -> dict:
    """One mq_run_layer step (A1..A8) on the headline layer, timed as replays of a graph of
    `sets_n` steps over rotating input sets (> 2x L2), and each of its calls alone."""
    import numpy as np
    import torch

    import synth
    from bit_quantized_gemm_zipperengine_b200 import mosaic
    wl = synth.WORKLOADS[wl_name]
    mat = wl.matrices[0]
    N, K, M, T = mat.N, mat.K, wl.Ms[0], wl.T
    budget = synth.budget_blocks(N, K, 0.10)
    L = synth.layer(wl, M=M)
    W0 = torch.from_numpy(L["W"].view(np.int16)).view(torch.bfloat16).to(dev)
    X0 = torch.from_numpy(L["X"].view(np.int16)).view(torch.bfloat16).to(dev)
    C0 = torch.from_numpy(L["Xcal"].view(np.int16)).view(torch.bfloat16).to(dev)
    sets = []
    for _ in range(sets_n):
        layer = mosaic.Layer(N, K, budget, dev, with_sf=False)
        sets.append({"layer": layer, "W": W0.clone(), "X": X0.clone(), "Xcal": C0.clone(),
                     "Y": layer.act_buffers(M)[1], "buf": layer.buffers(M, T)})

    def step(s):
        mosaic.mq_run_layer(s["W"], s["X"], s["Xcal"], s["Y"], M, N, K, T, budget, 0, False, s["buf"])
    c0 = mosaic.mq_launch_count()
    step(sets[0])
    launches = mosaic.mq_launch_count() - c0
    for s in sets:
        step(s)
    torch.cuda.synchronize()
    assert mosaic.mq_get_error() == 0
    us_step = graph_time_us(lambda: [step(s) for s in sets], sets_n, max(3, steps // sets_n), stream)
    per_call = step_bytes(M, N, K, T, budget)

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
    hbm = load_peaks()["hbm_gbs"]
    kern = {}
    for c in ("hessian_diag", "quantize_weight_delta", "quantize_act", "topk_blocks", "pack_residual", "gemm"):
        us = graph_time_us(lambda: [issue(c, s) for _ in range(4) for s in sets], 4 * sets_n, 20, stream)
        gbs = per_call[c] / (us * 1e-6) / 1e9
        kern[c] = {"us": round(us, 3), "alg_bytes": per_call[c], "gbs": round(gbs, 1), "frac_hbm": round(gbs / hbm, 4),
                   "traffic": dram_traffic(c, wl_name)}
    bytes_step = sum(per_call.values())
    out = {"workload": wl_name, "us_per_step": round(us_step, 3), "alg_bytes": bytes_step,
           "gbs": round(bytes_step / (us_step * 1e-6) / 1e9, 1), "launches_per_step": int(launches),
           "timing": f"graph of {sets_n} mq_run_layer steps over rotating input sets, replayed",
           "calls": kern}
    for s in sets:
        s.clear()
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-sweep", action="store_true", help="skip the GEMM sweep over every workload")
    ap.add_argument("--no-path", action="store_true", help="skip the whole-path step")
    ap.add_argument("--no-fp4-peak", action="store_true", help="skip the FP4 MMA-loop probe")
    ap.add_argument("--traffic-from", metavar="CSV",
                    help="write profiles/traffic.json from an ncu DRAM-bytes capture and exit (no GPU)")
    ap.add_argument("--traffic-call", default="gemm", choices=sorted(TRAFFIC_KERNELS),
                    help="with --traffic-from: the call whose kernels the capture holds")
    ap.add_argument("--traffic-skip", type=int, default=0, metavar="N",
                    help="with --traffic-from: leave out the first N captured calls (warm-up)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.traffic_from:
        print(json.dumps(write_traffic(args.traffic_from, call=args.traffic_call, skip=args.traffic_skip,
                                       workload=args.workload)))
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
    stream = torch.cuda.current_stream(dev)
    peaks = load_peaks()

    # ---- the headline layer, prepared once (A1..A5), its activations quantized (A6)
    wl = synth.WORKLOADS[args.workload]
    mat = wl.matrices[0]
    N, K, M, T = mat.N, mat.K, wl.Ms[0], wl.T
    budget = synth.budget_blocks(N, K, 0.10)
    L = synth.layer(wl, M=M)
    W0 = torch.from_numpy(L["W"].view(np.int16)).view(torch.bfloat16)
    X0 = torch.from_numpy(L["X"].view(np.int16)).view(torch.bfloat16)
    C0 = torch.from_numpy(L["Xcal"].view(np.int16)).view(torch.bfloat16)
    layer = mosaic.Layer(N, K, budget, dev, with_sf=False)
    layer.prepare_path(W0.to(dev), C0.to(dev))
    xq, Y, ws = layer.act_buffers(M)
    mosaic.mq_quantize_act(X0.to(dev), xq)
    torch.cuda.synchronize()
    assert mosaic.mq_get_error() == 0
    per_call = gemm_bytes(M, N, K, budget)
    copies = operand_copies(layer, xq, Y, ws, per_call)
    R = len(copies)

    def call(k):
        b, p, a, y, w = copies[k % R]
        mosaic.mq_gemm(a, b, p, y, M, N, K, 0, w)

    c0 = mosaic.mq_launch_count()
    for k in range(R):
        call(k)
    launches_per_step = (mosaic.mq_launch_count() - c0) / R
    torch.cuda.synchronize()
    # the timed steps: a graph of R consecutive calls (copies 0..R-1) replayed back to back,
    # and single-call graphs for a remainder; step k always uses copy k % R
    gall = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gall):
        for k in range(R):
            call(k)
    singles = []
    for k in range(R):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            call(k)
        singles.append(g)

    def run_steps(n):
        for _ in range(n // R):
            gall.replay()
        for k in range(n - n % R, n):
            singles[k % R].replay()

    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    warmup_done = max(args.warmup, R)  # every graph replayed before the timed region
    run_steps(warmup_done)
    for g in singles:
        g.replay()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    run_steps(args.steps)
    ev1.record(stream)
    torch.cuda.synchronize()
    t_wall1 = time.time()
    # the same steps for three more seconds, so the SM clock has about 15 samples under
    # this load even when the timed region is shorter than the sampling interval
    while time.time() - t_wall1 < 3.0:
        run_steps(R * 50)
        torch.cuda.synchronize()
    t_wall2 = time.time()
    if world > 1:
        dist.barrier()
    ms_total = max_over_ranks(ev0.elapsed_time(ev1), world, dev)
    err = mosaic.mq_get_error()
    if err != 0:
        raise RuntimeError(f"device error word {err}")
    ms_step = ms_total / args.steps
    us = ms_step * 1e3
    value = replica_gbs(per_call, world, ms_step)
    clocks = sampler.summary(t_wall0, t_wall2)
    if clocks:
        clocks["window"] = "timed region + 3 s of the same steps"
    fl_exec, fl_dense = gemm_flops(M, N, K, budget)
    gbs_rank = per_call / (us * 1e-6) / 1e9
    fp4_burst = peaks["bf16_tflops"] * FP4_PER_BF16
    tf = fl_exec / (us * 1e-6) / 1e12
    gemm = {"us": round(us, 3), "alg_bytes": per_call, "gbs": round(gbs_rank, 1),
            "frac_hbm": round(gbs_rank / peaks["hbm_gbs"], 4), "tflops_executed": round(tf, 2),
            "tflops_dense_equiv": round(fl_dense / (us * 1e-6) / 1e12, 2),
            "frac_fp4_burst": round(tf / fp4_burst, 5), "rotating_copies": R,
            "kernel": "%s (%s)" % gemm_kernel(M, N, K)}
    roofline = {"bound": "hbm", "kernel": f"gemm ({gemm_kernel(M, N, K)[0]})",
                "timing": f"CUDA events around {args.steps} back-to-back calls over {R} operand copies",
                "achieved": round(gbs_rank, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(gbs_rank / peaks["hbm_gbs"], 4), "traffic": dram_traffic("gemm", args.workload),
                "peak_source": f"{peaks['source']} (copy bandwidth)"}
    # the same calls with MQ_GEMM_WEIGHTS_READY (a layer's weights at inference: the next
    # call's W is requested before it waits for the current one)
    def issue_wr():
        for k in range(R):
            b, p, a, y, w = copies[k]
            mosaic.mq_gemm(a, b, p, y, M, N, K, mosaic.MQ_GEMM_WEIGHTS_READY, w)
    us_wr = graph_time_us(issue_wr, R, max(1, args.steps // R), stream)
    gemm["us_weights_ready"] = round(us_wr, 3)
    gemm["gbs_weights_ready"] = round(per_call / (us_wr * 1e-6) / 1e9, 1)
    gemm["frac_hbm_weights_ready"] = round(per_call / (us_wr * 1e-6) / 1e9 / peaks["hbm_gbs"], 4)
    for g in singles:
        del g
    del gall, singles

    # ---- end to end: inference on the prepared layer through mq_run_layer with pinned
    # host buffers (H2D of X, activation quantizer, GEMM, D2H of Y in every step). Two steps
    # are in flight: step i runs on stream i % 2 with its own activation and staging buffers
    # and its own pinned X and Y (the layer's weights are shared), so one step's copies
    # overlap the other's kernels, as a server overlaps consecutive requests. Step i reads
    # the weight copy i % R of the timed region's rotation (more than 2x the L2). The calls
    # are captured once in a CUDA graph (R steps rounded up to a multiple of 2, the streams
    # forked and joined) and the graph is replayed. The same steps issued one after another
    # on one stream are timed too.
    e2e = None
    if not args.no_e2e:
        import ctypes
        S = 2
        G = (R + S - 1) // S
        streams = [torch.cuda.Stream(device=dev) for _ in range(S)]  # graphs are not captured on the default stream
        hbs = [layer.buffers(M, T, staging=True, slot=j) for j in range(S)]
        Xhs = [X0.pin_memory() for _ in range(S)]
        Yhs = [torch.empty((M, N), dtype=torch.bfloat16).pin_memory() for _ in range(S)]

        def step_buffers(k, j):
            b = mosaic.LayerBuffers()
            ctypes.memmove(ctypes.byref(b), ctypes.byref(hbs[j]), ctypes.sizeof(b))
            b.base, b.packed = mosaic.mat(copies[k][0]), mosaic.packed_struct(copies[k][1])
            return b
        sbufs = {(k, j): step_buffers(k, j) for k in range(R) for j in range(S)}

        def run_step(i, j=None):
            j = i % S if j is None else j
            mosaic.mq_run_layer(None, Xhs[j], None, Yhs[j], M, N, K, T, budget, mosaic.MQ_LAYER_PREPARED, True,
                                sbufs[(i % R, j)], streams[j])
        for i in range(2 * S):
            run_step(i)
        torch.cuda.synchronize()
        ke = max(20, min(args.steps, 2000))
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        a0.record(streams[0])
        for i in range(ke):
            run_step(i, 0)
        a1.record(streams[0])
        torch.cuda.synchronize()
        ms_one = max_over_ranks(a0.elapsed_time(a1) / ke, world, dev)
        one = {"value": round(replica_gbs(per_call, world, ms_one), 2), "ms_per_step": ms_one, "steps": ke}
        e2e = {"value": one["value"], "unit": "GB/s", "ms_per_step": ms_one,
               "h2d_bytes_per_step": 2 * M * K, "d2h_bytes_per_step": 2 * M * N, "steps": ke,
               "call": "mq_run_layer(host=1, MQ_LAYER_PREPARED): H2D X, quantize X, GEMM, D2H Y",
               "overlap": "none (one stream)", "l2": f"steps rotate over {R} weight copies (> 2x L2)",
               "one_stream": one}
        try:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=streams[0]):
                for st in streams[1:]:
                    st.wait_stream(streams[0])
                for i in range(S * G):
                    run_step(i)
                for st in streams[1:]:
                    streams[0].wait_stream(st)
            with torch.cuda.stream(streams[0]):
                g.replay()
            torch.cuda.synchronize()
            reps = max(5, ke // (S * G))
            if world > 1:
                dist.barrier()
            torch.cuda.synchronize()
            with torch.cuda.stream(streams[0]):
                a0.record(streams[0])
                for _ in range(reps):
                    g.replay()
                a1.record(streams[0])
            torch.cuda.synchronize()
            ms_e = max_over_ranks(a0.elapsed_time(a1) / (reps * S * G), world, dev)
            del g
            e2e.update({"value": round(replica_gbs(per_call, world, ms_e), 2), "ms_per_step": ms_e,
                        "steps": reps * S * G,
                        "overlap": f"{S} steps in flight on {S} streams, own buffers each; CUDA graph of {S * G} steps"})
        except RuntimeError as ex:  # keep the one-stream figure, say why the other is missing
            torch.cuda.synchronize()
            e2e["overlap"] = f"not measured: {str(ex).splitlines()[0][:200]}"
        err = mosaic.mq_get_error()
        if err != 0:
            raise RuntimeError(f"device error word {err}")
    del copies, layer
    torch.cuda.empty_cache()

    path = None
    if world == 1 and not args.no_path:
        path = whole_path(dev, args.workload, 6, 600, stream)
    peak = None
    if world == 1 and not args.no_fp4_peak:
        peak = fp4_peak(sampler)
    sampler.stop()
    sweep = drows = None
    if world == 1 and not args.no_sweep:
        torch.cuda.empty_cache()
        sweep, drows = gemm_sweep(peaks, peak["tflops"] if peak else None)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(args.workload)
    if peak:
        gemm["frac_fp4_measured"] = round(tf / peak["tflops"], 5)

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {"metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "warmup_steps_run": warmup_done, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "nvfp4 (e2m1 x e2m1, e4m3 scales, fp32 accumulate)",
            "data": "synthetic",
            "config": {"workload": f"{args.workload} fused GEMM", "M": M, "N": N, "K": K, "budget_frac": 0.10,
                       "budget_blocks": budget, "parallelism": f"replicas x{world}",
                       "l2": f"{R} rotating operand copies ({R * per_call / 1e6:.0f} MB) > 2x L2; no flush",
                       "graphs": f"{R} calls per graph replay (one per copy)"},
            "roofline": roofline, "gemm": gemm, "fp4_peak": peak, "gemm_sweep": sweep, "delta_topk": drows,
            "whole_path": path, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": int(round(launches_per_step * args.steps)), "clocks": clocks}
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
