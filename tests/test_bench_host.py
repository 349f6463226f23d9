"""bench.py's host-side bookkeeping, without a GPU: the algorithmic bytes per call, the
ingestion of an ncu DRAM-bytes capture into traffic.json, and the clock summary."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_step_bytes_decode_workload():
    # LLaMA3-8B q_proj decode: M=16, N=K=4096, T=512, 409 selected blocks
    b = bench.step_bytes(16, 4096, 4096, 512, 409)
    NK, B = 4096 * 4096, 64 * 64
    assert b["quantize_weight_delta"] == 2 * NK + 4 * 4096 + NK // 2 + NK // 16 + 4 + 8 * B == 43040772
    assert b["hessian_diag"] == 2 * 512 * 4096 + 4 * 4096
    assert b["topk_blocks"] == 8 * B + 8 * 409
    # the selected blocks' bf16 W (8 KB each) in, the packed 2048 + 512 B out
    assert b["pack_residual"] > 409 * (8192 + 2560)
    # the per-call figures bench.py reports for this workload, and the step's 62.4 MB
    assert (b["pack_residual"], b["quantize_act"], b["gemm"]) == (4401616, 196672, 10548296)
    assert sum(b.values()) == 62434084


def _row(i, kernel, metric, value):
    return (f'"{i}","1","python","h","{kernel}","1","7","(256, 1, 1)","(444, 1, 1)","0","10.0",'
            f'"Command line profiler metrics","{metric}","byte","{value}"\n')


def test_traffic_ingestion(tmp_path):
    hdr = ('"ID","Process ID","Process Name","Host Name","Kernel Name","Context","Stream","Block Size",'
           '"Grid Size","Device","CC","Section Name","Metric Name","Metric Unit","Metric Value"\n')
    lines = ["==PROF== Connected to process 1\n", hdr]
    calls = [(33554432, 100, 2000, 3000000), (33550000, 200, 50000, 2900000), (33560000, 0, 10, 3100000)]
    for c, (ar, aw, qr, qw) in enumerate(calls):
        lines += [_row(2 * c, "k_amax_partial(const unsigned short *, long, float *)", "dram__bytes_read.sum", ar),
                  _row(2 * c, "k_amax_partial(const unsigned short *, long, float *)", "dram__bytes_write.sum", aw),
                  _row(2 * c + 1, "void k_quant_delta<1, 0>(CUtensorMap_st, ...)", "dram__bytes_read.sum", qr),
                  _row(2 * c + 1, "void k_quant_delta<1, 0>(CUtensorMap_st, ...)", "dram__bytes_write.sum", qw)]
    csv_path = tmp_path / "traffic.csv"
    csv_path.write_text("".join(lines))
    out = tmp_path / "traffic.json"
    e = bench.write_traffic(str(csv_path), skip=1, out_path=str(out), workload="qwen3_32b")
    want = sum(sum(c) for c in calls[1:]) / 2
    assert e["calls"] == 2 and abs(e["bytes_per_call"] - want) <= 1
    d = json.loads(out.read_text())
    assert d["quantize_weight_delta"]["source_hash"] == bench.source_hash()
    assert d["quantize_weight_delta"]["workload"] == "qwen3_32b"


def test_traffic_belongs_to_its_workload():
    # a capture taken on one workload is never reported for another
    assert bench.dram_traffic("gemm", "llama3_8b_mlp_prefill") is None
    assert bench.dram_traffic("gemm", "no such workload") is None


def test_clock_summary():
    cs = bench.ClockSampler(0)
    row = lambda sm, pc: ["t", "0", str(sm), "1965", "900", "0x0", "Not Active", "Not Active", "Not Active", pc]
    cs.samples = [(1.0, row(1965, "Not Active")), (1.2, row(1800, "Active")), (1.4, row(1965, "Not Active")),
                  (9.0, row(100, "Not Active"))]
    s = cs.summary(1.0, 1.4)
    assert s["samples"] == 3 and s["sm_mhz"] == 1965.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"]
