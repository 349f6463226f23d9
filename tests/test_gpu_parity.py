"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the same seeded
inputs. Codes, scales, H, Delta (fp64 bits), ranking, selection and the packed store are
compared bit for bit; the GEMM within the stated tolerance."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_path import check_gemm, gpu_run, oracle_ref, prepare, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


_cache = {}
_oracle = {}


def _pair(name, dev, M=None, fused=False):
    key = (name, M, fused)
    if key not in _cache:
        L = synth.layer(name, M=M)
        budget = synth.budget_blocks(L["N"], L["K"], 0.10)
        if (name, M) not in _oracle:
            _oracle[(name, M)] = oracle_ref(L, budget)
        _cache[key] = (L, budget, gpu_run(L, budget, dev, fused=fused), _oracle[(name, M)])
    return _cache[key]


WORKLOADS = ["tiny", "llama3_8b_qproj_decode"]
PATHS = [pytest.param(False, id="separate"), pytest.param(True, id="fused"), pytest.param("path", id="path")]


@pytest.mark.parametrize("fused", PATHS)
@pytest.mark.parametrize("name", WORKLOADS)
def test_quantize_weight_bit_exact(name, fused, dev):
    L, budget, g, o = _pair(name, dev, fused=fused)
    wq = o["wq"]
    assert g["g"] == wq["g"]
    assert np.array_equal(g["codes"], wq["codes"])
    assert np.array_equal(g["sf"], wq["sf"])
    assert np.array_equal(g["sf_swz"], oracle.sf_tile(wq["sf"], L["N"], L["K"]))
    if fused != "path":  # the run_layer route does not store the full residual
        assert np.array_equal(g["r_codes"], wq["r_codes"])
        assert np.array_equal(g["r_sf"], wq["r_sf"])


@pytest.mark.parametrize("fused", PATHS)
@pytest.mark.parametrize("name", WORKLOADS)
def test_hessian_bit_exact(name, fused, dev):
    L, budget, g, o = _pair(name, dev, fused=fused)
    assert np.array_equal(g["H"].view(np.uint32), o["H"].view(np.uint32))


@pytest.mark.parametrize("fused", PATHS)
@pytest.mark.parametrize("name", WORKLOADS)
def test_delta_and_selection_bit_exact(name, fused, dev):
    L, budget, g, o = _pair(name, dev, fused=fused)
    assert np.array_equal(g["delta"].view(np.uint64), o["delta"].view(np.uint64))
    assert np.array_equal(g["rank"], o["rank"])
    assert np.array_equal(g["sel"], o["sel"])


@pytest.mark.parametrize("fused", PATHS)
@pytest.mark.parametrize("name", WORKLOADS)
def test_pack_bit_exact(name, fused, dev):
    L, budget, g, o = _pair(name, dev, fused=fused)
    for k in ("blk_codes", "blk_sf", "blk_kt", "tile_ptr"):
        assert np.array_equal(g["packed"][k], o["packed"][k]), k
    assert np.array_equal(g["packed"]["bitmap"].view(np.uint32), o["packed"]["bitmap"])


@pytest.mark.parametrize("name", WORKLOADS)
def test_quantize_act_bit_exact(name, dev):
    L, budget, g, o = _pair(name, dev)
    xq = o["xq"]
    assert np.array_equal(g["xq_codes"], xq["codes"])
    assert np.array_equal(g["xq_g"], xq["g"])
    assert np.array_equal(g["xq_swz"], oracle.sf_tile(xq["sf"], L["M"], L["K"]))


@pytest.mark.parametrize("fused", PATHS)
@pytest.mark.parametrize("name", WORKLOADS)
def test_gemm_fused_within_tolerance(name, fused, dev):
    L, budget, g, o = _pair(name, dev, fused=fused)
    check_gemm(g["Y"], o["y"], o["yabs"], name)


@pytest.mark.parametrize("M", [1, 5, 16, 37, 64, 100, 128, 130, 300])
def test_gemm_ragged_token_counts(M, dev):
    """Token counts that are not a multiple of the token tile (ragged tail), across the
    16/32/64/128 token tiles and several token tiles."""
    L = synth.layer("tiny", M=M)
    budget = synth.budget_blocks(L["N"], L["K"], 0.10)
    g = gpu_run(L, budget, dev)
    o = oracle_ref(L, budget)
    assert np.array_equal(g["xq_codes"], o["xq"]["codes"])
    check_gemm(g["Y"], o["y"], o["yabs"], f"M={M}")


@pytest.mark.parametrize("M", [129, 256, 300, 1000])
@pytest.mark.parametrize("flags_name", ["AUTO", "PREFILL", "DECODE"])
def test_gemm_prefill_kernel(M, flags_name, dev):
    """Large token counts through the prefill kernel (tokens as the MMA's M side, 256-row
    weight tiles, N = 64 residual MMAs), with a ragged last token tile; the decode kernel
    forced on the same inputs must agree with the oracle too."""
    from bit_quantized_gemm_zipperengine_b200 import mosaic
    N, K = 512, 1024
    L = {"N": N, "K": K, "M": M, "T": 128,
         "W": synth.weight(N, K, 701, 704, 0.02, int(0.005 * N * K), 6, 20.0),
         "X": synth.act(M, K, 702, 704, 10, 30.0), "Xcal": synth.act(128, K, 703, 704, 10, 30.0)}
    budget = synth.budget_blocks(N, K, 0.10)
    flags = getattr(mosaic, "MQ_GEMM_" + flags_name)
    g = gpu_run(L, budget, dev, flags=flags, fused=True)
    o = oracle_ref(L, budget)
    check_gemm(g["Y"], o["y"], o["yabs"], f"M={M} {flags_name}")


def test_gemm_prefill_modes(dev):
    """Prefill kernel: base-only equals the oracle's dense base; residual-only the
    oracle's residual; r = NULL equals base-only bit for bit."""
    from bit_quantized_gemm_zipperengine_b200 import mosaic
    N, K, M = 512, 1024, 384
    L = {"N": N, "K": K, "M": M, "T": 128,
         "W": synth.weight(N, K, 711, 714, 0.02, int(0.005 * N * K), 6, 20.0),
         "X": synth.act(M, K, 712, 714, 10, 30.0), "Xcal": synth.act(128, K, 713, 714, 10, 30.0)}
    budget = synth.budget_blocks(N, K, 0.10)
    g = gpu_run(L, budget, dev, fused=True)
    o = oracle_ref(L, budget)
    layer = g["layer"]
    xq = layer.act_buffers(M)[0]
    outs = {}
    for name, flags, packed in (("base", mosaic.MQ_GEMM_BASE_ONLY, layer.packed), ("none", 0, None),
                                ("resid", mosaic.MQ_GEMM_RESIDUAL_ONLY, layer.packed)):
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        mosaic.mq_gemm(xq, layer.base, packed, Y, M, N, K, flags | mosaic.MQ_GEMM_PREFILL, None)
        outs[name] = Y
    torch.cuda.synchronize()
    assert torch.equal(outs["base"], outs["none"])
    yb, yba = oracle.gemm_rows(o["xq"], o["wq"], o["sel"], M, N, K, 1)
    check_gemm(outs["base"].float().cpu().numpy().astype(np.float64), yb, yba, "prefill base only")
    yr, yra = oracle.gemm_rows(o["xq"], o["wq"], o["sel"], M, N, K, 2)
    check_gemm(outs["resid"].float().cpu().numpy().astype(np.float64), yr, yra, "prefill residual only")


@pytest.mark.parametrize("mode", ["fused", "BASE_ONLY", "RESIDUAL_ONLY"])
def test_gemm_prefill_pairs_many_tiles(mode, dev):
    """The large-M kernel on CTA pairs with several tiles per pair and more K stages than
    pipeline stages (128 tiles of 256 x 256 over at most 74 pairs, 8 stages of K each):
    the stage and accumulator barriers cycle through many phases, including stages that
    carry no copies for one CTA of the pair (residual-only stages without a selected
    block). Sampled token rows against the oracle, and a repeat bit for bit."""
    from bit_quantized_gemm_zipperengine_b200 import mosaic
    N, K, M = 4096, 2048, 2048
    L = {"N": N, "K": K, "M": M, "T": 128,
         "W": synth.weight(N, K, 721, 724, 0.02, int(0.005 * N * K), (N // 64) * (K // 64) // 20, 20.0),
         "X": synth.act(M, K, 722, 724, 20, 30.0), "Xcal": synth.act(128, K, 723, 724, 20, 30.0)}
    budget = synth.budget_blocks(N, K, 0.10)
    flags = mosaic.MQ_GEMM_PREFILL | (0 if mode == "fused" else getattr(mosaic, "MQ_GEMM_" + mode))
    layer = mosaic.Layer(N, K, budget, dev)
    layer.prepare(to_dev(L["W"], dev), to_dev(L["Xcal"], dev))
    X = to_dev(L["X"], dev)
    outs = []
    for _ in range(2):
        layer.act_buffers(M, flags)[1].fill_(float("nan"))
        outs.append(layer.forward(X, flags).clone())
    torch.cuda.synchronize()
    assert mosaic.mq_get_error() == 0
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))
    rows = np.array(sorted(set(list(range(0, M, 97)) + [127, 128, 255, 256, M - 1])), dtype=np.int32)
    wq = oracle.quantize_weight(L["W"])
    H = oracle.hessian_diag(L["Xcal"])
    _, sel = oracle.topk(oracle.delta_score(L["W"], H, wq), budget)
    assert np.array_equal(layer.sel[:budget].cpu().numpy(), sel)
    xo = oracle.quantize_act(L["X"])
    y, ya = oracle.gemm_rows(xo, wq, sel, M, N, K, {"fused": 0, "BASE_ONLY": 1, "RESIDUAL_ONLY": 2}[mode], rows)
    got = outs[0][torch.from_numpy(rows).long().to(dev)].float().cpu().numpy().astype(np.float64)
    check_gemm(got, y, ya, f"pairs {mode}")


@pytest.mark.parametrize("M", [16, 100, 128])
def test_gemm_narrow_layer_workspace_split_k(M, dev):
    """A 1024 x 4096 layer: 8 weight tiles, so K is split 16 ways and the partials are
    added through the global workspace (the path above the cluster size)."""
    from bit_quantized_gemm_zipperengine_b200 import mosaic
    N, K = 1024, 4096
    L = {"N": N, "K": K, "M": M, "T": 128,
         "W": synth.weight(N, K, 801, 804, 0.02, int(0.005 * N * K), 51, 20.0),
         "X": synth.act(M, K, 802, 804, 40, 30.0), "Xcal": synth.act(128, K, 803, 804, 40, 30.0)}
    budget = synth.budget_blocks(N, K, 0.10)
    assert mosaic.lib().mq_gemm_workspace_bytes(M, N, K, 0) > 0
    g = gpu_run(L, budget, dev, fused=True)
    o = oracle_ref(L, budget)
    assert np.array_equal(g["sel"], o["sel"])
    check_gemm(g["Y"], o["y"], o["yabs"], f"narrow M={M}")


def test_gemm_base_only_paths_identical(dev):
    """r = NULL, a zero budget and the BASE_ONLY flag all give the dense base, bit for bit,
    and match the oracle's base-only GEMM."""
    from bit_quantized_gemm_zipperengine_b200 import mosaic
    L, budget, g, o = _pair("llama3_8b_qproj_decode", dev)
    layer = g["layer"]
    M, N, K = L["M"], L["N"], L["K"]
    xq, _, ws = layer.act_buffers(M)
    outs = []
    for packed, flags in ((None, 0), (layer.packed, mosaic.MQ_GEMM_BASE_ONLY)):
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        mosaic.mq_gemm(xq, layer.base, packed, Y, M, N, K, flags, ws)
        outs.append(Y)
    zero = mosaic.alloc_packed(N, K, 0, dev)
    mosaic.mq_pack_residual(layer.resid, layer.sel, 0, zero)
    Y0 = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    mosaic.mq_gemm(xq, layer.base, zero, Y0, M, N, K, 0, ws)
    torch.cuda.synchronize()
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[0], Y0)
    yb, yba = oracle.gemm_rows(o["xq"], o["wq"], o["sel"], M, N, K, 1)
    check_gemm(outs[0].float().cpu().numpy().astype(np.float64), yb, yba, "base only")


def test_gemm_linearity(dev):
    """Fused = base-only + residual-only (one accumulator, summed by linearity)."""
    from bit_quantized_gemm_zipperengine_b200 import mosaic
    L, budget, g, o = _pair("llama3_8b_qproj_decode", dev)
    layer = g["layer"]
    M, N, K = L["M"], L["N"], L["K"]
    xq, _, ws = layer.act_buffers(M)
    Yr = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    mosaic.mq_gemm(xq, layer.base, layer.packed, Yr, M, N, K, mosaic.MQ_GEMM_RESIDUAL_ONLY, ws)
    torch.cuda.synchronize()
    yr, yra = oracle.gemm_rows(o["xq"], o["wq"], o["sel"], M, N, K, 2)
    check_gemm(Yr.float().cpu().numpy().astype(np.float64), yr, yra, "residual only")
    assert np.abs(yr).max() > 0


def test_repeat_calls_deterministic(dev):
    """Same inputs twice: quantization, Delta, selection and the GEMM output repeat bit for
    bit (the split-K partials are added in a fixed order)."""
    L, budget, g, o = _pair("llama3_8b_qproj_decode", dev)
    g2 = gpu_run(L, budget, dev)
    for k in ("codes", "sf", "r_codes", "r_sf", "H", "rank", "sel"):
        assert np.array_equal(g[k], g2[k]), k
    assert np.array_equal(g["delta"].view(np.uint64), g2["delta"].view(np.uint64))
    assert np.array_equal(g["Y"], g2["Y"])


def test_topk_blocks_alone_and_large_budgets(dev):
    """A4 alone on many blocks and budgets (the one-CTA radix selection and the split rank
    kernel; keys in shared or global memory, a threshold inside a bucket of one tied value,
    every block selected), with ties, against the oracle's sort."""
    from bit_quantized_gemm_zipperengine_b200 import mosaic
    rng = np.random.default_rng(12)
    cases = [(32, (0, 1, 3, 32), False), (4096, (409, 767, 768, 769, 1024, 1025), False),
             (57344, (500, 2867, 11468, 57344), False), (4096, (300, 500, 700), True),
             (4096, (1000, 2000, 4096), True), (40000, (1300, 6000), True)]
    for B, budgets, many_ties in cases:
        d = rng.standard_normal(B) * np.exp2(rng.integers(-20, 5, B))
        d[rng.choice(B, B // 10, replace=False)] = 0.0      # ties at zero
        d[rng.choice(B, B // 50, replace=False)] = d[0]     # ties at an arbitrary value
        d[:3] = -0.0
        if many_ties:
            # mostly negative, ~400 positive, 1000 zeros: a threshold inside a bucket of one
            # value shared by far more keys than the candidate list holds
            d = -np.abs(d)
            d[rng.choice(B, 400, replace=False)] *= -1.0
            z = rng.choice(np.flatnonzero(d < 0), 1000, replace=False)
            d[z] = 0.0
        dd = torch.from_numpy(d).to(dev)
        for k in budgets:
            rank = torch.empty(max(k, 1), dtype=torch.int32, device=dev)
            sel = torch.empty(max(k, 1), dtype=torch.int32, device=dev)
            mosaic.mq_topk_blocks(dd, k, rank, sel)
            torch.cuda.synchronize()
            r_ref, s_ref = oracle.topk(d, k)
            assert np.array_equal(rank[:k].cpu().numpy(), r_ref), (B, k)
            assert np.array_equal(sel[:k].cpu().numpy(), s_ref), (B, k)


def test_topk_cluster_sizes_and_ties_across_ctas(dev):
    """Key counts that take the cluster selection (more keys than one CTA holds, spread over
    eight CTAs): just above one CTA's capacity (a ragged last CTA), LLaMA3-70B MLP's 57344
    blocks, the largest count the cluster holds and one key more (the one-CTA kernel with
    keys in global memory); one value tied across every CTA with the threshold inside it,
    and all keys equal; budgets 1 .. B. Against the oracle's sort."""
    from bit_quantized_gemm_zipperengine_b200 import mosaic
    rng = np.random.default_rng(77)
    for B in (20481, 57344, 163840, 163841):
        for mode in ("spread", "tied", "equal"):
            d = rng.standard_normal(B) * np.exp2(rng.integers(-20, 5, B))
            if mode == "tied":
                d[rng.choice(B, B // 3, replace=False)] = 0.5
            elif mode == "equal":
                d[:] = 1.25
            dd = torch.from_numpy(d).to(dev)
            # rank counts over the selected set (budget squared comparisons): the full
            # budget range on the smaller key counts only
            ks = (1, 7, B // 20, B // 3, B - 1, B) if B <= 60000 else (1, 7, B // 20, B // 3)
            for k in ks:
                rank = torch.empty(k, dtype=torch.int32, device=dev)
                sel = torch.empty(k, dtype=torch.int32, device=dev)
                mosaic.mq_topk_blocks(dd, k, rank, sel)
                torch.cuda.synchronize()
                assert mosaic.mq_get_error() == 0
                r_ref, s_ref = oracle.topk(d, k)
                assert np.array_equal(sel.cpu().numpy(), s_ref), (B, mode, k)
                assert np.array_equal(rank.cpu().numpy(), r_ref), (B, mode, k)


@pytest.mark.parametrize("host", [False, True])
def test_run_layer_whole_path(host, dev):
    """mq_run_layer (the whole path in one C call), with device buffers and with pinned
    host buffers copied inside the call, against the oracle."""
    from bit_quantized_gemm_zipperengine_b200 import mosaic
    L = synth.layer("llama3_8b_qproj_decode")
    M, N, K, T = L["M"], L["N"], L["K"], L["T"]
    budget = synth.budget_blocks(N, K, 0.10)
    o = _oracle.get(("llama3_8b_qproj_decode", None)) or oracle_ref(L, budget)
    layer = mosaic.Layer(N, K, budget, dev, with_sf=False)
    buf = layer.buffers(M, T, staging=host)
    if host:
        W = torch.from_numpy(L["W"].view(np.int16)).view(torch.bfloat16).pin_memory()
        X = torch.from_numpy(L["X"].view(np.int16)).view(torch.bfloat16).pin_memory()
        C = torch.from_numpy(L["Xcal"].view(np.int16)).view(torch.bfloat16).pin_memory()
        Y = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
    else:
        W, X, C = to_dev(L["W"], dev), to_dev(L["X"], dev), to_dev(L["Xcal"], dev)
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    mosaic.mq_run_layer(W, X, C, Y, M, N, K, T, budget, 0, host, buf)
    torch.cuda.synchronize()
    assert mosaic.mq_get_error() == 0
    assert np.array_equal(layer.sel[:budget].cpu().numpy(), o["sel"])
    # every intermediate the call leaves behind, bit for bit (the activation quantizer runs
    # ahead of the selection and quantizes before waiting for the Delta pass)
    xq_ref = o["xq"]
    xq = layer.act_buffers(M)[0]
    assert np.array_equal(xq["codes"].cpu().numpy(), xq_ref["codes"])
    assert np.array_equal(xq["sf_swz"].cpu().numpy(), oracle.sf_tile(xq_ref["sf"], M, K))
    assert np.array_equal(xq["gscale"].cpu().numpy().view(np.uint32), xq_ref["g"].view(np.uint32))
    assert np.array_equal(layer.H.cpu().numpy().view(np.uint32), o["H"].view(np.uint32))
    assert np.array_equal(layer.rank[:budget].cpu().numpy(), o["rank"])
    check_gemm(Y.float().cpu().numpy().astype(np.float64), o["y"], o["yabs"], f"run_layer host={host}")
    # inference on the prepared layer (A6 + GEMM only; W and Xcal not passed): the same Y
    Y2 = torch.full_like(Y, float("nan"))
    mosaic.mq_run_layer(None, X, None, Y2, M, N, K, T, budget, mosaic.MQ_LAYER_PREPARED, host, buf)
    torch.cuda.synchronize()
    assert mosaic.mq_get_error() == 0
    assert torch.equal(Y2.view(torch.int16), Y.view(torch.int16))


RUN_LAYER_CASES = [
    ("qwen3_32b", "q", 1, 0.10),                        # one token
    ("qwen3_32b", "up", 16, 0.10),                      # wide N
    ("llama3_70b_mlp", "down", 16, 0.10),               # K = 28672: split-K through the workspace
    ("llama3_8b_qproj_decode", "q_proj", 128, 0.10),    # 128-token tile
    ("llama3_8b_qproj_decode", "q_proj", 16, 0.0),      # no budget: no top-K kernel, no residual
    ("llama3_8b_qproj_decode", "q_proj", 16, 0.50),     # budget past the one-CTA top-K
    ("llama3_8b_mlp_prefill", "up", 384, 0.10),         # prefill kernel
]


@pytest.mark.parametrize("wl,mat,M,frac", RUN_LAYER_CASES)
def test_run_layer_shapes(wl, mat, M, frac, dev):
    """mq_run_layer across the GEMM's kernels and plans, with and without a residual: the
    whole-path call overlaps the decode GEMM's base pass with top-K and the pack (the
    residual blocks follow the wait for the pack). Selection and ranking bit for bit, Y on
    sampled token rows within the GEMM tolerance."""
    from bit_quantized_gemm_zipperengine_b200 import mosaic
    L = synth.layer(wl, matrix=mat, M=M)
    N, K, T = L["N"], L["K"], L["T"]
    budget = synth.budget_blocks(N, K, frac)
    rows = np.array(sorted({0, M // 2, M - 1}), dtype=np.int32)
    o = oracle_ref(L, budget, rows)
    layer = mosaic.Layer(N, K, budget, dev, with_sf=False)
    buf = layer.buffers(M, T)
    W, X, C = to_dev(L["W"], dev), to_dev(L["X"], dev), to_dev(L["Xcal"], dev)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    for _ in range(2):  # the second call runs behind the first one's kernels
        mosaic.mq_run_layer(W, X, C, Y, M, N, K, T, budget, 0, False, buf)
    torch.cuda.synchronize()
    assert mosaic.mq_get_error() == 0
    what = f"{wl}/{mat} M={M} budget={budget}"
    if budget:
        assert np.array_equal(layer.rank[:budget].cpu().numpy(), o["rank"]), what
        assert np.array_equal(layer.sel[:budget].cpu().numpy(), o["sel"]), what
    assert torch.isfinite(Y.float()).all(), what
    y = Y[torch.from_numpy(rows).long().to(dev)].float().cpu().numpy().astype(np.float64)
    check_gemm(y, o["y"], o["yabs"], what)


@pytest.mark.parametrize("fused", PATHS)
def test_odd_block_rows_bit_exact(fused, dev):
    """N / 64 odd (5 block rows): the quantize+Delta pass works on strips of two block rows,
    and the last strip holds a single block; codes, tiled scales, Delta, the selection and
    the packed store must still match the oracle bit for bit."""
    from bit_quantized_gemm_zipperengine_b200 import mosaic
    N, K, T = 320, 512, 64
    Wb = synth.weight(N, K, 801, 804, 0.02, int(0.005 * N * K), 4, 20.0)
    Cb = synth.act(T, K, 803, 804, 8, 30.0)
    budget = synth.budget_blocks(N, K, 0.10)
    wq = oracle.quantize_weight(Wb)
    H = oracle.hessian_diag(Cb)
    delta = oracle.delta_score(Wb, H, wq)
    rank, sel = oracle.topk(delta, budget)
    packed = oracle.pack_residual(wq, sel, N, K)
    layer = mosaic.Layer(N, K, budget, dev)
    prepare(layer, to_dev(Wb, dev), to_dev(Cb, dev), fused)
    torch.cuda.synchronize()
    assert mosaic.mq_get_error() == 0
    assert layer.base["gscale"].cpu().numpy()[0] == wq["g"]
    assert np.array_equal(layer.base["codes"].cpu().numpy(), wq["codes"])
    assert np.array_equal(layer.base["sf_swz"].cpu().numpy(), oracle.sf_tile(wq["sf"], N, K))
    assert np.array_equal(layer.delta.cpu().numpy().view(np.uint64), delta.ravel().view(np.uint64))
    assert np.array_equal(layer.rank[:budget].cpu().numpy(), rank)
    assert np.array_equal(layer.sel[:budget].cpu().numpy(), sel)
    for k in ("blk_codes", "blk_sf", "blk_kt"):
        assert np.array_equal(layer.packed[k][:budget].cpu().numpy(), packed[k]), k
    assert np.array_equal(layer.packed["tile_ptr"].cpu().numpy(), packed["tile_ptr"])
    assert np.array_equal(layer.packed["bitmap"].cpu().numpy().view(np.uint32), packed["bitmap"])


@pytest.mark.parametrize("N,K", [(4096, 4096), (1024, 4096), (512, 1024), (25600, 512)])
@pytest.mark.parametrize("M", [1, 5, 16, 37, 64, 100, 128])
def test_gemm_act_fused_quantization(N, K, M, dev):
    """The decode GEMM quantizing bf16 X itself (A6 inside the pipeline) against
    mq_quantize_act + mq_gemm: per-token scales bit-exact with the oracle, and both
    outputs within the GEMM tolerance of the oracle (mq_gemm's decode kernel splits K at
    other points, so its fp32 sums may round differently), across token tiles and the
    three split-K regimes of this kernel (no split: N = 25600; split in a cluster:
    N = 4096 and 512; more than 8 splits through the workspace: N = 1024)."""
    from bit_quantized_gemm_zipperengine_b200 import mosaic
    Wb = synth.weight(N, K, 901, 904, 0.02, int(0.005 * N * K), max(1, (N // 64) * (K // 64) // 20), 20.0)
    Xb = synth.act(M, K, 902, 904, max(1, K // 100), 30.0)
    Cb = synth.act(64, K, 903, 904, max(1, K // 100), 30.0)
    budget = synth.budget_blocks(N, K, 0.10)
    layer = mosaic.Layer(N, K, budget, dev, with_sf=False)
    layer.prepare_path(to_dev(Wb, dev), to_dev(Cb, dev))
    X = to_dev(Xb, dev)
    flags = mosaic.MQ_GEMM_DECODE
    xq, Y2, ws = layer.act_buffers(M, flags)
    mosaic.mq_quantize_act(X, xq)
    mosaic.mq_gemm(xq, layer.base, layer.packed, Y2, M, N, K, flags, ws)
    Y1 = torch.empty_like(Y2)
    gx = torch.empty(M, dtype=torch.float32, device=dev)
    ws1 = mosaic.gemm_workspace(M, N, K, flags, dev)
    for _ in range(2):  # twice: the scratch counters reset themselves
        mosaic.mq_gemm_act(X, layer.base, layer.packed, Y1, M, N, K, flags, ws1, gx)
    torch.cuda.synchronize()
    assert mosaic.mq_get_error() == 0
    xo = oracle.quantize_act(Xb)
    assert np.array_equal(gx.cpu().numpy().view(np.uint32), xo["g"].view(np.uint32))
    assert np.array_equal(xq["codes"].cpu().numpy(), xo["codes"])
    wq = oracle.quantize_weight(Wb)
    sel = layer.sel[:budget].cpu().numpy()
    y_ref, yabs = oracle.gemm_rows(xo, wq, sel, M, N, K)
    check_gemm(Y1.float().cpu().numpy().astype(np.float64), y_ref, yabs, f"gemm_act N={N} K={K} M={M}")
    check_gemm(Y2.float().cpu().numpy().astype(np.float64), y_ref, yabs, f"two calls N={N} K={K} M={M}")


@pytest.mark.parametrize("T", [1, 7, 16, 33, 128, 500, 512, 513, 1000, 1024])
def test_hessian_token_counts(T, dev):
    """A2 alone across calibration token counts (the kernel pads the tree to 512 or 1024
    leaves, the oracle to the next power of two; rows past T are not read): bit-exact with
    the oracle; more than 1024 tokens is refused."""
    from bit_quantized_gemm_zipperengine_b200 import mosaic
    K = 256
    Xb = synth.act(T, K, 911, 914, 3, 30.0)
    H = torch.empty(K, dtype=torch.float32, device=dev)
    mosaic.mq_hessian_diag(to_dev(Xb, dev), H)
    torch.cuda.synchronize()
    assert np.array_equal(H.cpu().numpy().view(np.uint32), oracle.hessian_diag(Xb).view(np.uint32))
    if T == 1024:
        big = to_dev(synth.act(1025, K, 915, 914, 3, 30.0), dev)
        with pytest.raises(mosaic.MosaicError):
            mosaic.mq_hessian_diag(big, H)
