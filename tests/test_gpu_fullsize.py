"""GPU parity at the workloads' full sizes, in the launch configuration bench.py times:
mq_run_layer's route (Hessian, quantize + Delta without storing the full residual, top-K,
pack from W, activation quantization, fused GEMM with the kernel chosen by AUTO).

Weight quantization, Delta, ranking, selection and the packed store are compared with
the oracle bit for bit over the whole matrix. The GEMM is compared on sampled output
rows (first, last, the first row of the second token tile, a middle one), which the
oracle computes one by one, within the GEMM tolerance; the other rows are checked for
being finite."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_path import check_gemm, to_dev

pytestmark = pytest.mark.gpu

CASES = [("llama3_8b_mlp_prefill", "up"), ("llama3_8b_mlp_prefill", "down"),
         ("qwen3_32b", "q"), ("qwen3_32b", "up"), ("qwen3_32b", "down"),
         ("llama3_70b_mlp", "up"), ("llama3_70b_mlp", "down")]


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def sample_rows(M: int) -> np.ndarray:
    rows = {0, M - 1, M // 2}
    if M > 128:
        rows.add(128)
    return np.array(sorted(rows), dtype=np.int32)


@pytest.mark.parametrize("wl,mat", CASES)
def test_full_size_path(wl, mat, dev):
    from bit_quantized_gemm_zipperengine_b200 import mosaic
    w = synth.WORKLOADS[wl]
    L = synth.layer(wl, matrix=mat, M=max(w.Ms))
    N, K = L["N"], L["K"]
    # the oracle over the whole matrix (budget-independent parts once)
    wq = oracle.quantize_weight(L["W"])
    H = oracle.hessian_diag(L["Xcal"])
    delta = oracle.delta_score(L["W"], H, wq)
    xq = oracle.quantize_act(L["X"])
    Wd, Cd, Xd = to_dev(L["W"], dev), to_dev(L["Xcal"], dev), to_dev(L["X"], dev)
    for frac in w.budgets:
        budget = synth.budget_blocks(N, K, frac)
        rank, sel = oracle.topk(delta, budget)
        packed = oracle.pack_residual(wq, sel, N, K)
        layer = mosaic.Layer(N, K, budget, dev, with_sf=False)
        layer.prepare_path(Wd, Cd)
        torch.cuda.synchronize()
        assert mosaic.mq_get_error() == 0
        what = f"{wl}/{mat} budget {budget}"
        assert layer.base["gscale"].cpu().numpy()[0] == wq["g"], what
        assert np.array_equal(layer.base["codes"].cpu().numpy(), wq["codes"]), what
        assert np.array_equal(layer.base["sf_swz"].cpu().numpy(), oracle.sf_tile(wq["sf"], N, K)), what
        assert np.array_equal(layer.H.cpu().numpy().view(np.uint32), H.view(np.uint32)), what
        assert np.array_equal(layer.delta.cpu().numpy().view(np.uint64), delta.ravel().view(np.uint64)), what
        assert np.array_equal(layer.rank[:budget].cpu().numpy(), rank), what
        assert np.array_equal(layer.sel[:budget].cpu().numpy(), sel), what
        for k in ("blk_codes", "blk_sf", "blk_kt"):
            assert np.array_equal(layer.packed[k][:budget].cpu().numpy(), packed[k]), (what, k)
        assert np.array_equal(layer.packed["tile_ptr"].cpu().numpy(), packed["tile_ptr"]), what
        assert np.array_equal(layer.packed["bitmap"].cpu().numpy().view(np.uint32), packed["bitmap"]), what
        for M in w.Ms:
            Y = layer.forward(Xd[:M].contiguous())
            torch.cuda.synchronize()
            assert mosaic.mq_get_error() == 0
            assert torch.isfinite(Y.float()).all(), (what, M)
            rows = sample_rows(M)
            y_ref, yabs = oracle.gemm_rows(xq, wq, sel, M, N, K, 0, rows)
            y = Y[torch.from_numpy(rows).long().to(dev)].float().cpu().numpy().astype(np.float64)
            check_gemm(y, y_ref, yabs, f"{what} M={M}")
        del layer
        torch.cuda.empty_cache()
