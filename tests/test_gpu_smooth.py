"""The equivalent transform on the GPU (SmoothQuant's per-channel rule, strength 1/2)
against the oracle: scales, smoothed weight and smoothed activations bit for bit, on the
tiny layer and the LLaMA3-8B q_proj layer; then the whole path on the smoothed operands
(the order the pages give: migrate outliers, then split into base and residual)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_path import check_gemm, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


@pytest.mark.parametrize("name", ["tiny", "llama3_8b_qproj_decode"])
def test_smooth_bit_exact_and_path(name, dev):
    from bit_quantized_gemm_zipperengine_b200 import mosaic
    L = synth.layer(name)
    N, K, M, T = L["N"], L["K"], L["M"], L["T"]
    W, X, C = to_dev(L["W"], dev), to_dev(L["X"], dev), to_dev(L["Xcal"], dev)
    s = torch.empty(K, dtype=torch.float32, device=dev)
    mosaic.mq_smooth_scales(C, W, s)
    Wp, Xp, Cp = torch.empty_like(W), torch.empty_like(X), torch.empty_like(C)
    mosaic.mq_smooth_apply(W, s, False, Wp)
    mosaic.mq_smooth_apply(X, s, True, Xp)
    mosaic.mq_smooth_apply(C, s, True, Cp)
    torch.cuda.synchronize()
    assert mosaic.mq_get_error() == 0
    s_ref = oracle.smooth_scales(L["Xcal"], L["W"])
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    Wr = oracle.smooth_apply(L["W"], s_ref, invert=False)
    Xr = oracle.smooth_apply(L["X"], s_ref, invert=True)
    Cr = oracle.smooth_apply(L["Xcal"], s_ref, invert=True)
    bits = lambda t: t.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(bits(Wp), Wr) and np.array_equal(bits(Xp), Xr) and np.array_equal(bits(Cp), Cr)
    # the path on the smoothed layer
    budget = synth.budget_blocks(N, K, 0.10)
    layer = mosaic.Layer(N, K, budget, dev)
    layer.prepare(Wp, Cp)
    Y = layer.forward(Xp)
    torch.cuda.synchronize()
    assert mosaic.mq_get_error() == 0
    ref = oracle.run_path(Wr, Xr, Cr, budget)
    assert np.array_equal(layer.sel[:budget].cpu().numpy(), ref["sel"])
    check_gemm(Y.float().cpu().numpy().astype(np.float64), ref["y"], ref["yabs"], f"smoothed {name}")
