"""mq_gemm_noalloc: the fused GEMM for callers that cannot allocate device memory.

Such callers (code embedded in a framework that owns all device memory, or paths where
an allocation is not allowed) cannot hand the library a workspace; this entry point
keeps its split-K scratch in a static buffer inside the library instead. The test
checks it through the C ABI against mq_gemm (which takes a caller workspace), within
the GEMM tolerance, on two calls in a row; that it picks the same kernel as mq_gemm for
every flag and shape (so its results match mq_gemm's bit for bit); and that a problem
needing more scratch than the static buffer holds is refused. This file is collected
last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth
from gpu_path import check_gemm, oracle_ref, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def _narrow_layer(M, N=1024):
    """A layer whose decode GEMM (the stream-K kernel at these token counts) splits tiles
    between CTAs, so its partials go through scratch memory (the case this entry point
    exists for): N = 1024 (8 tiles) at 64 tokens, N = 19200 (150 tiles) at 16."""
    K = 4096
    return {"N": N, "K": K, "M": M, "T": 128,
            "W": synth.weight(N, K, 901, 904, 0.02, int(0.005 * N * K), (N // 64) * (K // 64) // 20, 20.0),
            "X": synth.act(M, K, 902, 904, 40, 30.0), "Xcal": synth.act(128, K, 903, 904, 40, 30.0)}


@pytest.mark.parametrize("M,N", [(16, 19200), (64, 1024)])
def test_noalloc_matches_workspace_gemm_twice(M, N, dev):
    from bit_quantized_gemm_zipperengine_b200 import mosaic
    L = _narrow_layer(M, N)
    N, K = L["N"], L["K"]
    name = f"narrow M={M}"
    assert mosaic.lib().mq_gemm_workspace_bytes(M, N, K, 0) > 0  # the scratch is really used
    budget = synth.budget_blocks(N, K, 0.10)
    layer = mosaic.Layer(N, K, budget, dev)
    layer.prepare(to_dev(L["W"], dev), to_dev(L["Xcal"], dev))
    X = to_dev(L["X"], dev)
    Y_ws = layer.forward(X).clone()          # mq_gemm with a caller workspace
    xq = layer.act_buffers(M)[0]
    ref = oracle_ref(L, budget)
    y_ws = Y_ws.float().cpu().numpy().astype(np.float64)
    for call in range(2):                     # two calls in a row share the static scratch
        Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=dev)
        mosaic.mq_gemm_noalloc(xq, layer.base, layer.packed, Y, M, N, K, 0)
        torch.cuda.synchronize()
        assert mosaic.mq_get_error() == 0
        y = Y.float().cpu().numpy().astype(np.float64)
        # within the GEMM tolerance of the workspace entry point's output
        check_gemm(y, y_ws, ref["yabs"], f"{name} noalloc call {call} vs mq_gemm")
        check_gemm(y, ref["y"], ref["yabs"], f"{name} noalloc call {call} vs oracle")


@pytest.mark.parametrize("M,flags", [(16, "DECODE"), (64, "DECODE"), (256, "AUTO"), (256, "PREFILL"),
                                     (16, "BASE_ONLY"), (16, "RESIDUAL_ONLY"), (256, "RESIDUAL_ONLY")])
def test_noalloc_follows_mq_gemm_kernel_choice(M, flags, dev):
    """Same flags, same kernel: the output equals mq_gemm's bit for bit (M=256 with
    N % 256 == 0 takes the large-M kernel, which needs no scratch at all)."""
    from bit_quantized_gemm_zipperengine_b200 import mosaic
    f = 0 if flags == "AUTO" else getattr(mosaic, "MQ_GEMM_" + flags)
    L = _narrow_layer(M)
    N, K = L["N"], L["K"]
    budget = synth.budget_blocks(N, K, 0.10)
    layer = mosaic.Layer(N, K, budget, dev)
    layer.prepare(to_dev(L["W"], dev), to_dev(L["Xcal"], dev))
    X = to_dev(L["X"], dev)
    Y_ws = layer.forward(X, f).clone()
    xq = layer.act_buffers(M, f)[0]
    for call in range(2):
        Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=dev)
        mosaic.mq_gemm_noalloc(xq, layer.base, layer.packed, Y, M, N, K, f)
        torch.cuda.synchronize()
        assert mosaic.mq_get_error() == 0
        assert torch.equal(Y.view(torch.int16), Y_ws.view(torch.int16)), (M, flags, call)


def test_noalloc_refuses_problems_beyond_the_static_scratch(dev):
    from bit_quantized_gemm_zipperengine_b200 import mosaic
    Lb = mosaic.lib()
    limit = Lb.mq_gemm_noalloc_scratch_limit()
    assert limit == 16 << 20
    # the first shape fits the static scratch; the second needs more than it holds and
    # must be refused before any launch
    assert 0 < Lb.mq_gemm_workspace_bytes(64, 1024, 16384, 0) <= limit
    M, N, K = 128, 1024, 16384
    assert Lb.mq_gemm_workspace_bytes(M, N, K, 0) > limit
    # real, correctly sized buffers: were the refusal to regress, the kernel would read
    # and write allocated memory, not a made-up address
    xm = mosaic.alloc_act(M, K, dev)
    wm, _ = mosaic.alloc_weight(N, K, dev, with_sf=False)
    Y = torch.zeros((M, N), dtype=torch.bfloat16, device=dev)
    st = Lb.mq_gemm_noalloc(ctypes.byref(mosaic.mat(xm)), ctypes.byref(mosaic.mat(wm)), None,
                            ctypes.c_void_p(Y.data_ptr()), M, N, K, 0, None)
    assert st == 3  # MQ_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert mosaic.mq_get_error() == 0
