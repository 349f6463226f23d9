"""mq_gemm_noalloc: the fused GEMM for callers that cannot allocate device memory.

Such callers (code embedded in a framework that owns all device memory, or paths where
an allocation is not allowed) cannot hand the library a workspace; this entry point
keeps its split-K scratch in a static buffer inside the library instead. The test
checks it through the C ABI against mq_gemm (which takes a caller workspace), within
the GEMM tolerance, on two calls in a row, and that a problem needing more scratch
than the static buffer holds is refused. This file is collected last on purpose.
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


def _narrow_layer(M):
    """A 1024 x 4096 layer: 8 weight tiles, so the decode GEMM splits K 16 ways and its
    partials go through scratch memory (the case this entry point exists for)."""
    N, K = 1024, 4096
    return {"N": N, "K": K, "M": M, "T": 128,
            "W": synth.weight(N, K, 901, 904, 0.02, int(0.005 * N * K), 51, 20.0),
            "X": synth.act(M, K, 902, 904, 40, 30.0), "Xcal": synth.act(128, K, 903, 904, 40, 30.0)}


@pytest.mark.parametrize("M", [16, 64])
def test_noalloc_matches_workspace_gemm_twice(M, dev):
    from bit_quantized_gemm_zipperengine_b200 import mosaic
    L = _narrow_layer(M)
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


def test_noalloc_refuses_problems_beyond_the_static_scratch(dev):
    from bit_quantized_gemm_zipperengine_b200 import mosaic
    Lb = mosaic.lib()
    limit = Lb.mq_gemm_noalloc_scratch_limit()
    assert limit == 8 << 20
    # M=16, N=1024, K=16384 needs 16 splits x 16 x 1024 fp32 partials = 1 MiB (fits);
    # M=128, N=1024, K=16384 needs 16 x 128 x 1024 x 4 B = 8 MiB plus the tile counters
    # and must be refused before any launch.
    assert 0 < Lb.mq_gemm_workspace_bytes(16, 1024, 16384, 0) <= limit
    M, N, K = 128, 1024, 16384
    assert Lb.mq_gemm_workspace_bytes(M, N, K, 0) > limit
    fake = ctypes.c_void_p(0x10000)
    xm = mosaic.NVFP4Mat(M, K, fake, None, fake, fake)
    wm = mosaic.NVFP4Mat(N, K, fake, None, fake, fake)
    st = Lb.mq_gemm_noalloc(ctypes.byref(xm), ctypes.byref(wm), None, fake, M, N, K, 0, None)
    assert st == 3  # MQ_ERR_WORKSPACE
