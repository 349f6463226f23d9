"""A pipeline wait that runs out (GPU), without faulting anything: the test hook makes CTA
0 of one decode-GEMM launch skip one stage's W copies and shortens every wait of that
launch to about a millisecond. The MMA issuer's wait for that stage then runs out with no
copy in flight; the kernel records MQ_ERR_TIMEOUT, stops issuing, releases its tensor
memory and returns, and mq_get_error() reports it. The context stays usable: the next
call (on a cleared workspace) matches the oracle."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_path import check_gemm, to_dev

pytestmark = pytest.mark.gpu

MQ_ERR_TIMEOUT = 5


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


@pytest.mark.parametrize("N,K,M,unit", [(4096, 4096, 16, 1), (1024, 4096, 16, 0),    # small-problem kernel
                                        (19200, 4096, 16, 1), (512, 1024, 100, 0)])  # stream-K kernel
def test_wait_runs_out_and_gpu_stays_usable(N, K, M, unit, dev):
    from bit_quantized_gemm_zipperengine_b200 import mosaic
    L = {"W": synth.weight(N, K, 951, 954, 0.02, int(0.005 * N * K), max(1, (N // 64) * (K // 64) // 20), 20.0),
         "X": synth.act(M, K, 952, 954, max(1, K // 100), 30.0),
         "Xcal": synth.act(128, K, 953, 954, max(1, K // 100), 30.0)}
    budget = synth.budget_blocks(N, K, 0.10)
    layer = mosaic.Layer(N, K, budget, dev)
    layer.prepare(to_dev(L["W"], dev), to_dev(L["Xcal"], dev))
    X = to_dev(L["X"], dev)
    xq, Y, ws = layer.act_buffers(M)
    mosaic.mq_quantize_act(X, xq)
    torch.cuda.synchronize()
    assert mosaic.mq_get_error() == 0
    Lb = mosaic.lib()
    assert Lb.mq_test_arm_wait_fault(unit, 1.0) == 0
    mosaic.mq_gemm(xq, layer.base, layer.packed, Y, M, N, K, 0, ws)   # the armed launch
    assert mosaic.mq_get_error() == MQ_ERR_TIMEOUT                     # synchronizes, reads, clears
    assert mosaic.mq_get_error() == 0                                  # cleared
    # the context is usable: clear the workspace's tile counters, run again, compare
    if ws is not None:
        ws.zero_()
    Y.fill_(float("nan"))
    mosaic.mq_gemm(xq, layer.base, layer.packed, Y, M, N, K, 0, ws)
    torch.cuda.synchronize()
    assert mosaic.mq_get_error() == 0
    wq = oracle.quantize_weight(L["W"])
    H = oracle.hessian_diag(L["Xcal"])
    _, sel = oracle.topk(oracle.delta_score(L["W"], H, wq), budget)
    y, ya = oracle.gemm_rows(oracle.quantize_act(L["X"]), wq, sel, M, N, K)
    check_gemm(Y.float().cpu().numpy().astype(np.float64), y, ya, f"after timeout {N}x{K} M={M}")
