"""The decode GEMM's two kernels and their work splits (GPU). Small problems: each 128-row
tile's K range split evenly among the CTAs of a cluster, the partials added through the
cluster's shared memory. Larger ones (stream-K): persistent CTAs take equal contiguous
ranges of (tile, 256-K stage) units, so tiles are cut into segments that different CTAs
finish and one of them adds in order. The cases cover both kernels with every token tile
(16/32/64/128 tokens, and several of them), every 64x64 block selected (the residual
ring full on every stage), and the base-only and residual-only modes (segments without
any residual block). Each runs twice on the same workspace: the tile counters must come
back to zero and the output repeat bit for bit."""
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


CASES = [
    # N, K, M, budget fraction, flags
    # the small-problem kernel (M <= 32, at most 74 tiles, short K ranges): each tile split
    # among the CTAs of a cluster
    (128, 256, 1, 0.50, "AUTO"),          # one tile, one K stage: one CTA
    (512, 4096, 16, 0.10, "AUTO"),        # 4 tiles x 8 splits
    (4096, 4096, 16, 1.00, "AUTO"),       # every block selected: 8 residual blocks per stage
    (4096, 4096, 16, 0.10, "RESIDUAL_ONLY"),
    (4096, 4096, 16, 0.10, "BASE_ONLY"),
    (5120, 5120, 32, 0.10, "AUTO"),       # 40 tiles x 3 splits of 6-7 stages, 32-token tile
    # the stream-K kernel
    (19200, 4096, 16, 0.10, "AUTO"),      # 150 tiles: 2400 units on 148 CTAs, tiles split
    (19200, 4096, 16, 1.00, "AUTO"),      # every block selected
    (4096, 14336, 16, 0.10, "RESIDUAL_ONLY"),  # long K: segments without residual blocks
    (4096, 14336, 16, 0.10, "BASE_ONLY"),
    (25600, 512, 33, 0.10, "AUTO"),       # 400 units, 2-3 per CTA, 64-token tile
    (1024, 8192, 100, 0.20, "AUTO"),      # 128-token tile
    (512, 1024, 300, 0.10, "DECODE"),     # three 128-token tiles
]


@pytest.mark.parametrize("N,K,M,frac,flags_name", CASES)
def test_decode_gemm_work_split(N, K, M, frac, flags_name, dev):
    from bit_quantized_gemm_zipperengine_b200 import mosaic
    seed = 900 + N % 97 + K % 89 + M
    L = {"N": N, "K": K, "M": M, "T": 128,
         "W": synth.weight(N, K, seed, seed + 3, 0.02, int(0.005 * N * K), max(1, (N // 64) * (K // 64) // 20),
                           20.0),
         "X": synth.act(M, K, seed + 1, seed + 3, max(1, K // 100), 30.0),
         "Xcal": synth.act(128, K, seed + 2, seed + 3, max(1, K // 100), 30.0)}
    budget = synth.budget_blocks(N, K, frac)
    flags = 0 if flags_name == "AUTO" else getattr(mosaic, "MQ_GEMM_" + flags_name)
    mode = {"BASE_ONLY": 1, "RESIDUAL_ONLY": 2}.get(flags_name, 0)
    layer = mosaic.Layer(N, K, budget, dev)
    layer.prepare(to_dev(L["W"], dev), to_dev(L["Xcal"], dev))
    X = to_dev(L["X"], dev)
    Ys = []
    for _ in range(2):
        # the output buffer is reused: fill it first, so that a tile the second call failed
        # to store (a counter left non-zero by the first) shows up
        layer.act_buffers(M, flags)[1].fill_(float("nan"))
        Ys.append(layer.forward(X, flags).clone())
    torch.cuda.synchronize()
    assert mosaic.mq_get_error() == 0
    assert torch.equal(Ys[0].view(torch.int16), Ys[1].view(torch.int16))
    wq = oracle.quantize_weight(L["W"])
    H = oracle.hessian_diag(L["Xcal"])
    _, sel = oracle.topk(oracle.delta_score(L["W"], H, wq), budget)
    assert np.array_equal(layer.sel[:budget].cpu().numpy(), sel)
    xq = oracle.quantize_act(L["X"])
    y, ya = oracle.gemm_rows(xq, wq, sel, M, N, K, mode)
    check_gemm(Ys[0].float().cpu().numpy().astype(np.float64), y, ya, f"{N}x{K} M={M} {flags_name}")
    if mode == 2:
        assert np.abs(y).max() > 0
