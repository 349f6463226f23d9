"""The distortion-recovery study's evaluation (bit_quantized_gemm_zipperengine_b200/study.py):
its dequantization against the oracle, its incremental exact distortion against a brute
force recomputation of ||X D_S^T||^2, its greedy step against the best single block, and
(on the GPU) the Delta-score of the CUDA path against the diagonal-Hessian surrogate of
the same exact distortion."""
import numpy as np
import pytest
import torch

import oracle
import synth
from bit_quantized_gemm_zipperengine_b200.study import Distortion, dequant_nvfp4, run


def test_dequant_matches_oracle():
    W = synth.weight(128, 256, 41, 42, 0.02, 200, 2, 20.0)
    wq = oracle.quantize_weight(W)
    g = torch.tensor([wq["g"]], dtype=torch.float32)
    for c, s in (("codes", "sf"), ("r_codes", "r_sf")):
        got = dequant_nvfp4(torch.from_numpy(wq[c]), torch.from_numpy(wq[s]), g).numpy()
        ref = oracle.nvfp4_dequantize(wq[c], wq[s], wq["g"])
        assert np.array_equal(got.view(np.uint32), ref.view(np.uint32)), c


def _brute(e, ep, X, S, b):
    D = e.clone()
    KB = e.shape[1] // b
    for blk in S:
        nt, kt = divmod(blk, KB)
        D[nt * b:(nt + 1) * b, kt * b:(kt + 1) * b] = ep[nt * b:(nt + 1) * b, kt * b:(kt + 1) * b]
    return float(((X @ D.T) ** 2).sum())


def _case(seed=3, N=16, K=24, T=10, b=4):
    g = torch.Generator().manual_seed(seed)
    e = torch.randn(N, K, generator=g, dtype=torch.float64)
    ep = e * 0.3 + 0.05 * torch.randn(N, K, generator=g, dtype=torch.float64)
    X = torch.randn(T, K, generator=g, dtype=torch.float64)
    X[:, 5] *= 8.0  # a hot channel, as in the synthetic activations
    return e, ep, X, b


def test_incremental_distortion_equals_brute_force():
    e, ep, X, b = _case()
    m = Distortion(e, ep, X, block=b)
    nblk = m.NB * m.KB
    assert m.E0 == pytest.approx(_brute(e, ep, X, [], b), rel=1e-12)
    assert m.E_all == pytest.approx(_brute(e, ep, X, list(range(nblk)), b), rel=1e-12)
    rng = np.random.default_rng(5)
    for _ in range(3):
        order = [int(v) for v in rng.permutation(nblk)[:10]]
        Es = m.curve(order)
        for k in range(len(order) + 1):
            assert Es[k] == pytest.approx(_brute(e, ep, X, order[:k], b), rel=1e-10), k
    # every block taken: the incremental value meets E(all)
    assert m.curve(list(range(nblk)))[-1] == pytest.approx(m.E_all, rel=1e-10)


def test_greedy_takes_the_best_block_each_step():
    e, ep, X, b = _case(seed=9)
    m = Distortion(e, ep, X, block=b)
    order, Es = m.greedy(4)
    S = []
    for step in range(4):
        cand = [blk for blk in range(m.NB * m.KB) if blk not in S]
        vals = [_brute(e, ep, X, S + [blk], b) for blk in cand]
        best = cand[int(np.argmin(vals))]
        assert order[step] == best, step
        S.append(best)
        assert Es[step + 1] == pytest.approx(min(vals), rel=1e-10)


def test_diagonal_gains_match_a_diagonal_gram():
    """With X^T X replaced by its diagonal, dE_b at S = {} is sum over the block of
    G_kk (e'^2 - e^2): the form the Delta-score scales by -1/T."""
    e, ep, X, b = _case(seed=11)
    m = Distortion(e, ep, X, block=b)
    Gd = torch.diagonal(X.T @ X)
    want = []
    for blk in range(m.NB * m.KB):
        nt, kt = divmod(blk, m.KB)
        r, c = slice(nt * b, (nt + 1) * b), slice(kt * b, (kt + 1) * b)
        want.append(float(((ep[r, c] ** 2 - e[r, c] ** 2) * Gd[c].reshape(1, -1)).sum()))
    assert np.allclose(m.diagonal_gains().numpy(), np.array(want), rtol=1e-12, atol=0)


@pytest.mark.gpu
def test_study_tiny_layer():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    out = run("tiny", fracs=(0.10, 0.25, 0.5))
    # the CUDA path's Delta equals -dE(diagonal Gram)/T up to its fp32 tau rounding
    assert out["delta_vs_diagonal_max_rel"] < 1e-5
    for r in out["budgets"]:
        assert np.isfinite(r["E_delta"]) and np.isfinite(r["E_greedy"])
        assert r["E_greedy"] < out["E_none"] and r["E_delta"] < out["E_none"]
