"""Pins for the oracle's Delta-score, top-K, pack and GEMM (CPU only).

The Delta-score is tied to the quantity it is defined to reduce: the diagonal-Hessian
output-distortion proxy E(S) = sum_k H_k sum_n (W - deq Q - [sel] deq R)^2 must fall by
exactly sum_{b in S} Delta_b. Top-K is checked by brute force over every subset; the
GEMM against a library matmul of independently dequantized operands and against the
plain matmul of the inputs in the lossless case.
"""
import itertools

import numpy as np
import pytest
import torch

import synth
from test_oracle_formats import E2M1_GRID, _decode_independent, e4m3_table, make_lossless_weight


def _bf16(x):
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(
        np.uint16)


def _f32(bits):
    return synth.bf16_to_f32(bits)


@pytest.fixture(scope="module")
def tiny(orc):
    L = synth.layer("tiny")
    out = orc.run_path(L["W"], L["X"], L["Xcal"], synth.budget_blocks(L["N"], L["K"], 0.10))
    out.update(L)
    return out


def _errors(W, wq):
    """e = fp32(W - deq Q), e' = fp32(e - deq R), from an independent dequantizer."""
    dq = _decode_independent(wq["codes"], wq["sf"], wq["g"])
    dr = _decode_independent(wq["r_codes"], wq["r_sf"], wq["g"])
    e = (_f32(W) - dq).astype(np.float32)
    e2 = (e - dr).astype(np.float32)
    return e, e2


def _distortion(H, e, e2, mask_elem):
    err = np.where(mask_elem, e2.astype(np.float64), e.astype(np.float64))
    return float(np.sum(H.astype(np.float64)[None, :] * err * err))


def _elem_mask(sel, N, K):
    bm = np.zeros((N // 64) * (K // 64), bool)
    bm[np.asarray(sel, dtype=np.int64)] = True
    return np.repeat(np.repeat(bm.reshape(N // 64, K // 64), 64, 0), 64, 1)


def test_tiny_budget_is_three_blocks():
    assert synth.budget_blocks(256, 512, 0.10) == 3
    assert synth.budget_blocks(4096, 4096, 0.10) == 409
    assert synth.budget_blocks(28672, 8192, 0.20) == 11468


def test_hessian_diag_against_numpy(orc):
    X = synth.act(100, 256, 5, 6, 3)
    H = orc.hessian_diag(X)
    x = _f32(X).astype(np.float64)
    ref = (np.sum(x * x, axis=0) / 100).astype(np.float32)
    assert np.all(np.abs(H.view(np.int32) - ref.view(np.int32)) <= 1)  # summation order: <= 1 ulp
    c = np.full((7, 64), 1.5, np.float32)
    assert np.all(orc.hessian_diag(_bf16(c)) == np.float32(2.25))


def test_hessian_diag_exact_when_no_rounding(orc):
    """Values of one binade ([1, 2), bf16): every square has at most 16 significant bits
    and every partial sum of up to 1024 of them fits in fp64 exactly, so whatever the
    summation order H_k must equal the exact mean rounded once to fp32 (Fractions)."""
    from fractions import Fraction
    rng = np.random.default_rng(7)
    for T in (1, 3, 100, 513, 1024):
        x = (1.0 + rng.integers(0, 128, size=(T, 64)) / 128.0).astype(np.float32)  # exact in bf16
        H = orc.hessian_diag(_bf16(x))
        for k in range(0, 64, 7):
            exact = sum(Fraction(float(v)) ** 2 for v in x[:, k]) / T
            # fp32(fp64(exact)): fp64 rounding of the exact mean, then to fp32 (the oracle's
            # division is the only rounding step here, in fp64, then the cast)
            assert H[k] == np.float32(float(exact)), (T, k)


def test_residual_is_base_error_and_shares_scale(orc, tiny):
    wq = tiny["wq"]
    w = _f32(tiny["W"])
    dq = _decode_independent(wq["codes"], wq["sf"], wq["g"])
    R = (w - dq).astype(np.float32)
    ref = orc.nvfp4_quantize(R, wq["g"])
    assert np.array_equal(ref["codes"], wq["r_codes"]) and np.array_equal(ref["sf"], wq["r_sf"])
    # the residual never increases any element's error: |e'| <= |e|
    e, e2 = _errors(tiny["W"], wq)
    assert np.all(np.abs(e2) <= np.abs(e) * (1 + 2 ** -22) + 1e-30)


def test_delta_nonnegative_and_distortion_identity(orc, tiny):
    N, K = tiny["N"], tiny["K"]
    H, delta, wq = tiny["H"], tiny["delta"], tiny["wq"]
    e, e2 = _errors(tiny["W"], wq)
    E0 = _distortion(H, e, e2, np.zeros((N, K), bool))
    # the squares are exact and every sum is fp64 (relative rounding 2^-53 per add), so
    # the identities below hold to ~1e-13 of the magnitudes involved; an fp32 tau or an
    # fp32 row tree (2^-24 per operation) misses these bounds by five orders of magnitude
    assert np.all(delta >= -1e-13 * E0)
    # E(S) = E(empty) - sum_{b in S} Delta_b for arbitrary S
    rng = np.random.default_rng(0)
    flat = delta.reshape(-1)
    for size in (1, 3, 7, flat.size):
        S = rng.choice(flat.size, size=size, replace=False)
        ES = _distortion(H, e, e2, _elem_mask(S, N, K))
        assert abs((E0 - ES) - flat[S].sum()) <= 1e-12 * E0
    # each block's Delta, written out element by element in fp64 (only the summation
    # order differs: bound by 1e-12 of the block's sum of H (e^2 + e'^2))
    worst = 0.0
    for b in range(flat.size):
        nt, kt = divmod(b, K // 64)
        sl = (slice(nt * 64, nt * 64 + 64), slice(kt * 64, kt * 64 + 64))
        h = H[kt * 64:kt * 64 + 64].astype(np.float64)[None, :]
        e64, e264 = e[sl].astype(np.float64), e2[sl].astype(np.float64)
        ref = np.sum(h * (e64 ** 2 - e264 ** 2))
        scale = np.sum(h * (e64 ** 2 + e264 ** 2))
        worst = max(worst, abs(ref - flat[b]) / (scale + 1e-300))
    assert worst <= 1e-12, worst


def test_outlier_blocks_score_highest(orc, tiny):
    """With uniform channel sensitivity (H = 1) the planted outlier blocks carry the
    concentrated error and rank first by a wide margin; with the calibration H, a block
    holding a hot activation channel can overtake one of them (the Hessian weighting)."""
    W = _f32(tiny["W"])
    N, K = tiny["N"], tiny["K"]
    big = (np.abs(W) > 0.2).reshape(N // 64, 64, K // 64, 64).any(axis=(1, 3)).reshape(-1)
    planted = set(np.flatnonzero(big).tolist())
    assert len(planted) == 3
    d1 = orc.delta_score(tiny["W"], np.ones(K, np.float32), tiny["wq"]).reshape(-1)
    order = np.argsort(-d1, kind="stable")
    assert set(order[:3].tolist()) == planted
    assert d1[order[2]] > 5 * d1[order[3]]
    hot_blocks = {int(k) // 64 for k in np.flatnonzero(tiny["H"] > 100)}
    assert set(tiny["sel"].tolist()) <= planted | {nt * (K // 64) + kt for nt in range(N // 64) for kt in hot_blocks}


def test_topk_brute_force_subsets(orc):
    rng = np.random.default_rng(2)
    for trial in range(40):
        B = 16
        d = rng.integers(0, 6, size=B).astype(np.float64) * (0.5 if trial % 2 else 1e-3)
        if trial % 5 == 0:
            d[:] = 0.0
        for k in (0, 1, 3, 4):
            rank, sel = orc.topk(d, k)
            best = None
            for S in itertools.combinations(range(B), k):  # lexicographic order
                s = sum(d[list(S)])
                if best is None or s > best[0]:
                    best = (s, S)
            assert tuple(sel.tolist()) == best[1]
            assert sorted(rank.tolist()) == sel.tolist()
            # rank order: Delta non-increasing, ties by ascending block index
            for a, b in zip(rank[:-1], rank[1:]):
                assert d[a] > d[b] or (d[a] == d[b] and a < b)


def test_larger_budget_never_raises_distortion(orc, tiny):
    N, K = tiny["N"], tiny["K"]
    e, e2 = _errors(tiny["W"], tiny["wq"])
    prev = None
    for k in range(0, (N // 64) * (K // 64) + 1, 3):
        _, sel = orc.topk(tiny["delta"], k)
        E = _distortion(tiny["H"], e, e2, _elem_mask(sel, N, K))
        assert prev is None or E <= prev * (1 + 1e-9)
        prev = E


def test_pack_round_trip(orc, tiny):
    N, K = tiny["N"], tiny["K"]
    wq, sel, p = tiny["wq"], tiny["sel"], tiny["packed"]
    KB = K // 64
    assert p["tile_ptr"][-1] == sel.size
    assert sum(bin(int(w)).count("1") for w in p["bitmap"].reshape(-1)) == sel.size
    for i, b in enumerate(sel):
        nt, kt = divmod(int(b), KB)
        assert p["blk_kt"][i] == kt
        assert p["tile_ptr"][nt] <= i < p["tile_ptr"][nt + 1]
        assert (p["bitmap"][nt, kt // 32] >> (kt % 32)) & 1
        blk = p["blk_codes"][i]
        for r in range(64):
            for j in range(32):
                off = (r // 8) * 256 + (j // 16) * 128 + (r % 8) * 16 + (j % 16)
                assert blk[off] == wq["r_codes"][nt * 64 + r, kt * 32 + j]
        sfc = p["blk_sf"][i]
        seen = np.zeros(512, bool)
        for r in range(64):
            t = 64 * (nt % 2) + r
            for q in range(4):
                off = (t % 32) * 16 + (t // 32) * 4 + q
                seen[off] = True
                assert sfc[off] == wq["r_sf"][nt * 64 + r, kt * 4 + q]
        assert not sfc[~seen].any()


def _gemm_numpy(xq, wq, sel, N, K, mode=0):
    """Library matmul of independently dequantized operands (fp64)."""
    t = e4m3_table()

    def deq_nog(codes, sf):
        lo, hi = codes & 15, codes >> 4
        c = np.stack([lo, hi], axis=-1).reshape(codes.shape[0], -1)
        mag = np.array(E2M1_GRID)[c & 7] * np.where(c & 8, -1.0, 1.0)
        return mag * np.repeat(t[sf], 16, axis=1)

    xh = deq_nog(xq["codes"], xq["sf"]) * xq["g"].astype(np.float64)[:, None]
    wh = np.zeros((N, K))
    if mode != 2:
        wh += deq_nog(wq["codes"], wq["sf"])
    if mode != 1 and sel is not None and len(sel):
        wh += np.where(_elem_mask(sel, N, K), deq_nog(wq["r_codes"], wq["r_sf"]), 0.0)
    return xh @ (wh * np.float64(wq["g"])).T


def test_gemm_matches_library_matmul(orc, tiny):
    N, K, M = tiny["N"], tiny["K"], tiny["M"]
    ref = _gemm_numpy(tiny["xq"], tiny["wq"], tiny["sel"], N, K)
    assert np.allclose(tiny["y"], ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    y1, _ = orc.gemm_rows(tiny["xq"], tiny["wq"], tiny["sel"], M, N, K, 1)
    assert np.allclose(y1, _gemm_numpy(tiny["xq"], tiny["wq"], None, N, K, 1), rtol=1e-12,
                       atol=1e-12 * np.abs(ref).max())
    rows = np.array([3, 0, 15], np.int32)
    ys, _ = orc.gemm_rows(tiny["xq"], tiny["wq"], tiny["sel"], M, N, K, 0, rows)
    assert np.array_equal(ys, tiny["y"][rows])


def test_gemm_budget_zero_and_linearity(orc, tiny):
    N, K, M = tiny["N"], tiny["K"], tiny["M"]
    y_none, _ = orc.gemm_rows(tiny["xq"], tiny["wq"], np.zeros(0, np.int32), M, N, K, 0)
    y_base, _ = orc.gemm_rows(tiny["xq"], tiny["wq"], tiny["sel"], M, N, K, 1)
    y_res, _ = orc.gemm_rows(tiny["xq"], tiny["wq"], tiny["sel"], M, N, K, 2)
    assert np.array_equal(y_none, y_base)  # budget 0 is the dense base, bit for bit
    assert np.allclose(tiny["y"], y_base + y_res, rtol=1e-12, atol=1e-13 * np.abs(tiny["y"]).max())
    assert np.abs(y_res).max() > 0


def test_lossless_path_is_plain_matmul(orc):
    rng = np.random.default_rng(4)
    N, K, M = 128, 256, 8
    Wb, w = make_lossless_weight(N, K, -10, rng)
    Xb, x = make_lossless_weight(M, K, -3, rng, per_row=True)
    r = orc.run_path(Wb, Xb, Xb, 3)
    assert not r["delta"].any()
    assert r["sel"].tolist() == [0, 1, 2]  # all Delta tie at 0: lowest block indices
    ref = x @ w.T
    assert np.allclose(r["y"], ref, rtol=1e-13, atol=1e-13 * np.abs(ref).max())


def test_synth_outliers_confined_to_blocks():
    W = synth.weight(256, 512, 1, 4, 0.02, 655, 3, 20.0)
    w = _f32(W)
    blocks = (np.abs(w) > 0.2).reshape(4, 64, 8, 64).any(axis=(1, 3))
    assert blocks.sum() == 3
    assert np.sum(np.abs(w) > 0.2) > 400
    assert np.array_equal(W, synth.weight(256, 512, 1, 4, 0.02, 655, 3, 20.0))
