"""Pins for the oracle's equivalent transform (SmoothQuant's per-channel rule, migration
strength 1/2; the MosaicQuant pages name the transform without defining it). CPU only.

The transform must leave the layer's product unchanged up to the two bf16 roundings:
X W^T = (X diag(s)^-1) (W diag(s))^T. It must also balance every input channel: after it,
the activation and weight maxima of channel k both equal sqrt(max|X_k| max|W_k|)."""
import numpy as np
import torch

import synth


def _bf16(x):
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(
        np.uint16)


def _f(bits):
    return synth.bf16_to_f32(bits).astype(np.float64)


def test_hand_worked_channels(orc):
    # channel 0: max|x| = 4, max|w| = 1 -> s = 2; channel 1: no activation -> s = 1;
    # channel 2: no weight -> s = 1; channel 3: equal maxima -> s = 1
    X = np.zeros((3, 64), np.float32)
    W = np.zeros((2, 64), np.float32)
    X[:, 0] = [1, -4, 2]
    W[:, 0] = [0.5, -1]
    W[:, 1] = [3, 1]
    X[:, 2] = [7, 0, 0]
    X[:, 3] = [0.25, -0.5, 0]
    W[:, 3] = [0.5, 0.125]
    s = orc.smooth_scales(_bf16(X), _bf16(W))
    assert s[0] == 2.0 and s[1] == 1.0 and s[2] == 1.0 and s[3] == 1.0
    assert np.all(s[4:] == 1.0)
    Wp = orc.smooth_apply(_bf16(W), s, invert=False)
    Xp = orc.smooth_apply(_bf16(X), s, invert=True)
    assert np.array_equal(_f(Wp)[:, 0], [1.0, -2.0]) and np.array_equal(_f(Xp)[:, 0], [0.5, -2.0, 1.0])


def test_product_unchanged_within_two_bf16_roundings(orc):
    L = synth.layer("tiny")
    X, W = L["X"], L["W"]            # outlier activation channels x30, outlier weights x20
    s = orc.smooth_scales(L["Xcal"], W)
    Xp = orc.smooth_apply(X, s, invert=True)
    Wp = orc.smooth_apply(W, s, invert=False)
    x, w, xp, wp = _f(X), _f(W), _f(Xp), _f(Wp)
    Y, Yp = x @ w.T, xp @ wp.T
    bound = np.abs(x) @ np.abs(w).T
    # each factor is rounded once to bf16 (relative error <= 2^-8, after an fp32 operation
    # with error <= 2^-24): |x'w' - xw| <= |xw| (2 (2^-8 + 2^-24) + (2^-8 + 2^-24)^2)
    u = 2.0 ** -8 + 2.0 ** -24
    assert np.all(np.abs(Yp - Y) <= (2 * u + u * u) * bound + 1e-30)
    # a transform applied the wrong way round is far outside that bound
    Wbad = orc.smooth_apply(W, s, invert=True)
    assert np.max(np.abs(xp @ _f(Wbad).T - Y) - (2 * u + u * u) * bound) > 0


def test_channels_balanced(orc):
    L = synth.layer("tiny")
    Xc, W = L["Xcal"], L["W"]
    s = orc.smooth_scales(Xc, W).astype(np.float64)
    ax, aw = np.abs(_f(Xc)).max(axis=0), np.abs(_f(W)).max(axis=0)
    assert np.allclose(s, np.sqrt(ax / aw), rtol=2 ** -23)
    target = np.sqrt(ax * aw)
    bx = np.abs(_f(orc.smooth_apply(Xc, s.astype(np.float32), invert=True))).max(axis=0)
    bw = np.abs(_f(orc.smooth_apply(W, s.astype(np.float32), invert=False))).max(axis=0)
    assert np.all(np.abs(bx - target) <= 2 ** -7 * target) and np.all(np.abs(bw - target) <= 2 ** -7 * target)
    # the hot activation channels (x30) give up most of their range to the weights
    hot = ax > 10 * np.median(ax)
    assert hot.any() and np.all(bx[hot] < ax[hot] / 3)


def test_power_of_two_scales_are_exact(orc):
    # when every ratio of maxima is a power of four, s is a power of two and the transform
    # only shifts exponents: the product is unchanged exactly
    rng = np.random.default_rng(5)
    K = 64
    e = rng.integers(-3, 4, size=K)
    W = (rng.integers(-8, 9, size=(32, K)) / 8.0).astype(np.float32)
    W[0, :] = 1.0
    X = (rng.integers(-8, 9, size=(16, K)) / 8.0).astype(np.float32) * (4.0 ** e)[None, :]
    X[0, :] = 4.0 ** e
    s = orc.smooth_scales(_bf16(X), _bf16(W))
    assert np.array_equal(s, (2.0 ** e).astype(np.float32))
    Xp = orc.smooth_apply(_bf16(X), s, invert=True)
    Wp = orc.smooth_apply(_bf16(W), s, invert=False)
    assert np.array_equal(_f(Xp) @ _f(Wp).T, _f(_bf16(X)) @ _f(_bf16(W)).T)
