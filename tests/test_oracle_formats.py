"""Pins for the oracle's number formats and NVFP4 quantization (CPU only).

Each check compares the oracle against something other than itself: hand-derived
fixtures in tests/golden, a brute-force nearest-value search over grids built from
the bit layouts, torch's float8 conversion, closed-form error bounds, and the
lossless special case.
"""
import math
import os

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")

# E2M1 grid as the NVFP4 format states it (value of codes 0..7).
E2M1_GRID = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                yield line.split()


def e4m3_table():
    """All 256 E4M3 byte values decoded by torch (NaN for 0x7F/0xFF)."""
    b = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn)
    return b.to(torch.float64).numpy()


def brute_e2m1(v: float) -> int:
    """Nearest grid value, ties to the even code, clamp to 6, sign kept."""
    a = abs(v)
    best = None
    for c, g in enumerate(E2M1_GRID):
        d = abs(a - g)
        if best is None or d < best[0] or (d == best[0] and c % 2 == 0):
            best = (d, c)
    c = best[1]
    return c | (8 if math.copysign(1.0, v) < 0 else 0)


def brute_e4m3(v: float, table) -> int:
    a = abs(v)
    best = None
    for c in range(0x7F):  # 0x00..0x7E: the non-negative finite values
        d = abs(a - table[c])
        if best is None or d < best[0] or (d == best[0] and c % 2 == 0):
            best = (d, c)
    c = best[1]
    return c | (0x80 if math.copysign(1.0, v) < 0 else 0)


def test_e2m1_grid_round_trip(orc):
    for c in range(16):
        v = orc.e2m1_value(c)
        expect = E2M1_GRID[c & 7] * (-1 if c & 8 else 1)
        assert v == expect
        # every grid value encodes to itself (including -0 -> 0x8)
        assert orc.e2m1_encode(np.float32(math.copysign(E2M1_GRID[c & 7], -1 if c & 8 else 1))) == c


def test_e2m1_golden_ties(orc):
    for v, code in _rows("e2m1_ties.txt"):
        assert orc.e2m1_encode(np.float32(float(v))) == int(code, 16), v


def test_e2m1_brute_force_sweep(orc):
    vals = set()
    for i in range(-8 * 256, 8 * 256 + 1):
        x = i / 256.0
        vals.update({x, float(np.nextafter(np.float32(x), np.float32(np.inf))),
                     float(np.nextafter(np.float32(x), np.float32(-np.inf)))})
    rng = np.random.default_rng(5)
    vals.update(rng.normal(0, 4, 2000).astype(np.float32).tolist())
    for v in vals:
        v = float(np.float32(v))
        assert orc.e2m1_encode(np.float32(v)) == brute_e2m1(v), v


def test_e4m3_decode_matches_torch(orc):
    t = e4m3_table()
    for c in range(256):
        if c in (0x7F, 0xFF):
            continue
        assert orc.e4m3_value(c) == t[c], hex(c)


def test_e4m3_golden_points(orc):
    for v, code in _rows("e4m3_points.txt"):
        assert orc.e4m3_encode(np.float32(float(v))) == int(code, 16), v


def test_e4m3_encode_round_trip_every_finite_value(orc):
    t = e4m3_table()
    for c in range(0x7F):
        assert orc.e4m3_encode(np.float32(t[c])) == c
        assert orc.e4m3_encode(np.float32(-t[c])) == (c | 0x80)


def test_e4m3_encode_vs_torch_and_brute_force(orc):
    t = e4m3_table()
    rng = np.random.default_rng(7)
    # log-uniform over [2^-12, 463] plus every midpoint between neighbours
    xs = list(np.exp2(rng.uniform(-12, math.log2(463), 3000)).astype(np.float32))
    fin = [t[c] for c in range(0x7F)]
    for a, b in zip(fin[:-1], fin[1:]):
        m = (a + b) / 2
        xs += [np.float32(m), np.nextafter(np.float32(m), np.float32(0)), np.nextafter(np.float32(m), np.float32(1e9))]
    xs = np.array(xs, dtype=np.float32)
    ref = torch.from_numpy(xs).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    for x, r in zip(xs, ref):
        got = orc.e4m3_encode(x)
        assert got == r, (float(x), hex(got), hex(r))
    for x in xs[::7]:
        assert orc.e4m3_encode(x) == brute_e4m3(float(x), t)
    # saturation beyond torch's finite range: clamp to 448, never NaN
    for x in (464.0, 500.0, 1e6, 3.0e38):
        assert orc.e4m3_encode(np.float32(x)) == 0x7E


def test_nvfp4_group_worked_example(orc):
    rows = {r[0]: r[1:] for r in _rows("nvfp4_group_example.txt")}
    g = np.float32(float(rows["g"][0]))
    a = np.array([float(v) for v in rows["a"]], np.float32)[None, :]
    q = orc.nvfp4_quantize(a, g)
    assert q["sf"][0, 0] == int(rows["sf"][0], 16)
    assert list(q["codes"][0]) == [int(v, 16) for v in rows["packed"]]
    unpacked = [(b >> (4 * (i % 2))) & 15 for i, b in enumerate(np.repeat(q["codes"][0], 2))]
    assert unpacked == [int(v, 16) for v in rows["codes"]]
    assert np.array_equal(q["deq"][0], np.array([float(v) for v in rows["deq"]], np.float32))


def _decode_independent(codes, sf, g):
    """Dequantize with the grid table and torch's E4M3 decode (not the oracle's)."""
    t = e4m3_table()
    lo = codes & 15
    hi = codes >> 4
    c = np.stack([lo, hi], axis=-1).reshape(codes.shape[0], -1)
    mag = np.array(E2M1_GRID)[c & 7] * np.where(c & 8, -1.0, 1.0)
    d = (t[sf].astype(np.float32) * np.float32(g)).astype(np.float32)
    return (mag.astype(np.float32) * np.repeat(d, 16, axis=1)).astype(np.float32)


def test_nvfp4_error_bound_and_scale_rule(orc):
    rng = np.random.default_rng(11)
    a = (rng.standard_normal((64, 256)) * np.exp2(rng.integers(-3, 4, (64, 1)))).astype(np.float32)
    a[3, 17] = 40.0
    g = orc.global_scale(a)
    assert g == np.float32(np.abs(a).max() / np.float32(2688.0))
    q = orc.nvfp4_quantize(a, g)
    t = e4m3_table()
    deq = _decode_independent(q["codes"], q["sf"], g)
    assert np.array_equal(deq, q["deq"])
    amax = np.abs(a.reshape(64, 16, 16)).max(-1)
    s_raw = (amax / np.float32(np.float32(6.0) * g)).astype(np.float32)
    sf_ref = torch.from_numpy(s_raw).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(q["sf"], sf_ref)
    d = np.repeat((t[q["sf"]].astype(np.float32) * g).astype(np.float32), 16, axis=1)
    normal = np.repeat(s_raw >= 2.0 ** -6, 16, axis=1)
    err = np.abs(a - deq)
    # nearest grid point: error <= half the widest gap (2) in units of d; the E4M3
    # rounding of the scale (<= 1/16 relative) keeps a saturated value within 0.375 d
    assert np.all(err[normal] <= d[normal] * (1 + 1e-6))


def test_nvfp4_zero_and_tiny_groups(orc):
    a = np.zeros((1, 32), np.float32)
    a[0, 16:] = -0.0
    q = orc.nvfp4_quantize(a, np.float32(1.0))
    assert q["sf"].tolist() == [[0, 0]]
    assert q["codes"][0, :8].tolist() == [0] * 8
    assert q["codes"][0, 8:].tolist() == [0x88] * 8  # signed zeros keep their sign
    assert orc.global_scale(a) == 1.0


def make_lossless_weight(N, K, p, rng, per_row=False):
    """A matrix whose every 16-group is E2M1 grid values times one E4M3 scale times 2^p,
    each group holding a +-6, and the tensor max 6 * 448 * 2^p, so that g = 2^p exactly
    and the quantization loses nothing."""
    t = e4m3_table()
    normal_codes = np.arange(0x08, 0x7F)  # positive normal E4M3 values
    G = K // 16
    sd = t[rng.choice(normal_codes, size=(N, G))]
    sd[0, 0] = 448.0
    if per_row:  # per-token scales: every row needs its own 6 * 448 * 2^p maximum
        sd[:, 0] = 448.0
    codes = rng.integers(0, 16, size=(N, K))
    codes.reshape(N, G, 16)[:, :, 0] = rng.choice([7, 15], size=(N, G))  # one +-6 per group
    mag = np.array(E2M1_GRID)[codes & 7] * np.where(codes & 8, -1.0, 1.0)
    w = mag * np.repeat(sd, 16, axis=1) * 2.0 ** p
    wb = torch.from_numpy(w).to(torch.bfloat16)
    assert torch.equal(wb.to(torch.float64), torch.from_numpy(w))  # exactly representable
    return wb.view(torch.int16).numpy().view(np.uint16), w


def test_lossless_weight_quantization(orc):
    rng = np.random.default_rng(3)
    Wb, w = make_lossless_weight(128, 256, -10, rng)
    q = orc.quantize_weight(Wb)
    assert q["g"] == np.float32(2.0 ** -10)
    deq = _decode_independent(q["codes"], q["sf"], q["g"])
    assert np.array_equal(deq.astype(np.float64), w)
    assert not q["r_codes"].any() and not q["r_sf"].any()  # residual is exactly zero


def test_quantize_act_per_token_scale(orc):
    rng = np.random.default_rng(9)
    x = rng.standard_normal((5, 128)).astype(np.float32)
    x[2] = 0.0
    xb = torch.from_numpy(x).to(torch.bfloat16)
    X = xb.view(torch.int16).numpy().view(np.uint16)
    xf = xb.to(torch.float32).numpy()
    q = orc.quantize_act(X)
    for m in range(5):
        amax = np.abs(xf[m]).max()
        assert q["g"][m] == (np.float32(1.0) if amax == 0 else np.float32(amax / np.float32(2688.0)))
        ref = orc.nvfp4_quantize(xf[m:m + 1], q["g"][m])
        assert np.array_equal(ref["codes"][0], q["codes"][m]) and np.array_equal(ref["sf"][0], q["sf"][m])


def test_sf_tile_independent_unswizzle(orc):
    rng = np.random.default_rng(1)
    for rows, cols in ((300, 512), (16, 256), (128, 64)):
        sf = rng.integers(1, 255, size=(rows, cols // 16)).astype(np.uint8)
        tiled = orc.sf_tile(sf, rows, cols)
        KS = cols // 64
        rt = (rows + 127) // 128
        assert tiled.size == rt * 128 * (cols // 16)
        back = np.zeros((rt * 128, cols // 16), np.uint8)
        for off in range(tiled.size):
            chunk, o = divmod(off, 512)
            r = (chunk // KS) * 128 + (o // 16) + 32 * ((o % 16) // 4)
            q = (chunk % KS) * 4 + o % 4
            back[r, q] = tiled[off]
        assert np.array_equal(back[:rows], sf)
        assert not back[rows:].any()
