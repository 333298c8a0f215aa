"""Pins of the oracle's FP8 E4M3 encoder/decoder (no GPU).

The encoder must give round-to-nearest-even with saturation to +-448 (the
"satfinite" convention the recipe uses for V and P).  It is pinned by the
format specification's reference points, by a brute-force nearest-even search
over the decoded code table, and by torch's float8_e4m3fn cast.
"""
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "e4m3_spec_points.txt")


def _spec_points():
    pts = []
    for line in open(GOLDEN):
        line = line.split("#")[0].strip()
        if line:
            c, v = line.split()
            pts.append((int(c, 16), float(v)))
    return pts


def test_decode_spec_points():
    for code, val in _spec_points():
        got = oracle.e4m3_decode([code])[0]
        if np.isnan(val):
            assert np.isnan(got)
        else:
            assert got == val and np.signbit(got) == np.signbit(val), hex(code)


def test_encode_spec_points():
    for code, val in _spec_points():
        if not np.isnan(val):
            assert oracle.e4m3_encode(np.array([val], np.float32))[0] == code


def _finite_table():
    codes = np.arange(256, dtype=np.uint8)
    vals = oracle.e4m3_decode(codes)
    keep = ~np.isnan(vals)
    return codes[keep], vals[keep]


def test_roundtrip_all_codes():
    codes, vals = _finite_table()
    back = oracle.e4m3_encode(vals.astype(np.float32))
    assert np.array_equal(back, codes)
    assert len(codes) == 254  # 256 minus the two NaN codes


def _brute_nearest_even(x):
    """Nearest representable by exhaustive search; ties to the even code."""
    codes, vals = _finite_table()
    pos = vals >= 0
    pc, pv = codes[pos & ~((vals == 0) & (codes == 0x80))], vals[pos & ~((vals == 0) & (codes == 0x80))]
    out = []
    for xi in x:
        a = min(abs(float(xi)), 448.0)
        dist = np.abs(pv - a)
        best = dist.min()
        cand = pc[dist == best]
        if len(cand) > 1:
            cand = [c for c in cand if (c & 1) == 0]
        c = int(cand[0])
        if np.signbit(xi):
            c |= 0x80
        out.append(c)
    return np.array(out, np.uint8)


def test_encoder_matches_brute_force_on_midpoints_and_random():
    codes, vals = _finite_table()
    pv = np.unique(vals[vals >= 0])
    mids = (pv[1:] + pv[:-1]) / 2
    xs = [mids, np.nextafter(mids.astype(np.float32), np.float32(0)),
          np.nextafter(mids.astype(np.float32), np.float32(1e9)),
          np.random.default_rng(7).uniform(0, 460, 3000),
          np.random.default_rng(8).uniform(0, 0.02, 3000),
          [448.0, 449.0, 464.0, 470.0, 1e6, 3e38, 2.0 ** -10, 2.0 ** -11, 1e-30]]
    x = np.concatenate([np.asarray(a, np.float64) for a in xs]).astype(np.float32)
    x = np.concatenate([x, -x])
    assert np.array_equal(oracle.e4m3_encode(x), _brute_nearest_even(x))


def test_encoder_matches_torch_cast_in_range():
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.standard_normal(200000).astype(np.float32) * 50,
                        rng.uniform(-448, 448, 200000).astype(np.float32),
                        (rng.standard_normal(20000) * 1e-3).astype(np.float32)])
    ours = oracle.e4m3_encode(x)
    theirs = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, theirs)


def test_saturation_and_nan():
    x = np.array([448.0, 460.0, 500.0, 1e30, np.inf, -np.inf, np.nan], np.float32)
    got = oracle.e4m3_encode(x)
    assert list(got[:4]) == [0x7E] * 4
    assert got[4] == 0x7E and got[5] == 0xFE
    assert got[6] & 0x7F == 0x7F
