"""Pins of the recipe's software exp2 (no GPU).

The oracle evaluates the exponentials of a fixed share of every KV tile's
columns with a software exp2 (a Cody-Waite style reduction to |f| <= 1/2,
a degree-3 polynomial fitted here for 2^f, and 2^j added to the exponent
field), exactly as the device does for those columns, so that both sides
agree bit for bit there.  Pinned here:

* against the mathematical exp2 (numpy, fp64): relative error at most
  2^-13.6 over the whole argument range the softmax produces, [-125, 9]
  (the fitted polynomial's minimax error with its fp32 evaluation is
  2^-13.7), dense grid plus every fp32 value of one binade;
* at integer arguments k the result is exactly 2^k times the polynomial's
  constant term (f = 0), and below -125 it saturates at 2^-125 p(0);
* in the attention, switching the polynomial on for some columns moves O by
  no more than the rounding slack computed with the polynomial's relative
  error (the slack itself is pinned in test_oracle_slack.py), and columns
  outside the share are untouched (all-off equals the default recipe).
"""
import numpy as np
import pytest

import oracle
from bit_quantized_attention_sage_b200 import synth

C0 = np.uint32(0x3F7FFB49).view(np.float32)  # the polynomial's constant term
POLY_REL = 2.0 ** -13.6


def test_relative_error_over_the_softmax_range():
    rng = np.random.default_rng(5)
    grid = np.concatenate([
        np.linspace(-125.0, 9.0, 4_000_001, dtype=np.float32),
        rng.uniform(-125.0, 9.0, 2_000_000).astype(np.float32),
        # every fp32 value in [1, 2) (one binade of f after the reduction)
        (np.arange(1 << 23, dtype=np.uint32) | np.uint32(0x3F800000)).view(np.float32),
    ])
    y = oracle.exp2_poly(grid).astype(np.float64)
    rel = np.abs(y / np.exp2(grid.astype(np.float64)) - 1.0)
    assert rel.max() <= POLY_REL, rel.max()


def test_integer_arguments_and_saturation():
    k = np.arange(-125, 10, dtype=np.float32)
    y = oracle.exp2_poly(k).astype(np.float64)
    assert np.array_equal(y, np.ldexp(float(C0), k.astype(np.int64)))
    low = oracle.exp2_poly(np.array([-125.0, -126.0, -1e30, -np.inf], np.float32))
    assert (low == np.float32(np.ldexp(float(C0), -125))).all()


def _head(nq, nkv, D, seed, off=4.0, mag=0.0):
    w = synth.Workload("t", 1, 1, nq, nkv, D, k_offset_var=off, outlier_mag=mag, seed=seed)
    return oracle.quant_head(*synth.head(w, 0, 0))


@pytest.mark.parametrize("first", [0, 64, 96, 112])
@pytest.mark.parametrize("mask,mb", [(oracle.MASK_NONE, 0), (oracle.MASK_BLOCK_CAUSAL, 100)])
def test_polynomial_columns_within_their_slack(first, mask, mb):
    qh = _head(90, 333, 64, 61)
    rows = np.arange(90)
    with oracle.exp2_poly_columns(128):
        o0, s0, l0 = oracle.attn_rows(qh, rows, mask, mb, eps=POLY_REL + 2.0 ** -24)
    with oracle.exp2_poly_columns(first):
        o1, _, l1 = oracle.attn_rows(qh, rows, mask, mb)
    r = np.exp(l0 - l1)[:, None]  # l0 / l1 (m is the same)
    bound = s0 * r + np.abs(o0) * np.abs(r - 1.0) + 1e-12
    assert (np.abs(o1 - o0) <= bound).all()
    assert np.abs(l1 - l0).max() < 1e-4


def test_no_polynomial_columns_is_the_exp2_recipe():
    qh = _head(64, 200, 128, 62)
    rows = np.arange(64)
    with oracle.exp2_poly_columns(128):
        a = oracle.attn_rows(qh, rows)
    with oracle.exp2_poly_columns(1000):
        b = oracle.attn_rows(qh, rows)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)
