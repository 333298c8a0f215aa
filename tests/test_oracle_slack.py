"""Pins of the oracle's quantized-mode arithmetic and of its rounding slack
(no GPU).

The slack is the part of the O tolerance that covers e4m3 rounding decisions
of y = 2^8 p which the device and the oracle may take differently, because
the device's exp2 differs from the oracle's by a small relative error.  It is
pinned here against what it claims to bound, with the oracle's exp2 result
perturbed (a test hook) by exactly such relative errors:

* any perturbation of every exp2 result by at most the stated relative
  uncertainty moves O by no more than the slack (plus the change of l, read
  from lse);
* the slack is attained: perturbing every element towards its larger or
  smaller admissible code, chosen per output channel by the sign of V, spans
  exactly the slack.

The quantized path itself is pinned against plain fp64 attention over the
dequantized operands (q8 * sq, k8 * sk, decoded v8 * sv), where the only
remaining difference is the e4m3 rounding of P: per output within the
rigorous bound sum_j (y_j / 16 + 2^-10) |v_j| / l, and lse (which P's
rounding does not enter) to 1e-5.

Each planted mistake (compiled into a separate copy of the oracle, see
sage_oracle.c) fails at least one of these pins, and the other admissible
reading of the 2^8 P scale (applied after exp2 instead of folded into its
argument) agrees with the adopted one within the slack.
"""
import math

import numpy as np
import pytest

import oracle
from bit_quantized_attention_sage_b200 import synth


def _bits(nq, nkv, D, seed, off=4.0, mag=0.0):
    w = synth.Workload("t", 1, 1, nq, nkv, D, k_offset_var=off, outlier_mag=mag, seed=seed)
    return synth.head(w, 0, 0)


def _visible(nq, nkv, mask, mb):
    g = np.arange(nq)[:, None] + (nkv - nq)
    j = np.arange(nkv)[None, :]
    if mask == oracle.MASK_CAUSAL:
        return j <= g
    if mask == oracle.MASK_BLOCK_CAUSAL:
        return (j // mb) <= (g // mb)
    return np.ones((nq, nkv), bool)


# small cases: several KV tiles and a ragged tail, every mask
CASES = [
    # nq, nkv, D, mask, mb, seed, k offset variance, outlier magnitude
    (96, 300, 64, oracle.MASK_NONE, 0, 31, 4.0, 0.0),
    (128, 400, 128, oracle.MASK_CAUSAL, 0, 32, 4.0, 0.0),
    (80, 333, 64, oracle.MASK_BLOCK_CAUSAL, 100, 33, 0.0, 20.0),
]


def _quant(case):
    nq, nkv, D, mask, mb, seed, off, mag = case
    q, k, v = _bits(nq, nkv, D, seed, off=off, mag=mag)
    return q, k, v, oracle.quant_head(q, k, v)


def _l_ratio(lse_a, lse_b):
    """l_a / l_b from the natural-log lse of the same rows (m does not move
    under exp2 perturbations, so lse differences are log l differences)."""
    return np.exp(lse_a - lse_b)[:, None]


# ------------------------------------------------------------------ checks
# Each returns (ok, detail); the tests assert ok, the planted-mistake test
# asserts that some check fails.

# The slack is computed the same way for any relative uncertainty eps; a
# large one (2^-10) makes about one element in fifty straddle a rounding
# boundary, so the pins below exercise many of them (with the device's eps,
# about 2^-21, a small case has almost none).
E_WIDE = 2.0 ** -10


def check_perturbations_within_slack(case, eps=E_WIDE, seed=0):
    _, _, _, qh = _quant(case)
    nq, nkv, D, mask, mb = case[:5]
    rows = np.arange(nq)
    o, slack, lse = oracle.attn_rows(qh, rows, mask, mb, eps=eps)
    rng = np.random.default_rng(seed)
    worst = 0.0
    moved = 0
    for _ in range(3):
        pert = rng.integers(-1, 2, size=(nq, nkv)).astype(np.int8)
        op, _, lsep = oracle.attn_rows(qh, rows, mask, mb, pert=pert, pert_eps=eps)
        r = _l_ratio(lse, lsep)  # l / l_perturbed
        bound = slack * r + np.abs(o) * np.abs(r - 1.0) + 1e-12
        worst = max(worst, float((np.abs(op - o) - bound).max()))
        moved += int((np.abs(op * _l_ratio(lsep, lse) - o) > 1e-12).sum())
    return worst <= 0.0, "worst excess over the slack %.3g (%d outputs moved)" % (worst, moved)


def check_slack_is_attained(case, E=E_WIDE):
    """Per output channel d, perturb every visible element by +E or -E
    (towards the larger or the smaller admissible code, by the sign of its V
    value): the two results span the slack computed with eps = E."""
    _, _, _, qh = _quant(case)
    nq, nkv, D, mask, mb = case[:5]
    rows = np.arange(nq)
    o, slack, lse = oracle.attn_rows(qh, rows, mask, mb, eps=E)
    if (slack > 0).sum() < 50:
        return False, "too few straddling elements to pin the slack"
    vis = _visible(nq, nkv, mask, mb)
    vsign = np.sign(oracle.e4m3_decode(qh["v8"]))  # [nkv, D]
    worst = 0.0
    for d in range(0, D, 7):
        up = np.where(vis, vsign[None, :, d], 0).astype(np.int8)
        oup, _, lup = oracle.attn_rows(qh, rows, mask, mb, pert=up, pert_eps=E)
        odn, _, ldn = oracle.attn_rows(qh, rows, mask, mb, pert=-up, pert_eps=E)
        # unnormalized sums in the units of the unperturbed l
        span = oup[:, d] * _l_ratio(lup, lse)[:, 0] - odn[:, d] * _l_ratio(ldn, lse)[:, 0]
        err = np.abs(span - slack[:, d])
        worst = max(worst, float((err - 1e-9 * (1.0 + slack[:, d])).max()))
    return worst <= 0.0, "worst |span - slack| excess %.3g" % worst


def _dequantized_reference(qh, nq, nkv, D, mask, mb):
    """Plain fp64 softmax attention over the dequantized operands; also the
    per-output bound of the e4m3 rounding of P and the lse."""
    qd = qh["q8"][:nq].astype(np.float64) * np.repeat(qh["qs"], 64)[:nq, None]
    kd = qh["k8"][:nkv].astype(np.float64) * np.repeat(qh["ks"], 64)[:nkv, None]
    vd = oracle.e4m3_decode(qh["v8"]) * qh["vs"][None, :].astype(np.float64)
    t = (qd @ kd.T) * (math.log2(math.e) / math.sqrt(D))  # log2 domain
    t = np.where(_visible(nq, nkv, mask, mb), t, -np.inf)
    mf = t.max(axis=1, keepdims=True)
    y = 256.0 * np.exp2(t - mf)  # y in the units of the final row maximum
    l = y.sum(axis=1, keepdims=True)
    o = (y @ vd) / l
    # |e4m3(y) - y| <= y / 16 for normal codes, 2^-10 below 2^-6; in the final
    # units every earlier tile's error only shrinks (factor 2^(m_k - m) <= 1)
    err = np.where(y > 0.0, y / 16.0 + 2.0 ** -10, 0.0)
    bound = (err @ np.abs(vd)) / l
    lse = (mf[:, 0] + np.log2(l[:, 0]) - 8.0) * math.log(2.0)
    return o, bound, lse


def check_dequantized_fp64(case):
    _, _, _, qh = _quant(case)
    nq, nkv, D, mask, mb = case[:5]
    rows = np.arange(nq)
    o, _, lse = oracle.attn_rows(qh, rows, mask, mb)
    ref, bound, lse_ref = _dequantized_reference(qh, nq, nkv, D, mask, mb)
    excess = float((np.abs(o - ref) - (bound * (1 + 1e-5) + 1e-6)).max())
    lse_err = float(np.abs(lse - lse_ref).max())
    ok = excess <= 0.0 and lse_err < 1e-5
    return ok, "bound excess %.3g, lse error %.3g" % (excess, lse_err)


def check_block_scales():
    """K blocks of very different magnitude: each key must use its own
    64-token block's scale."""
    nq, nkv, D = 64, 320, 64
    q, k, v = _bits(nq, nkv, D, 12, off=0.0)
    kf = oracle.bf16_bits_to_f64(k)
    kf[64:128] *= 8.0
    kf[192:256] *= 0.125
    k = synth.f32_to_bf16_bits(kf.astype(np.float32))
    qh = oracle.quant_head(q, k, v)
    o, _, lse = oracle.attn_rows(qh, np.arange(nq))
    ref, bound, lse_ref = _dequantized_reference(qh, nq, nkv, D, oracle.MASK_NONE, 0)
    excess = float((np.abs(o - ref) - (bound * (1 + 1e-5) + 1e-6)).max())
    lse_err = float(np.abs(lse - lse_ref).max())
    return excess <= 0.0 and lse_err < 1e-5, "excess %.3g, lse error %.3g" % (excess, lse_err)


# ------------------------------------------------------------------ tests

@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("eps", [oracle.EPS, E_WIDE])
def test_exp2_perturbations_stay_within_slack(case, eps):
    ok, detail = check_perturbations_within_slack(case, eps)
    assert ok, detail


@pytest.mark.parametrize("case", CASES)
def test_slack_is_attained(case):
    ok, detail = check_slack_is_attained(case)
    assert ok, detail


@pytest.mark.parametrize("case", CASES)
def test_quantized_path_against_dequantized_fp64(case):
    ok, detail = check_dequantized_fp64(case)
    assert ok, detail


def test_block_scales_against_dequantized_fp64():
    ok, detail = check_block_scales()
    assert ok, detail


def test_slack_statistics_are_small():
    # the slack is non-zero only where an element lies within eps of an
    # e4m3 rounding boundary: a small share of the outputs, far below 2e-3
    case = (128, 1024, 128, oracle.MASK_NONE, 0, 41, 4.0, 0.0)
    _, _, _, qh = _quant(case)
    _, slack, _ = oracle.attn_rows(qh, np.arange(case[0]))
    share = float((slack > 0).mean())
    assert share < 0.25, share
    assert float(slack.max()) < 2e-3


@pytest.mark.parametrize("plant", [1, 2, 3, 4, 5])
def test_planted_mistakes_fail_a_pin(plant):
    names = {1: "K scale from block j / 128", 2: "l from decoded codes",
             3: "slack not rescaled by alpha", 4: "slack gap in code units",
             5: "slack not divided by l"}
    results = []
    with oracle.variant(ORC_PLANT=plant):
        for case in CASES:
            results.append(check_perturbations_within_slack(case)[0])
            results.append(check_slack_is_attained(case)[0])
            results.append(check_dequantized_fp64(case)[0])
        results.append(check_block_scales()[0])
    assert not all(results), "planted mistake not detected: " + names[plant]


def test_folded_and_unfolded_p_scale_agree_within_the_slack():
    # y = exp2(fmaf(S, c, fp32(8 - m))) (adopted) against
    # y' = 2^8 exp2(fmaf(S, c, -m)): both are 2^8 exp2(S c - m) up to the
    # rounding of the exponent argument, a relative difference below 2^-16
    # for these scores; every e4m3 decision they may take differently is
    # inside the slack computed with eps = 2^-16
    E = 2.0 ** -16
    for case in CASES[:2]:
        _, _, _, qh = _quant(case)
        nq, nkv, D, mask, mb = case[:5]
        rows = np.arange(nq)
        o, slack, lse = oracle.attn_rows(qh, rows, mask, mb, eps=E)
        with oracle.variant(ORC_PSCALE_UNFOLDED=1):
            ou, _, lseu = oracle.attn_rows(qh, rows, mask, mb, eps=E)
        r = _l_ratio(lse, lseu)
        bound = slack * r + np.abs(o) * np.abs(r - 1.0) + 1e-12
        assert (np.abs(ou - o) <= bound).all()
        assert np.abs(lse - lseu).max() < 1e-5
