"""Pins of the channel-equalised quantization variant (no GPU).

A labelled accuracy variant, kept apart from the pages' recipe (which stays
the default): before the per-block INT8 quantization, channel d of Q is
multiplied and channel d of the mean-smoothed K divided by the same power of
two 2^e[d].  The scores are unchanged in exact arithmetic, while a K channel
with outliers no longer sets the scale of every K block alone: the INT8
error of Q K^T is what dominates the recipe's error on such data (the pages
call the 8-bit result nearly lossless for video models, TurboDiffusion notes,
"几乎无损"; the per-block INT8 recipe alone is not on outlier channels).

* The exponent rule, restated here with numpy's frexp: e = floor((E(ak) -
  E(aq)) / 2), E(x) = floor(log2 x), ak and aq the channel maxima of the
  smoothed K and of Q; after scaling the two maxima lie within (1/2, 4).
* The dequantized scores approximate the plain scores Q (K - mu)^T (fp64)
  within the INT8 error bound of the equalised operands: a sign error in the
  scaling (K multiplied too) breaks it.
* Balanced channels (every e = 0) give the default recipe bit for bit; the K
  mean and the V codes are never touched.
* Against fp64 attention, accuracy improves on data with x20 outlier K
  channels and does not degrade without outliers.
* Planted mistakes (K multiplied by 2^e; e not halved) fail a pin.
"""
import numpy as np
import pytest

import oracle
from bit_quantized_attention_sage_b200 import synth

EQ_MAX = 32


def _head(nq, nkv, D, mag, seed, k_offset_var=0.0):
    w = synth.Workload("eq", 1, 1, nq, nkv, D, outlier_mag=mag, k_offset_var=k_offset_var,
                       seed=seed)
    return synth.head(w, 0, 0)


def _f32(bits):
    return oracle.bf16_bits_to_f64(bits).astype(np.float32)


def expected_exponents(q, k, mu):
    """e[d] from the definition, with numpy: channel maxima of Q and of the
    fp32 smoothed key, binary exponents by frexp, floor division by 2."""
    qf, kf = _f32(q), _f32(k)
    ks = kf - mu[None, :].astype(np.float32)  # fp32 subtraction
    aq, ak = np.abs(qf).max(0), np.abs(ks).max(0)
    e = np.zeros(q.shape[1], np.int64)
    nz = (aq > 0) & (ak > 0)
    eq_ = np.frexp(aq[nz].astype(np.float64))[1] - 1
    ek_ = np.frexp(ak[nz].astype(np.float64))[1] - 1
    e[nz] = np.clip((ek_ - eq_) // 2, -EQ_MAX, EQ_MAX)
    return e, aq, ak


def check_exponent_rule(q, k, v):
    h = oracle.quant_head(q, k, v, eq=True)
    e, aq, ak = expected_exponents(q, k, h["mu"])
    ok = np.array_equal(h["eq_exp"].astype(np.int64), e)
    nz = (aq > 0) & (ak > 0) & (np.abs(e) < EQ_MAX)
    ratio = (ak[nz] * np.exp2(-e[nz])) / (aq[nz] * np.exp2(e[nz]))
    ok = ok and bool(((ratio > 0.5) & (ratio < 4.0)).all())
    return ok, h


def check_scores_within_int8_bound(q, k, v):
    """|dequantized score - Q (K - mu)^T| within the INT8 bound of the
    equalised operands, every (i, j)."""
    h = oracle.quant_head(q, k, v, eq=True)
    nq, D = q.shape
    nkv = k.shape[0]
    qf, kf = _f32(q).astype(np.float64), _f32(k).astype(np.float64)
    km = kf - h["mu"].astype(np.float64)[None, :]
    true = qf @ km.T
    sq = np.repeat(h["qs"].astype(np.float64), 64)[:nq]
    sk = np.repeat(h["ks"].astype(np.float64), 64)[:nkv]
    deq = (h["q8"][:nq].astype(np.int64) @ h["k8"][:nkv].astype(np.int64).T).astype(np.float64)
    deq *= sq[:, None] * sk[None, :]
    s = np.exp2(h["eq_exp"].astype(np.float64))
    qa, ka = np.abs(qf) * s[None, :], np.abs(km) / s[None, :]
    # sum_d (|Q'| sk / 2 + |K'| sq / 2 + sq sk / 4): half a step of each code
    bound = (qa.sum(1)[:, None] * sk[None, :] / 2 + sq[:, None] * ka.sum(1)[None, :] / 2 +
             D * sq[:, None] * sk[None, :] / 4)
    # the fp32 rounding of K - mu and of x * inv, relative 2^-23 of |Q||K - mu|
    bound = bound * (1 + 1e-5) + (np.abs(qf) @ np.abs(km).T) * 2.0 ** -22 + 1e-30
    return bool((np.abs(deq - true) <= bound).all()), h


CASES = [(130, 300, 64, 20.0, 1), (70, 650, 128, 20.0, 2), (200, 200, 128, 5.0, 3),
         (64, 129, 64, 0.0, 4)]


@pytest.mark.parametrize("nq,nkv,D,mag,seed", CASES)
def test_exponent_rule(nq, nkv, D, mag, seed):
    q, k, v = _head(nq, nkv, D, mag, seed)
    ok, h = check_exponent_rule(q, k, v)
    assert ok
    if mag >= 20:  # the outlier channels are equalised
        assert (h["eq_exp"] >= 1).sum() >= 4


@pytest.mark.parametrize("nq,nkv,D,mag,seed", CASES)
def test_scores_within_the_int8_bound(nq, nkv, D, mag, seed):
    q, k, v = _head(nq, nkv, D, mag, seed, k_offset_var=2.0)
    assert check_scores_within_int8_bound(q, k, v)[0]


def test_extreme_channel_ratios_clamp():
    rng = np.random.default_rng(5)
    qf = rng.standard_normal((64, 64)).astype(np.float32)
    kf = rng.standard_normal((128, 64)).astype(np.float32)
    qf[:, 0] *= 2.0 ** -80   # K/Q ratio 2^80: e clamps at +32
    kf[:, 1] *= 2.0 ** -90   # ratio 2^-90: e clamps at -32
    qf[:, 2] = 0.0           # a zero channel: e = 0
    q, k = synth.f32_to_bf16_bits(qf), synth.f32_to_bf16_bits(kf)
    v = synth.f32_to_bf16_bits(rng.standard_normal((128, 64)).astype(np.float32))
    ok, h = check_exponent_rule(q, k, v)
    assert ok
    assert h["eq_exp"][0] == EQ_MAX and h["eq_exp"][1] == -EQ_MAX and h["eq_exp"][2] == 0


def test_balanced_channels_give_the_default_recipe():
    # every channel's maxima of Q and of the smoothed K in [2, 4): e = 0
    rng = np.random.default_rng(6)
    qf = np.clip(rng.standard_normal((150, 64)), -1.9, 1.9).astype(np.float32)
    kf = np.clip(rng.standard_normal((260, 64)), -1.9, 1.9).astype(np.float32)
    qf[3, :] = 3.5
    kf[5, :], kf[6, :] = 3.25, -3.25
    q, k = synth.f32_to_bf16_bits(qf), synth.f32_to_bf16_bits(kf)
    v = synth.f32_to_bf16_bits(rng.standard_normal((260, 64)).astype(np.float32))
    a, b = oracle.quant_head(q, k, v), oracle.quant_head(q, k, v, eq=True)
    assert not b["eq_exp"].any()
    for key in ("q8", "qs", "k8", "ks", "mu", "v8", "vs"):
        assert np.array_equal(a[key], b[key]), key


@pytest.mark.parametrize("nq,nkv,D,mag,seed", CASES[:3])
def test_mean_and_v_untouched(nq, nkv, D, mag, seed):
    q, k, v = _head(nq, nkv, D, mag, seed)
    a, b = oracle.quant_head(q, k, v), oracle.quant_head(q, k, v, eq=True)
    for key in ("mu", "v8", "vs"):
        assert np.array_equal(a[key], b[key]), key


def _accuracy(q, k, v, eq):
    rows = np.arange(q.shape[0])
    h = oracle.quant_head(q, k, v, eq=eq)
    o, _, _ = oracle.attn_rows(h, rows)
    return oracle.accuracy(o, oracle.attn_fp64_rows(q, k, v, rows))


def test_accuracy_improves_with_outlier_channels():
    q, k, v = _head(192, 2048, 128, 20.0, 7)
    cos0, rel0 = _accuracy(q, k, v, False)
    cos1, rel1 = _accuracy(q, k, v, True)
    assert rel1 < rel0 / 1.5 and cos1 > cos0, (cos0, rel0, cos1, rel1)
    assert cos1 >= 0.999


def test_accuracy_unchanged_without_outliers():
    q, k, v = _head(192, 2048, 128, 0.0, 8)
    cos0, rel0 = _accuracy(q, k, v, False)
    cos1, rel1 = _accuracy(q, k, v, True)
    assert rel1 < rel0 * 1.02 and cos1 > cos0 - 1e-4, (cos0, rel0, cos1, rel1)


@pytest.mark.parametrize("plant", [6, 7])
def test_planted_mistakes_are_caught(plant):
    results = []
    with oracle.variant(ORC_PLANT=plant):
        for nq, nkv, D, mag, seed in CASES:
            q, k, v = _head(nq, nkv, D, mag, seed, k_offset_var=2.0)
            results.append(check_exponent_rule(q, k, v)[0])
            results.append(check_scores_within_int8_bound(q, k, v)[0])
    assert not all(results), "planted mistake %d not detected" % plant
