"""GPU parity of the channel-equalised quantization (sage_quant_qk_equalized),
a labelled accuracy variant outside the recipe: channel d of Q is multiplied
and channel d of the smoothed K divided by 2^e[d] before the per-block INT8
codes.

* Codes, scales, the K mean, the V codes and the exponents e equal the
  oracle's orc_quant_head_eq bit for bit: D = 64 and 128, ragged token
  counts, Nq != Nkv both ways, x20 outlier channels, zero and tiny channels,
  ratios that clamp.
* Attention over the equalised quantization matches the oracle's
  same-quantization attention on every row (all masks).
* At the full 720p and 480p workloads (x20 outlier K channels), sampled heads
  are bit-exact and the sampled rows' accuracy against fp64 attention is
  better than the recipe's on the same rows.
"""
import numpy as np
import pytest
import torch

import bit_quantized_attention_sage_b200 as sage
import oracle
from bit_quantized_attention_sage_b200 import synth

from gpu_helpers import check_quant_head, check_rows, rows_of, to_dev

pytestmark = pytest.mark.gpu


def _run_eq(q, k, v, mask=0, mb=0):
    B, H, Nq, D = q.shape
    e = torch.full((B, H, D), 99, dtype=torch.int8, device="cuda")
    qkv = sage.quant_qk_equalized(to_dev(q), to_dev(k), to_dev(v), eq_exp=e)
    o32 = torch.empty((B, H, Nq, D), dtype=torch.float32, device="cuda")
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device="cuda")
    o = sage.attn_fwd(qkv, mask, mb, o_f32=o32, lse=lse)
    assert sage.sync_status() == 0
    return qkv, e.cpu().numpy(), o, o32, lse


CASES = [  # B, H, Nq, Nkv, D, outlier magnitude, mask, mask block
    (1, 2, 130, 300, 64, 20.0, 0, 0),
    (1, 2, 300, 129, 128, 20.0, 0, 0),
    (2, 1, 65, 1000, 128, 5.0, 2, 40),
    (1, 3, 257, 257, 128, 0.0, 1, 0),
    (1, 1, 1, 700, 64, 20.0, 0, 0),
]


@pytest.mark.parametrize("case", CASES)
def test_equalised_quantization_and_attention(case):
    B, H, Nq, Nkv, D, mag, mask, mb = case
    w = synth.Workload("eqg", B, H, Nq, Nkv, D, outlier_mag=mag, k_offset_var=2.0,
                       seed=300 + Nq + Nkv)
    q, k, v = synth.full(w)
    qkv, e, o, o32, lse = _run_eq(q, k, v, mask, mb)
    for b in range(B):
        for h in range(H):
            ref = oracle.quant_head(q[b, h], k[b, h], v[b, h], eq=True)
            check_quant_head(qkv, b, h, ref)
            assert np.array_equal(e[b, h], ref["eq_exp"]), "eq_exp differs"
            rows = np.arange(Nq)
            check_rows(ref, rows, rows_of(o, b, h, rows), rows_of(o32, b, h, rows),
                       rows_of(lse, b, h, rows), mask, mb)


def test_extreme_channels():
    # a zero Q channel, ratios that clamp at +-32, tiny and subnormal-range
    # magnitudes: the exponent decisions and the codes stay bit-exact
    rng = np.random.default_rng(31)
    qf = rng.standard_normal((1, 2, 200, 64)).astype(np.float32)
    kf = rng.standard_normal((1, 2, 333, 64)).astype(np.float32)
    qf[..., 0] = 0.0
    qf[..., 1] *= 2.0 ** -90
    kf[..., 2] *= 2.0 ** -100
    kf[..., 3] *= 2.0 ** -130   # bf16 subnormals
    qf[..., 4] *= 2.0 ** 60
    kf[..., 5] = 7.0            # constant channel: K - mu = 0
    q, k = synth.f32_to_bf16_bits(qf), synth.f32_to_bf16_bits(kf)
    v = synth.f32_to_bf16_bits(rng.standard_normal((1, 2, 333, 64)).astype(np.float32))
    qkv, e, _, _, _ = _run_eq(q, k, v)
    for h in range(2):
        ref = oracle.quant_head(q[0, h], k[0, h], v[0, h], eq=True)
        check_quant_head(qkv, 0, h, ref)
        assert np.array_equal(e[0, h], ref["eq_exp"])
    assert e[0, 0, 0] == 0 and e[0, 0, 5] == 0


def test_default_recipe_unchanged_by_the_variant():
    # the same inputs through sage_quant_qk give the recipe's codes: the two
    # calls share kernels but not their outputs
    w = synth.Workload("eqd", 1, 2, 200, 450, 128, outlier_mag=20.0, seed=77)
    q, k, v = synth.full(w)
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    sage.quant_qk_equalized(qd, kd, vd)
    plain = sage.quant_qk(qd, kd, vd)
    assert sage.sync_status() == 0
    for h in range(2):
        check_quant_head(plain, 0, h, oracle.quant_head(q[0, h], k[0, h], v[0, h]))


@pytest.mark.parametrize("w", [synth.P480, synth.P720], ids=lambda w: w.name)
def test_full_size_sampled_and_more_accurate(w):
    q, k, v = synth.full(w)
    qkv, e, o, o32, lse = _run_eq(q, k, v, w.mask, w.mask_block)
    plain = sage.quant_qk(to_dev(q), to_dev(k), to_dev(v))
    o_plain = torch.empty_like(o32)
    sage.attn_fwd(plain, w.mask, w.mask_block, o_f32=o_plain)
    assert sage.sync_status() == 0
    rng = np.random.default_rng(w.seed + 1)
    heads = sorted(set([0, w.B * w.H - 1]) | set(rng.choice(w.B * w.H, 1).tolist()))
    got_eq, got_plain, truth = [], [], []
    for bh in heads:
        b, h = divmod(bh, w.H)
        ref = oracle.quant_head(q[b, h], k[b, h], v[b, h], eq=True)
        check_quant_head(qkv, b, h, ref)
        assert np.array_equal(e[b, h], ref["eq_exp"])
        rows = np.sort(rng.choice(w.Nq, 48, replace=False))
        check_rows(ref, rows, rows_of(o, b, h, rows), rows_of(o32, b, h, rows),
                   rows_of(lse, b, h, rows), w.mask, w.mask_block)
        got_eq.append(rows_of(o32, b, h, rows))
        got_plain.append(rows_of(o_plain, b, h, rows))
        truth.append(oracle.attn_fp64_rows(q[b, h], k[b, h], v[b, h], rows, w.mask, w.mask_block))
    t = np.concatenate(truth)
    cos_e, rel_e = oracle.accuracy(np.concatenate(got_eq), t)
    cos_p, rel_p = oracle.accuracy(np.concatenate(got_plain), t)
    print("%s: recipe cos %.5f relL1 %.4f; equalised cos %.5f relL1 %.4f" % (
        w.name, cos_p, rel_p, cos_e, rel_e))
    assert rel_e < rel_p and cos_e > cos_p
