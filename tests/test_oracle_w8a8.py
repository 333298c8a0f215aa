"""Pins of the oracle's per-block W8A8 linear layer (no GPU).

* Quantizers: the largest code of every non-zero group is 127, every value is
  reconstructed within half a step, all-zero groups get scale 0, ties round to
  even, and the block shapes are right (a token x 128 channels for X, 128 x 128
  for W).
* GEMM with integer-valued inputs whose groups have absmax 127 (so every scale
  is exactly 1 and the codes are the values): Y equals the integer product
  computed by numpy int64 brute force, exactly.  This pins the indexing of both
  operands, the grouping and the transposition.
* GEMM on random inputs: Y equals the fp64 definition sum_g P_g sx sw within
  the fp32 accumulation bound.
"""
import numpy as np
import pytest

import oracle
from bit_quantized_attention_sage_b200 import synth

G = 128


def bf16(a):
    return synth.f32_to_bf16_bits(np.asarray(a, np.float32))


def _rand(shape, seed, outliers=0):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal(shape).astype(np.float32)
    if outliers:
        cols = rng.choice(shape[1], outliers, replace=False)
        x[:, cols] *= 30.0
    return bf16(x)


@pytest.mark.parametrize("M,K,seed", [(3, 128, 1), (17, 512, 2), (64, 384, 3)])
def test_act_quant_invariants(M, K, seed):
    x = _rand((M, K), seed, outliers=3)
    xq, sx = oracle.w8a8_quant_act(x)
    xf = oracle.bf16_bits_to_f64(x).reshape(M, K // G, G)
    q = xq.reshape(M, K // G, G).astype(np.int64)
    assert sx.shape == (M, K // G)
    a = np.abs(xf).max(2)
    np.testing.assert_array_equal(sx, (a / 127.0).astype(np.float32))
    assert np.all(np.abs(q).max(2) == 127)
    err = np.abs(xf - q * sx[..., None].astype(np.float64))
    assert np.all(err <= 0.5 * sx[..., None] * (1 + 1e-5) + 1e-30)


def test_weight_quant_blocks():
    N, K = 256, 384
    w = _rand((N, K), 4, outliers=2)
    wq, sw = oracle.w8a8_quant_weight(w)
    wf = oracle.bf16_bits_to_f64(w)
    assert sw.shape == (N // G, K // G)
    for nb in range(N // G):
        for g in range(K // G):
            blk = wf[nb * G:(nb + 1) * G, g * G:(g + 1) * G]
            assert sw[nb, g] == np.float32(np.abs(blk).max() / 127.0)
            q = wq[nb * G:(nb + 1) * G, g * G:(g + 1) * G]
            assert np.abs(q).max() == 127


def test_zero_groups_and_ties():
    x = np.zeros((2, 256), np.float32)
    x[1, 128] = 127.0  # group absmax 127: scale 1, codes are the values
    x[1, 129:133] = [0.5, 1.5, 2.5, -2.5]
    xq, sx = oracle.w8a8_quant_act(bf16(x))
    assert sx[0, 0] == 0 and sx[0, 1] == 0 and sx[1, 0] == 0 and sx[1, 1] == 1.0
    assert not xq[0].any() and not xq[1, :128].any()
    np.testing.assert_array_equal(xq[1, 128:133], [127, 0, 2, 2, -2])


@pytest.mark.parametrize("M,N,K,seed", [(5, 128, 128, 5), (33, 256, 512, 6)])
def test_gemm_exact_on_unit_scales(M, N, K, seed):
    rng = np.random.default_rng(seed)
    xi = rng.integers(-127, 128, (M, K)).astype(np.int64)
    wi = rng.integers(-127, 128, (N, K)).astype(np.int64)
    xi.reshape(M, K // G, G)[:, :, 0] = 127  # every activation group: absmax 127
    wi.reshape(N // G, G, K // G, G)[:, 0, :, 0] = 127  # every weight block: absmax 127
    xq, sx = oracle.w8a8_quant_act(bf16(xi))
    wq, sw = oracle.w8a8_quant_weight(bf16(wi))
    assert np.all(sx == 1.0) and np.all(sw == 1.0)
    np.testing.assert_array_equal(xq, xi)
    np.testing.assert_array_equal(wq, wi)
    y = oracle.w8a8_gemm_rows(xq, sx, wq, sw, np.arange(M))
    ref = xi @ wi.T  # |ref| < 2^24: exact in fp32 whatever the order
    assert np.abs(ref).max() < 2 ** 24
    np.testing.assert_array_equal(y.astype(np.int64), ref)


@pytest.mark.parametrize("M,N,K,seed", [(9, 128, 256, 7), (40, 384, 640, 8)])
def test_gemm_matches_blockwise_definition(M, N, K, seed):
    x = _rand((M, K), seed, outliers=4)
    w = _rand((N, K), seed + 50)
    xq, sx = oracle.w8a8_quant_act(x)
    wq, sw = oracle.w8a8_quant_weight(w)
    rows = np.arange(M)[::-1].copy()  # any row order
    y = oracle.w8a8_gemm_rows(xq, sx, wq, sw, rows)
    Gn = K // G
    P = np.einsum("mgc,ngc->mng", xq.reshape(M, Gn, G).astype(np.int64),
                  wq.reshape(N, Gn, G).astype(np.int64)).astype(np.float64)
    s = sx[:, None, :].astype(np.float64) * np.repeat(sw, G, axis=0)[None, :, :]
    terms = P * s.astype(np.float32).astype(np.float64)
    ref = terms.sum(2)[rows]
    bound = Gn * 2.0 ** -23 * np.abs(terms).sum(2)[rows] + 1e-30
    assert np.all(np.abs(y - ref) <= bound)
