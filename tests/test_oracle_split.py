"""Pins of the oracle's split-KV form (no GPU).

The KV tiles that a 128-query tile visits are cut into S contiguous ranges.
Each range runs its own online softmax, and the partial results are merged
(the standard split-KV evaluation of flash-style attention, used to fill the
GPU when there are few query tiles).

* One split is the plain oracle, bit for bit.
* Identity quantizers: any split count equals textbook softmax attention to
  1e-12, for every mask and ragged sizes.  The merge is exact mathematics.
* More splits than tiles leaves a single non-empty range, so the result is
  the plain oracle's bit for bit.
* Quantized, no mask: the split result equals a merge, done here in fp64, of
  the plain oracle run on each range's keys alone, with range r covering
  tiles [floor(r nk / S), floor((r + 1) nk / S)).  This pins the range
  boundaries and the merge.
"""
import numpy as np
import pytest

import oracle
from test_oracle_attn import MASKS, _bits, visible_matrix
from test_oracle_block_sparse import textbook_masked

T = 128


@pytest.mark.parametrize("mask,mb", MASKS)
def test_one_split_is_plain(mask, mb):
    q, k, v = _bits(300, 700, 128, seed=31, mag=5.0)
    qh = oracle.quant_head(q, k, v)
    rows = np.arange(300)
    a = oracle.attn_rows(qh, rows, mask, mb)
    b = oracle.attn_rows(qh, rows, mask, mb, kv_splits=1)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


@pytest.mark.parametrize("mask,mb", MASKS)
@pytest.mark.parametrize("nq,nkv,splits", [(300, 700, 2), (130, 1000, 3), (1, 900, 5), (256, 256, 4)])
def test_identity_split_equals_textbook(mask, mb, nq, nkv, splits):
    rng = np.random.default_rng(nq + nkv + splits)
    D = 64
    q, k, v = (rng.standard_normal((n, D)) for n in (nq, nkv, nkv))
    rows = np.arange(nq)
    o, lse = oracle.attn_rows_identity(q, k, v, rows, mask, mb, kv_splits=splits)
    vis = visible_matrix(nq, nkv, mask, mb)
    ref, ref_lse = textbook_masked(q, k, v, vis)
    assert np.abs(o - ref).max() < 1e-12
    assert np.abs(lse - ref_lse).max() < 1e-12


def test_more_splits_than_tiles_is_plain():
    q, k, v = _bits(200, 100, 128, seed=32)
    qh = oracle.quant_head(q, k, v)
    rows = np.arange(200)
    a = oracle.attn_rows(qh, rows)
    b = oracle.attn_rows(qh, rows, kv_splits=3)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def _slice_head(qh, t0, t1):
    """The quantized head restricted to the keys of tiles [t0, t1)."""
    j0, j1 = t0 * T, min(t1 * T, qh["nkv"])
    out = dict(qh)
    out["k8"] = np.ascontiguousarray(qh["k8"][j0:j0 + -(-(j1 - j0) // 64) * 64])
    out["ks"] = np.ascontiguousarray(qh["ks"][j0 // 64:-(-j1 // 64)])
    out["v8"] = np.ascontiguousarray(qh["v8"][j0:j1])
    out["nkv"] = j1 - j0
    return out


@pytest.mark.parametrize("nkv,splits", [(1000, 3), (1280, 4), (700, 2)])
def test_quantized_split_is_merge_of_ranges(nkv, splits):
    nq = 150
    q, k, v = _bits(nq, nkv, 128, seed=nkv + splits, mag=5.0)
    qh = oracle.quant_head(q, k, v)
    rows = np.arange(nq)
    o, _, lse = oracle.attn_rows(qh, rows, kv_splits=splits)
    nk = -(-nkv // T)
    parts = []
    for s in range(splits):
        t0, t1 = nk * s // splits, nk * (s + 1) // splits
        if t1 > t0:
            po, _, pl = oracle.attn_rows(_slice_head(qh, t0, t1), rows)
            parts.append((po, pl))
    L = np.logaddexp.reduce(np.stack([pl for _, pl in parts]), axis=0)
    ref = sum(po * np.exp(pl - L)[:, None] for po, pl in parts)
    assert np.abs(lse - L).max() < 1e-5
    assert np.abs(o - ref).max() < 1e-5 * max(1.0, np.abs(ref).max())
    # and close to the plain oracle (different P rounding points only)
    o1, _, _ = oracle.attn_rows(qh, rows)
    assert np.abs(o - o1).max() < 0.05
