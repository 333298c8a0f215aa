"""Pins of the windowed quantization of the streaming cache (no GPU).

Reading: a sliding-window step quantizes only the keys it attends to -- the
reference context and the union of its query rows' windows -- so the K mean
and the V channel scales are those of these keys, and the window attention
then runs over the gathered keys with the same frame / window / reference
parameters.  The gathered keys are the cache's reference context and one
contiguous range of whole frames ("Vidu S1" digest, section "Infra": every
step attends to the reference context and a fixed-length window of the
cache).

* The gathered index set equals the union of the explicit per-row masks.
* Identity quantizers: window attention over the gathered keys equals window
  attention over the whole cache to 1e-12 (every row sees the same keys).
* When the window reaches back over the whole cache, the gathered set is the
  cache and the quantized result is the whole-cache recipe, bit for bit.
* Quantized: the windowed statistics (fewer tokens per V channel maximum and
  per K mean) are at least as accurate against fp64 attention.
"""
import numpy as np
import pytest

import oracle
from test_oracle_attn import _bits
from test_oracle_window import window_visible

W = oracle.MASK_SLIDING_WINDOW
CASES = [  # nq, nkv, frame, win, sink
    (40, 700, 40, 3, 40),
    (100, 1300, 100, 4, 100),
    (130, 1000, 64, 4, 300),
    (96, 2100, 96, 5, 500),
    (1, 900, 100, 2, 64),
]


@pytest.mark.parametrize("nq,nkv,frame,win,sink", CASES)
def test_gathered_keys_are_the_union_of_visible_keys(nq, nkv, frame, win, sink):
    idx = oracle.window_keys(nq, nkv, frame, win, sink)
    vis = window_visible(nq, nkv, frame, win, sink).any(axis=0)
    assert np.array_equal(idx, np.flatnonzero(vis))
    gap = (idx[np.searchsorted(idx, sink) if sink < nkv else 0] - sink) if sink < idx.size else 0
    assert gap % frame == 0


@pytest.mark.parametrize("nq,nkv,frame,win,sink", CASES)
def test_identity_attention_over_gathered_keys(nq, nkv, frame, win, sink):
    D = 64
    q, k, v = (np.random.default_rng(7).standard_normal((n, D)) for n in (nq, nkv, nkv))
    idx = oracle.window_keys(nq, nkv, frame, win, sink)
    rows = np.arange(nq)
    full, _ = oracle.attn_rows_identity(q, k, v, rows, window=(frame, win, sink))
    gath, _ = oracle.attn_rows_identity(q, k[idx], v[idx], rows, window=(frame, win, sink))
    assert np.abs(full - gath).max() < 1e-12


def test_window_over_the_whole_cache_is_the_whole_cache_recipe():
    nq, nkv, frame, win, sink = 120, 600, 120, 10, 0
    q, k, v = _bits(nq, nkv, 64, 81)
    idx = oracle.window_keys(nq, nkv, frame, win, sink)
    assert np.array_equal(idx, np.arange(nkv))
    a = oracle.quant_head(q, k[idx], v[idx])
    b = oracle.quant_head(q, k, v)
    for key in a:
        if isinstance(a[key], np.ndarray):
            assert np.array_equal(a[key], b[key]), key


@pytest.mark.parametrize("nq,nkv,frame,win,sink", CASES[:4])
def test_windowed_statistics_accuracy(nq, nkv, frame, win, sink):
    q, k, v = _bits(nq, nkv, 128, 82, off=4.0)
    idx = oracle.window_keys(nq, nkv, frame, win, sink)
    rows = np.arange(nq)
    ref = oracle.attn_fp64_rows(q, k, v, rows, window=(frame, win, sink))
    whole = oracle.attn_rows(oracle.quant_head(q, k, v), rows, window=(frame, win, sink))[0]
    gath = oracle.attn_rows(oracle.quant_head(q, k[idx], v[idx]), rows,
                            window=(frame, win, sink))[0]
    cw, rw = oracle.accuracy(whole, ref)
    cg, rg = oracle.accuracy(gath, ref)
    assert cg > 0.995 and rg < 0.06, (cg, rg)
    assert rg <= rw * 1.05, (rg, rw)
