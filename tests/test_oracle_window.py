"""Pins of the oracle's sliding-window mask with a persistent reference context (no GPU).

Streaming generation attends, at every step, to a fixed window: the reference
context (tokens taken once from the first frame and kept for the whole stream,
the role of a sink token), the cached history frames inside the window and the
frame being denoised (Vidu S1 digest, section "Infra", sliding-window
paragraph).  Reading: the cache holds the reference context at positions
[0, sink), then frames of `frame` tokens.  A query in frame f sees the
reference context and frames f - win + 1 .. f.  A query inside the reference
context sees the reference context only.

* The visible-key description of every row equals an explicit boolean mask
  built here from frame indices.
* Identity quantizers: the oracle equals textbook softmax attention under that
  mask to 1e-12, for any split count.  For the last frame it also equals
  unmasked attention over the gathered window keys (the pages' formulation).
* Quantized, sink = 0 with a window wider than the cache: bit for bit the
  block-causal result (block = frame).
* Quantized, tile-aligned frames and reference context: bit for bit the
  block-sparse oracle with the equivalent tile mask.  In split form it equals
  an fp64 merge of block-sparse runs over each range's tiles; the ranges cut
  the query tile's tile sequence, which skips the gap between the reference
  context and the window.
* Quantized against fp64 attention under the same mask: the recipe's accuracy.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from test_oracle_attn import _bits
from test_oracle_block_sparse import textbook_masked

T = 128
W = oracle.MASK_SLIDING_WINDOW


def window_visible(nq, nkv, frame, win, sink):
    """Explicit [nq, nkv] mask from frame indices (the reference context is frame -1)."""
    s0 = min(sink, nkv)
    g = np.arange(nq)[:, None] + (nkv - nq)
    j = np.arange(nkv)[None, :]
    fg = np.where(g < s0, -1, (g - s0) // frame)
    fj = np.where(j < s0, -1, (j - s0) // frame)
    in_ref = fj == -1
    in_window = (fj >= 0) & (fj <= fg) & (fj > fg - win)
    return np.where(fg == -1, in_ref, in_ref | in_window)


CASES = [  # nq, nkv, frame, win, sink
    (300, 700, 40, 3, 0),
    (300, 700, 40, 3, 17),
    (1, 900, 100, 2, 64),
    (256, 1000, 200, 1, 150),
    (130, 1000, 64, 4, 300),
    (500, 500, 70, 2, 90),
    (96, 2100, 96, 5, 500),
]


@pytest.mark.parametrize("nq,nkv,frame,win,sink", CASES + [(50, 50, 7, 100, 0), (20, 60, 5, 2, 80)])
def test_row_window_matches_explicit_mask(nq, nkv, frame, win, sink):
    vis = window_visible(nq, nkv, frame, win, sink)
    j = np.arange(nkv)
    for i in range(nq):
        se, lo, hi = oracle.row_window(i, nq, nkv, W, frame, win, sink)
        got = (j < se) | ((j >= lo) & (j < hi))
        assert np.array_equal(got, vis[i]), i
        assert vis[i].any()  # every row sees at least its own frame


@pytest.mark.parametrize("nq,nkv,frame,win,sink", CASES)
@pytest.mark.parametrize("splits", [1, 2, 3])
def test_identity_equals_textbook_under_window(nq, nkv, frame, win, sink, splits):
    rng = np.random.default_rng(nq + nkv + frame + sink + splits)
    D = 64
    q, k, v = (rng.standard_normal((n, D)) for n in (nq, nkv, nkv))
    rows = np.arange(nq)
    o, lse = oracle.attn_rows_identity(q, k, v, rows, window=(frame, win, sink),
                                       kv_splits=splits)
    ref, ref_lse = textbook_masked(q, k, v, window_visible(nq, nkv, frame, win, sink))
    assert np.abs(o - ref).max() < 1e-12
    assert np.abs(lse - ref_lse).max() < 1e-12


def test_last_frame_equals_attention_over_the_gathered_window():
    # one streaming step: the newest frame against reference context + window
    rng = np.random.default_rng(5)
    frame, win, sink, D = 120, 3, 200, 64
    nkv = sink + 9 * frame
    q = rng.standard_normal((frame, D))
    k, v = rng.standard_normal((nkv, D)), rng.standard_normal((nkv, D))
    keep = np.r_[0:sink, nkv - win * frame:nkv]
    o, lse = oracle.attn_rows_identity(q, k, v, np.arange(frame), window=(frame, win, sink))
    kt, vt = torch.from_numpy(k[keep]), torch.from_numpy(v[keep])
    s = torch.from_numpy(q) @ kt.T / math.sqrt(D)
    ref = torch.softmax(s, -1) @ vt
    assert np.abs(o - ref.numpy()).max() < 1e-12
    assert np.abs(lse - torch.logsumexp(s, -1).numpy()).max() < 1e-12


def test_fp64_window_equals_textbook():
    q, k, v = _bits(200, 900, 64, seed=41, mag=3.0)
    frame, win, sink = 130, 2, 70
    rows = np.arange(200)
    o = oracle.attn_fp64_rows(q, k, v, rows, window=(frame, win, sink))
    f = [oracle.bf16_bits_to_f64(a) for a in (q, k, v)]
    ref, _ = textbook_masked(*f, window_visible(200, 900, frame, win, sink))
    assert np.abs(o - ref).max() < 1e-12


@pytest.mark.parametrize("nq,nkv,frame", [(300, 700, 40), (256, 1000, 200), (130, 1000, 64)])
@pytest.mark.parametrize("splits", [1, 3])
def test_wide_window_without_reference_is_block_causal(nq, nkv, frame, splits):
    q, k, v = _bits(nq, nkv, 128, seed=nq + frame, mag=5.0)
    qh = oracle.quant_head(q, k, v)
    rows = np.arange(nq)
    a = oracle.attn_rows(qh, rows, window=(frame, nkv // frame + 1, 0), kv_splits=splits)
    b = oracle.attn_rows(qh, rows, oracle.MASK_BLOCK_CAUSAL, frame, kv_splits=splits)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def aligned_tile_mask(nq, nkv, frame, win, sink):
    """Block mask (query tile x KV tile) equal to the window mask when frame
    and sink are multiples of 128 and the queries start on a tile boundary."""
    n_qt, n_kt = -(-nq // T), -(-nkv // T)
    g0 = nkv - nq
    bm = np.zeros((n_qt, n_kt), np.uint8)
    for qt in range(n_qt):
        g = g0 + qt * T
        bm[qt, :sink // T] = 1
        if g < sink:
            continue
        f = (g - sink) // frame
        lo = sink + max(f - win + 1, 0) * frame
        bm[qt, lo // T:min(sink + (f + 1) * frame, nkv + T - 1) // T] = 1
    return bm


ALIGNED = [(512, 1536, 256, 2, 128), (256, 2048, 128, 3, 256), (384, 1280, 256, 1, 0),
           (300, 1324, 128, 2, 128)]


@pytest.mark.parametrize("nq,nkv,frame,win,sink", ALIGNED)
def test_aligned_window_equals_block_sparse(nq, nkv, frame, win, sink):
    q, k, v = _bits(nq, nkv, 128, seed=nkv + win, mag=5.0)
    qh = oracle.quant_head(q, k, v)
    rows = np.arange(nq)
    bm = aligned_tile_mask(nq, nkv, frame, win, sink)
    a = oracle.attn_rows(qh, rows, window=(frame, win, sink))
    b = oracle.attn_rows(qh, rows, block_mask=bm)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


@pytest.mark.parametrize("nq,nkv,frame,win,sink,splits", [(256, 2048, 128, 3, 256, 2),
                                                          (128, 3072, 256, 4, 512, 3),
                                                          (128, 1664, 128, 5, 128, 4)])
def test_aligned_window_split_is_merge_of_ranges(nq, nkv, frame, win, sink, splits):
    # each query tile's tiles: the reference context's, then (after a gap) the
    # window's; the ranges cut that sequence, not the tile index space
    q, k, v = _bits(nq, nkv, 128, seed=nkv + splits, mag=5.0)
    qh = oracle.quant_head(q, k, v)
    rows = np.arange(nq)
    o, _, lse = oracle.attn_rows(qh, rows, window=(frame, win, sink), kv_splits=splits)
    bm = aligned_tile_mask(nq, nkv, frame, win, sink)
    ref = np.empty_like(o)
    ref_lse = np.empty_like(lse)
    for qt in range(bm.shape[0]):
        seq = np.flatnonzero(bm[qt])
        nk = seq.size
        parts = []
        for s in range(splits):
            part = seq[nk * s // splits:nk * (s + 1) // splits]
            if part.size == 0:
                continue
            pm = np.zeros_like(bm)
            pm[qt, part] = 1
            r = rows[qt * T:(qt + 1) * T]
            po, _, pl = oracle.attn_rows(qh, r, block_mask=pm)
            parts.append((po, pl))
        L = np.logaddexp.reduce(np.stack([pl for _, pl in parts]), axis=0)
        ref[qt * T:(qt + 1) * T] = sum(po * np.exp(pl - L)[:, None] for po, pl in parts)
        ref_lse[qt * T:(qt + 1) * T] = L
    assert np.abs(lse - ref_lse).max() < 1e-5
    assert np.abs(o - ref).max() < 1e-5 * max(1.0, np.abs(ref).max())


def test_gap_is_skipped_in_split_ranges():
    # reference context = tile 0; the query tile (positions 3968..4095, frame
    # 15) sees frames 14 and 15 = tiles 29..31.  Its sequence is [0, 29, 30,
    # 31]; 2 ranges are {0, 29} and {30, 31} (a cut of the tile index space
    # would give {0} and {29, 30, 31}).
    nq, nkv, frame, win, sink = 128, 4096, 256, 2, 128
    q, k, v = _bits(nq, nkv, 128, seed=77, mag=5.0)
    qh = oracle.quant_head(q, k, v)
    rows = np.arange(nq)
    bm = aligned_tile_mask(nq, nkv, frame, win, sink)
    assert list(np.flatnonzero(bm[0])) == [0, 29, 30, 31]
    o, _, _ = oracle.attn_rows(qh, rows, window=(frame, win, sink), kv_splits=2)
    p0 = np.zeros_like(bm)
    p0[0, [0, 29]] = 1
    p1 = np.zeros_like(bm)
    p1[0, [30, 31]] = 1
    a, _, la = oracle.attn_rows(qh, rows, block_mask=p0)
    b, _, lb = oracle.attn_rows(qh, rows, block_mask=p1)
    L = np.logaddexp(la, lb)
    ref = a * np.exp(la - L)[:, None] + b * np.exp(lb - L)[:, None]
    assert np.abs(o - ref).max() < 1e-5 * max(1.0, np.abs(ref).max())
    # the cut of the tile index space, {0} and {29, 30, 31}, is measurably different
    p0[0, 29] = 0
    p1[0, 29] = 1
    a, _, la = oracle.attn_rows(qh, rows, block_mask=p0)
    b, _, lb = oracle.attn_rows(qh, rows, block_mask=p1)
    L = np.logaddexp(la, lb)
    other = a * np.exp(la - L)[:, None] + b * np.exp(lb - L)[:, None]
    assert np.abs(o - other).max() > 10 * np.abs(o - ref).max()


@pytest.mark.parametrize("nq,nkv,frame,win,sink", [(300, 1500, 130, 3, 70), (128, 2000, 256, 2, 300)])
def test_quantized_window_accuracy(nq, nkv, frame, win, sink):
    q, k, v = _bits(nq, nkv, 128, seed=nkv, mag=3.0)
    qh = oracle.quant_head(q, k, v)
    rows = np.arange(nq)
    o, _, _ = oracle.attn_rows(qh, rows, window=(frame, win, sink))
    ref = oracle.attn_fp64_rows(q, k, v, rows, window=(frame, win, sink))
    cos, rel = oracle.accuracy(o, ref)[:2]
    assert cos > 0.999 and rel < 0.05


def test_invalid_window_arguments():
    q, k, v = _bits(64, 256, 64, seed=1)
    qh = oracle.quant_head(q, k, v)
    for bad in [(0, 1, 0), (64, 0, 0), (64, 1, -1)]:
        with pytest.raises(ValueError):
            oracle.attn_rows(qh, np.arange(4), window=bad)
    qh2 = oracle.quant_head(*_bits(300, 256, 64, seed=2))
    with pytest.raises(ValueError):  # a window mask needs Nkv >= Nq
        oracle.attn_rows(qh2, np.arange(4), window=(64, 1, 0))
