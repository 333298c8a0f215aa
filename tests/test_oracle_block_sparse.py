"""Pins of the oracle's block-sparse skipping (no GPU).

A caller-supplied block mask switches 128-query x 128-key tiles off (the
skipping that sparse attention layers such as SLA put on top of quantized
attention; the TurboDiffusion notes' hybrid-attention bullet).  Key j is
visible to query i iff the row mask allows it AND the tile (i // 128, j // 128)
is on.

* Identity mode (quantizers replaced by identity, fp64) equals textbook
  softmax attention under that combined element mask to 1e-12, for all row
  masks and ragged sizes: this pins which tiles are skipped and that the
  running max / rescale / sum stay correct across skipped tiles.
* A row that sees no key at all has O = 0 and lse = -inf (both modes).
* An all-ones mask reproduces the dense quantized result bit for bit.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from bit_quantized_attention_sage_b200 import synth

from test_oracle_attn import MASKS, _bits, visible_matrix

T = 128


def combined_visible(nq, nkv, mask, mb, bm):
    vis = visible_matrix(nq, nkv, mask, mb)
    tiles = bm[np.arange(nq)[:, None] // T, np.arange(nkv)[None, :] // T].astype(bool)
    return vis & tiles


def random_block_mask(nq, nkv, density, seed):
    rng = np.random.default_rng(seed)
    return (rng.random((-(-nq // T), -(-nkv // T))) < density).astype(np.uint8)


def textbook_masked(q, k, v, vis):
    q, k, v = (torch.from_numpy(np.asarray(a, np.float64)) for a in (q, k, v))
    s = q @ k.T / math.sqrt(q.shape[1])
    s = s.masked_fill(~torch.from_numpy(vis), float("-inf"))
    any_vis = torch.from_numpy(vis.any(1))
    p = torch.softmax(s, dim=-1)
    o = torch.where(any_vis[:, None], p @ v, torch.zeros(()))
    lse = torch.where(any_vis, torch.logsumexp(s, dim=-1), torch.tensor(float("-inf")))
    return o.numpy(), lse.numpy()


@pytest.mark.parametrize("mask,mb", MASKS)
@pytest.mark.parametrize("nq,nkv,density,seed", [(300, 700, 0.5, 1), (1, 900, 0.4, 2),
                                                 (256, 256, 0.7, 3), (130, 1000, 0.3, 4)])
def test_identity_equals_textbook_under_block_mask(mask, mb, nq, nkv, density, seed):
    rng = np.random.default_rng(seed)
    D = 64
    q, k, v = (rng.standard_normal((n, D)) for n in (nq, nkv, nkv))
    bm = random_block_mask(nq, nkv, density, seed + 100)
    rows = np.arange(nq)
    o, lse = oracle.attn_rows_identity(q, k, v, rows, mask, mb, block_mask=bm)
    vis = combined_visible(nq, nkv, mask, mb, bm)
    ref, ref_lse = textbook_masked(q, k, v, vis)
    assert np.abs(o - ref).max() < 1e-12
    seen = vis.any(1)
    assert np.abs(lse[seen] - ref_lse[seen]).max() < 1e-12
    assert np.all(np.isneginf(lse[~seen])) and not o[~seen].any()


def test_rows_without_keys_quantized():
    q, k, v = _bits(200, 400, 128, seed=5)
    qh = oracle.quant_head(q, k, v)
    bm = np.ones((2, 4), np.uint8)
    bm[1, :] = 0  # query tile 1 (rows 128..199) sees nothing
    rows = np.arange(200)
    o, slack, lse = oracle.attn_rows(qh, rows, block_mask=bm)
    assert not o[128:].any() and not slack[128:].any() and np.all(np.isneginf(lse[128:]))
    assert np.all(np.isfinite(lse[:128])) and np.abs(o[:128]).max() > 0


@pytest.mark.parametrize("mask,mb", MASKS)
def test_all_ones_mask_is_dense_bit_exact(mask, mb):
    q, k, v = _bits(300, 700, 128, seed=6, mag=20.0)
    qh = oracle.quant_head(q, k, v)
    rows = np.arange(300)
    o0, s0, l0 = oracle.attn_rows(qh, rows, mask, mb)
    o1, s1, l1 = oracle.attn_rows(qh, rows, mask, mb, block_mask=np.ones((3, 6), np.uint8))
    assert np.array_equal(o0, o1) and np.array_equal(s0, s1) and np.array_equal(l0, l1)


def test_quantized_block_mask_restricts_to_enabled_keys():
    # Quantized mode, one query row that may see all 300 keys, only KV tile 2
    # (keys 256..299) switched on: the result is softmax attention over those
    # 44 keys, within the quantization error.
    q, k, v = _bits(1, 300, 64, seed=7)
    qh = oracle.quant_head(q, k, v)
    bm = np.array([[0, 0, 1]], np.uint8)
    o, _, lse = oracle.attn_rows(qh, np.array([0]), oracle.MASK_NONE, 0, block_mask=bm)
    vis = np.zeros((1, 300), bool)
    vis[0, 256:] = True
    ref, _ = textbook_masked(oracle.bf16_bits_to_f64(q), oracle.bf16_bits_to_f64(k),
                             oracle.bf16_bits_to_f64(v), vis)
    assert np.abs(o - ref).max() < 0.1
    assert np.isfinite(lse).all()
