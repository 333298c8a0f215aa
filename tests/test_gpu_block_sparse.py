"""GPU parity of block-sparse skipping (sage_attn_fwd_block_sparse) against
the oracle given the same 128 x 128 tile mask: every row of small cases
(random masks over several tiles and ragged tails, every row mask, D 64 and
128), CTAs whose tiles are all switched off, rows that see no key inside a
CTA that does visit tiles, the all-ones mask against the dense call, and
sampled rows of a 480p-shaped workload at 50 % tile density."""
import numpy as np
import pytest
import torch

import oracle
from bit_quantized_attention_sage_b200 import synth

from gpu_helpers import check_quant_head, check_rows, rows_of, run

pytestmark = pytest.mark.gpu

W = synth.Workload


def random_mask(w, density, seed):
    rng = np.random.default_rng(seed)
    shape = (w.B, w.H, -(-w.Nq // 128), -(-w.Nkv // 128))
    return (rng.random(shape) < density).astype(np.uint8)


CASES = [
    (W("bs_none_d128", 1, 2, 700, 900, 128, k_offset_var=4.0, seed=51), 0.5),
    (W("bs_causal_d64", 2, 1, 300, 1000, 64, mask=1, outlier_mag=20.0, seed=52), 0.6),
    (W("bs_blockcausal", 1, 2, 520, 1300, 128, mask=2, mask_block=200, seed=53), 0.4),
    (W("bs_single_row", 1, 1, 1, 1000, 128, seed=54), 0.5),
    (W("bs_dense_tail_16", 1, 1, 256, 1168, 128, outlier_mag=5.0, seed=55), 0.7),
]


def _check_all(w, q, k, v, bm, outs):
    qkv, o, o32, lse = outs
    for b in range(w.B):
        for h in range(w.H):
            ref = oracle.quant_head(q[b, h], k[b, h], v[b, h])
            check_quant_head(qkv, b, h, ref)
            r = np.arange(w.Nq)
            check_rows(ref, r, rows_of(o, b, h, r), rows_of(o32, b, h, r), rows_of(lse, b, h, r),
                       w.mask, w.mask_block, block_mask=bm[b, h])


@pytest.mark.parametrize("w,density", CASES, ids=lambda c: c.name if hasattr(c, "name") else "")
def test_small_all_rows(w, density):
    q, k, v = synth.full(w)
    bm = random_mask(w, density, w.seed)
    _check_all(w, q, k, v, bm, run(q, k, v, w.mask, w.mask_block, block_mask=bm))


def test_empty_ctas_and_rows():
    # causal, Nq = 200, Nkv = 300 (queries are keys 100..299): query tile 0
    # visits only KV tile 1, so its rows 0..27 (limits 101..128) see no key;
    # query tile 1 has every tile off (a CTA with nothing to visit)
    w = W("bs_empty", 1, 1, 200, 300, 128, mask=1, seed=56)
    q, k, v = synth.full(w)
    bm = np.zeros((1, 1, 2, 3), np.uint8)
    bm[0, 0, 0, 1] = 1
    qkv, o, o32, lse = run(q, k, v, w.mask, w.mask_block, block_mask=bm)
    lse_h = lse[0, 0].cpu().numpy()
    assert np.all(np.isneginf(lse_h[:28])) and np.all(np.isfinite(lse_h[28:128]))
    assert np.all(np.isneginf(lse_h[128:]))
    assert not o32[0, 0, :28].any() and not o32[0, 0, 128:].any()
    assert not o[0, 0, 128:].float().any()
    _check_all(w, q, k, v, bm, (qkv, o, o32, lse))


def test_all_ones_equals_dense():
    w = W("bs_ones", 1, 2, 640, 1100, 128, mask=2, mask_block=300, outlier_mag=20.0, seed=57)
    q, k, v = synth.full(w)
    bm = np.ones((1, 2, 5, 9), np.uint8)
    _, o1, a1, l1 = run(q, k, v, w.mask, w.mask_block, block_mask=bm)
    _, o0, a0, l0 = run(q, k, v, w.mask, w.mask_block)
    assert torch.equal(o0, o1) and torch.equal(a0, a1) and torch.equal(l0, l1)


def test_480p_half_density_sampled():
    w = synth.P480
    q, k, v = synth.full(w)
    bm = random_mask(w, 0.5, 58)
    qkv, o, o32, lse = run(q, k, v, w.mask, w.mask_block, block_mask=bm)
    rng = np.random.default_rng(58)
    for bh in (0, w.B * w.H - 1):
        b, h = divmod(bh, w.H)
        ref = oracle.quant_head(q[b, h], k[b, h], v[b, h])
        rows = np.sort(rng.choice(w.Nq, 48, replace=False))
        check_rows(ref, rows, rows_of(o, b, h, rows), rows_of(o32, b, h, rows),
                   rows_of(lse, b, h, rows), w.mask, w.mask_block, block_mask=bm[b, h])
