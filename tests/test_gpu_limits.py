"""GPU parity at the largest sizes the library accepts.

* B*H = 65535 heads (the largest the shape check accepts; the quantizer and
  attention grids put the heads on their y dimension, whose limit this is),
  one token each: sampled heads' quantized tensors are bit-exact, O matches
  the oracle, unsplit and in split-KV form with more ranges than KV tiles.
* A block-sparse call over 6144 KV tiles (786432 keys, the most its tile
  bitmap holds): sampled rows match the oracle's block-sparse form.
* The rotary quantizer at its token limit, 65535 blocks of 64 keys (its
  grid puts the blocks on the y dimension): bit-exact with the oracle.
"""
import numpy as np
import pytest
import torch

import bit_quantized_attention_sage_b200 as sage
import oracle
from bit_quantized_attention_sage_b200 import synth

from gpu_helpers import check_quant_head, check_rows, rows_of, to_dev

pytestmark = pytest.mark.gpu

MAX_HEADS = 65535
MAX_SPARSE_KEYS = 6144 * 128
MAX_ROPE_TOKENS = 65535 * 64


def test_most_heads_one_token_each():
    rng = np.random.default_rng(65535)
    shape = (1, MAX_HEADS, 1, 64)
    q = synth.f32_to_bf16_bits(rng.standard_normal(shape).astype(np.float32))
    k = synth.f32_to_bf16_bits((rng.standard_normal(shape) + 3.0).astype(np.float32))
    v = synth.f32_to_bf16_bits(rng.standard_normal(shape).astype(np.float32))
    qkv = sage.quant_qk(to_dev(q), to_dev(k), to_dev(v))
    outs = {}
    for splits in (1, 2):
        o32 = torch.empty(shape, dtype=torch.float32, device="cuda")
        lse = torch.empty(shape[:3], dtype=torch.float32, device="cuda")
        o = sage.attn_fwd(qkv, 0, 0, o_f32=o32, lse=lse, kv_splits=splits)
        assert sage.sync_status() == 0
        outs[splits] = (o, o32, lse)
    heads = sorted({0, 1, MAX_HEADS - 1} | set(rng.choice(MAX_HEADS, 5).tolist()))
    rows = np.arange(1)
    for h in heads:
        ref = oracle.quant_head(q[0, h], k[0, h], v[0, h])
        check_quant_head(qkv, 0, h, ref)
        for splits, (o, o32, lse) in outs.items():
            check_rows(ref, rows, rows_of(o, 0, h, rows), rows_of(o32, 0, h, rows),
                       rows_of(lse, 0, h, rows), 0, 0, kv_splits=splits)


def test_block_sparse_at_its_tile_limit():
    w = synth.Workload("limit_sparse", 1, 1, 200, MAX_SPARSE_KEYS, 64, seed=6144)
    q, k, v = synth.full(w)
    n_qt, n_kt = -(-w.Nq // 128), MAX_SPARSE_KEYS // 128
    rng = np.random.default_rng(7)
    bm = (rng.random((1, 1, n_qt, n_kt)) < 0.5).astype(np.uint8)
    bm[0, 0, :, -1] = 1  # the last tile is visited
    qkv = sage.quant_qk(to_dev(q), to_dev(k), to_dev(v))
    o32 = torch.empty((1, 1, w.Nq, 64), dtype=torch.float32, device="cuda")
    lse = torch.empty((1, 1, w.Nq), dtype=torch.float32, device="cuda")
    o = sage.attn_fwd(qkv, 0, 0, o_f32=o32, lse=lse, block_mask=torch.from_numpy(bm).cuda())
    assert sage.sync_status() == 0
    ref = oracle.quant_head(q[0, 0], k[0, 0], v[0, 0])
    rows = np.array([0, 1, 127, 128, 150, 199])
    check_rows(ref, rows, rows_of(o, 0, 0, rows), rows_of(o32, 0, 0, rows),
               rows_of(lse, 0, 0, rows), 0, 0, block_mask=bm[0, 0])
    # one tile more is refused before anything is enqueued
    w2 = synth.Workload("limit_sparse2", 1, 1, 64, MAX_SPARSE_KEYS + 1, 64, seed=1)
    q2, k2, v2 = synth.full(w2)
    qkv2 = sage.quant_qk(to_dev(q2), to_dev(k2), to_dev(v2))
    bm2 = torch.ones((1, 1, 1, n_kt + 1), dtype=torch.uint8, device="cuda")
    with pytest.raises(RuntimeError):
        sage.attn_fwd(qkv2, 0, 0, block_mask=bm2)
    assert sage.sync_status() == 0


def test_rotary_quantizer_at_its_token_limit():
    rng = np.random.default_rng(4194240)
    nq, nkv, D = 64, MAX_ROPE_TOKENS, 64
    q = synth.f32_to_bf16_bits(rng.standard_normal((1, 1, nq, D), dtype=np.float32))
    k = synth.f32_to_bf16_bits(rng.standard_normal((1, 1, nkv, D), dtype=np.float32))
    v = synth.f32_to_bf16_bits(rng.standard_normal((1, 1, nkv, D), dtype=np.float32))
    ang_q = rng.uniform(-np.pi, np.pi, (nq, D // 2))
    ang_k = rng.uniform(-np.pi, np.pi, (nkv, D // 2)).astype(np.float32)
    tabs = (np.cos(ang_q).astype(np.float32), np.sin(ang_q).astype(np.float32),
            np.cos(ang_k), np.sin(ang_k))
    qkv = sage.quant_qk(to_dev(q), to_dev(k), to_dev(v),
                        rope=[torch.from_numpy(t).cuda() for t in tabs])
    assert sage.sync_status() == 0
    check_quant_head(qkv, 0, 0, oracle.quant_head(q[0, 0], k[0, 0], v[0, 0], rope=tabs))
