"""GPU parity of the split-KV attention (sage_attn_fwd_split) against the
oracle's split-KV form: every row of small ragged cases under each mask and
several range counts (including more ranges than KV tiles, i.e. empty
ranges), and sampled rows of a streaming-frame shape with the suggested
split count."""
import numpy as np
import pytest
import torch

import bit_quantized_attention_sage_b200 as sage
import oracle
from bit_quantized_attention_sage_b200 import synth

from gpu_helpers import check_rows, rows_of, to_dev

pytestmark = pytest.mark.gpu


def run_split(q, k, v, mask, mb, splits):
    B, H, Nq, D = q.shape
    qkv = sage.quant_qk(to_dev(q), to_dev(k), to_dev(v))
    o32 = torch.empty((B, H, Nq, D), dtype=torch.float32, device="cuda")
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device="cuda")
    o = sage.attn_fwd(qkv, mask, mb, o_f32=o32, lse=lse, kv_splits=splits)
    assert sage.sync_status() == 0
    return o, o32, lse


@pytest.mark.parametrize("mask,mb", [(0, 0), (1, 0), (2, 100)])
@pytest.mark.parametrize("Nq,Nkv,D,splits", [(300, 700, 128, 2), (130, 1000, 64, 3),
                                             (1, 900, 128, 4), (200, 200, 128, 5)])
def test_small_all_rows(mask, mb, Nq, Nkv, D, splits):
    w = synth.Workload("split", 1, 2, Nq, Nkv, D, mask=mask, mask_block=mb, outlier_mag=5.0,
                       seed=Nq + Nkv + splits)
    q, k, v = synth.full(w)
    o, o32, lse = run_split(q, k, v, mask, mb, splits)
    rows = np.arange(Nq)
    for h in range(2):
        ref = oracle.quant_head(q[0, h], k[0, h], v[0, h])
        check_rows(ref, rows, rows_of(o, 0, h, rows), rows_of(o32, 0, h, rows),
                   rows_of(lse, 0, h, rows), mask, mb, kv_splits=splits)


def test_streaming_frame_sampled():
    # one latent frame of queries against a long cache (block-causal), few
    # query tiles: the shape split-KV is for
    w = synth.Workload("split_stream", 1, 4, 2040, 26520, 128, mask=2, mask_block=2040,
                       outlier_mag=5.0, seed=91)
    q, k, v = synth.full(w)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    splits = sage.suggest_kv_splits(1, 4, 2040, 26520, sms)
    assert splits > 1
    o, o32, lse = run_split(q, k, v, 2, 2040, splits)
    rng = np.random.default_rng(5)
    rows = np.unique(np.concatenate([[0, 127, 128, 2039], rng.choice(2040, 40, replace=False)]))
    for h in (0, 3):
        ref = oracle.quant_head(q[0, h], k[0, h], v[0, h])
        check_rows(ref, rows, rows_of(o, 0, h, rows), rows_of(o32, 0, h, rows),
                   rows_of(lse, 0, h, rows), 2, 2040, kv_splits=splits)


def test_drop_in_attention_picks_the_split_form():
    w = synth.Workload("split_dropin", 1, 4, 2040, 26520, 128, mask=2, mask_block=2040, seed=92)
    q, k, v = synth.full(w)
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    splits = sage.suggest_kv_splits(1, 4, 2040, 26520, sms)
    o_auto = sage.attention(qd, kd, vd, mask=("block_causal", 2040))
    qkv = sage.quant_qk(qd, kd, vd)
    o_split = sage.attn_fwd(qkv, 2, 2040, kv_splits=splits)
    o_one = sage.attention(qd, kd, vd, mask=("block_causal", 2040), kv_splits=1)
    o_plain = sage.attn_fwd(qkv, 2, 2040)
    assert sage.sync_status() == 0
    assert torch.equal(o_auto, o_split) and torch.equal(o_one, o_plain)
