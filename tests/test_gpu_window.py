"""GPU parity of the sliding-window attention with a persistent reference
context (sage_attn_fwd_window) against the oracle's window mask.

* Every row of small ragged cases: frames shorter and longer than a KV tile,
  reference contexts that do and do not end on a tile boundary, query tiles
  inside the reference context, a gap of skipped tiles between the reference
  context and the window, D = 64 and 128, one and several KV ranges.
* sink = 0 with a window wider than the cache: the block-causal kernel's
  output, bit for bit (same tiles, same order, same arithmetic).
* Sampled rows of a streaming step: the newest 2040-token frame against a
  26520-token cache, reference context = the first frame, window = 4 frames,
  with the suggested KV split count and unsplit.
* The drop-in attention() with mask=("window", ...).
"""
import numpy as np
import pytest
import torch

import bit_quantized_attention_sage_b200 as sage
import oracle
from bit_quantized_attention_sage_b200 import synth

from gpu_helpers import bf16_half_ulp, check_rows, rows_of, to_dev

pytestmark = pytest.mark.gpu


def run_window(q, k, v, window, splits=1):
    B, H, Nq, D = q.shape
    qkv = sage.quant_qk(to_dev(q), to_dev(k), to_dev(v))
    o32 = torch.empty((B, H, Nq, D), dtype=torch.float32, device="cuda")
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device="cuda")
    o = sage.attn_fwd(qkv, o_f32=o32, lse=lse, kv_splits=splits, window=window)
    assert sage.sync_status() == 0
    return qkv, o, o32, lse


CASES = [  # Nq, Nkv, D, frame, win, sink, splits
    (300, 700, 128, 40, 3, 17, 1),       # frames shorter than a tile, ragged
    (300, 700, 128, 40, 3, 17, 3),
    (256, 1000, 64, 200, 1, 150, 1),     # window = the query's own frame
    (130, 1000, 128, 64, 4, 300, 2),
    (500, 500, 128, 70, 2, 90, 1),       # early query tiles inside the reference context
    (500, 500, 64, 70, 2, 90, 4),
    (96, 2100, 128, 96, 5, 500, 1),      # gap of skipped tiles after the reference context
    (128, 4096, 128, 256, 2, 128, 2),    # tile-aligned, gap, 2 ranges
    (1, 900, 128, 100, 2, 64, 1),        # a single query row
    (200, 3000, 128, 300, 3, 0, 3),      # no reference context
]


@pytest.mark.parametrize("Nq,Nkv,D,frame,win,sink,splits", CASES)
def test_small_all_rows(Nq, Nkv, D, frame, win, sink, splits):
    w = synth.Workload("window", 1, 2, Nq, Nkv, D, outlier_mag=5.0,
                       seed=Nq + Nkv + frame + sink + splits)
    q, k, v = synth.full(w)
    _, o, o32, lse = run_window(q, k, v, (frame, win, sink), splits)
    rows = np.arange(Nq)
    for h in range(2):
        ref = oracle.quant_head(q[0, h], k[0, h], v[0, h])
        check_rows(ref, rows, rows_of(o, 0, h, rows), rows_of(o32, 0, h, rows),
                   rows_of(lse, 0, h, rows), 0, 0, kv_splits=splits, window=(frame, win, sink))


@pytest.mark.parametrize("Nq,Nkv,frame,splits", [(300, 700, 40, 1), (1000, 3000, 330, 1),
                                                 (300, 2000, 256, 3)])
def test_wide_window_without_reference_equals_block_causal(Nq, Nkv, frame, splits):
    w = synth.Workload("window_bc", 1, 2, Nq, Nkv, 128, outlier_mag=5.0, seed=Nkv + frame)
    q, k, v = synth.full(w)
    qkv, o, o32, lse = run_window(q, k, v, (frame, Nkv // frame + 1, 0), splits)
    o32b = torch.empty_like(o32)
    lseb = torch.empty_like(lse)
    ob = sage.attn_fwd(qkv, sage.MASK_BLOCK_CAUSAL, frame, o_f32=o32b, lse=lseb,
                       kv_splits=splits)
    assert sage.sync_status() == 0
    assert torch.equal(o, ob) and torch.equal(o32, o32b) and torch.equal(lse, lseb)


@pytest.mark.parametrize("auto", [False, True])
def test_streaming_step_sampled(auto):
    w = synth.STREAMING_WINDOW
    w = synth.Workload(w.name, 1, 4, w.Nq, w.Nkv, w.D, mask=3, mask_block=w.mask_block,
                       k_offset_var=4.0, outlier_mag=5.0, seed=93, win=w.win, sink=w.sink)
    q, k, v = synth.full(w)
    window = (w.mask_block, w.win, w.sink)
    splits = "auto" if auto else 1
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    qkv = sage.quant_qk(qd, kd, vd)
    o32 = torch.empty((1, 4, w.Nq, w.D), dtype=torch.float32, device="cuda")
    lse = torch.empty((1, 4, w.Nq), dtype=torch.float32, device="cuda")
    o = sage.attn_fwd(qkv, o_f32=o32, lse=lse, kv_splits=splits, window=window)
    assert sage.sync_status() == 0
    if auto:
        sms = torch.cuda.get_device_properties(0).multi_processor_count
        nkv = min(w.Nkv, w.sink + (w.win + 1) * w.mask_block + 128)
        n = sage.suggest_kv_splits(1, 4, w.Nq, nkv, sms)
        assert n > 1
    else:
        n = 1
    rng = np.random.default_rng(7)
    rows = np.unique(np.concatenate([[0, 127, 128, w.Nq - 1], rng.choice(w.Nq, 40, replace=False)]))
    for h in (0, 3):
        ref = oracle.quant_head(q[0, h], k[0, h], v[0, h])
        check_rows(ref, rows, rows_of(o, 0, h, rows), rows_of(o32, 0, h, rows),
                   rows_of(lse, 0, h, rows), 0, 0, kv_splits=n, window=window)


def test_drop_in_attention_window():
    w = synth.Workload("window_dropin", 1, 3, 640, 5000, 128, outlier_mag=5.0, seed=17)
    q, k, v = synth.full(w)
    window = (320, 3, 400)
    o = sage.attention(to_dev(q), to_dev(k), to_dev(v), mask=("window",) + window)
    assert sage.sync_status() == 0
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    n = sage.suggest_kv_splits(1, 3, 640, min(5000, 400 + 4 * 320 + 128), sms)
    rows = np.arange(0, 640, 7)
    ref = oracle.quant_head(q[0, 1], k[0, 1], v[0, 1])
    o_ref, slack, _ = oracle.attn_rows(ref, rows, kv_splits=n, window=window)
    got = o[0, 1].float().cpu().numpy()[rows].astype(np.float64)
    assert np.all(np.abs(got - o_ref) <= 2e-3 + slack + bf16_half_ulp(o_ref))
