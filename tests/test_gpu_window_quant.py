"""GPU parity of the windowed quantization of the streaming cache
(sage_quant_qk_window): only the keys a sliding-window step attends to -- the
reference context and the window -- are quantized, with their own K mean and
V channel scales, optionally rotated at their current positions.

* The codes, scales and mean equal the oracle's quantizer on the gathered
  keys (oracle.window_keys) bit for bit: ragged frames, a reference context
  that does and does not end on a 64-token block, D = 64 and 128, with and
  without RoPE, a block straddling the gap.
* The window attention over the gathered quantization matches the oracle's
  same-quantization window attention on every row.
* Sampled rows of the streaming step (2040-token frame, 26520-token cache,
  reference context = the first frame, window = 4 frames).
"""
import numpy as np
import pytest
import torch

import bit_quantized_attention_sage_b200 as sage
import oracle
from bit_quantized_attention_sage_b200 import synth

from gpu_helpers import check_quant_head, check_rows, rows_of, to_dev

pytestmark = pytest.mark.gpu


def _angles(n, D, pos0):
    pos = np.arange(pos0, pos0 + n, dtype=np.float64)[:, None]
    inv = 10000.0 ** (-2.0 * np.arange(D // 2) / D)
    ang = pos * inv[None, :]
    return np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)


CASES = [  # B, H, Nq, Nkv, D, frame, win, sink, rope
    (1, 2, 40, 700, 128, 40, 3, 40, False),
    (1, 2, 130, 1000, 64, 64, 4, 300, False),   # block straddles the gap
    (2, 1, 96, 2100, 128, 96, 5, 500, True),
    (1, 1, 1, 900, 128, 100, 2, 64, True),
    (1, 3, 300, 700, 128, 40, 3, 17, False),
]


@pytest.mark.parametrize("case", CASES)
def test_windowed_quantization_and_attention(case):
    B, H, Nq, Nkv, D, frame, win, sink, rope = case
    w = synth.Workload("winq", B, H, Nq, Nkv, D, k_offset_var=4.0, seed=120 + Nkv)
    q, k, v = synth.full(w)
    idx = oracle.window_keys(Nq, Nkv, frame, win, sink)
    tabs = None
    if rope:
        qc, qs = _angles(Nq, D, len(idx) - Nq)
        kc, ks = _angles(len(idx), D, 0)
        tabs = tuple(torch.from_numpy(t).cuda() for t in (qc, qs, kc, ks))
    qkv = sage.quant_qk_window(to_dev(q), to_dev(k), to_dev(v), frame, win, sink, rope=tabs)
    assert qkv.shape.Nkv == len(idx)
    o32 = torch.empty((B, H, Nq, D), dtype=torch.float32, device="cuda")
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device="cuda")
    o = sage.attn_fwd(qkv, o_f32=o32, lse=lse, window=(frame, win, sink))
    assert sage.sync_status() == 0
    rows = np.arange(Nq)
    for b in range(B):
        for h in range(H):
            r = (qc, qs, kc, ks) if rope else None
            ref = oracle.quant_head(q[b, h], k[b, h][idx], v[b, h][idx], rope=r)
            check_quant_head(qkv, b, h, ref)
            check_rows(ref, rows, rows_of(o, b, h, rows), rows_of(o32, b, h, rows),
                       rows_of(lse, b, h, rows), 0, 0, window=(frame, win, sink))


def test_streaming_step_sampled_rows():
    w = synth.STREAMING_WINDOW
    q, k, v = synth.full(w)
    qkv = sage.quant_qk_window(to_dev(q), to_dev(k), to_dev(v), w.mask_block, w.win, w.sink)
    idx = oracle.window_keys(w.Nq, w.Nkv, w.mask_block, w.win, w.sink)
    assert qkv.shape.Nkv == len(idx) == 10200
    rng = np.random.default_rng(5)
    rows = np.sort(rng.choice(w.Nq, size=96, replace=False))
    refs = {h: oracle.quant_head(q[0, h], k[0, h][idx], v[0, h][idx]) for h in (0, 11, 23)}
    for h, ref in refs.items():
        check_quant_head(qkv, 0, h, ref)
    for splits in (1, 3):  # unsplit and the benchmark's KV ranges
        o32 = torch.empty((w.B, w.H, w.Nq, w.D), dtype=torch.float32, device="cuda")
        lse = torch.empty((w.B, w.H, w.Nq), dtype=torch.float32, device="cuda")
        o = sage.attn_fwd(qkv, o_f32=o32, lse=lse, kv_splits=splits,
                          window=(w.mask_block, w.win, w.sink))
        assert sage.sync_status() == 0
        for h, ref in refs.items():
            check_rows(ref, rows, rows_of(o, 0, h, rows), rows_of(o32, 0, h, rows),
                       rows_of(lse, 0, h, rows), 0, 0, kv_splits=splits,
                       window=(w.mask_block, w.win, w.sink))
