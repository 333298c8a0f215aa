"""The benchmark's TOPS numerator counts visible (query, key) pairs
(synth.Workload.visible_pairs).  It must equal the count of the explicit
boolean masks the oracle tests build from the mask definitions (no GPU)."""
import pytest

from bit_quantized_attention_sage_b200 import synth
from test_oracle_attn import visible_matrix
from test_oracle_window import window_visible

W = synth.Workload


@pytest.mark.parametrize("nq,nkv,mask,mb", [(300, 700, 0, 0), (300, 700, 1, 0), (77, 333, 2, 100),
                                            (640, 640, 1, 0), (2040, 4080, 2, 2040)])
def test_prefix_masks(nq, nkv, mask, mb):
    w = W("c", 1, 1, nq, nkv, 64, mask=mask, mask_block=mb)
    assert w.visible_pairs() == int(visible_matrix(nq, nkv, mask, mb).sum())


@pytest.mark.parametrize("nq,nkv,frame,win,sink", [(300, 700, 40, 3, 17), (500, 500, 70, 2, 90),
                                                   (2040, 26520, 2040, 4, 2040), (96, 2100, 96, 5, 0),
                                                   (20, 60, 5, 2, 80)])
def test_sliding_window(nq, nkv, frame, win, sink):
    w = W("c", 1, 1, nq, nkv, 64, mask=3, mask_block=frame, win=win, sink=sink)
    assert w.visible_pairs() == int(window_visible(nq, nkv, frame, win, sink).sum())


def test_ops_scale_with_heads_and_d():
    w = W("c", 2, 3, 100, 200, 128)
    assert w.ops() == 4 * 128 * 2 * 3 * 100 * 200
