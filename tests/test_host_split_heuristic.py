"""Host logic of the split-KV choice (no GPU): suggest_kv_splits picks 1 when
the query tiles already fill the GPU in well-balanced waves, and otherwise the
smallest count whose waves are at least 90 % full with at least 8 KV tiles
per range."""
import math

import pytest

import bit_quantized_attention_sage_b200 as sage

SMS = 148  # B200


def wave_fill(ctas, slots):
    w = ctas / slots
    return w / math.ceil(w)


@pytest.mark.parametrize("B,H,Nq,Nkv", [(1, 12, 32760, 32760), (1, 40, 75600, 75600),
                                         (1, 16, 131072, 131072)])
def test_video_shapes_are_not_split(B, H, Nq, Nkv):
    assert sage.suggest_kv_splits(B, H, Nq, Nkv, SMS) == 1


def test_streaming_frame_is_split_in_three():
    # 16 query tiles x 24 heads = 384 CTAs for 296 slots: 1.3 waves unsplit
    assert sage.suggest_kv_splits(1, 24, 2040, 26520, SMS) == 3


@pytest.mark.parametrize("B,H,Nq,Nkv", [(1, 1, 128, 1 << 20), (1, 4, 2040, 26520),
                                         (2, 3, 500, 70000), (1, 1, 1, 4096), (1, 8, 64, 2048)])
def test_choice_obeys_its_rules(B, H, Nq, Nkv):
    s = sage.suggest_kv_splits(B, H, Nq, Nkv, SMS)
    ctas = B * H * -(-Nq // 128)
    tiles = -(-Nkv // 128)
    assert 1 <= s <= 16
    if s > 1:
        assert tiles // s >= 8                        # enough tiles per range
        # no smaller count already filled its waves to 90 %
        for t in range(1, s):
            assert wave_fill(ctas * t, 2 * SMS) < 0.9


def test_few_tiles_are_never_split():
    # fewer than 16 KV tiles: no count keeps 8 tiles per range
    assert sage.suggest_kv_splits(1, 1, 128, 15 * 128, SMS) == 1
