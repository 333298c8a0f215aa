"""The hardware-ceiling microbenchmarks (sage_ceiling) run, report through the
status word, and give rates in the range the B200's units allow (broad
bounds: these are measurements, not parity)."""
import pytest
import torch

import bit_quantized_attention_sage_b200 as sage

pytestmark = pytest.mark.gpu

BOUNDS = {  # per SM per clock
    "ex2": (4, 64),
    "ffma2": (32, 1024),
    "cvt_e4m3x2": (2, 256),
    "copy": (2, 256),
    "mma_i8": (2000, 40000),
    "mma_e4m3": (2000, 40000),
}


@pytest.mark.parametrize("kind", sorted(BOUNDS))
def test_ceiling_runs_and_is_plausible(kind):
    scratch = torch.empty(256 << 20, dtype=torch.uint8, device="cuda") if kind == "copy" else None
    r = sage.ceiling(kind, iters=512, n=256, scratch=scratch)
    assert sage.sync_status() == 0
    lo, hi = BOUNDS[kind]
    assert lo <= r["per_sm_per_clock"] <= hi, r
    assert r["per_second"] > 0 and r["blocks"] >= r["blocks_per_sm"] >= 1


def test_mma_rate_scales_with_n():
    # the same number of MMAs with half the N does about half the work
    a = sage.ceiling("mma_i8", iters=1024, n=256)
    b = sage.ceiling("mma_i8", iters=1024, n=64)
    assert sage.sync_status() == 0
    assert b["per_sm_per_clock"] <= a["per_sm_per_clock"] * 1.05
