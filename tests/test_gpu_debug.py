"""GPU checks of the pieces under the parity tests: the int32 score tiles the
attention kernel leaves in tensor memory (bit-exact vs int64 brute force),
the device e4m3 conversion (bit-exact vs the oracle encoder), the device
exp2 error bound the oracle's rounding slack assumes, and the bounded-wait
timeout path."""
import numpy as np
import pytest
import torch

import bit_quantized_attention_sage_b200 as sage
import oracle
from bit_quantized_attention_sage_b200 import synth

from gpu_helpers import run, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("D", [128, 64])
def test_qk_int32_tiles_bit_exact(D):
    w = synth.Workload("s_dump", 1, 3, 300, 700, D, k_offset_var=4.0, outlier_mag=20.0, seed=51)
    q, k, v = synth.full(w)
    qkv = sage.quant_qk(to_dev(q), to_dev(k), to_dev(v))
    nqt, nkt = -(-(-(-w.Nq // 64) * 64) // 128), -(-(-(-w.Nkv // 64) * 64) // 128)
    rng = np.random.default_rng(3)
    tiles = [(0, 0, 0), (2, nqt - 1, nkt - 1), (1, 1, 1), (1, nqt - 1, 0)]
    tiles += [(int(rng.integers(3)), int(rng.integers(nqt)), int(rng.integers(nkt)))
              for _ in range(16)]
    got = sage.debug_qk_int32(qkv, tiles).cpu().numpy()
    assert sage.sync_status() == 0
    refs = {}
    for t, (bh, qt, kt) in enumerate(tiles):
        if bh not in refs:
            refs[bh] = oracle.quant_head(q[0, bh], k[0, bh], v[0, bh])
        r = refs[bh]
        q8 = np.zeros((nqt * 128, D), np.int8)
        k8 = np.zeros((nkt * 128, D), np.int8)
        q8[:r["q8"].shape[0]] = r["q8"]
        k8[:r["k8"].shape[0]] = r["k8"]
        ref = oracle.qk_int32(q8, k8, qt * 128, 128, kt * 128, 128)
        assert np.array_equal(got[t], ref), "tile %s" % (tiles[t],)


def test_e4m3_conversion_matches_oracle():
    rng = np.random.default_rng(5)
    codes = np.arange(256, dtype=np.uint8)
    vals = oracle.e4m3_decode(codes)
    pos = np.unique(vals[(vals >= 0) & ~np.isnan(vals)])
    mids = ((pos[1:] + pos[:-1]) / 2).astype(np.float32)
    parts = [mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(1e9)),
             pos.astype(np.float32)]
    for e in range(-24, 12):
        parts.append((rng.random(200000, dtype=np.float32) + 1) * np.float32(2.0 ** e))
    parts.append(rng.integers(0, 2 ** 32, 2_000_000, dtype=np.uint64).astype(np.uint32).view(np.float32))
    x = np.concatenate(parts).astype(np.float32)
    x = np.concatenate([x, -x])
    x = x[~np.isnan(x)]
    got = sage.debug_e4m3(torch.from_numpy(x).cuda()).cpu().numpy()
    assert sage.sync_status() == 0
    ref = oracle.e4m3_encode(x)
    assert np.array_equal(got, ref), "%d mismatches" % (got != ref).sum()


def test_exp2_error_within_oracle_bound():
    # the softmax's argument range: x <= 0 (p = 2^(x) with x = score - max)
    rng = np.random.default_rng(6)
    k = np.arange(0, 127, dtype=np.float64)
    f = np.linspace(0, 1, 1 << 15, endpoint=False)
    grid = -(k[:, None] + f[None, :]).ravel()
    x = np.concatenate([grid, -rng.random(4_000_000) * 126.0]).astype(np.float32)
    got = sage.debug_exp2(torch.from_numpy(x).cuda()).cpu().numpy().astype(np.float64)
    assert sage.sync_status() == 0
    ref = np.exp2(x.astype(np.float64))
    normal = ref >= 2.0 ** -126
    rel = np.abs(got[normal] - ref[normal]) / ref[normal]
    print("max relative error of device exp2: 2^%.2f" % np.log2(rel.max()))
    assert rel.max() <= oracle.EXP2_REL_ERR
    # subnormal results are flushed to zero (such p round to 0 in e4m3 anyway)
    assert np.all(got[~normal] <= 2.0 ** -126)


def test_timeout_path_reports_and_context_survives():
    sage.timeout_probe(2_000_000)        # ~1 ms of SM clock
    assert sage.sync_status() == 4       # SAGE_ERR_TIMEOUT, then cleared
    assert sage.sync_status() == 0
    w = synth.Workload("after_timeout", 1, 1, 128, 256, 128, seed=52)
    q, k, v = synth.full(w)
    run(q, k, v)                         # the context is still usable
