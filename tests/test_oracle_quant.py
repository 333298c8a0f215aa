"""Pins of the oracle's quantizers and integer scores (no GPU).

The quantized tensors must satisfy the properties that define symmetric
per-block INT8 and per-channel e4m3 quantization, the K channel mean must be
the arithmetic mean, and the integer scores must equal brute-force int64 dot
products.
"""
import numpy as np
import pytest

import oracle
from bit_quantized_attention_sage_b200 import synth


def _head(nq=200, nkv=333, D=64, seed=5, off=4.0, mag=0.0):
    w = synth.Workload("t", 1, 1, nq, nkv, D, k_offset_var=off, outlier_mag=mag, seed=seed)
    return synth.head(w, 0, 0)


def _f(bits):
    return oracle.bf16_bits_to_f64(bits)


@pytest.mark.parametrize("nq,nkv,D", [(200, 333, 64), (64, 64, 128), (1, 1, 128), (129, 65, 64)])
def test_block_int8_invariants(nq, nkv, D):
    q, k, v = _head(nq, nkv, D)
    r = oracle.quant_head(q, k, v)
    x = _f(q)
    nb = -(-nq // 64)
    assert r["q8"].shape == (nb * 64, D) and r["qs"].shape == (nb,)
    for b in range(nb):
        blk = x[b * 64:(b + 1) * 64]
        qb = r["q8"][b * 64:b * 64 + blk.shape[0]].astype(np.float64)
        s = float(r["qs"][b])
        a = np.abs(blk).max()
        assert s == np.float32(np.float32(a) / np.float32(127))
        assert np.abs(qb).max() == 127
        assert np.all(np.abs(qb) <= 127)
        # reconstruction within half a step, plus |x| * (s * inv - 1) <= 127 * 2^-22 * s
        assert np.all(np.abs(blk - qb * s) <= s * (0.5 + 127 * 2.0 ** -21))
    assert not r["q8"][nq:].any()  # padding rows are zero


def test_zero_block_gives_zero_scale():
    q, k, v = _head(130, 130, 64)
    q[64:128] = 0
    r = oracle.quant_head(q, k, v)
    assert r["qs"][1] == 0 and not r["q8"][64:128].any()
    assert r["qs"][0] > 0 and r["qs"][2] > 0


def test_rounding_is_half_to_even():
    # one block whose absmax is 127 gives inv = 1 exactly, so q = rne(x)
    D = 64
    x = np.zeros((64, D), np.float32)
    x[0, 0] = 127.0
    x[1, :6] = [0.5, 1.5, 2.5, -0.5, -1.5, -2.5]
    bits = synth.f32_to_bf16_bits(x)
    r = oracle.quant_head(bits, bits, bits)
    assert r["qs"][0] == 1.0
    assert list(r["q8"][1, :6]) == [0, 2, 2, 0, -2, -2]


def test_k_mean_is_the_mean():
    q, k, v = _head(100, 1000, 128, off=4.0)
    r = oracle.quant_head(q, k, v)
    ref = _f(k).mean(axis=0)
    # canonical fp64 order vs numpy pairwise: equal up to one fp32 rounding step
    ulp = np.spacing(np.abs(ref).astype(np.float32))
    assert np.all(np.abs(r["mu"].astype(np.float64) - ref) <= ulp)


def test_k_is_quantized_after_smoothing():
    q, k, v = _head(64, 500, 64, off=4.0)
    r = oracle.quant_head(q, k, v)
    ks = (_f(k).astype(np.float32) - r["mu"][None, :]).astype(np.float64)
    for b in range(-(-500 // 64)):
        blk = ks[b * 64:(b + 1) * 64]
        s = float(r["ks"][b])
        kb = r["k8"][b * 64:b * 64 + blk.shape[0]].astype(np.float64)
        assert np.all(np.abs(blk - kb * s) <= s * (0.5 + 127 * 2.0 ** -21))
        assert np.abs(kb).max() == 127
    # smoothing removes the large per-channel offset: scales shrink
    raw = oracle.quant_head(q, k - 0, v)  # same call, sanity of determinism
    assert np.array_equal(raw["k8"], r["k8"])


def test_v_per_channel_e4m3():
    q, k, v = _head(64, 300, 64)
    r = oracle.quant_head(q, k, v)
    x = _f(v)
    dec = oracle.e4m3_decode(r["v8"])
    a = np.abs(x).max(axis=0)
    assert np.array_equal(r["vs"], (a.astype(np.float32) / np.float32(448)).astype(np.float32))
    # the absmax element of each channel lands exactly on 448
    assert np.all(np.abs(dec).max(axis=0) == 448.0)
    rec = dec * r["vs"][None, :].astype(np.float64)
    # 3 mantissa bits: half-step relative error 2^-4 in the normal range,
    # absolute 2^-10 * scale in the subnormal range
    tol = np.maximum(np.abs(x) * 2.0 ** -4, 2.0 ** -10 * r["vs"][None, :]) * (1 + 1e-6)
    assert np.all(np.abs(rec - x) <= tol)


def test_v_zero_channel():
    q, k, v = _head(64, 100, 64)
    v[:, 3] = 0
    r = oracle.quant_head(q, k, v)
    assert r["vs"][3] == 0 and not r["v8"][:, 3].any()


def test_qk_int32_brute_force():
    q, k, v = _head(150, 260, 128, off=4.0, mag=20.0)
    r = oracle.quant_head(q, k, v)
    got = oracle.qk_int32(r["q8"], r["k8"], 10, 100, 30, 200)
    ref = r["q8"][10:110].astype(np.int64) @ r["k8"][30:230].astype(np.int64).T
    assert np.array_equal(got, ref.astype(np.int32))
    assert np.abs(ref).max() <= 127 * 127 * 128
