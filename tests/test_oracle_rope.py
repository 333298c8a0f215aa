"""Pins of the oracle's rotary quantization (``quant_head(..., rope=...)``), no GPU.

The features are quantized after RoPE is applied at their current positions
(the RoPE Repositioning bullet of the "Vidu S1" digest, Infra).  Channel
pairs (2p, 2p+1) are rotated by caller-supplied angles, then quantized exactly
as without rotation.

* Zero angles (cos 1, sin 0) give the unrotated result bit for bit.
* A quarter turn (cos 0, sin 1) maps a pair (x0, x1) to (-x1, x0) exactly, so
  the result equals the plain quantizer on that permuted and negated bf16
  input.  This pins the pair indexing, the sign convention, and that the K
  mean is taken over the rotated keys.
* A half turn (cos -1, sin 0) negates Q and K: the codes and the K mean
  change sign and the scales stay.
* Each row uses its own table row: quarter turns on some rows and none on
  the others equal the plain quantizer on the correspondingly transformed
  input.
* Random angles: every dequantized Q and K value is within half a
  quantization step of the fp64 rotation of the input, and V is untouched.
"""
import numpy as np
import pytest

import oracle
from bit_quantized_attention_sage_b200 import synth

KEYS = ("q8", "qs", "k8", "ks", "mu", "v8", "vs")


def _bits(n, D, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    return synth.f32_to_bf16_bits((rng.standard_normal((n, D)) * scale).astype(np.float32))


def _tables(n, D, cos, sin):
    return (np.full((n, D // 2), cos, np.float32), np.full((n, D // 2), sin, np.float32))


def _f(bits):
    return oracle.bf16_bits_to_f64(bits)


def _quarter(bits):
    """bf16 bits of (x0, x1) -> (-x1, x0) per channel pair (exact in bf16)."""
    x = bits.reshape(bits.shape[0], -1, 2)
    out = np.empty_like(x)
    out[..., 0] = x[..., 1] ^ np.uint16(0x8000)
    out[..., 1] = x[..., 0]
    return out.reshape(bits.shape)


@pytest.mark.parametrize("nq,nkv,D", [(100, 70, 64), (130, 200, 128)])
def test_zero_angles_are_identity(nq, nkv, D):
    q, k, v = _bits(nq, D, 1), _bits(nkv, D, 2), _bits(nkv, D, 3)
    a = oracle.quant_head(q, k, v)
    b = oracle.quant_head(q, k, v, rope=(*_tables(nq, D, 1.0, 0.0), *_tables(nkv, D, 1.0, 0.0)))
    for key in KEYS:
        assert np.array_equal(a[key], b[key]), key


@pytest.mark.parametrize("nq,nkv,D", [(65, 129, 64), (200, 130, 128)])
def test_quarter_turn_is_pair_swap(nq, nkv, D):
    q, k, v = _bits(nq, D, 4), _bits(nkv, D, 5, 3.0), _bits(nkv, D, 6)
    rot = oracle.quant_head(q, k, v, rope=(*_tables(nq, D, 0.0, 1.0), *_tables(nkv, D, 0.0, 1.0)))
    ref = oracle.quant_head(_quarter(q), _quarter(k), v)
    for key in KEYS:
        assert np.array_equal(rot[key], ref[key]), key


def test_half_turn_negates():
    nq, nkv, D = 90, 150, 128
    q, k, v = _bits(nq, D, 7), _bits(nkv, D, 8), _bits(nkv, D, 9)
    a = oracle.quant_head(q, k, v)
    b = oracle.quant_head(q, k, v, rope=(*_tables(nq, D, -1.0, 0.0), *_tables(nkv, D, -1.0, 0.0)))
    assert np.array_equal(b["q8"], -a["q8"]) and np.array_equal(b["qs"], a["qs"])
    assert np.array_equal(b["k8"], -a["k8"]) and np.array_equal(b["ks"], a["ks"])
    assert np.array_equal(b["mu"], -a["mu"])
    assert np.array_equal(b["v8"], a["v8"]) and np.array_equal(b["vs"], a["vs"])


def test_each_row_uses_its_own_angles():
    nq, nkv, D = 130, 77, 64
    q, k, v = _bits(nq, D, 10), _bits(nkv, D, 11), _bits(nkv, D, 12)
    rq = np.arange(nq) % 3 == 0
    rk = np.arange(nkv) % 2 == 1
    qc, qs = _tables(nq, D, 1.0, 0.0)
    kc, ks = _tables(nkv, D, 1.0, 0.0)
    qc[rq], qs[rq] = 0.0, 1.0
    kc[rk], ks[rk] = 0.0, 1.0
    qt, kt = q.copy(), k.copy()
    qt[rq], kt[rk] = _quarter(q[rq]), _quarter(k[rk])
    rot = oracle.quant_head(q, k, v, rope=(qc, qs, kc, ks))
    ref = oracle.quant_head(qt, kt, v)
    for key in KEYS:
        assert np.array_equal(rot[key], ref[key]), key


def _rotate64(x, c, s):
    x0, x1 = x[:, 0::2], x[:, 1::2]
    out = np.empty_like(x)
    out[:, 0::2] = x0 * c - x1 * s
    out[:, 1::2] = x0 * s + x1 * c
    return out


@pytest.mark.parametrize("nq,nkv,D,seed", [(150, 260, 128, 13), (64, 65, 64, 14)])
def test_random_angles_within_half_step(nq, nkv, D, seed):
    rng = np.random.default_rng(seed)
    q, k, v = _bits(nq, D, seed), _bits(nkv, D, seed + 1, 2.0), _bits(nkv, D, seed + 2)
    aq = rng.uniform(-np.pi, np.pi, (nq, D // 2))
    ak = rng.uniform(-np.pi, np.pi, (nkv, D // 2))
    tabs = (np.cos(aq).astype(np.float32), np.sin(aq).astype(np.float32),
            np.cos(ak).astype(np.float32), np.sin(ak).astype(np.float32))
    out = oracle.quant_head(q, k, v, rope=tabs)
    c64 = [t.astype(np.float64) for t in tabs]
    qr = _rotate64(_f(q), c64[0], c64[1])
    kr = _rotate64(_f(k), c64[2], c64[3])
    # Q: |q8 * qs - rot(q)| <= qs / 2, up to the fp32 rounding of the rotation
    qs = np.repeat(out["qs"].astype(np.float64), 64)[:nq, None]
    dq = out["q8"][:nq].astype(np.float64) * qs
    assert np.all(np.abs(dq - qr) <= 0.5 * qs * (1 + 1e-5) + 1e-6 * np.abs(qr).max())
    # K: the mean of the rotated keys, then the same bound on k8 * ks + mu
    assert np.allclose(out["mu"], kr.mean(0), rtol=0, atol=1e-6 * np.abs(kr).max())
    ks = np.repeat(out["ks"].astype(np.float64), 64)[:nkv, None]
    dk = out["k8"][:nkv].astype(np.float64) * ks + out["mu"].astype(np.float64)
    assert np.all(np.abs(dk - kr) <= 0.5 * ks * (1 + 1e-5) + 1e-5 * np.abs(kr).max())
    # V is not rotated
    plain = oracle.quant_head(q, k, v)
    assert np.array_equal(out["v8"], plain["v8"]) and np.array_equal(out["vs"], plain["vs"])
