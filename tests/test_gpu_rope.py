"""GPU parity of sage_quant_qk_rope (RoPE applied to Q and K inside the
quantizer) against the oracle: the quantized tensors bit for bit on ragged
shapes, both head sizes, several heads, per-token angles of a 1D RoPE and of
random angles; the attention output on the rotated quantization within the
usual tolerance."""
import numpy as np
import pytest
import torch

import bit_quantized_attention_sage_b200 as sage
import oracle
from bit_quantized_attention_sage_b200 import synth

from gpu_helpers import check_quant_head, check_rows, rows_of, to_dev

pytestmark = pytest.mark.gpu


def rope_tables(n, D, pos0=0, base=10000.0, rng=None):
    """cos/sin [n, D/2] float32: 1D RoPE angles pos * base^(-2p/D), or random
    angles when rng is given."""
    if rng is not None:
        ang = rng.uniform(-np.pi, np.pi, (n, D // 2))
    else:
        pos = np.arange(pos0, pos0 + n, dtype=np.float64)[:, None]
        ang = pos * base ** (-2.0 * np.arange(D // 2) / D)[None, :]
    return np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)


def run_rope(q, k, v, tabs):
    dev = [torch.from_numpy(t).cuda() for t in tabs]
    qkv = sage.quant_qk(to_dev(q), to_dev(k), to_dev(v), rope=dev)
    assert sage.sync_status() == 0
    return qkv


@pytest.mark.parametrize("B,H,Nq,Nkv,D,random", [(1, 2, 200, 300, 128, False),
                                                (2, 1, 65, 129, 64, True),
                                                (1, 3, 1, 1000, 128, True),
                                                (1, 1, 2040, 4080, 128, False)])
def test_quantized_tensors_bit_exact(B, H, Nq, Nkv, D, random):
    w = synth.Workload("rope", B, H, Nq, Nkv, D, outlier_mag=5.0, seed=Nq + Nkv)
    q, k, v = synth.full(w)
    rng = np.random.default_rng(Nkv) if random else None
    # keys at positions 0 .. Nkv-1, queries at the newest positions
    tabs = (*rope_tables(Nq, D, Nkv - Nq, rng=rng), *rope_tables(Nkv, D, 0, rng=rng))
    qkv = run_rope(q, k, v, tabs)
    for b in range(B):
        for h in range(H):
            check_quant_head(qkv, b, h, oracle.quant_head(q[b, h], k[b, h], v[b, h], rope=tabs))


def test_attention_on_rotated_quantization():
    w = synth.Workload("rope_attn", 1, 2, 300, 700, 128, mask=2, mask_block=100, seed=77)
    q, k, v = synth.full(w)
    tabs = (*rope_tables(300, 128, 400), *rope_tables(700, 128, 0))
    qkv = run_rope(q, k, v, tabs)
    o32 = torch.empty((1, 2, 300, 128), dtype=torch.float32, device="cuda")
    lse = torch.empty((1, 2, 300), dtype=torch.float32, device="cuda")
    o = sage.attn_fwd(qkv, 2, 100, o_f32=o32, lse=lse)
    assert sage.sync_status() == 0
    rows = np.arange(300)
    for h in range(2):
        ref = oracle.quant_head(q[0, h], k[0, h], v[0, h], rope=tabs)
        check_rows(ref, rows, rows_of(o, 0, h, rows), rows_of(o32, 0, h, rows),
                   rows_of(lse, 0, h, rows), 2, 100)


def test_zero_angles_equal_plain_quantizer():
    w = synth.Workload("rope0", 1, 1, 130, 260, 64, seed=5)
    q, k, v = synth.full(w)
    one = (np.ones((130, 32), np.float32), np.zeros((130, 32), np.float32),
           np.ones((260, 32), np.float32), np.zeros((260, 32), np.float32))
    a = run_rope(q, k, v, one)
    b = sage.quant_qk(to_dev(q), to_dev(k), to_dev(v))
    for name in ("q_i8", "q_scale", "k_i8", "k_scale", "k_mean", "v_f8", "v_scale"):
        assert torch.equal(a.view(name), b.view(name)), name
