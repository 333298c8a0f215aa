"""Shared helpers of the GPU parity tests: run the library through its C ABI
and compare with the CPU oracle on the same seeded inputs."""
import numpy as np
import torch

import bit_quantized_attention_sage_b200 as sage
import oracle

# Tolerances: O within 2e-3 (absolute) of the oracle's same-quantization
# output plus the per-element e4m3 rounding slack of P; bf16 O additionally
# within half a bf16 ulp of the oracle value; lse within 1e-4.
O_ATOL = 2e-3
LSE_ATOL = 1e-4


def to_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def run(q, k, v, mask=0, mb=0, block_mask=None):
    """Quantize + attend on the GPU (block-sparse when `block_mask`, a numpy
    uint8 [B, H, n_qt, n_kt], is given).  Returns (qkv, o_bf16, o_f32, lse)."""
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    B, H, Nq, D = q.shape
    qkv = sage.quant_qk(qd, kd, vd)
    o_f32 = torch.empty((B, H, Nq, D), dtype=torch.float32, device="cuda")
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device="cuda")
    bm = None if block_mask is None else torch.from_numpy(
        np.ascontiguousarray(block_mask, np.uint8)).cuda()
    o = sage.attn_fwd(qkv, mask, mb, o_f32=o_f32, lse=lse, block_mask=bm)
    st = sage.sync_status()
    assert st == 0, "device status %d" % st
    return qkv, o, o_f32, lse


def f32_bits(a):
    return np.ascontiguousarray(a, np.float32).view(np.int32)


def check_quant_head(qkv, b, h, ref):
    """Bit-exact comparison of one head's quantized tensors with the oracle's."""
    s = qkv.shape
    q8 = qkv.view("q_i8")[b, h].cpu().numpy()
    k8 = qkv.view("k_i8")[b, h].cpu().numpy()
    assert np.array_equal(q8, ref["q8"]), "q_i8 differs"
    assert np.array_equal(k8, ref["k8"]), "k_i8 differs"
    for name, key in (("q_scale", "qs"), ("k_scale", "ks"), ("k_mean", "mu"), ("v_scale", "vs")):
        got = qkv.view(name)[b, h].cpu().numpy()
        assert np.array_equal(f32_bits(got), f32_bits(ref[key])), name + " differs"
    v8 = qkv.view("v_f8")[b, h].cpu().numpy()  # [Nkv_pad, D]
    assert np.array_equal(v8[:s.Nkv], ref["v8"]), "v_f8 differs"
    assert not v8[s.Nkv:].any(), "v_f8 padding not zero"


def bf16_half_ulp(x):
    a = np.abs(np.asarray(x, np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return 0.5 * 2.0 ** (e - 7)


def check_rows(ref_head, rows, o_bf16_rows, o_f32_rows, lse_rows, mask, mb, block_mask=None,
               kv_splits=1, window=None):
    """O and lse of the given rows against the oracle (same quantized inputs;
    `block_mask`: this head's [n_qt, n_kt] tile mask, if any; `kv_splits`:
    the split-KV form's range count; `window`: (frame, win, sink) of the
    sliding-window mask)."""
    o_ref, slack, lse_ref = oracle.attn_rows(ref_head, rows, mask, mb, block_mask=block_mask,
                                             kv_splits=kv_splits, window=window)
    tol = O_ATOL + slack
    # the rounding slack's share of the tolerance, for the test log
    print("slack: max %.3g, mean %.3g, share of outputs with slack %.5f (%d rows)" % (
        float(slack.max(initial=0.0)), float(slack.mean()) if slack.size else 0.0,
        float((slack > 0).mean()) if slack.size else 0.0, len(rows)))
    err32 = np.abs(o_f32_rows.astype(np.float64) - o_ref)
    bad = err32 > tol
    assert not bad.any(), "fp32 O: %d elements out of tolerance, worst excess %.3g" % (
        bad.sum(), (err32 - tol).max())
    errb = np.abs(o_bf16_rows.astype(np.float64) - o_ref)
    tolb = tol + bf16_half_ulp(o_ref)
    assert not (errb > tolb).any(), "bf16 O out of tolerance"
    empty = np.isneginf(lse_ref)  # rows that see no key (block masks only)
    assert np.all(np.isneginf(lse_rows[empty])), "lse of rows without keys is not -inf"
    assert np.abs(lse_rows[~empty].astype(np.float64) - lse_ref[~empty]).max(initial=0.0) \
        <= LSE_ATOL
    return o_ref, slack


def rows_of(t, b, h, rows):
    return t[b, h].float().cpu().numpy()[rows] if t.dim() == 4 else t[b, h].cpu().numpy()[rows]
