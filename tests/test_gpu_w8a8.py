"""GPU parity of the per-block W8A8 linear layer against the oracle: the
quantized activations, weights and their scales bit for bit, and the GEMM's
fp32 output bit for bit (same exact group products, same fp32 promotion
order), its bf16 output equal to the oracle's value rounded to bf16.  Small
shapes compare every row (ragged M, one and several groups, zero groups,
more tiles than SMs); DiT-sized shapes compare sampled rows."""
import numpy as np
import pytest
import torch

import bit_quantized_attention_sage_b200 as sage
import oracle
from bit_quantized_attention_sage_b200 import synth

pytestmark = pytest.mark.gpu


def bits(shape, seed, outliers=0):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal(shape).astype(np.float32)
    if outliers:
        x[:, rng.choice(shape[1], outliers, replace=False)] *= 30.0
    return synth.f32_to_bf16_bits(x)


def dev(b):
    return torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).view(torch.bfloat16).cuda()


def run(x, w):
    xq, sx = sage.w8a8_quant_act(dev(x))
    wq, sw = sage.w8a8_quant_weight(dev(w))
    y32 = torch.empty((x.shape[0], w.shape[0]), dtype=torch.float32, device="cuda")
    y = sage.w8a8_gemm(xq, sx, wq, sw, y_f32=y32)
    assert sage.sync_status() == 0
    return xq, sx, wq, sw, y, y32


def check(x, w, rows=None):
    xq, sx, wq, sw, y, y32 = run(x, w)
    rxq, rsx = oracle.w8a8_quant_act(x)
    rwq, rsw = oracle.w8a8_quant_weight(w)
    np.testing.assert_array_equal(xq.cpu().numpy(), rxq)
    np.testing.assert_array_equal(sx.cpu().numpy().view(np.int32), rsx.view(np.int32))
    np.testing.assert_array_equal(wq.cpu().numpy(), rwq)
    np.testing.assert_array_equal(sw.cpu().numpy().view(np.int32), rsw.view(np.int32))
    rows = np.arange(x.shape[0]) if rows is None else rows
    ry = oracle.w8a8_gemm_rows(rxq, rsx, rwq, rsw, rows)
    got32 = y32.cpu().numpy()[rows]
    np.testing.assert_array_equal(got32.view(np.int32), ry.view(np.int32))
    gotb = y.view(torch.int16).cpu().numpy().view(np.uint16)[rows]
    np.testing.assert_array_equal(gotb, synth.f32_to_bf16_bits(ry))


@pytest.mark.parametrize("M,N,K,seed", [(1, 128, 128, 1), (200, 256, 384, 2), (333, 384, 1536, 3),
                                        (129, 128, 640, 4)])
def test_small_all_rows(M, N, K, seed):
    check(bits((M, K), seed, outliers=3), bits((N, K), seed + 100))


@pytest.mark.parametrize("M,N,K,seed", [(2100, 1280, 256, 9), (1900, 1408, 640, 10)])
def test_many_tiles_per_cta_all_rows(M, N, K, seed):
    # more output tiles than SMs: each persistent CTA computes several tiles,
    # with the pipeline steps (odd counts here) running on across them
    check(bits((M, K), seed, outliers=2), bits((N, K), seed + 100))


def test_zero_groups():
    x = bits((150, 384), 5)
    x[:, 128:256] = 0      # a zero activation group in every row
    x[7] = 0               # a zero row
    w = bits((256, 384), 6)
    w[128:, :128] = 0      # a zero weight block
    check(x, w)


@pytest.mark.parametrize("M,N,K", [(4096, 1536, 1536), (2040, 5120, 5120)])
def test_dit_shapes_sampled(M, N, K):
    rng = np.random.default_rng(M + N)
    rows = np.sort(np.concatenate([[0, M - 1], rng.choice(M, 30, replace=False)]))
    check(bits((M, K), 7, outliers=8), bits((N, K), 8), rows=np.unique(rows))


def test_bf16_output_alone():
    # without the optional fp32 output (the layer's usual call): the bf16 tile
    # stores alone, on a shape with an M tail and several tiles per CTA
    M, N, K = 2500, 1152, 384
    x, w = bits((M, K), 21, outliers=2), bits((N, K), 22)
    xq, sx = sage.w8a8_quant_act(dev(x))
    wq, sw = sage.w8a8_quant_weight(dev(w))
    y = sage.w8a8_gemm(xq, sx, wq, sw)
    assert sage.sync_status() == 0
    rxq, rsx = oracle.w8a8_quant_act(x)
    rwq, rsw = oracle.w8a8_quant_weight(w)
    ry = oracle.w8a8_gemm_rows(rxq, rsx, rwq, rsw, np.arange(M))
    gotb = y.view(torch.int16).cpu().numpy().view(np.uint16)
    np.testing.assert_array_equal(gotb, synth.f32_to_bf16_bits(ry))


@pytest.mark.parametrize("M,H,K,keep_y", [(300, 2, 256, True), (1000, 3, 640, False),
                                          (2040, 4, 1536, True)])
def test_q_quantization_fused_in_the_epilogue(M, H, K, keep_y):
    # the Q projection with attention's per-64-token INT8 Q quantization in the
    # GEMM epilogue: equal to sage_quant_qk's Q of the bf16 Y, bit for bit
    N = 128 * H
    x, w = bits((M, K), M + 1, outliers=3), bits((N, K), M + 2)
    xq, sx = sage.w8a8_quant_act(dev(x))
    wq, sw = sage.w8a8_quant_weight(dev(w))
    y = sage.w8a8_gemm(xq, sx, wq, sw)
    yq = torch.empty_like(y) if keep_y else None
    q8, qs, yq = sage.w8a8_gemm_q(xq, sx, wq, sw, y=yq)
    assert sage.sync_status() == 0
    if keep_y:
        assert torch.equal(yq, y)
    qh = y.view(M, H, 128).permute(1, 0, 2).contiguous().unsqueeze(0)  # [1, H, M, 128]
    ref = sage.quant_qk(qh, qh, qh)
    assert torch.equal(q8, ref.view("q_i8")[0])
    assert torch.equal(qs.view(torch.int32), ref.view("q_scale")[0].view(torch.int32))
    # and the oracle: its fp32 Y, rounded to bf16, quantized as Q
    rxq, rsx = oracle.w8a8_quant_act(x)
    rwq, rsw = oracle.w8a8_quant_weight(w)
    ry = synth.f32_to_bf16_bits(oracle.w8a8_gemm_rows(rxq, rsx, rwq, rsw, np.arange(M)))
    for h in range(H):
        qb = np.ascontiguousarray(ry[:, h * 128:(h + 1) * 128])
        rq = oracle.quant_head(qb, qb[:64], qb[:64])
        np.testing.assert_array_equal(q8[h].cpu().numpy(), rq["q8"])
        np.testing.assert_array_equal(qs[h].cpu().numpy().view(np.int32), rq["qs"].view(np.int32))
