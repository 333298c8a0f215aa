"""The path captured in a CUDA graph: quantization + attention (dense and
split-KV), the streaming step (RoPE in the quantizer, sliding-window
attention) and the W8A8 layer replay bit-identically to eager calls, and a
replay after new inputs are copied into the captured buffers recomputes."""
import numpy as np
import pytest
import torch

import bit_quantized_attention_sage_b200 as sage
from bit_quantized_attention_sage_b200 import synth

from gpu_helpers import to_dev

pytestmark = pytest.mark.gpu


def _capture(fn):
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):  # warm-up on the capture's side stream
        fn()
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


@pytest.mark.parametrize("splits", [1, 3])
def test_attention_step_replays(splits):
    w = synth.Workload("graph", 1, 4, 700, 3000, 128, mask=1, outlier_mag=5.0, seed=17)
    w2 = synth.Workload("graph2", 1, 4, 700, 3000, 128, mask=1, outlier_mag=5.0, seed=18)
    (q, k, v), (q2, k2, v2) = synth.full(w), synth.full(w2)
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    qkv = sage.quant_qk(qd, kd, vd)  # eager (also the library's one-time set-up)
    ws = torch.empty(max(sage.workspace_bytes(qkv.shape), 16), dtype=torch.uint8, device="cuda")
    sws = None
    if splits > 1:
        sws = torch.empty(sage.attn_split_workspace_bytes(qkv.shape, splits), dtype=torch.uint8,
                          device="cuda")
    o = torch.empty((1, 4, 700, 128), dtype=torch.bfloat16, device="cuda")

    def step():
        sage.quant_qk(qd, kd, vd, out=qkv, workspace=ws)
        sage.attn_fwd(qkv, 1, 0, out=o, kv_splits=splits, workspace=sws)

    step()
    torch.cuda.synchronize()
    ref = o.clone()
    g = _capture(step)
    o.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert sage.sync_status() == 0
    assert torch.equal(o, ref)
    # new inputs in the captured buffers
    qd.copy_(to_dev(q2)); kd.copy_(to_dev(k2)); vd.copy_(to_dev(v2))
    g.replay()
    torch.cuda.synchronize()
    got = o.clone()
    step()
    torch.cuda.synchronize()
    assert torch.equal(got, o) and not torch.equal(got, ref)


def test_w8a8_layer_replays():
    rng = np.random.default_rng(3)
    x = torch.from_numpy(rng.standard_normal((1000, 1536)).astype(np.float32)).cuda().to(torch.bfloat16)
    w = torch.from_numpy(rng.standard_normal((768, 1536)).astype(np.float32)).cuda().to(torch.bfloat16)
    wq, sw = sage.w8a8_quant_weight(w)
    xq, sx = sage.w8a8_quant_act(x)
    y = sage.w8a8_gemm(xq, sx, wq, sw)
    torch.cuda.synchronize()
    ref = y.clone()

    def layer():
        sage.w8a8_quant_act(x, xq, sx)
        sage.w8a8_gemm(xq, sx, wq, sw, out=y)

    g = _capture(layer)
    y.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert sage.sync_status() == 0
    assert torch.equal(y, ref)


@pytest.mark.parametrize("splits", [1, 3])
def test_streaming_window_step_replays(splits):
    # the streaming step of the pages: RoPE applied to Q and K at their
    # positions inside the quantizer, then attention under the sliding window
    # with a reference context; captured once, replayed per step
    Nq, Nkv, D = 600, 4000, 128
    w = synth.Workload("graph_win", 1, 3, Nq, Nkv, D, outlier_mag=5.0, seed=21)
    w2 = synth.Workload("graph_win2", 1, 3, Nq, Nkv, D, outlier_mag=5.0, seed=22)
    (q, k, v), (q2, k2, v2) = synth.full(w), synth.full(w2)
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    inv = 1.0 / (10000.0 ** (np.arange(D // 2) / (D // 2)))
    ang_k = np.arange(Nkv)[:, None] * inv[None, :]
    ang_q = ang_k[Nkv - Nq:]
    rope = tuple(torch.from_numpy(np.ascontiguousarray(f(a)).astype(np.float32)).cuda()
                 for a, f in ((ang_q, np.cos), (ang_q, np.sin), (ang_k, np.cos), (ang_k, np.sin)))
    window = (600, 3, 400)
    qkv = sage.quant_qk(qd, kd, vd, rope=rope)
    ws = torch.empty(max(sage.workspace_bytes(qkv.shape), 16), dtype=torch.uint8, device="cuda")
    sws = None
    if splits > 1:
        sws = torch.empty(sage.attn_split_workspace_bytes(qkv.shape, splits), dtype=torch.uint8,
                          device="cuda")
    o = torch.empty((1, 3, Nq, D), dtype=torch.bfloat16, device="cuda")

    def step():
        sage.quant_qk(qd, kd, vd, out=qkv, workspace=ws, rope=rope)
        sage.attn_fwd(qkv, out=o, kv_splits=splits, workspace=sws, window=window)

    step()
    torch.cuda.synchronize()
    ref = o.clone()
    g = _capture(step)
    o.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert sage.sync_status() == 0
    assert torch.equal(o, ref)
    qd.copy_(to_dev(q2)); kd.copy_(to_dev(k2)); vd.copy_(to_dev(v2))
    g.replay()
    torch.cuda.synchronize()
    got = o.clone()
    step()
    torch.cuda.synchronize()
    assert torch.equal(got, o) and not torch.equal(got, ref)
