"""sage_quant_qk_noalloc -- the quantizer for callers that cannot allocate
device memory (code inside a pre-sized, locked memory pool, a real-time loop
that must not enter the allocator, or a plugin that only receives its input
and output buffers).  Called through the C ABI, its outputs must equal those
of sage_quant_qk (bit for bit, the tolerance every quantized tensor is held
to) on two calls in a row that share its fixed scratch array, and shapes
whose scratch would not fit must be refused."""
import ctypes

import numpy as np
import pytest
import torch

import bit_quantized_attention_sage_b200 as sage
from bit_quantized_attention_sage_b200 import synth

pytestmark = pytest.mark.gpu


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _noalloc(q, k, v, out):
    L = sage.lib()
    st = out.struct()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return L.sage_quant_qk_noalloc(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                                   ctypes.c_void_p(v.data_ptr()), ctypes.byref(out.shape),
                                   ctypes.byref(st), stream)


def _inputs(w):
    q, k, v = synth.full(w)
    return _dev(q), _dev(k), _dev(v)


def test_noalloc_matches_quant_qk_on_two_calls_in_a_row():
    # two different problems back to back: the second call finds the first
    # call's leftovers in the shared scratch
    w1 = synth.Workload("noalloc_stream", 1, 24, 2040, 26520, 128, mask=2, mask_block=2040,
                        k_offset_var=4.0, seed=71)
    w2 = synth.Workload("noalloc_ragged", 2, 3, 333, 1000, 64, outlier_mag=20.0, seed=72)
    ins = [_inputs(w1), _inputs(w2)]
    outs = []
    for (q, k, v), w in zip(ins, (w1, w2)):
        out = sage.QuantizedQKV(sage.make_shape(w.B, w.H, w.Nq, w.Nkv, w.D), q.device)
        for t in out.bufs.values():
            t.fill_(0xA5)  # stale bytes that must all be overwritten
        assert _noalloc(q, k, v, out) == 0
        outs.append(out)
    assert sage.sync_status() == 0
    for (q, k, v), out in zip(ins, outs):
        ref = sage.quant_qk(q, k, v)  # the existing entry point, with its own workspace
        assert sage.sync_status() == 0
        for name in sage.BUFFERS:
            assert torch.equal(out.bufs[name], ref.bufs[name]), name


def test_noalloc_allocates_nothing():
    # after a warm-up call (which looks up the scratch array's address), two
    # more calls change neither the device's free memory nor torch's pool
    w = synth.Workload("noalloc_mem", 1, 4, 500, 700, 128, k_offset_var=4.0, seed=73)
    q, k, v = _inputs(w)
    out = sage.QuantizedQKV(sage.make_shape(w.B, w.H, w.Nq, w.Nkv, w.D), q.device)
    assert _noalloc(q, k, v, out) == 0
    torch.cuda.synchronize()
    free0, alloc0 = torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated()
    for _ in range(2):
        assert _noalloc(q, k, v, out) == 0
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert torch.cuda.memory_allocated() == alloc0
    assert sage.sync_status() == 0


def test_python_wrapper_matches_quant_qk():
    w = synth.Workload("noalloc_py", 1, 2, 200, 450, 64, outlier_mag=5.0, seed=74)
    q, k, v = _inputs(w)
    out = sage.QuantizedQKV(sage.make_shape(w.B, w.H, w.Nq, w.Nkv, w.D), q.device)
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        sage.quant_qk_noalloc(q, k, v, out, stream=stream)
    torch.cuda.current_stream().wait_stream(stream)
    ref = sage.quant_qk(q, k, v)
    assert sage.sync_status() == 0
    for name in sage.BUFFERS:
        assert torch.equal(out.bufs[name], ref.bufs[name]), name


def test_noalloc_refuses_shapes_beyond_its_scratch():
    w = synth.P720  # needs about 72 MB of scratch, more than the fixed 16 MiB
    shape = sage.make_shape(w.B, w.H, w.Nq, w.Nkv, w.D)
    assert sage.workspace_bytes(shape) > sage.NOALLOC_SCRATCH_BYTES
    small = torch.zeros(1 << 12, dtype=torch.uint8, device="cuda")  # never touched
    L = sage.lib()
    ptrs = sage._QKV(*([small.data_ptr()] * 7))
    p = ctypes.c_void_p(small.data_ptr())
    rc = L.sage_quant_qk_noalloc(p, p, p, ctypes.byref(shape), ctypes.byref(ptrs), None)
    assert rc == 2  # SAGE_ERR_UNSUPPORTED, nothing enqueued
    assert sage.sync_status() == 0
    assert not small.any()
