"""The C-ABI library loads and exports every symbol include/sage.h declares,
and its host-side logic (sizes, argument validation, status strings) works
without a GPU."""
import ctypes
import os
import re

import pytest

import bit_quantized_attention_sage_b200 as sage
from bit_quantized_attention_sage_b200 import build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "sage.h")


@pytest.fixture(scope="module")
def L():
    build.build()
    return sage.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sage_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(L, n), n


def test_abi_version_and_status_strings(L):
    assert L.sage_abi_version() == 1
    for code in range(5):
        assert L.sage_status_string(code)
    assert L.sage_status_string(99) == b"unknown status"


def test_buffer_and_workspace_sizes(L):
    s = sage.make_shape(1, 2, 1000, 3000, 128)
    b = sage.buffer_bytes(s)
    nqp, nkp = 1024, 3008
    assert b["q_i8"] == 2 * nqp * 128 and b["q_scale"] == 2 * 16 * 4
    assert b["k_i8"] == 2 * nkp * 128 and b["k_scale"] == 2 * 47 * 4
    assert b["k_mean"] == 2 * 128 * 4 and b["v_scale"] == 2 * 128 * 4
    assert b["v_f8"] == 2 * 128 * nkp
    assert sage.workspace_bytes(s) == 2 * 47 * 128 * 12 + 2 * 128 * 4
    # equalised variant: + |Q| maxima per Q block, K maxima and minima per K
    # block, the two factors per channel
    assert sage.equalized_workspace_bytes(s) == (sage.workspace_bytes(s) +
                                                 2 * 128 * 4 * (16 + 2 * 47 + 2))


@pytest.mark.parametrize("shape", [(0, 1, 8, 8, 128), (1, 1, 8, 8, 96), (1, 1, 0, 8, 64),
                                   (300, 300, 8, 8, 64)])
def test_invalid_shapes(L, shape):
    s = sage.make_shape(*shape)
    sizes = (ctypes.c_size_t * 7)()
    assert L.sage_quant_buffer_bytes(ctypes.byref(s), sizes) == 1
    assert L.sage_quant_workspace_bytes(ctypes.byref(s)) == 0
    assert L.sage_quant_equalized_workspace_bytes(ctypes.byref(s)) == 0


def test_invalid_arguments_are_rejected_before_any_launch(L):
    s = sage.make_shape(1, 1, 64, 64, 128)
    null = sage._QKV()
    assert L.sage_quant_qk(None, None, None, ctypes.byref(s), ctypes.byref(null), None, 0,
                           None) == 1
    assert L.sage_attn_fwd(ctypes.byref(null), ctypes.byref(s), 0, 0, None, None, None, None) == 1
    # misaligned pointers
    fake = sage._QKV(*([16 * 1024 + 4] * 7))
    assert L.sage_attn_fwd(ctypes.byref(fake), ctypes.byref(s), 0, 0, ctypes.c_void_p(4096),
                           None, None, None) == 1
    ok = sage._QKV(*([16 * 1024] * 7))
    # bad mask, causal with Nkv < Nq, block-causal without a block length
    assert L.sage_attn_fwd(ctypes.byref(ok), ctypes.byref(s), 7, 0, ctypes.c_void_p(4096),
                           None, None, None) == 1
    s2 = sage.make_shape(1, 1, 128, 64, 128)
    assert L.sage_attn_fwd(ctypes.byref(ok), ctypes.byref(s2), 1, 0, ctypes.c_void_p(4096),
                           None, None, None) == 1
    assert L.sage_attn_fwd(ctypes.byref(ok), ctypes.byref(s), 2, 0, ctypes.c_void_p(4096),
                           None, None, None) == 1
    assert L.sage_debug_timeout_probe(0, None) == 1
    # tile outside the shape
    tiles = (ctypes.c_int * 3)(0, 5, 0)
    assert L.sage_debug_qk_int32(ctypes.byref(ok), ctypes.byref(s), tiles, 1,
                                 ctypes.c_void_p(4096), None) == 1


def test_block_sparse_and_w8a8_arguments_are_rejected_before_any_launch(L):
    s = sage.make_shape(1, 1, 64, 64, 128)
    ok = sage._QKV(*([16 * 1024] * 7))
    out = ctypes.c_void_p(4096)
    # block-sparse: the mask pointer is required; more than 6144 KV tiles is unsupported
    assert L.sage_attn_fwd_block_sparse(ctypes.byref(ok), ctypes.byref(s), 0, 0, None, out,
                                        None, None, None) == 1
    big = sage.make_shape(1, 1, 64, 6144 * 128 + 1, 128)
    assert L.sage_attn_fwd_block_sparse(ctypes.byref(ok), ctypes.byref(big), 0, 0,
                                        ctypes.c_void_p(4096), out, None, None, None) == 2
    p = ctypes.c_void_p(4096)
    # W8A8: K and N must be multiples of 128, M >= 1, pointers 16-byte aligned
    assert L.sage_w8a8_quant_act(p, 4, 100, p, p, None) == 1
    assert L.sage_w8a8_quant_act(p, 0, 128, p, p, None) == 1
    assert L.sage_w8a8_quant_weight(p, 130, 128, p, p, None) == 1
    assert L.sage_w8a8_gemm(p, p, p, p, 8, 128, 200, p, None, None) == 1
    assert L.sage_w8a8_gemm(p, p, p, p, 8, 64, 128, p, None, None) == 1
    assert L.sage_w8a8_gemm(ctypes.c_void_p(4100), p, p, p, 8, 128, 128, p, None, None) == 1
    # the Q-fused form: q codes and scales required and aligned
    assert L.sage_w8a8_gemm_q(p, p, p, p, 8, 128, 128, None, None, p, None) == 1
    assert L.sage_w8a8_gemm_q(p, p, p, p, 8, 128, 128, None, ctypes.c_void_p(4100), p, None) == 1
    assert L.sage_w8a8_gemm_q(p, p, p, p, 8, 128, 128, None, p, None, None) == 1
    assert L.sage_w8a8_gemm_q(p, p, p, p, 8, 128, 128, None, p, ctypes.c_void_p(4098), None) == 1


def test_rope_quantizer_arguments_are_rejected_before_any_launch(L):
    s = sage.make_shape(1, 1, 64, 64, 128)
    ok = sage._QKV(*([16 * 1024] * 7))
    p = ctypes.c_void_p(4096)
    ws = L.sage_quant_workspace_bytes(ctypes.byref(s))
    tabs = [p, p, p, p]
    # every table is required and 16-byte aligned
    for i in range(4):
        t = list(tabs)
        t[i] = None
        assert L.sage_quant_qk_rope(p, p, p, ctypes.byref(s), *t, ctypes.byref(ok), p, ws,
                                    None) == 1
        t[i] = ctypes.c_void_p(4100)
        assert L.sage_quant_qk_rope(p, p, p, ctypes.byref(s), *t, ctypes.byref(ok), p, ws,
                                    None) == 1
    # more than 65535 blocks of 64 tokens is unsupported
    big = sage.make_shape(1, 1, 64, 65535 * 64 + 1, 128)
    assert L.sage_quant_qk_rope(p, p, p, ctypes.byref(big), *tabs, ctypes.byref(ok), p, 1 << 40,
                                None) == 2
    # the checks of sage_quant_qk still apply (workspace too small)
    assert L.sage_quant_qk_rope(p, p, p, ctypes.byref(s), *tabs, ctypes.byref(ok), p, ws - 1,
                                None) == 1


def test_split_attention_arguments_are_rejected_before_any_launch(L):
    s = sage.make_shape(1, 2, 300, 700, 128)
    ok = sage._QKV(*([16 * 1024] * 7))
    p = ctypes.c_void_p(4096)
    need = L.sage_attn_split_workspace_bytes(ctypes.byref(s), 3)
    assert need == 3 * 2 * 384 * 130 * 4
    assert L.sage_attn_split_workspace_bytes(ctypes.byref(s), 1) == 0
    assert L.sage_attn_split_workspace_bytes(ctypes.byref(s), 17) == 0
    for splits in (0, 17):
        assert L.sage_attn_fwd_split(ctypes.byref(ok), ctypes.byref(s), 0, 0, splits, p, need, p,
                                     None, None, None) == 1
    # workspace missing, misaligned or too small
    assert L.sage_attn_fwd_split(ctypes.byref(ok), ctypes.byref(s), 0, 0, 3, None, need, p,
                                 None, None, None) == 1
    assert L.sage_attn_fwd_split(ctypes.byref(ok), ctypes.byref(s), 0, 0, 3, ctypes.c_void_p(4100),
                                 need, p, None, None, None) == 1
    assert L.sage_attn_fwd_split(ctypes.byref(ok), ctypes.byref(s), 0, 0, 3, p, need - 1, p,
                                 None, None, None) == 1


def test_window_attention_arguments_are_rejected_before_any_launch(L):
    s = sage.make_shape(1, 2, 300, 700, 128)
    ok = sage._QKV(*([16 * 1024] * 7))
    p = ctypes.c_void_p(4096)
    need = L.sage_attn_split_workspace_bytes(ctypes.byref(s), 3)

    def call(frame, win, sink, splits=1, ws=None, nbytes=0, shape=s):
        return L.sage_attn_fwd_window(ctypes.byref(ok), ctypes.byref(shape), frame, win, sink,
                                      splits, ws, nbytes, p, None, None, None)

    for frame, win, sink in [(0, 1, 0), (64, 0, 0), (64, 1, -1), (-5, 2, 10)]:
        assert call(frame, win, sink) == 1
    for splits in (0, 17):
        assert call(64, 2, 0, splits, p, need) == 1
    # a window needs Nkv >= Nq
    assert call(64, 2, 0, shape=sage.make_shape(1, 2, 701, 700, 128)) == 1
    # workspace missing, misaligned or too small when kv_splits > 1
    assert call(64, 2, 0, 3, None, need) == 1
    assert call(64, 2, 0, 3, ctypes.c_void_p(4100), need) == 1
    assert call(64, 2, 0, 3, p, need - 1) == 1
    # the window mask id is not a public sage_mask value
    assert L.sage_attn_fwd(ctypes.byref(ok), ctypes.byref(s), 3, 64, p, None, None, None) == 1
    assert L.sage_attn_fwd_split(ctypes.byref(ok), ctypes.byref(s), 3, 64, 3, p, need, p,
                                 None, None, None) == 1
    assert L.sage_attn_fwd_block_sparse(ctypes.byref(ok), ctypes.byref(s), 3, 64, p, p, None,
                                        None, None) == 1


def test_ceiling_arguments_are_rejected_before_any_launch(L):
    blocks, bps, opb = ctypes.c_int(), ctypes.c_int(), ctypes.c_double()
    cyc = ctypes.c_void_p(4096)

    def call(kind, iters=10, n=256, scratch=None, nbytes=0, cycles=cyc):
        return L.sage_ceiling(kind, iters, n, scratch, nbytes, cycles, ctypes.byref(blocks),
                              ctypes.byref(bps), ctypes.byref(opb), None)

    assert call(-1) == 1 and call(6) == 1               # unknown kinds
    assert call(0, iters=0) == 1 and call(1, iters=(1 << 24) + 1) == 1
    assert call(4, n=100) == 1 and call(5, n=512) == 1  # MMA N must be 64, 128 or 256
    assert call(3, scratch=None, nbytes=1 << 30) == 1   # copy needs a scratch buffer
    assert call(3, scratch=ctypes.c_void_p(4096), nbytes=1 << 19) == 1  # of at least 1 MiB
    assert call(3, scratch=ctypes.c_void_p(4104), nbytes=1 << 30) == 1  # 16-byte aligned
    assert call(0, cycles=None) == 1 and call(0, cycles=ctypes.c_void_p(4100)) == 1


def test_noalloc_wrapper_refuses_oversized_shapes_before_any_launch(L):
    # the Python wrapper checks the scratch size on the host and raises
    # before it touches the tensors or the C entry point
    class _Out:
        shape = sage.make_shape(1, 40, 75600, 75600, 128)

    assert sage.workspace_bytes(_Out.shape) > sage.NOALLOC_SCRATCH_BYTES
    with pytest.raises(sage.SageError):
        sage.quant_qk_noalloc(None, None, None, _Out())
