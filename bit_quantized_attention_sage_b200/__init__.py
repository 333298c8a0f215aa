"""B200-native SageAttention-style quantized attention.

Thin ctypes binding of ``libsage_b200.so`` (the C ABI in ``include/sage.h``).
This module only marshals arguments: torch provides device memory and the
stream, every step of the computation runs in the library's CUDA kernels.
There is no CPU fallback -- if the library is missing or the device is not an
sm_100a GPU the calls raise.

One-line use, in place of a FlashAttention call on [B, H, N, D] bf16 tensors:

    o = attention(q, k, v)                          # bidirectional
    o = attention(q, k, v, mask="causal")
    o = attention(q, k, v, mask=("block_causal", 2040))   # streaming KV cache
"""
import ctypes
import math
import os

MASK_NONE, MASK_CAUSAL, MASK_BLOCK_CAUSAL = 0, 1, 2
TILE_M, TILE_N = 128, 128   # attention kernel's query rows per CTA / keys per KV tile

STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported", 3: "CUDA error",
          4: "device wait timed out"}

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsage_b200.so")
_lib = None


class SageError(RuntimeError):
    def __init__(self, code, what):
        super().__init__("%s: %s (status %d)" % (what, STATUS.get(code, "?"), code))
        self.code = code


class Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("Nq", ctypes.c_int),
                ("Nkv", ctypes.c_int), ("D", ctypes.c_int)]


class _QKV(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("q_i8", "q_scale", "k_i8", "k_scale", "k_mean", "v_f8", "v_scale")]


BUFFERS = ("q_i8", "q_scale", "k_i8", "k_scale", "k_mean", "v_f8", "v_scale")


def lib():
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError("libsage_b200.so is not built; run "
                              "`python -m bit_quantized_attention_sage_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        L.sage_abi_version.restype = I
        L.sage_status_string.restype = ctypes.c_char_p
        L.sage_status_string.argtypes = [I]
        L.sage_quant_buffer_bytes.restype = I
        L.sage_quant_buffer_bytes.argtypes = [P, P]
        L.sage_quant_workspace_bytes.restype = SZ
        L.sage_quant_workspace_bytes.argtypes = [P]
        L.sage_quant_qk.restype = I
        L.sage_quant_qk.argtypes = [P, P, P, P, P, P, SZ, P]
        L.sage_quant_qk_rope.restype = I
        L.sage_quant_qk_rope.argtypes = [P, P, P, P, P, P, P, P, P, P, SZ, P]
        L.sage_quant_equalized_workspace_bytes.restype = SZ
        L.sage_quant_equalized_workspace_bytes.argtypes = [P]
        L.sage_quant_qk_equalized.restype = I
        L.sage_quant_qk_equalized.argtypes = [P, P, P, P, P, P, P, SZ, P]
        L.sage_window_keys.restype = I
        L.sage_window_keys.argtypes = [P, I, I, I, P, P, P]
        L.sage_quant_qk_window.restype = I
        L.sage_quant_qk_window.argtypes = [P, P, P, P, I, I, I, P, P, P, P, P, P, SZ, P]
        L.sage_quant_qk_noalloc.restype = I
        L.sage_quant_qk_noalloc.argtypes = [P, P, P, P, P, P]
        L.sage_attn_fwd.restype = I
        L.sage_attn_fwd.argtypes = [P, P, I, I, P, P, P, P]
        L.sage_attn_fwd_split.restype = I
        L.sage_attn_fwd_split.argtypes = [P, P, I, I, I, P, SZ, P, P, P, P]
        L.sage_attn_split_workspace_bytes.restype = SZ
        L.sage_attn_split_workspace_bytes.argtypes = [P, I]
        L.sage_ceiling.restype = I
        L.sage_ceiling.argtypes = [I, I, I, P, SZ, P, P, P, P, P]
        L.sage_attn_fwd_window.restype = I
        L.sage_attn_fwd_window.argtypes = [P, P, I, I, I, I, P, SZ, P, P, P, P]
        L.sage_attn_fwd_block_sparse.restype = I
        L.sage_attn_fwd_block_sparse.argtypes = [P, P, I, I, P, P, P, P, P]
        L.sage_debug_qk_int32.restype = I
        L.sage_debug_qk_int32.argtypes = [P, P, P, I, P, P]
        L.sage_debug_timeout_probe.restype = I
        L.sage_debug_timeout_probe.argtypes = [ctypes.c_longlong, P]
        L.sage_debug_e4m3.restype = I
        L.sage_debug_e4m3.argtypes = [P, P, SZ, P]
        L.sage_debug_exp2.restype = I
        L.sage_debug_exp2.argtypes = [P, P, SZ, P]
        LL = ctypes.c_longlong
        L.sage_w8a8_quant_act.restype = I
        L.sage_w8a8_quant_act.argtypes = [P, LL, LL, P, P, P]
        L.sage_w8a8_quant_weight.restype = I
        L.sage_w8a8_quant_weight.argtypes = [P, LL, LL, P, P, P]
        L.sage_w8a8_gemm_q.restype = I
        L.sage_w8a8_gemm_q.argtypes = [P, P, P, P, LL, LL, LL, P, P, P, P]
        L.sage_w8a8_gemm.restype = I
        L.sage_w8a8_gemm.argtypes = [P, P, P, P, LL, LL, LL, P, P, P]
        L.sage_sync_status.restype = I
        L.sage_sync_status.argtypes = [P]
        _lib = L
    return _lib


def _check(code, what):
    if code != 0:
        raise SageError(code, what)


def _stream(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def make_shape(B, H, Nq, Nkv, D):
    return Shape(int(B), int(H), int(Nq), int(Nkv), int(D))


def buffer_bytes(shape):
    sizes = (ctypes.c_size_t * 7)()
    _check(lib().sage_quant_buffer_bytes(ctypes.byref(shape), sizes), "sage_quant_buffer_bytes")
    return dict(zip(BUFFERS, (int(x) for x in sizes)))


def workspace_bytes(shape):
    return int(lib().sage_quant_workspace_bytes(ctypes.byref(shape)))


class QuantizedQKV:
    """The seven device buffers sage_quant_qk fills (torch uint8 storage)."""

    def __init__(self, shape, device):
        import torch
        self.shape = shape
        self.bufs = {n: torch.empty(b, dtype=torch.uint8, device=device)
                     for n, b in buffer_bytes(shape).items()}

    def struct(self):
        return _QKV(*(self.bufs[n].data_ptr() for n in BUFFERS))

    # typed views (for inspection and tests)
    def view(self, name):
        import torch
        s = self.shape
        bh = s.B * s.H
        nqp, nkp = -(-s.Nq // 64) * 64, -(-s.Nkv // 64) * 64
        t = self.bufs[name]
        if name == "q_i8":
            return t.view(torch.int8).view(s.B, s.H, nqp, s.D)
        if name == "k_i8":
            return t.view(torch.int8).view(s.B, s.H, nkp, s.D)
        if name == "v_f8":
            return t.view(s.B, s.H, nkp, s.D)
        if name == "q_scale":
            return t.view(torch.float32).view(s.B, s.H, nqp // 64)
        if name == "k_scale":
            return t.view(torch.float32).view(s.B, s.H, nkp // 64)
        return t.view(torch.float32).view(s.B, s.H, s.D)


def quant_qk(q, k, v, out=None, workspace=None, stream=None, rope=None):
    """sage_quant_qk on bf16 CUDA tensors [B, H, N, D]; returns QuantizedQKV.

    rope: None, or (q_cos, q_sin, k_cos, k_sin), contiguous float32 CUDA
    tensors [Nq, D/2] and [Nkv, D/2]: Q and K are rotated pairwise by those
    angles before quantization (sage_quant_qk_rope)."""
    import torch
    B, H, Nq, D = q.shape
    Nkv = k.shape[2]
    shape = make_shape(B, H, Nq, Nkv, D)
    for t in (q, k, v):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous bf16 CUDA tensors")
    if rope is not None:
        for t, n in zip(rope, (Nq, Nq, Nkv, Nkv)):
            if (t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous()
                    or tuple(t.shape) != (n, D // 2)):
                raise ValueError("rotation tables must be contiguous float32 CUDA tensors "
                                 "[Nq, D/2], [Nq, D/2], [Nkv, D/2], [Nkv, D/2]")
    if out is None:
        out = QuantizedQKV(shape, q.device)
    ws_need = workspace_bytes(shape)
    if workspace is None:
        workspace = torch.empty(max(ws_need, 16), dtype=torch.uint8, device=q.device)
    qs = out.struct()
    if rope is None:
        _check(lib().sage_quant_qk(_ptr(q), _ptr(k), _ptr(v), ctypes.byref(shape),
                                   ctypes.byref(qs), _ptr(workspace), workspace.numel(),
                                   _stream(stream)),
               "sage_quant_qk")
    else:
        _check(lib().sage_quant_qk_rope(_ptr(q), _ptr(k), _ptr(v), ctypes.byref(shape),
                                        *[_ptr(t) for t in rope], ctypes.byref(qs),
                                        _ptr(workspace), workspace.numel(), _stream(stream)),
               "sage_quant_qk_rope")
    return out


def equalized_workspace_bytes(shape):
    """sage_quant_equalized_workspace_bytes."""
    return int(lib().sage_quant_equalized_workspace_bytes(ctypes.byref(shape)))


def quant_qk_equalized(q, k, v, out=None, eq_exp=None, workspace=None, stream=None):
    """sage_quant_qk_equalized (a labelled accuracy variant outside the
    recipe): channel d of Q times 2^e[d] and of the smoothed K times 2^-e[d]
    before the block codes.  q, k, v bf16 CUDA [B, H, N, D]; eq_exp: None or
    an int8 CUDA tensor [B, H, D] that receives e.  Returns QuantizedQKV."""
    import torch
    B, H, Nq, D = q.shape
    shape = make_shape(B, H, Nq, k.shape[2], D)
    for t in (q, k, v):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous bf16 CUDA tensors")
    if eq_exp is not None and (eq_exp.dtype != torch.int8 or not eq_exp.is_cuda
                               or not eq_exp.is_contiguous() or tuple(eq_exp.shape) != (B, H, D)):
        raise ValueError("eq_exp must be a contiguous int8 CUDA tensor [B, H, D]")
    if out is None:
        out = QuantizedQKV(shape, q.device)
    if workspace is None:
        workspace = torch.empty(max(equalized_workspace_bytes(shape), 16), dtype=torch.uint8,
                                device=q.device)
    qs = out.struct()
    _check(lib().sage_quant_qk_equalized(_ptr(q), _ptr(k), _ptr(v), ctypes.byref(shape),
                                         ctypes.byref(qs), None if eq_exp is None else _ptr(eq_exp),
                                         _ptr(workspace), workspace.numel(), _stream(stream)),
           "sage_quant_qk_equalized")
    return out


def window_keys(shape, frame, win, sink):
    """sage_window_keys: (n_sink, lo, hi) -- a sliding-window step over a
    cache of `shape` attends to keys [0, n_sink) and [lo, hi)."""
    a, b, c = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    _check(lib().sage_window_keys(ctypes.byref(shape), int(frame), int(win), int(sink),
                                  ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)),
           "sage_window_keys")
    return a.value, b.value, c.value


def quant_qk_window(q, k_cache, v_cache, frame, win, sink, rope=None, out=None, workspace=None,
                    stream=None):
    """sage_quant_qk_window: quantize only the keys a sliding-window step
    attends to (the reference context and the window, gathered in cache
    order).  q [B, H, Nq, D], k_cache / v_cache [B, H, Nkv, D] bf16 CUDA;
    rope: None or (q_cos, q_sin, k_cos, k_sin) float32 [Nq, D/2] and
    [Nkv', D/2] (the gathered keys' positions).  Returns QuantizedQKV of the
    gathered shape (Nkv' = n_sink + hi - lo keys)."""
    import torch
    B, H, Nq, D = q.shape
    cache = make_shape(B, H, Nq, k_cache.shape[2], D)
    for t in (q, k_cache, v_cache):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError("q, k_cache, v_cache must be contiguous bf16 CUDA tensors")
    n_sink, lo, hi = window_keys(cache, frame, win, sink)
    shape = make_shape(B, H, Nq, n_sink + hi - lo, D)
    if rope is not None:
        for t, n in zip(rope, (Nq, Nq, shape.Nkv, shape.Nkv)):
            if (t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous()
                    or tuple(t.shape) != (n, D // 2)):
                raise ValueError("rotation tables must be contiguous float32 CUDA tensors "
                                 "[Nq, D/2], [Nq, D/2], [Nkv', D/2], [Nkv', D/2]")
    if out is None:
        out = QuantizedQKV(shape, q.device)
    if workspace is None:
        workspace = torch.empty(max(workspace_bytes(shape), 16), dtype=torch.uint8,
                                device=q.device)
    qs = out.struct()
    tabs = [None] * 4 if rope is None else [_ptr(t) for t in rope]
    _check(lib().sage_quant_qk_window(_ptr(q), _ptr(k_cache), _ptr(v_cache), ctypes.byref(cache),
                                      int(frame), int(win), int(sink), *tabs, ctypes.byref(qs),
                                      _ptr(workspace), workspace.numel(), _stream(stream)),
           "sage_quant_qk_window")
    return out


NOALLOC_SCRATCH_BYTES = 16 << 20  # SAGE_NOALLOC_SCRATCH_BYTES in include/sage.h


def quant_qk_noalloc(q, k, v, out, stream=None):
    """sage_quant_qk_noalloc: quantize into caller-provided outputs without
    any workspace, for callers that cannot allocate device memory (the
    library's fixed 16 MiB scratch array is used instead; calls on one device
    share it, so do not overlap them across streams)."""
    shape = out.shape
    need = workspace_bytes(shape)
    if need > NOALLOC_SCRATCH_BYTES:
        raise SageError(2, "sage_quant_qk_noalloc: this shape needs %d bytes of scratch, more "
                           "than the fixed %d-byte array" % (need, NOALLOC_SCRATCH_BYTES))
    qs = out.struct()
    _check(lib().sage_quant_qk_noalloc(_ptr(q), _ptr(k), _ptr(v), ctypes.byref(shape),
                                       ctypes.byref(qs), _stream(stream)),
           "sage_quant_qk_noalloc")
    return out


def block_mask_shape(B, H, Nq, Nkv):
    """Shape of a block mask: one byte per 128-query x 128-key tile."""
    return (B, H, -(-Nq // 128), -(-Nkv // 128))


def suggest_kv_splits(B, H, Nq, Nkv, sm_count, max_splits=16):
    """A KV split count for sage_attn_fwd_split: 1 when the 128-query tiles
    already fill the GPU (two CTAs per SM) in well-balanced waves, else the
    smallest count whose waves are at least 90 % full, keeping at least 8 KV
    tiles per range."""
    ctas = B * H * -(-Nq // 128)
    slots = 2 * sm_count
    tiles = -(-Nkv // 128)
    best, best_eff = 1, 0.0
    for sp in range(1, max_splits + 1):
        if sp > 1 and tiles // sp < 8:
            break
        waves = ctas * sp / slots
        eff = waves / math.ceil(waves)
        if eff >= 0.9:
            return sp
        if eff > best_eff + 1e-9:
            best, best_eff = sp, eff
    return best


def attn_split_workspace_bytes(shape, kv_splits):
    return lib().sage_attn_split_workspace_bytes(ctypes.byref(shape), int(kv_splits))


def attn_fwd(qkv, mask=MASK_NONE, mask_block=0, out=None, o_f32=None, lse=None, stream=None,
             block_mask=None, kv_splits=1, workspace=None, window=None):
    """sage_attn_fwd on a QuantizedQKV; returns the bf16 output tensor.

    block_mask: optional contiguous uint8 CUDA tensor of block_mask_shape();
    tiles whose byte is 0 are skipped (sage_attn_fwd_block_sparse).
    kv_splits: > 1 runs the split-KV form (sage_attn_fwd_split) with that
    many KV ranges per query tile; "auto" picks one with suggest_kv_splits.
    workspace: its device scratch (allocated here when None).
    window: (frame_len, window_frames, sink_tokens) runs the sliding-window
    mask with a reference context (sage_attn_fwd_window; mask and mask_block
    are then ignored)."""
    import torch
    s = qkv.shape
    dev = qkv.bufs["q_i8"].device
    if out is None:
        out = torch.empty((s.B, s.H, s.Nq, s.D), dtype=torch.bfloat16, device=dev)
    st = qkv.struct()
    if kv_splits == "auto":
        sms = torch.cuda.get_device_properties(dev).multi_processor_count
        nkv = s.Nkv
        if window is not None:  # keys a query tile visits, at most
            frame, win, sink = (int(x) for x in window)
            nkv = min(s.Nkv, sink + (win + 1) * frame + 128)
        kv_splits = suggest_kv_splits(s.B, s.H, s.Nq, nkv, sms)
    if window is not None:
        if block_mask is not None:
            raise ValueError("window and block_mask are not combined")
        frame, win, sink = (int(x) for x in window)
        ws_ptr, ws_bytes = None, 0
        if kv_splits != 1:
            need = attn_split_workspace_bytes(s, kv_splits)
            if need == 0:
                raise ValueError("kv_splits must be in 1..16")
            if workspace is None:
                workspace = torch.empty(need, dtype=torch.uint8, device=dev)
            ws_ptr, ws_bytes = _ptr(workspace), workspace.numel() * workspace.element_size()
        _check(lib().sage_attn_fwd_window(ctypes.byref(st), ctypes.byref(s), frame, win, sink,
                                          int(kv_splits), ws_ptr, ws_bytes, _ptr(out),
                                          _ptr(o_f32), _ptr(lse), _stream(stream)),
               "sage_attn_fwd_window")
        return out
    if kv_splits != 1:
        if block_mask is not None:
            raise ValueError("kv_splits and block_mask are not combined")
        need = attn_split_workspace_bytes(s, kv_splits)
        if need == 0:
            raise ValueError("kv_splits must be in 1..16")
        if workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=dev)
        _check(lib().sage_attn_fwd_split(ctypes.byref(st), ctypes.byref(s), int(mask),
                                         int(mask_block), int(kv_splits), _ptr(workspace),
                                         workspace.numel() * workspace.element_size(), _ptr(out),
                                         _ptr(o_f32), _ptr(lse), _stream(stream)),
               "sage_attn_fwd_split")
        return out
    if block_mask is None:
        _check(lib().sage_attn_fwd(ctypes.byref(st), ctypes.byref(s), int(mask), int(mask_block),
                                   _ptr(out), _ptr(o_f32), _ptr(lse), _stream(stream)),
               "sage_attn_fwd")
        return out
    if (block_mask.dtype != torch.uint8 or not block_mask.is_cuda
            or not block_mask.is_contiguous()
            or tuple(block_mask.shape) != block_mask_shape(s.B, s.H, s.Nq, s.Nkv)):
        raise ValueError("block_mask must be a contiguous uint8 CUDA tensor of shape %s"
                         % (block_mask_shape(s.B, s.H, s.Nq, s.Nkv),))
    _check(lib().sage_attn_fwd_block_sparse(ctypes.byref(st), ctypes.byref(s), int(mask),
                                            int(mask_block), _ptr(block_mask), _ptr(out),
                                            _ptr(o_f32), _ptr(lse), _stream(stream)),
           "sage_attn_fwd_block_sparse")
    return out


def attention(q, k, v, mask=None, stream=None, kv_splits="auto"):
    """Drop-in quantized attention: bf16 [B, H, N, D] in, bf16 out.

    mask: None, "causal", ("block_causal", n) or ("window", frame_len,
    window_frames, sink_tokens) -- the sliding window with a reference context
    of streaming generation (sage_attn_fwd_window).
    kv_splits: "auto" runs the split-KV form when the query tiles alone would
    leave the GPU idle (e.g. one streaming frame against a long cache); an
    int forces a split count (1: never split)."""
    window = None
    if mask is None or mask == "none":
        m, mb = MASK_NONE, 0
    elif mask == "causal":
        m, mb = MASK_CAUSAL, 0
    elif isinstance(mask, tuple) and mask[0] == "block_causal":
        m, mb = MASK_BLOCK_CAUSAL, int(mask[1])
    elif isinstance(mask, tuple) and mask[0] == "window" and len(mask) == 4:
        m, mb, window = MASK_NONE, 0, tuple(int(x) for x in mask[1:])
    else:
        raise ValueError("mask must be None, 'causal', ('block_causal', n) or "
                         "('window', frame_len, window_frames, sink_tokens)")
    qkv = quant_qk(q, k, v, stream=stream)
    return attn_fwd(qkv, m, mb, stream=stream, kv_splits=kv_splits, window=window)


def debug_qk_int32(qkv, tiles, stream=None):
    """int32 score tiles left in tensor memory by the attention kernel.

    tiles: sequence of (bh, qt, kt); returns a torch int32 [n, 128, 128]."""
    import torch
    n = len(tiles)
    flat = (ctypes.c_int * (3 * n))(*[int(x) for t in tiles for x in t])
    out = torch.empty((n, TILE_M, TILE_N), dtype=torch.int32, device=qkv.bufs["q_i8"].device)
    st = qkv.struct()
    _check(lib().sage_debug_qk_int32(ctypes.byref(st), ctypes.byref(qkv.shape), flat, n,
                                     _ptr(out), _stream(stream)), "sage_debug_qk_int32")
    return out


def debug_e4m3(x, stream=None):
    """Device e4m3 codes of a float32 CUDA tensor (the kernels' conversion)."""
    import torch
    x = x.contiguous()
    y = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    _check(lib().sage_debug_e4m3(_ptr(x), _ptr(y), x.numel(), _stream(stream)), "sage_debug_e4m3")
    return y


def debug_exp2(x, stream=None):
    """Device 2^x of a float32 CUDA tensor (the softmax's exp2)."""
    import torch
    x = x.contiguous()
    y = torch.empty_like(x)
    _check(lib().sage_debug_exp2(_ptr(x), _ptr(y), x.numel(), _stream(stream)), "sage_debug_exp2")
    return y


def timeout_probe(budget_cycles, stream=None):
    _check(lib().sage_debug_timeout_probe(int(budget_cycles), _stream(stream)),
           "sage_debug_timeout_probe")


def sync_status(stream=None):
    """Synchronize the stream and return (and clear) the device status code."""
    return int(lib().sage_sync_status(_stream(stream)))


# ---------------------------------------------------------------- W8A8 linear layer

W8A8_GROUP = 128


CEILINGS = {"ex2": 0, "ffma2": 1, "cvt_e4m3x2": 2, "copy": 3, "mma_i8": 4, "mma_e4m3": 5}


def ceiling(kind, iters=4096, n=256, scratch=None, stream=None):
    """Run one hardware-ceiling microbenchmark (sage_ceiling) and return
    {"per_sm_per_clock": median over blocks of ops_per_block * blocks_per_sm
    / cycles, "per_second": ops of the whole launch / its CUDA-event time,
    "ms": that time, "blocks": ...}.  kind: a key of CEILINGS.  scratch: the
    copy's device buffer (its two halves), required for "copy"."""
    import torch
    k = CEILINGS[kind]
    dev = torch.device("cuda", torch.cuda.current_device())
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    cycles = torch.zeros(8 * sms, dtype=torch.int64, device=dev)
    blocks, bps, opb = ctypes.c_int(), ctypes.c_int(), ctypes.c_double()
    st = torch.cuda.current_stream(dev) if stream is None else stream
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(st)
    _check(lib().sage_ceiling(k, int(iters), int(n), _ptr(scratch),
                              0 if scratch is None else scratch.numel() * scratch.element_size(),
                              _ptr(cycles), ctypes.byref(blocks), ctypes.byref(bps),
                              ctypes.byref(opb), _stream(st)), "sage_ceiling")
    b.record(st)
    b.synchronize()
    ms = a.elapsed_time(b)
    cyc = cycles[:blocks.value].float().cpu()
    if bool((cyc <= 0).any()):
        raise SageError(3, "sage_ceiling: a block did not record its cycles")
    med = float(cyc.median())
    return {"kind": kind, "per_sm_per_clock": opb.value * bps.value / med,
            "per_second": opb.value * blocks.value / (ms / 1e3), "ms": ms,
            "blocks": blocks.value, "blocks_per_sm": bps.value, "median_cycles": med}


def w8a8_quant_act(x, xq=None, sx=None, stream=None):
    """X bf16 [M, K] (CUDA, contiguous) -> (xq int8 [M, K], sx f32 [M, K/128])."""
    import torch
    M, K = x.shape
    if x.dtype != torch.bfloat16 or not x.is_cuda or not x.is_contiguous():
        raise ValueError("x must be a contiguous bf16 CUDA tensor")
    xq = torch.empty((M, K), dtype=torch.int8, device=x.device) if xq is None else xq
    sx = torch.empty((M, K // W8A8_GROUP), dtype=torch.float32, device=x.device) if sx is None else sx
    _check(lib().sage_w8a8_quant_act(_ptr(x), M, K, _ptr(xq), _ptr(sx), _stream(stream)),
           "sage_w8a8_quant_act")
    return xq, sx


def w8a8_quant_weight(w, stream=None):
    """W bf16 [N, K] (CUDA, contiguous) -> (wq int8 [N, K], sw f32 [N/128, K/128])."""
    import torch
    N, K = w.shape
    if w.dtype != torch.bfloat16 or not w.is_cuda or not w.is_contiguous():
        raise ValueError("w must be a contiguous bf16 CUDA tensor")
    wq = torch.empty((N, K), dtype=torch.int8, device=w.device)
    sw = torch.empty((N // W8A8_GROUP, K // W8A8_GROUP), dtype=torch.float32, device=w.device)
    _check(lib().sage_w8a8_quant_weight(_ptr(w), N, K, _ptr(wq), _ptr(sw), _stream(stream)),
           "sage_w8a8_quant_weight")
    return wq, sw


def w8a8_gemm(xq, sx, wq, sw, out=None, y_f32=None, stream=None):
    """Y bf16 [M, N] = dequant(X) dequant(W)^T from the quantized operands."""
    import torch
    M, K = xq.shape
    N = wq.shape[0]
    out = torch.empty((M, N), dtype=torch.bfloat16, device=xq.device) if out is None else out
    _check(lib().sage_w8a8_gemm(_ptr(xq), _ptr(sx), _ptr(wq), _ptr(sw), M, N, K, _ptr(out),
                                _ptr(y_f32), _stream(stream)), "sage_w8a8_gemm")
    return out


def w8a8_gemm_q(xq, sx, wq, sw, q_i8=None, q_scale=None, y=None, stream=None):
    """sage_w8a8_gemm_q: the Q projection with Q's per-64-token INT8
    quantization in the GEMM epilogue.  Returns (q_i8 [N/128, M_pad, 128],
    q_scale [N/128, M_pad/64], y) where y is the optional bf16 Y passed in."""
    import torch
    M, K = xq.shape
    N = wq.shape[0]
    mpad = -(-M // 64) * 64
    if q_i8 is None:
        q_i8 = torch.empty((N // 128, mpad, 128), dtype=torch.int8, device=xq.device)
    if q_scale is None:
        q_scale = torch.empty((N // 128, mpad // 64), dtype=torch.float32, device=xq.device)
    _check(lib().sage_w8a8_gemm_q(_ptr(xq), _ptr(sx), _ptr(wq), _ptr(sw), M, N, K, _ptr(y),
                                  _ptr(q_i8), _ptr(q_scale), _stream(stream)), "sage_w8a8_gemm_q")
    return q_i8, q_scale, y


def linear_w8a8(x, wq, sw, stream=None):
    """A W8A8 linear layer on bf16 activations [..., K] with pre-quantized
    weights (from w8a8_quant_weight): quantize X per token and 128-channel
    group, then the INT8 GEMM; returns bf16 [..., N]."""
    lead = x.shape[:-1]
    x2 = x.reshape(-1, x.shape[-1])
    xq, sx = w8a8_quant_act(x2.contiguous(), stream=stream)
    return w8a8_gemm(xq, sx, wq, sw, stream=stream).reshape(*lead, wq.shape[0])
