"""CPU oracle for the quantized-attention hot path (ctypes over ``liboracle.so``).

TEST INFRASTRUCTURE: only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference arm import this package.  The product
path (the CUDA library and its binding) never imports it and shares no code
with it.

Every array here is numpy.  bf16 tensors travel as their uint16 bit patterns.
Layouts follow the library's logical layout [B, H, N, D]; V codes are
token-major [N_kv, D] here (the device library stores them in its own order).
"""
import contextlib
import ctypes
import math
import os

import numpy as np

from . import build as _build

MASK_NONE, MASK_CAUSAL, MASK_BLOCK_CAUSAL, MASK_SLIDING_WINDOW = 0, 1, 2, 3
BLK = 64          # Q/K quantization block (tokens)
TKV = 128         # KV tile width of the online softmax (the device kernel's)
BQ = 128          # query rows per block of a block-sparse mask (one query tile)

# Relative uncertainty of the device's exp2 result plus one fp32 rounding of
# the oracle's own exp2.  The device uses the hardware ex2.approx.ftz.f32; its
# measured worst relative error over the softmax's argument range is checked
# by a GPU test to stay below EXP2_REL_ERR.  The slack derived from EPS marks
# every e4m3 rounding of p*256 that the two sides may take differently.
EXP2_REL_ERR = 2.0 ** -21
EPS = EXP2_REL_ERR + 2.0 ** -24

_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = _load(_build.build())
    return _lib


@contextlib.contextmanager
def variant(**defines):
    """Within the block, every function of this module runs on a separately
    compiled copy of the oracle with the given preprocessor defines (the
    planted mistakes and the alternative P-scale reading listed in
    sage_oracle.c).  Test-suite only."""
    global _lib
    saved = lib()
    _lib = _load(_build.build_variant(defines))
    try:
        yield
    finally:
        _lib = saved


def _load(path):
    L = ctypes.CDLL(path)
    P = ctypes.c_void_p
    i64, i32, f64 = ctypes.c_long, ctypes.c_int, ctypes.c_double
    L.orc_e4m3_decode.restype = f64
    L.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
    L.orc_e4m3_encode.restype = ctypes.c_uint8
    L.orc_e4m3_encode.argtypes = [ctypes.c_float]
    L.orc_e4m3_encode_n.restype = None
    L.orc_e4m3_encode_n.argtypes = [P, i64, P]
    L.orc_quant_head.restype = i32
    L.orc_quant_head.argtypes = [P, P, P, i64, i64, i32, P, P, P, P, P, P, P]
    L.orc_quant_head_eq.restype = i32
    L.orc_quant_head_eq.argtypes = [P, P, P, i64, i64, i32, P, P, P, P, P, P, P, P]
    L.orc_quant_head_rope.restype = i32
    L.orc_quant_head_rope.argtypes = [P, P, P, i64, i64, i32, P, P, P, P, P, P, P, P, P, P, P]
    L.orc_qk_int32.restype = None
    L.orc_qk_int32.argtypes = [P, P, i32, i64, i64, i64, i64, P]
    L.orc_row_limit.restype = i64
    L.orc_row_limit.argtypes = [i64, i64, i64, i32, i64]
    L.orc_attn_rows.restype = i32
    L.orc_attn_rows.argtypes = [P, P, P, P, P, P, i64, i64, i32, i32, i64, i64, f64,
                                P, i64, P, P, P, i32]
    L.orc_attn_rows_identity.restype = i32
    L.orc_attn_rows_identity.argtypes = [P, P, P, i64, i64, i32, i32, i64, i64,
                                         P, i64, P, P, i32]
    L.orc_attn_rows_bs.restype = i32
    L.orc_attn_rows_bs.argtypes = [P, P, P, P, P, P, i64, i64, i32, i32, i64, i64, f64,
                                   P, i64, i64, P, i64, P, P, P, i32]
    L.orc_attn_rows_identity_bs.restype = i32
    L.orc_attn_rows_identity_bs.argtypes = [P, P, P, i64, i64, i32, i32, i64, i64,
                                            P, i64, i64, P, i64, P, P, i32]
    L.orc_attn_rows_split.restype = i32
    L.orc_attn_rows_split.argtypes = [P, P, P, P, P, P, i64, i64, i32, i32, i64, i64, f64,
                                      i32, i64, P, i64, P, P, P, i32]
    L.orc_attn_rows_identity_split.restype = i32
    L.orc_attn_rows_identity_split.argtypes = [P, P, P, i64, i64, i32, i32, i64, i64, i32, i64,
                                               P, i64, P, P, i32]
    L.orc_w8a8_quant_act.restype = i32
    L.orc_w8a8_quant_act.argtypes = [P, i64, i64, P, P]
    L.orc_w8a8_quant_weight.restype = i32
    L.orc_w8a8_quant_weight.argtypes = [P, i64, i64, P, P]
    L.orc_w8a8_gemm_rows.restype = i32
    L.orc_w8a8_gemm_rows.argtypes = [P, P, P, P, i64, i64, i64, P, i64, P, i32]
    L.orc_attn_fp64_rows.restype = i32
    L.orc_attn_fp64_rows.argtypes = [P, P, P, i64, i64, i32, i32, i64, P, i64, P, i32]
    L.orc_attn_fp64_rows_win.restype = i32
    L.orc_attn_fp64_rows_win.argtypes = [P, P, P, i64, i64, i32, i64, i64, i64, P, i64, P,
                                         i32]
    L.orc_attn_rows_win.restype = i32
    L.orc_attn_rows_win.argtypes = [P, P, P, P, P, P, i64, i64, i32, i64, i64, i64, i64, f64,
                                    i32, i64, P, i64, P, P, P, i32]
    L.orc_attn_rows_identity_win.restype = i32
    L.orc_attn_rows_identity_win.argtypes = [P, P, P, i64, i64, i32, i64, i64, i64, i64, i32,
                                             i64, P, i64, P, P, i32]
    L.orc_row_window_export.restype = None
    L.orc_row_window_export.argtypes = [i64, i64, i64, i32, i64, i64, i64, P]
    L.orc_exp2_poly.restype = ctypes.c_float
    L.orc_exp2_poly.argtypes = [ctypes.c_float]
    L.orc_exp2_poly_n.restype = None
    L.orc_exp2_poly_n.argtypes = [P, i64, P]
    L.orc_set_exp2_poly_from.restype = None
    L.orc_set_exp2_poly_from.argtypes = [i32]
    L.orc_get_exp2_poly_from.restype = i32
    L.orc_get_exp2_poly_from.argtypes = []
    L.orc_attn_rows_pert.restype = i32
    L.orc_attn_rows_pert.argtypes = [P, P, P, P, P, P, i64, i64, i32, i32, i64, i64, f64, P,
                                     f64, P, i64, P, P, P, i32]
    return L


def exp2_poly(x):
    """The recipe's software exp2 (``orc_exp2_poly``), elementwise on fp32."""
    x = np.ascontiguousarray(x, np.float32)
    y = np.empty_like(x)
    lib().orc_exp2_poly_n(_p(x), x.size, _p(y))
    return y


def exp2_poly_from():
    """The first KV-tile column whose exponentials use the software exp2."""
    return int(lib().orc_get_exp2_poly_from())


@contextlib.contextmanager
def exp2_poly_columns(first):
    """Within the block the oracle evaluates the exponentials of tile columns
    >= `first` with the software exp2 (tkv or more: none); afterwards the
    recipe's own value is restored.  Test-suite only."""
    saved = exp2_poly_from()
    lib().orc_set_exp2_poly_from(int(first))
    try:
        yield
    finally:
        lib().orc_set_exp2_poly_from(saved)


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _threads(n):
    return int(n) if n else (os.cpu_count() or 1)


# ---------------------------------------------------------------- e4m3

def e4m3_encode(x):
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, np.uint8)
    lib().orc_e4m3_encode_n(_p(x), x.size, _p(out))
    return out


def e4m3_decode(codes):
    L = lib()
    table = np.array([L.orc_e4m3_decode(c) for c in range(256)], np.float64)
    return table[np.asarray(codes, dtype=np.uint8)]


# ---------------------------------------------------------------- quantization

def quant_head(q, k, v, rope=None, eq=False):
    """Quantize one head.  q [nq, D], k/v [nkv, D] as uint16 bf16 bits.

    rope: None, or (q_cos, q_sin, k_cos, k_sin), float32 [nq, D/2] and
    [nkv, D/2]: Q and K are first rotated pairwise by those angles
    (``orc_quant_head_rope``).
    eq: the channel-equalised variant (``orc_quant_head_eq``; no rotation):
    channel d of Q is multiplied and channel d of the smoothed K divided by
    2^eq_exp[d] before the block quantization.

    Returns a dict: q8 [nq_pad, D] int8, qs [nq_blk] f32, k8 [nkv_pad, D] int8,
    ks [nkv_blk] f32, mu [D] f32, v8 [nkv, D] uint8 e4m3 codes, vs [D] f32
    (and eq_exp [D] int8 with eq).
    """
    q = np.ascontiguousarray(q, np.uint16)
    k = np.ascontiguousarray(k, np.uint16)
    v = np.ascontiguousarray(v, np.uint16)
    nq, D = q.shape
    nkv = k.shape[0]
    nqb, nkb = -(-nq // BLK), -(-nkv // BLK)
    out = dict(q8=np.empty((nqb * BLK, D), np.int8), qs=np.empty(nqb, np.float32),
               k8=np.empty((nkb * BLK, D), np.int8), ks=np.empty(nkb, np.float32),
               mu=np.empty(D, np.float32), v8=np.empty((nkv, D), np.uint8),
               vs=np.empty(D, np.float32))
    outs = [_p(out[key]) for key in ("q8", "qs", "k8", "ks", "mu", "v8", "vs")]
    if eq:
        if rope is not None:
            raise ValueError("the equalised variant takes no rotation")
        out["eq_exp"] = np.empty(D, np.int8)
        rc = lib().orc_quant_head_eq(_p(q), _p(k), _p(v), nq, nkv, D, *outs, _p(out["eq_exp"]))
    elif rope is None:
        rc = lib().orc_quant_head(_p(q), _p(k), _p(v), nq, nkv, D, *outs)
    else:
        tabs = [np.ascontiguousarray(t, np.float32) for t in rope]
        for t, n in zip(tabs, (nq, nq, nkv, nkv)):
            if t.shape != (n, D // 2):
                raise ValueError("rotation table shape %s, expected %s" % (t.shape, (n, D // 2)))
        rc = lib().orc_quant_head_rope(_p(q), _p(k), _p(v), nq, nkv, D,
                                       *[_p(t) for t in tabs], *outs)
    if rc:
        raise MemoryError("oracle quantization failed")
    out["nq"], out["nkv"], out["D"] = nq, nkv, D
    return out


def quant(q, k, v, rope=None, eq=False):
    """Quantize [B, H, N, D] bf16-bit tensors head by head; returns stacked arrays.
    rope, eq: as for quant_head (the same tables for every batch entry and head)."""
    B, H = q.shape[:2]
    heads = [quant_head(q[b, h], k[b, h], v[b, h], rope, eq) for b in range(B) for h in range(H)]
    out = {}
    for key in ("q8", "qs", "k8", "ks", "mu", "v8", "vs") + (("eq_exp",) if eq else ()):
        a = np.stack([hd[key] for hd in heads])
        out[key] = a.reshape((B, H) + a.shape[1:])
    return out


def qk_int32(q8, k8, i0, ni, j0, nj):
    q8 = np.ascontiguousarray(q8, np.int8)
    k8 = np.ascontiguousarray(k8, np.int8)
    out = np.empty((ni, nj), np.int32)
    lib().orc_qk_int32(_p(q8), _p(k8), q8.shape[1], i0, ni, j0, nj, _p(out))
    return out


def row_limit(i, nq, nkv, mask, mb):
    return lib().orc_row_limit(i, nq, nkv, mask, mb)


def row_window(i, nq, nkv, mask, mb, win=0, sink=0):
    """(sink_end, lo, hi): query row i sees keys [0, sink_end) and [lo, hi)."""
    out = np.empty(3, np.int64)
    lib().orc_row_window_export(i, nq, nkv, mask, mb, win, sink, _p(out))
    return tuple(int(x) for x in out)


def window_keys(nq, nkv, frame, win, sink):
    """The keys a sliding-window step attends to: the union over its nq query
    rows (the newest nq of nkv cache tokens) of the visible keys, as indices
    into the cache, ascending: the reference context [0, min(sink, nkv)) and
    the window [lo(first row), hi(last row)).  Quantizing only these keys
    (gathered in this order) is the windowed reading of the streaming cache;
    the window attention over the gathered keys, with the same (frame, win,
    sink), gives every query row the same visible keys (the gap removed
    between the reference context and the window is a whole number of
    frames)."""
    se0, lo0, _ = row_window(0, nq, nkv, MASK_SLIDING_WINDOW, frame, win, sink)
    se1, _, hi1 = row_window(nq - 1, nq, nkv, MASK_SLIDING_WINDOW, frame, win, sink)
    se = min(int(sink), int(nkv))
    lo = max(int(lo0), se)
    return np.concatenate([np.arange(se), np.arange(lo, int(hi1))]).astype(np.int64)


def _window(window):
    frame, win, sink = (int(x) for x in window)
    return frame, win, sink


# ---------------------------------------------------------------- attention

def _block_mask(block_mask, nkv, tkv):
    """(pointer, bq, n_kt) of an optional block mask [n_qt, n_kt] of one head."""
    if block_mask is None:
        return None, 0, 0, None
    bm = np.ascontiguousarray(block_mask, np.uint8)
    if bm.ndim != 2 or bm.shape[1] < -(-nkv // tkv):
        raise ValueError("block mask must be [n_qtiles, ceil(Nkv / tkv)]")
    return _p(bm), BQ, bm.shape[1], bm


def attn_rows(qh, rows, mask=MASK_NONE, mb=0, tkv=TKV, eps=EPS, with_slack=True,
              threads=None, block_mask=None, kv_splits=1, window=None, pert=None,
              pert_eps=0.0):
    """Same-quantization attention of one quantized head on the given rows.

    block_mask: optional uint8 [ceil(Nq / 128), ceil(Nkv / tkv)] of this head;
    query row i visits KV tile t only if block_mask[i // 128, t] != 0.
    kv_splits > 1: the split-KV form (``orc_attn_rows_split``): the KV tiles of
    each 128-query tile in that many ranges, each its own online softmax,
    merged (not combined with a block mask).
    window: (frame, win, sink) for the sliding-window mask with a reference
    context (``orc_attn_rows_win``; mask and mb are then ignored).
    pert, pert_eps (test hook, dense form only): int8 [Nq, Nkv] of -1, 0, +1;
    the exp2 result y of row i and key j becomes the fp32 value nearest to
    y (1 + pert[i, j] pert_eps) on y's side (``orc_attn_rows_pert``).
    Returns (o [n, D] float64 of the fp32 recipe, slack [n, D] or None, lse [n]).
    """
    rows = np.ascontiguousarray(rows, np.int64)
    n, D = rows.size, qh["D"]
    o = np.empty((n, D), np.float64)
    slack = np.empty((n, D), np.float64) if with_slack else None
    lse = np.empty(n, np.float64)
    q8 = np.ascontiguousarray(qh["q8"])
    k8 = np.ascontiguousarray(qh["k8"])
    v8 = np.ascontiguousarray(qh["v8"])
    qs = np.ascontiguousarray(qh["qs"])
    ks = np.ascontiguousarray(qh["ks"])
    vs = np.ascontiguousarray(qh["vs"])
    if pert is not None:
        if window is not None or block_mask is not None or kv_splits > 1:
            raise ValueError("pert is supported on the dense form only")
        pert = np.ascontiguousarray(pert, np.int8)
        if pert.shape != (qh["nq"], qh["nkv"]):
            raise ValueError("pert must be int8 [Nq, Nkv]")
        rc = lib().orc_attn_rows_pert(_p(q8), _p(qs), _p(k8), _p(ks), _p(v8), _p(vs),
                                      qh["nq"], qh["nkv"], D, mask, mb, tkv, eps, _p(pert),
                                      float(pert_eps), _p(rows), n, _p(o),
                                      _p(slack) if slack is not None else None, _p(lse),
                                      _threads(threads))
    elif window is not None:
        if block_mask is not None:
            raise ValueError("window and block_mask are not combined")
        frame, win, sink = _window(window)
        rc = lib().orc_attn_rows_win(_p(q8), _p(qs), _p(k8), _p(ks), _p(v8), _p(vs),
                                     qh["nq"], qh["nkv"], D, frame, win, sink, tkv, eps,
                                     max(int(kv_splits), 1), BQ, _p(rows), n, _p(o),
                                     _p(slack) if slack is not None else None, _p(lse),
                                     _threads(threads))
    elif kv_splits > 1:
        if block_mask is not None:
            raise ValueError("kv_splits and block_mask are not combined")
        rc = lib().orc_attn_rows_split(_p(q8), _p(qs), _p(k8), _p(ks), _p(v8), _p(vs),
                                       qh["nq"], qh["nkv"], D, mask, mb, tkv, eps, kv_splits, BQ,
                                       _p(rows), n, _p(o),
                                       _p(slack) if slack is not None else None, _p(lse),
                                       _threads(threads))
    else:
        bptr, bq, n_kt, _keep = _block_mask(block_mask, qh["nkv"], tkv)
        rc = lib().orc_attn_rows_bs(_p(q8), _p(qs), _p(k8), _p(ks), _p(v8), _p(vs),
                                    qh["nq"], qh["nkv"], D, mask, mb, tkv, eps, bptr, bq, n_kt,
                                    _p(rows), n, _p(o), _p(slack) if slack is not None else None,
                                    _p(lse), _threads(threads))
    if rc:
        raise ValueError("orc_attn_rows: invalid arguments")
    return o, slack, lse


def attn_rows_identity(q, k, v, rows, mask=MASK_NONE, mb=0, tkv=TKV, threads=None,
                       block_mask=None, kv_splits=1, window=None):
    """The oracle's tiled loop with identity quantizers, fp64 throughout
    (kv_splits > 1: the split-KV form; window: the sliding-window mask; as
    for attn_rows)."""
    q = np.ascontiguousarray(q, np.float64)
    k = np.ascontiguousarray(k, np.float64)
    v = np.ascontiguousarray(v, np.float64)
    rows = np.ascontiguousarray(rows, np.int64)
    n, D = rows.size, q.shape[1]
    o = np.empty((n, D), np.float64)
    lse = np.empty(n, np.float64)
    if window is not None:
        if block_mask is not None:
            raise ValueError("window and block_mask are not combined")
        frame, win, sink = _window(window)
        rc = lib().orc_attn_rows_identity_win(_p(q), _p(k), _p(v), q.shape[0], k.shape[0], D,
                                              frame, win, sink, tkv, max(int(kv_splits), 1), BQ,
                                              _p(rows), n, _p(o), _p(lse), _threads(threads))
    elif kv_splits > 1:
        if block_mask is not None:
            raise ValueError("kv_splits and block_mask are not combined")
        rc = lib().orc_attn_rows_identity_split(_p(q), _p(k), _p(v), q.shape[0], k.shape[0], D,
                                                mask, mb, tkv, kv_splits, BQ, _p(rows), n, _p(o),
                                                _p(lse), _threads(threads))
    else:
        bptr, bq, n_kt, _keep = _block_mask(block_mask, k.shape[0], tkv)
        rc = lib().orc_attn_rows_identity_bs(_p(q), _p(k), _p(v), q.shape[0], k.shape[0], D,
                                             mask, mb, tkv, bptr, bq, n_kt, _p(rows), n, _p(o),
                                             _p(lse), _threads(threads))
    if rc:
        raise ValueError("orc_attn_rows_identity: invalid arguments")
    return o, lse


def attn_fp64_rows(q, k, v, rows, mask=MASK_NONE, mb=0, threads=None, window=None):
    """Full-precision softmax attention of one head from bf16 bits, fp64
    (window: (frame, win, sink), the sliding-window mask)."""
    q = np.ascontiguousarray(q, np.uint16)
    k = np.ascontiguousarray(k, np.uint16)
    v = np.ascontiguousarray(v, np.uint16)
    rows = np.ascontiguousarray(rows, np.int64)
    n, D = rows.size, q.shape[1]
    o = np.empty((n, D), np.float64)
    if window is not None:
        frame, win, sink = _window(window)
        rc = lib().orc_attn_fp64_rows_win(_p(q), _p(k), _p(v), q.shape[0], k.shape[0], D, frame,
                                          win, sink, _p(rows), n, _p(o), _threads(threads))
    else:
        rc = lib().orc_attn_fp64_rows(_p(q), _p(k), _p(v), q.shape[0], k.shape[0], D, mask, mb,
                                      _p(rows), n, _p(o), _threads(threads))
    if rc:
        raise ValueError("orc_attn_fp64_rows: invalid arguments")
    return o


def bf16_bits_to_f64(x):
    return (np.asarray(x, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def accuracy(o, ref):
    """cosine similarity and mean relative L1 of o against ref (flattened)."""
    o = np.asarray(o, np.float64).ravel()
    ref = np.asarray(ref, np.float64).ravel()
    cos = float(o @ ref / (np.linalg.norm(o) * np.linalg.norm(ref)))
    rel_l1 = float(np.abs(o - ref).sum() / np.abs(ref).sum())
    return cos, rel_l1


def c0(D):
    """fp32(log2(e)/sqrt(D)) as the recipe defines it (for tests)."""
    return np.float32(math.log2(math.e) / math.sqrt(D))


# ---------------------------------------------------------------- W8A8 linear layer

W8A8_G = 128  # channels per quantization group along K


def w8a8_quant_act(x):
    """X [M, K] bf16 bits -> (xq [M, K] int8, sx [M, K/128] f32): one scale
    per token and 128-channel group."""
    x = np.ascontiguousarray(x, np.uint16)
    M, K = x.shape
    xq = np.empty((M, K), np.int8)
    sx = np.empty((M, K // W8A8_G), np.float32)
    if lib().orc_w8a8_quant_act(_p(x), M, K, _p(xq), _p(sx)):
        raise ValueError("orc_w8a8_quant_act: K must be a multiple of 128")
    return xq, sx


def w8a8_quant_weight(w):
    """W [N, K] bf16 bits -> (wq [N, K] int8, sw [N/128, K/128] f32): one
    scale per 128 x 128 block."""
    w = np.ascontiguousarray(w, np.uint16)
    N, K = w.shape
    wq = np.empty((N, K), np.int8)
    sw = np.empty((N // W8A8_G, K // W8A8_G), np.float32)
    if lib().orc_w8a8_quant_weight(_p(w), N, K, _p(wq), _p(sw)):
        raise ValueError("orc_w8a8_quant_weight: N and K must be multiples of 128")
    return wq, sw


def w8a8_gemm_rows(xq, sx, wq, sw, rows, threads=None):
    """Rows of Y = X W^T from the quantized operands (fp32, before the bf16
    rounding), promoting each 128-channel group's exact integer dot product
    into an fp32 running sum with one fma, in ascending group order."""
    xq, sx, wq, sw = (np.ascontiguousarray(a) for a in (xq, sx, wq, sw))
    rows = np.ascontiguousarray(rows, np.int64)
    M, K = xq.shape
    N = wq.shape[0]
    y = np.empty((rows.size, N), np.float32)
    if lib().orc_w8a8_gemm_rows(_p(xq), _p(sx), _p(wq), _p(sw), M, N, K, _p(rows), rows.size,
                                _p(y), _threads(threads)):
        raise ValueError("orc_w8a8_gemm_rows: invalid arguments")
    return y
