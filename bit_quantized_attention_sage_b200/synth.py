"""Seeded synthetic inputs for the quantized-attention workloads.

This module only draws random tensors; it holds none of the method's
arithmetic.  Both the device path (through the tests and the benchmark) and
the CPU oracle are fed from it.

Every (tensor, batch, head) slice has its own counter-keyed stream
(numpy ``default_rng([seed, tensor_id, b, h])``), so one head can be
regenerated on its own without drawing the others.

Value recipe (the pages' video-DiT workloads, with their shapes):
  * Q, V ~ N(0, 1); K ~ N(0, 1)
  * optional per-(b, h, channel) K offset ~ N(0, var) with var = 4 (std 2),
    constant over tokens, added before rounding to bf16
  * optional 4 distinct K outlier channels per (b, h), multiplied by ``mag``
  * everything rounded to bf16 with round-to-nearest-even.
"""
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

TID_Q, TID_K, TID_V, TID_OFFSET, TID_OUTLIER = 0, 1, 2, 3, 4


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    Nq: int
    Nkv: int
    D: int
    mask: int = 0          # 0 none, 1 causal, 2 block-causal, 3 sliding window
    mask_block: int = 0    # block (2) or frame (3) length
    k_offset_var: float = 0.0
    outlier_mag: float = 0.0
    seed: int = 0
    extra: dict = field(default_factory=dict, compare=False, hash=False)
    win: int = 0           # sliding window: frames per window
    sink: int = 0          # sliding window: reference-context tokens

    def visible_pairs(self) -> int:
        """Number of (query, key) pairs that the mask leaves visible, per head."""
        nq, nkv, off = self.Nq, self.Nkv, self.Nkv - self.Nq
        g = np.arange(nq, dtype=np.int64) + off
        if self.mask == 1:
            lim = g + 1
        elif self.mask == 2:
            lim = (g // self.mask_block + 1) * self.mask_block
        elif self.mask == 3:
            s0 = min(self.sink, nkv)
            f = np.maximum(g - s0, 0) // self.mask_block
            hi = np.minimum(s0 + (f + 1) * self.mask_block, nkv)
            lo = s0 + np.maximum(f - self.win + 1, 0) * self.mask_block
            return int(np.where(g < s0, s0, s0 + hi - lo).sum())
        else:
            lim = np.full(nq, nkv, np.int64)
        return int(np.minimum(lim, nkv).sum())

    def ops(self) -> int:
        """Algorithmic 8-bit tensor operations: 4 * D per visible pair per head."""
        return 4 * self.D * self.B * self.H * self.visible_pairs()


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    u = np.ascontiguousarray(x, np.float32).view(np.uint32)
    return ((u + (((u >> 16) & 1) + 0x7FFF)) >> 16).astype(np.uint16)


def _rng(seed, tid, b, h):
    return np.random.default_rng([int(seed), int(tid), int(b), int(h)])


def head_q(w: Workload, b: int, h: int) -> np.ndarray:
    return f32_to_bf16_bits(_rng(w.seed, TID_Q, b, h).standard_normal((w.Nq, w.D), np.float32))


def head_v(w: Workload, b: int, h: int) -> np.ndarray:
    return f32_to_bf16_bits(_rng(w.seed, TID_V, b, h).standard_normal((w.Nkv, w.D), np.float32))


def head_k(w: Workload, b: int, h: int) -> np.ndarray:
    k = _rng(w.seed, TID_K, b, h).standard_normal((w.Nkv, w.D), np.float32)
    if w.outlier_mag > 0:
        ch = _rng(w.seed, TID_OUTLIER, b, h).choice(w.D, 4, replace=False)
        k[:, ch] *= np.float32(w.outlier_mag)
    if w.k_offset_var > 0:
        off = _rng(w.seed, TID_OFFSET, b, h).standard_normal(w.D) * np.sqrt(w.k_offset_var)
        k += off.astype(np.float32)[None, :]
    return f32_to_bf16_bits(k)


def head(w: Workload, b: int, h: int):
    return head_q(w, b, h), head_k(w, b, h), head_v(w, b, h)


def full(w: Workload, threads: int = 8):
    """All heads: (q, k, v) uint16 arrays [B, H, N, D] of bf16 bits."""
    q = np.empty((w.B, w.H, w.Nq, w.D), np.uint16)
    k = np.empty((w.B, w.H, w.Nkv, w.D), np.uint16)
    v = np.empty((w.B, w.H, w.Nkv, w.D), np.uint16)

    def one(bh):
        b, h = divmod(bh, w.H)
        q[b, h], k[b, h], v[b, h] = head(w, b, h)

    with ThreadPoolExecutor(max_workers=threads) as ex:
        list(ex.map(one, range(w.B * w.H)))
    return q, k, v


# The five workload families: a tiny parity case, a streaming block-causal
# step, the 480p and 720p bidirectional video-DiT shapes, and the sweep.
TINY = Workload("tiny_b1h2_n1024_d128", 1, 2, 1024, 1024, 128, k_offset_var=4.0, seed=1001)
STREAMING = Workload("streaming_b1h24_nq2040_nkv26520_d128_blockcausal2040", 1, 24, 2040, 26520,
                     128, mask=2, mask_block=2040, k_offset_var=4.0, seed=1002)
# one streaming step under the sliding window: the newest frame (2040
# tokens) against a cache whose first frame is the reference context,
# attending to it and the 4 newest frames (its own included)
STREAMING_WINDOW = Workload("streaming_window_b1h24_nq2040_nkv26520_d128_frame2040_win4_sink2040",
                            1, 24, 2040, 26520, 128, mask=3, mask_block=2040, k_offset_var=4.0,
                            seed=1005, win=4, sink=2040)
# the same step with the windowed quantization of the cache: only the
# reference context and the window (10200 of the 26520 keys) are quantized
STREAMING_WINDOW_Q = Workload(
    "streaming_window_winquant_b1h24_nq2040_nkv26520_d128_frame2040_win4_sink2040",
    1, 24, 2040, 26520, 128, mask=3, mask_block=2040, k_offset_var=4.0, seed=1005, win=4,
    sink=2040, extra={"window_quant": True})
P480 = Workload("video480p_b1h12_n32760_d128", 1, 12, 32760, 32760, 128, outlier_mag=20.0,
                seed=1003)
P720 = Workload("video720p_b1h40_n75600_d128", 1, 40, 75600, 75600, 128, outlier_mag=20.0,
                seed=1004)


def sweep():
    pts = []
    idx = 0
    for n in (4096, 8192, 16384, 32768, 65536, 131072):
        for D in (64, 128):
            for mask in (0, 2):
                for mag in (0.0, 5.0, 20.0):
                    pts.append(Workload("sweep_n%d_d%d_%s_mag%d" % (n, D, "bc" if mask else "nc",
                                                                   int(mag)),
                                        1, 16, n, n, D, mask=mask,
                                        mask_block=2040 if mask else 0,
                                        outlier_mag=mag, seed=2000 + idx))
                    idx += 1
    return pts


WORKLOADS = {w.name: w for w in (TINY, STREAMING, STREAMING_WINDOW, STREAMING_WINDOW_Q,
                                  P480, P720)}
