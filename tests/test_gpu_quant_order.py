"""The K mean's ordered fp64 sum on the GPU.

The recipe's mean adds each channel's per-block fp64 sums in ascending block
order, every addition rounded.  On normal data most orders give the same sum;
here some channels hold values whose magnitudes span far more than fp64's 53
bits, so their block sums cancel and round, and only the ascending order
gives the oracle's mean bit for bit.  The inputs also cover some extreme
bf16 magnitudes (2^-60 .. 2^60) in the Q/K block quantization.
"""
import numpy as np
import pytest

import oracle
from bit_quantized_attention_sage_b200 import synth

from gpu_helpers import check_quant_head, run

pytestmark = pytest.mark.gpu


def _wide_range_k(k, seed):
    """Channels 0-3 of every head: values of random sign with magnitudes
    2^U(-60, 60) (channel 0), alternating +-2^50 and +-2^-50 (channel 1),
    a huge value early and tiny ones after it (channel 2), large cancelling
    pairs with a small remainder (channel 3)."""
    rng = np.random.default_rng(seed)
    kf = oracle.bf16_bits_to_f64(k).astype(np.float32)
    B, H, N, D = kf.shape
    sign = rng.choice([-1.0, 1.0], size=(B, H, N))
    kf[..., 0] = sign * np.exp2(rng.uniform(-60, 60, size=(B, H, N)))
    alt = np.where(np.arange(N) % 2 == 0, 2.0 ** 50, 2.0 ** -50)
    kf[..., 1] = sign * alt
    kf[..., 2] = sign * 2.0 ** -40
    kf[:, :, 5, 2] = 2.0 ** 60
    kf[..., 3] = np.where(np.arange(N) % 2 == 0, 3.0 * 2.0 ** 45, -3.0 * 2.0 ** 45) + sign
    return synth.f32_to_bf16_bits(kf)


@pytest.mark.parametrize("n,D", [(1000, 128), (4100, 64), (9000, 128)])
def test_mean_matches_the_ordered_sum(n, D):
    w = synth.Workload("order_%d_%d" % (n, D), 1, 2, 300, n, D, k_offset_var=4.0, seed=90 + n)
    q, k, v = synth.full(w)
    k = _wide_range_k(k, 91 + n)
    qkv, _, _, _ = run(q, k, v)
    for h in range(w.H):
        check_quant_head(qkv, 0, h, oracle.quant_head(q[0, h], k[0, h], v[0, h]))
