"""Write tests/golden/oracle_tiny_regression.txt and
tests/golden/oracle_window_regression.txt from the CPU oracle only.

A regression fixture: a later change of the oracle's arithmetic shows up as a
mismatch, and the commit that changes it must name the passage (or the
reading of it) that justifies the change.

Run:  python tests/golden/make_golden.py
"""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from bit_quantized_attention_sage_b200 import synth  # noqa: E402

CASE = synth.Workload("golden_tiny", 1, 1, 96, 160, 64, mask=2, mask_block=48,
                      k_offset_var=4.0, outlier_mag=5.0, seed=77)
ROWS = [0, 1, 47, 48, 63, 64, 95]
OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_tiny_regression.txt")


WIN_CASE = synth.Workload("golden_window", 1, 1, 200, 900, 64, k_offset_var=4.0,
                          outlier_mag=5.0, seed=78)
WINDOW = (130, 2, 70)  # frame tokens, frames per window, reference-context tokens
WIN_ROWS = [0, 1, 69, 70, 127, 128, 199]
OUT_WIN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_window_regression.txt")


def compute_window():
    """The sliding-window form, unsplit and in 3 KV ranges."""
    q, k, v = synth.head(WIN_CASE, 0, 0)
    qh = oracle.quant_head(q, k, v)
    rows = np.array(WIN_ROWS)
    o1, _, l1 = oracle.attn_rows(qh, rows, window=WINDOW, threads=1)
    o3, _, l3 = oracle.attn_rows(qh, rows, window=WINDOW, kv_splits=3, threads=1)
    return o1, l1, o3, l3


def compute():
    q, k, v = synth.head(CASE, 0, 0)
    qh = oracle.quant_head(q, k, v)
    o, _, lse = oracle.attn_rows(qh, np.array(ROWS), CASE.mask, CASE.mask_block, threads=1)
    return qh, o, lse


def main():
    qh, o, lse = compute()
    with open(OUT, "w") as f:
        f.write("# written by tests/golden/make_golden.py from the CPU oracle only\n")
        f.write("# case: B1 H1 Nq96 Nkv160 D64 block-causal 48, K offset var 4, outliers x5, seed 77\n")
        f.write("qs %s\n" % " ".join("%.9g" % x for x in qh["qs"]))
        f.write("ks %s\n" % " ".join("%.9g" % x for x in qh["ks"]))
        f.write("mu %s\n" % " ".join("%.9g" % x for x in qh["mu"][:8]))
        f.write("vs %s\n" % " ".join("%.9g" % x for x in qh["vs"][:8]))
        f.write("q8sum %d\n" % int(qh["q8"].astype(np.int64).sum()))
        f.write("k8sum %d\n" % int(qh["k8"].astype(np.int64).sum()))
        f.write("v8sum %d\n" % int(qh["v8"].astype(np.int64).sum()))
        for r, row in enumerate(ROWS):
            f.write("o %d %s\n" % (row, " ".join("%.9g" % x for x in o[r, :8])))
            f.write("lse %d %.12g\n" % (row, lse[r]))
    o1, l1, o3, l3 = compute_window()
    with open(OUT_WIN, "w") as f:
        f.write("# written by tests/golden/make_golden.py from the CPU oracle only\n")
        f.write("# case: B1 H1 Nq200 Nkv900 D64, sliding window: frame 130, 2 frames, reference "
                "context 70; K offset var 4, outliers x5, seed 78\n")
        for tag, o, lse in (("s1", o1, l1), ("s3", o3, l3)):
            for r, row in enumerate(WIN_ROWS):
                f.write("o %s %d %s\n" % (tag, row, " ".join("%.9g" % x for x in o[r, :8])))
                f.write("lse %s %d %.12g\n" % (tag, row, lse[r]))


if __name__ == "__main__":
    main()
