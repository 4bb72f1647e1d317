"""Calibrate the background-head gate magnitude gamma of the synthetic workloads.

TEST INFRASTRUCTURE.  For each (H, d) this bisects gamma so that, with gate
weights w_j = +1/H on signal heads and -gamma/H on background heads, about 1%
of pure background keys reach I >= 0.5.  The 1% is the small false-positive
leakage the pages report for the sigmoid gate (gist.science section 5,
"Context-Independent Overhead"; blog page, limitation 3).  Scores come from the
oracle only.  Prints the table that ``synth.GATE_GAMMA`` stores.

    python -m oracle.calibrate_gate
"""
from __future__ import annotations

import sys

import numpy as np
import torch

import synth
from oracle import index_score

TARGET = 0.01


def pass_rate(gamma, q, keys, H, d):
    w = synth.gate_weights(H, gamma)[None, :]
    z = index_score(q, "bf16", w, keys, "bf16", None, np.array([0, keys.shape[0]], np.int64), H, d,
                    want_I=False)
    return float(np.mean(z >= 0.0))


def calibrate(H, d, n=65536, seed=12345, iters=30):
    g = torch.Generator().manual_seed(seed + 131 * H + d)
    u = synth.unit(g, d)
    q = synth.bf16_bits(synth.indexer_queries(g, H, d, u)[None])
    keys = synth.bf16_bits(synth.background_keys(g, n, d))
    lo, hi = 0.0, 64.0          # pass_rate is non-increasing in gamma
    for _ in range(iters):
        mid = 0.5 * (lo + hi)
        if pass_rate(mid, q, keys, H, d) > TARGET:
            lo = mid
        else:
            hi = mid
    return round(hi, 3), pass_rate(hi, q, keys, H, d)


def main(argv=None):
    shapes = sorted(synth.GATE_GAMMA) if not argv else [tuple(map(int, a.split("x"))) for a in argv]
    for H, d in shapes:
        gamma, rate = calibrate(H, d)
        print(f"    ({H}, {d}): {gamma},   # background pass rate {rate:.4f}")


if __name__ == "__main__":
    main(sys.argv[1:])
