"""Calibrate the strength kappa of the Zipf router bias.

The skewed workloads route tokens of the full-size layer (hidden 6144, 256
experts, top-8) through a router whose per-expert bias is
    b_e = kappa * (-1.1 ln rank_e - mean),
rank_e being a seeded popularity permutation. kappa is chosen by bisection so
that a least-squares fit of ln(selection count) against ln(popularity rank),
over 8192 tokens (seed 0, step 0), has slope -1.10: expert popularity then
follows Zipf(s = 1.1).

Routing uses only the oracle. Writes ``synth/zipf_kappa.txt``.
Run: python tests/golden/calibrate_zipf.py
"""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import synth  # noqa: E402

H, E, K, TOKENS, SEED = 6144, 256, 8, 8192, 0


def slope(logits0, b_unit, rank, kappa):
    lg = logits0 + kappa * b_unit.astype(np.float64)[None, :]
    ids, _ = oracle.topk(lg, K)
    cnt = np.bincount(ids.ravel(), minlength=E)
    r = rank.astype(np.float64)
    m = cnt > 0
    return np.polyfit(np.log(r[m]), np.log(cnt[m].astype(np.float64)), 1)[0]


def main():
    wr = synth.router(SEED, 0, E, H)
    x = synth.x_f32(SEED, 0, TOKENS, H)
    logits0 = oracle.router_logits(wr, None, x)
    b_unit, rank = synth.zipf_bias(SEED, 0, E, kappa=1.0)
    lo, hi = 0.0, 4.0
    for _ in range(40):
        mid = 0.5 * (lo + hi)
        if slope(logits0, b_unit, rank, mid) > -1.1:
            lo = mid
        else:
            hi = mid
    kappa = 0.5 * (lo + hi)
    s = slope(logits0, b_unit, rank, kappa)
    out = os.path.join(ROOT, "synth", "zipf_kappa.txt")
    with open(out, "w") as f:
        f.write(f"{kappa:.6f}  # slope {s:.4f} over {TOKENS} tokens, seed {SEED}\n")
    print(f"kappa={kappa:.6f} slope={s:.4f} -> {out}")


if __name__ == "__main__":
    main()
