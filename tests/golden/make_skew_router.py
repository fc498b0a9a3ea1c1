"""Writes tests/golden/skew_router_scale.txt: per-expert router row scales that
give the skewed-routing workload its expert popularity.

The workload: T = 4096 tokens at K2 shapes, correction bias ~N(0, 0.05), and
router rows W_g[e] = s_e * u_e (u_e the seeded N(0, 0.02) rows). Popularity
is shaped by the row scales: a larger row gives a token-dependent logit of
larger spread, which wins the top 8 more often. Exact per-expert targets
cannot be hit this way (large rows saturate the sigmoid at 1.0 in fp32, and
among saturated experts the bias alone decides), so the scales follow a
two-parameter law s = A * rank^-gamma over a seeded random permutation of the
experts, plus 16 zero rows (logit 0, score 0.5: never in a token's top 8, so
those experts are empty). A and gamma are picked on a grid so that the
oracle's routing (oracle.moe.route, float64) of the seeded CPU tokens gives
counts whose log-log slope against popularity rank over ranks 8..128 is
closest to the Zipf exponent -1.2, with the hottest expert above 800 tokens.
Only the scale table is stored; the GPU tests draw their own tokens and check
the skew that results (hottest expert over 800 tokens, empty experts).

Run from the repository root: python tests/golden/make_skew_router.py
"""
from __future__ import annotations

import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import synth  # noqa: E402
from oracle import moe as orc  # noqa: E402

T = 4096
E = 384
K = 8
EMPTY = 16
BIAS_STD = 0.05
OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "skew_router_scale.txt")


def scales_for(A, gamma):
    perm = np.random.default_rng(1234).permutation(E)
    s = np.zeros(E)
    live = perm[: E - EMPTY]
    s[live] = A * np.arange(1, E - EMPTY + 1, dtype=np.float64) ** -gamma
    return s


def slope(counts):
    c = np.sort(counts)[::-1][7:128].astype(np.float64)
    r = np.arange(8, 8 + len(c), dtype=np.float64)
    keep = c > 0
    return np.polyfit(np.log(r[keep]), np.log(c[keep]), 1)[0]


def route_counts(x, scale):
    W, b = synth.make_router(synth.K2, bias_std=BIAS_STD, row_scale=torch.from_numpy(scale))
    r = orc.route(x, W.numpy().astype(np.float64), b.numpy().astype(np.float64), K)
    return np.bincount(r.ids.ravel(), minlength=E)


def main():
    x = synth.make_tokens(synth.K2, T).float().numpy().astype(np.float64)
    best = None
    for A in (0.4, 0.5, 0.7, 1.0):
        for gamma in (0.2, 0.25, 0.3, 0.35, 0.4):
            c = route_counts(x, scales_for(A, gamma))
            sl = slope(c)
            ok = c.max() > 800
            print(f"A {A:3.1f} gamma {gamma:3.1f}: max {c.max():5d} empty {int((c == 0).sum()):3d} "
                  f"slope {sl:6.2f}{'' if ok else '  (max <= 800)'}")
            if ok and (best is None or abs(sl + 1.2) < abs(best[0] + 1.2)):
                best = (sl, A, gamma)
    assert best is not None, "no grid point gives a hottest expert above 800 tokens"
    sl, A, gamma = best
    scale = scales_for(A, gamma)
    c = route_counts(x, scale)
    with open(OUT, "w") as f:
        f.write("# per-expert router row scales for the skewed-routing workload "
                "(written by make_skew_router.py)\n")
        f.write(f"# A {A} gamma {gamma}; realised on the seeded CPU tokens: max {c.max()}, "
                f"empty {(c == 0).sum()}, slope over ranks 8..128 {sl:.2f}, "
                f"top5 {[int(v) for v in np.sort(c)[::-1][:5]]}\n")
        for v in scale:
            f.write(f"{v:.9g}\n")
    print("wrote", OUT, "A", A, "gamma", gamma, "slope", round(sl, 2))


if __name__ == "__main__":
    main()
