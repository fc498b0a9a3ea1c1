"""The same layer definition as oracle.moe, written as explicit scalar loops.

Test infrastructure only. For tiny shapes (a few tokens, d and f of a few
dozen): every dot product is a Python loop over float64 scalars, top-k is
repeated arg-max scanning, e4m3 goes through the scalar codec. It shares no
vectorised code with oracle.moe, so an index, sign or transpose slip in
either one shows up as a mismatch.
"""
from __future__ import annotations

import math

import numpy as np

from . import e4m3

GROUP = 128


def _f32(v: float) -> float:
    return float(np.float32(v))


def _dot(a, b) -> float:
    s = 0.0
    for i in range(len(a)):
        s += float(a[i]) * float(b[i])
    return s


def _sig(z: float) -> float:
    if z < -700.0:
        return 0.0
    return 1.0 / (1.0 + math.exp(-z))


def _best(vals, allowed, taken):
    """Index of the largest allowed, untaken value; ties to the lower index."""
    best = -1
    for i in range(len(vals)):
        if not allowed[i] or taken[i]:
            continue
        if best < 0 or vals[i] > vals[best]:
            best = i
    return best


def route_token(xt, Wg, bias, k, scale=2.827, norm=True, n_group=1, topk_group=1):
    """Returns (ids list, weights list) for one token. With n_group > 1 the
    experts form n_group contiguous groups; a group scores the float32 sum of
    its two largest keys; only the topk_group best groups' experts compete."""
    E = len(Wg)
    logits = [_dot(xt, Wg[e]) for e in range(E)]
    scores = [_sig(l) for l in logits]
    keys = [_f32(_f32(_sig(_f32(logits[e]))) + _f32(bias[e])) for e in range(E)]
    gs = E // n_group
    gscore = []
    for g in range(n_group):
        members = keys[g * gs:(g + 1) * gs]
        first = _best(members, [True] * gs, [False] * gs)
        rest = [i != first for i in range(gs)]
        second = _best(members, rest, [False] * gs)
        gscore.append(members[first] if second < 0 else _f32(members[first] + members[second]))
    kept_groups = [False] * n_group
    for _ in range(topk_group):
        kept_groups[_best(gscore, [True] * n_group, kept_groups)] = True
    allowed = [kept_groups[e // gs] for e in range(E)]
    taken = [False] * E
    ids = []
    for _ in range(k):
        best = _best(keys, allowed, taken)
        taken[best] = True
        ids.append(best)
    total = sum(scores[e] for e in ids) if norm else 1.0
    w = [scores[e] / total * scale for e in ids]
    return ids, w


def _matvec(W, v):
    return [_dot(W[r], v) for r in range(len(W))]


def _quant_row(v):
    """Per-128 group e4m3 quantise then dequantise one row (float32 decisions)."""
    out = []
    for g0 in range(0, len(v), GROUP):
        grp = [np.float32(t) for t in v[g0:g0 + GROUP]]
        amax = np.float32(0.0)
        for t in grp:
            if abs(t) > amax:
                amax = np.float32(abs(t))
        s = np.float32(1.0) if amax == 0 else np.float32(amax / np.float32(448.0))
        for t in grp:
            q = e4m3.encode_scalar(float(np.float32(t / s)))
            out.append(e4m3.decode_scalar(q) * float(s))
    return out


def expert_token(xt, Wgate, Wup, Wdown, fp8=False):
    xin = _quant_row(xt) if fp8 else [float(t) for t in xt]
    g = _matvec(Wgate, xin)
    u = _matvec(Wup, xin)
    h = [(g[i] / (1.0 + math.exp(-g[i])) if g[i] > -700 else 0.0) * u[i] for i in range(len(g))]
    if fp8:
        h = _quant_row([_f32(t) for t in h])
    return _matvec(Wdown, h)


def layer_token(xt, Wg, bias, experts, shared, k, scale=2.827, norm=True, fp8=False):
    """y for one token; experts[e] and shared are (gate, up, down) float64
    matrices (already dequantised for FP8)."""
    ids, w = route_token(xt, Wg, bias, k, scale, norm)
    d = len(xt)
    y = [0.0] * d
    for j, e in enumerate(ids):
        o = expert_token(xt, *experts[e], fp8=fp8)
        for i in range(d):
            y[i] += w[j] * o[i]
    if shared is not None:
        o = expert_token(xt, *shared, fp8=fp8)
        for i in range(d):
            y[i] += o[i]
    return y, ids, w
