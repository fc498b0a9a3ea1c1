"""The parity tests' own checks, on the CPU: the permutation check accepts
the row order the dispatch is specified to produce and rejects each plausible
mistake in it; the routing check accepts valid near-tie choices and rejects
wrong ones; the token sample covers what the parity contract asks for."""
import numpy as np
import pytest

from oracle import moe as orc
from tests import gpu_util as gu


def _reference_rows(ids: np.ndarray, E: int):
    """Rows grouped by expert, ascending token order inside an expert (a
    stable sort of the pairs by expert), and the offsets of each expert."""
    T, k = ids.shape
    flat = ids.ravel()
    order = np.argsort(flat, kind="stable")  # pair index t*k + j, grouped by expert
    rows = np.empty(T * k, np.int64)
    rows[order] = np.arange(T * k)
    counts = np.bincount(flat, minlength=E)
    offsets = np.concatenate([[0], np.cumsum(counts)])
    return offsets, rows.reshape(T, k)


def _ids(T=200, E=16, k=4, seed=0):
    rng = np.random.default_rng(seed)
    ids = np.stack([rng.choice(E - 3, k, replace=False) for _ in range(T)])  # 3 experts empty
    return ids, E


def test_permutation_check_accepts_the_specified_order():
    ids, E = _ids()
    off, rows = _reference_rows(ids, E)
    msg = gu.check_permutation(ids, off, rows)
    assert "3 empty experts" in msg


@pytest.mark.parametrize("mistake", ["swap_within_expert", "swap_across_experts", "duplicate",
                                     "offsets_shifted", "empty_expert_gets_a_row"])
def test_permutation_check_catches_planted_mistakes(mistake):
    ids, E = _ids()
    off, rows = _reference_rows(ids, E)
    rows = rows.copy()
    off = off.copy()
    flat = rows.ravel()
    if mistake == "swap_within_expert":
        e = ids[0, 0]
        p = np.nonzero(ids.ravel() == e)[0][:2]  # two pairs of one expert
        flat[p[0]], flat[p[1]] = flat[p[1]], flat[p[0]]
    elif mistake == "swap_across_experts":
        a, b = 0, 1  # slots 0 and 1 of token 0 hold different experts
        flat[a], flat[b] = flat[b], flat[a]
    elif mistake == "duplicate":
        flat[5] = flat[6]
    elif mistake == "offsets_shifted":
        off[3] += 1
    else:
        empty = np.setdiff1d(np.arange(E), ids.ravel())[0]
        off[empty + 1:] += 0  # keep offsets, but claim the last row for the empty expert
        off[empty + 1] += 1
    with pytest.raises(AssertionError):
        gu.check_permutation(ids, off, flat.reshape(rows.shape))


def _route(T=64, E=16, k=4, d=32, seed=1):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, d))
    W = rng.standard_normal((E, d)) * 0.3
    b = rng.standard_normal(E) * 0.01
    return orc.route(x, W, b, k)


def test_routing_check_accepts_the_oracle_and_slot_swaps_within_the_band():
    r = _route()
    rc = gu.check_routing(r, r.ids, r.weights, 16, 2.827, True)
    assert rc.mismatch == 0 and rc.invalid == 0 and rc.weight_max_rel < 1e-12
    # a near-tie token may take the (k+1)-th expert instead of the k-th
    r.margin[3] = 0.0
    kth_plus = np.argsort(-r.keys[3].astype(np.float64), kind="stable")[4]
    r.keys[3, kth_plus] = r.keys[3, r.ids[3, 3]]  # make the two keys equal
    gid = r.ids.copy()
    gid[3, 3] = kth_plus
    w = orc.routing_weights(r.scores, gid)
    rc = gu.check_routing(r, gid, w, 16, 2.827, True)
    assert rc.mismatch == 0 and rc.invalid == 0
    assert rc.same_set[3] == False and rc.tie[3]


def test_routing_check_rejects_wrong_choices_and_weights():
    r = _route()
    gid = r.ids.copy()
    t = int(np.argmax(r.margin))  # a clear-cut token
    worst = np.argsort(-r.keys[t].astype(np.float64))[-1]
    gid[t, 0] = worst
    rc = gu.check_routing(r, gid, orc.routing_weights(r.scores, gid), 16, 2.827, True)
    assert rc.mismatch == 1 and rc.invalid >= 1
    # slots out of key order
    gid = r.ids.copy()
    gid[t] = gid[t][::-1]
    rc = gu.check_routing(r, gid, orc.routing_weights(r.scores, gid), 16, 2.827, True)
    assert rc.invalid == 1
    # biased keys used as weights
    wk = np.take_along_axis(r.keys.astype(np.float64), r.ids, axis=1)
    rc = gu.check_routing(r, r.ids, 2.827 * wk / wk.sum(1, keepdims=True), 16, 2.827, True)
    assert rc.weight_max_rel > 1e-5
    # an id out of range
    gid = r.ids.copy()
    gid[0, 0] = 99
    rc = gu.check_routing(r, gid, r.weights, 16, 2.827, True)
    assert rc.invalid == 1


@pytest.mark.parametrize("T", [1, 64, 512, 513, 1024, 8192, 16384])
def test_token_sample(T):
    s = gu.sample_tokens(T)
    assert np.all(np.diff(s) > 0) and s[0] == 0 and s[-1] == T - 1
    assert len(s) == min(T, 512)
