"""Expert parallelism on CPU ranks (gloo): the partition of the experts, the
dispatch plan and both exchanges of sparse_moe_sigmoid_b200.ep, checked
against the single-process oracle.

Each rank owns a contiguous slice of the routed experts and routes its own
tokens (token counts differ by rank, one rank may have none). The arithmetic
callables are the oracle's here (route, the owner's experts on the rows it
receives, the shared expert, the combine), so what is tested is where every
(token, slot) pair goes and how its output comes back: the layer's output on
every rank must equal the oracle's forward of that rank's tokens.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import moe as orc

D, F, E, K = 32, 16, 8, 3


def _layer(seed=5):
    r = np.random.default_rng(seed)
    Wg = r.standard_normal((E, D)) * 0.3
    b = r.standard_normal(E) * 0.01
    ex = [{n: r.standard_normal(s) * 0.2 for n, s in (("gate", (F, D)), ("up", (F, D)),
                                                      ("down", (D, F)))} for _ in range(E)]
    sh = {n: r.standard_normal(s) * 0.2 for n, s in (("gate", (F, D)), ("up", (F, D)),
                                                     ("down", (D, F)))}
    return Wg, b, ex, sh


def _tokens(rank, n):
    return np.random.default_rng(100 + rank).standard_normal((n, D))


def _worker(rank, world, port, counts, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from sparse_moe_sigmoid_b200 import ep  # the module under test (no library needed)
        Wg, b, ex, sh = _layer()
        per = E // world
        x = torch.from_numpy(_tokens(rank, counts[rank]))

        def route(xx):
            r = orc.route(xx.numpy(), Wg, b, K)
            return torch.from_numpy(r.ids), torch.from_numpy(r.weights)

        def experts(rows, local):
            out = torch.zeros_like(rows)
            for li in torch.unique(local).tolist():
                sel = (local == li).nonzero().view(-1)
                m = ex[rank * per + li]
                out[sel] = torch.from_numpy(orc.swiglu_expert(rows[sel].numpy(), m["gate"],
                                                              m["up"], m["down"]))
            return out

        def shared(xx):
            return torch.from_numpy(orc.swiglu_expert(xx.numpy(), sh["gate"], sh["up"],
                                                      sh["down"]))

        def combine(pair_out, w, s):
            T = w.shape[0]
            return torch.from_numpy(orc.combine(pair_out.view(T, K, D).numpy(), w.numpy(),
                                                s.numpy()))

        y = ep.ep_forward(x, route, experts, shared, combine, E, K)
        want, _ = orc.forward(x.numpy(), Wg, b, lambda e: ex[e], lambda: sh, K)
        err = float(np.max(np.abs(y.numpy() - want))) if counts[rank] else 0.0
        q.put((rank, err, tuple(y.shape)))
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("counts", [(5, 7), (0, 6), (4, 1, 9, 3)])
def test_ep_matches_the_single_process_oracle(counts):
    world = len(counts)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    mp.spawn(_worker, args=(world, _free_port(), counts, q), nprocs=world, join=True)
    res = sorted(q.get() for _ in range(world))
    for rank, err, shape in res:
        assert shape == (counts[rank], D)
        assert err < 1e-12, (rank, err)


@pytest.mark.parametrize("world", [1, 2, 4, 8])
def test_plan_partitions_every_pair_once(world):
    """The plan sends every (token, slot) pair exactly once, to the rank that
    owns its expert (contiguous slices of E / world), grouped by rank in rank
    order and by pair index inside a rank, with the expert's index inside the
    owner's slice."""
    from sparse_moe_sigmoid_b200 import ep
    E, k, T = 16, 4, 50
    rng = np.random.default_rng(world)
    ids = torch.from_numpy(np.stack([rng.choice(E, k, replace=False) for _ in range(T)]))
    p = ep.make_plan(ids, E, world)
    per = E // world
    flat = ids.reshape(-1).numpy()
    order = p.order.numpy()
    assert np.array_equal(np.sort(order), np.arange(T * k))
    assert sum(p.send_counts) == T * k
    owner = flat[order] // per
    assert np.all(np.diff(owner) >= 0)
    bounds = np.cumsum([0] + p.send_counts)
    for r in range(world):
        seg = order[bounds[r]:bounds[r + 1]]
        assert np.all(owner[bounds[r]:bounds[r + 1]] == r)
        assert np.all(np.diff(seg) > 0)
    assert np.array_equal(p.local_id.numpy(), flat[order] - owner * per)


def test_plan_rejects_uneven_slices_and_bad_ids():
    from sparse_moe_sigmoid_b200 import ep
    with pytest.raises(ValueError):
        ep.make_plan(torch.zeros((2, 2), dtype=torch.int64), 10, 4)
    with pytest.raises(ValueError):
        ep.make_plan(torch.tensor([[0, 16]]), 16, 2)


def test_library_ep_refuses_what_its_router_cannot_do():
    # the checks run before any device work, so no GPU is needed
    import sparse_moe_sigmoid_b200 as smoe
    from sparse_moe_sigmoid_b200 import ep
    cfg = smoe.moe_config_init_k2(n_group=8, topk_group=4)
    with pytest.raises(ValueError, match="n_group"):
        ep.LibraryEP(smoe, cfg, None, None, None, None, None)
    cfg = smoe.moe_config_init_k2(weight_format=smoe.MOE_WEIGHT_FP8_E4M3_BLOCK)
    with pytest.raises(ValueError, match="block scales"):
        ep.LibraryEP(smoe, cfg, None, None, None, None, None)
