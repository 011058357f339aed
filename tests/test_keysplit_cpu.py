"""Key-range split of one sequence's cache (the multi-device variant of the
decode step) on CPU: the oracle's partial-and-merge is pinned to attention
over the whole key set (the log-sum-exp identity), the prompt is cut into
shares as stated, and the exchange runs as two gloo ranks on 127.0.0.1.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_partial_merge_equals_whole_attention():
    g = np.random.default_rng(0)
    q = g.standard_normal(64)
    k = g.standard_normal((300, 64))
    v = g.standard_normal((300, 64))
    whole = oracle.attend(q, k, v, 0.125)
    for cuts in ([0, 300], [0, 100, 300], [0, 1, 2, 299, 300], [0, 0, 150, 150, 300]):
        parts = [oracle.attend_partial(q, k[a:b], v[a:b], 0.125) for a, b in zip(cuts, cuts[1:])]
        assert np.max(np.abs(oracle.combine_partials(parts) - whole)) < 1e-13
    # one part: o / l is the attention itself; an empty part changes nothing
    m, l, o = oracle.attend_partial(q, k, v, 0.125)
    assert np.max(np.abs(o / l - whole)) < 1e-13
    assert oracle.attend_partial(q, k[:0], v[:0], 0.125)[0] == -np.inf


def test_share_bounds():
    sys.path.insert(0, ROOT)
    from ring_sliding_window_b200.keysplit import share_bounds
    assert share_bounds(10, 3) == [(0, 4), (4, 7), (7, 10)]
    assert share_bounds(2, 3) == [(0, 1), (1, 2), (2, 2)]
    assert share_bounds(0, 2) == [(0, 0), (0, 0)]
    with pytest.raises(ValueError):
        share_bounds(5, 0)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import oracle as orc
    from ring_sliding_window_b200.keysplit import gather_partials, share_bounds
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        g = np.random.default_rng(5)
        B, H, d, n = 2, 3, 16, 50
        q = g.standard_normal((B, H, d))
        k = g.standard_normal((B, H, n, d))
        v = g.standard_normal((B, H, n, d))
        lo, hi = share_bounds(n, world)[rank]
        ml = torch.zeros(B, H, 2, dtype=torch.float64)
        o = torch.zeros(B, H, d, dtype=torch.float64)
        for b in range(B):
            for h in range(H):
                m, l, oo = orc.attend_partial(q[b, h], k[b, h, lo:hi], v[b, h, lo:hi], 0.25)
                ml[b, h] = torch.tensor([m, l], dtype=torch.float64)
                o[b, h] = torch.tensor(oo, dtype=torch.float64)
        all_ml, all_o = gather_partials(ml, o)
        err = 0.0
        for b in range(B):
            for h in range(H):
                parts = [(float(all_ml[r, b, h, 0]), float(all_ml[r, b, h, 1]), all_o[r, b, h].numpy())
                         for r in range(world)]
                got = orc.combine_partials(parts)
                err = max(err, float(np.max(np.abs(got - orc.attend(q[b, h], k[b, h], v[b, h], 0.25)))))
        results[rank] = (tuple(all_ml.shape), err)
    finally:
        dist.destroy_process_group()


def test_gather_and_merge_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    results = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, results)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    for r in range(2):
        shape, err = results[r]
        assert shape == (2, 2, 3, 2)
        assert err < 1e-12
