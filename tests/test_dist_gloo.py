"""Multi-rank host logic (world size 2, gloo, CPU): branch sharding and the
distributed normalisation of the loss (SpecOPD review §3.2: numerators and
counts gathered separately) reproduce the single-process oracle exactly,
including when the ranks hold different numbers of branches.

The per-rank compute here is the oracle (CPU), and the loss is finished on
the host; tests/test_gpu_dist.py runs the same exchange around the library
(specopd_e2e_tv per shard, specopd_e2e_tv_finalize after the sum).
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import tv as otv
from tree_attention_specopd_b200 import dist as sdist


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _problem(nb, W, V, seed=0):
    rng = np.random.default_rng(seed)
    zt = rng.standard_normal((nb * W, V)) * 2
    zd = zt + rng.standard_normal((nb * W, V))
    return zt, zd


def _worker(rank, world, port, nb, W, V, out_q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        zt, zd = _problem(nb, W, V)
        start, cnt = sdist.shard_branches(nb, rank, world)
        rows = slice(start * W, (start + cnt) * W)
        n_global = sdist.global_count(cnt * W)
        res = otv.e2e_tv(zt[rows], None, zd[rows], cnt, W, norm_count=n_global)
        numer = torch.tensor([res["numer"]], dtype=torch.float64)
        loss = 1.0 - sdist.global_numer(numer).item() / n_global
        out_q.put((rank, start, cnt, float(loss), res["g"].tolist(), n_global))
    finally:
        dist.destroy_process_group()


def test_shard_branches_partition():
    for nb in (1, 5, 64, 1024):
        for world in (1, 2, 3, 8):
            owned = []
            for r in range(world):
                s, c = sdist.shard_branches(nb, r, world)
                owned.extend(range(s, s + c))
            assert owned == list(range(nb))


@pytest.mark.parametrize("nb", [6, 7])  # 7: ranks hold 4 and 3 branches
def test_two_rank_normalisation_matches_single_process(nb):
    W, V, world = 3, 40, 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, nb, W, V, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    zt, zd = _problem(nb, W, V)
    full = otv.e2e_tv(zt, None, zd, nb, W)
    g = np.empty(nb * W)
    for rank, start, cnt, loss, g_local, n_global in results:
        assert n_global == nb * W
        assert abs(loss - full["loss"]) < 1e-14
        g[start * W:(start + cnt) * W] = g_local
    np.testing.assert_allclose(g, full["g"], rtol=1e-14, atol=0)
