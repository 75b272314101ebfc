"""The sharded E2E-TV path through the library, two ranks (SpecOPD review
§3.2, distributed normalisation: numerators and counts are gathered
separately and the loss normalised once).

Two processes, spawned, both on cuda:0 (this host has one GPU); gloo carries
the host-side exchange.  No kernel of one process waits on the other's: each
rank scores its own branches with specopd_e2e_tv (norm_count = the global
position count, so its gradient already carries the global 1/N), the ranks
all-reduce their `numer` outputs, and specopd_e2e_tv_finalize writes the
loss on the device.  Every rank's overlaps, prefix products and gradient rows
and the common loss must match the single-process fp64 oracle, also when the
ranks hold different numbers of branches.  The same holds for the call with
the LM heads fused in front (specopd_e2e_tv_lmhead), each rank holding the
hidden rows of its own positions.
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import synth
from oracle import lmhead as olm
from oracle import tv as otv

pytestmark = pytest.mark.gpu


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _data(nb, W, V):
    rng = np.random.default_rng(nb * 100 + W)
    zt = (2.0 * rng.standard_normal((nb * W, V))).astype(np.float32)
    zd = (zt + rng.standard_normal((nb * W, V))).astype(np.float32)
    return synth.round_bf16(zt), synth.round_bf16(zd)


def _lm_data(nb, W, V):
    return synth.lmhead_inputs(nb * 100 + W, nb, W, V, 128)


def _rank(rank, world, port, nb, W, V, out_q, fused=False):
    import datetime

    import torch.distributed as dist

    from tree_attention_specopd_b200 import api
    from tree_attention_specopd_b200 import dist as sdist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        torch.cuda.set_device(0)
        zt, zd = _data(nb, W, V)
        start, cnt = sdist.shard_branches(nb, rank, world)
        rows = slice(start * W, (start + cnt) * W)
        n_global = sdist.global_count(cnt * W)
        t = lambda x: torch.from_numpy(np.ascontiguousarray(x)).to("cuda").to(torch.bfloat16)  # noqa
        if fused:
            x = _lm_data(nb, W, V)
            ht = x.h_target[x.target_row[rows]]  # this rank's scoring rows, in position order
            desc = api.lmhead_tv_desc(cnt, W, V, x.w_target.shape[1], cnt * W, "f32", True,
                                      norm_count=n_global)
            res = api.specopd_e2e_tv_lmhead(desc, t(ht), None, t(x.w_target), t(x.h_draft[rows]),
                                            t(x.w_draft))
        else:
            desc = api.tv_desc(cnt, W, V, cnt * W, "bf16", "f32", True, norm_count=n_global)
            res = api.specopd_e2e_tv(desc, t(zt[rows]), None, t(zd[rows]))
        loss = sdist.global_loss(res["numer"], n_global)
        torch.cuda.synchronize()
        status = api.specopd_get_device_status()
        out_q.put((rank, start, cnt, n_global, float(loss.item()), res["a"].cpu().numpy(),
                   res["prefix"].cpu().numpy(), res["grad"].cpu().numpy(), status))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("nb,fused", [(10, False), (11, False), (11, True)])  # 11: 6 and 5 branches
def test_two_ranks_through_the_library(lib, nb, fused):
    W, V, world = 4, 4096, 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, nb, W, V, q, fused))
             for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=300) for _ in range(world)]
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    if fused:
        x = _lm_data(nb, W, V)
        full = olm.e2e_tv_lmhead(x.h_target, x.target_row, x.w_target, x.h_draft, x.w_draft, nb, W)
        # logits formed on the tensor cores (fp32 sums of 128 bf16 products):
        # the fused call's bound, 1e-5 + 2 sqrt(d) 2^-24 zmax with zmax < 40
        rtol = 1e-5 + 2.0 * np.sqrt(128) * 2.0 ** -24 * 40.0
    else:
        zt, zd = _data(nb, W, V)
        full = otv.e2e_tv(zt, None, zd, nb, W)
        rtol = 1e-5
    for rank, start, cnt, n_global, loss, a, prefix, grad, status in results:
        assert status == 0
        assert n_global == nb * W
        assert abs(loss - full["loss"]) <= 1e-4 * abs(full["loss"])
        rows = range(start * W, (start + cnt) * W)
        ref_a = full["a"][start * W:(start + cnt) * W]
        ref_p = full["prefix"][start * W:(start + cnt) * W]
        assert np.all(np.abs(a - ref_a) <= rtol * np.abs(ref_a) + 1e-7)
        assert np.all(np.abs(prefix - ref_p) <= rtol * np.abs(ref_p) + 1e-7)
        for k, n in enumerate(rows):
            gr = full["grad"][n]
            err = np.max(np.abs(grad[k] - gr)) / np.max(np.abs(gr))
            assert err < 1e-3, (rank, n, err)
