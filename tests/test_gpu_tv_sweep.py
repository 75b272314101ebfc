"""E2E-TV on the overlap-sweep workload at full size (GPU vs the fp64 oracle).

N = 4096 positions (512 branches x W = 8), V = 151,936, bf16 logits, draft
noise sigma in {0, 0.25, 1, 4}, plus 5 % of the rows bit-identical between
target and draft and 5 % with disjoint top-k supports (synth.tv_config).
The kernel scores all positions in the launch configuration the benchmark
uses.  The oracle recomputes every overlap (row chunks, so host memory stays
bounded), hence the loss, and the gradient rows of a sample of whole
branches (a branch's gradient needs only its own W overlaps and the global
position count).

Tolerances (fp32 accumulation against fp64): overlaps and prefix products
1e-5 relative per element (1e-7 floor for values at or near zero), loss
1e-4 relative, gradient rows 1e-3 relative (normwise per row: near-ties of
q and p may take the other side of the subgradient of min).
"""

import numpy as np
import pytest
import torch

import synth
from oracle import tv as otv
from tests._util import assert_close_elementwise, rel_err, to_np

CHUNK = 256  # positions per host-side chunk


def _upload(cfg):
    N = cfg.nbranch * cfg.W
    zt = torch.empty((N, cfg.V), dtype=torch.bfloat16, device="cuda")
    zd = torch.empty((N, cfg.V), dtype=torch.bfloat16, device="cuda")
    a_ref = np.empty(N)
    for n0 in range(0, N, CHUNK):
        n1 = min(N, n0 + CHUNK)
        t, d = synth.logits(cfg, positions=range(n0, n1))  # bf16-exact fp32
        zt[n0:n1] = torch.from_numpy(t).to("cuda").to(torch.bfloat16)
        zd[n0:n1] = torch.from_numpy(d).to("cuda").to(torch.bfloat16)
        for k in range(n1 - n0):
            p = otv.softmax(t[k].astype(np.float64))
            q = otv.softmax(d[k].astype(np.float64))
            a_ref[n0 + k] = otv.overlap(p, q)
    return zt, zd, a_ref


@pytest.mark.gpu
@pytest.mark.parametrize("sigma_index", [0, 1, 2, 3])
def test_tv_overlap_sweep_full_size(lib, sigma_index):
    cfg = synth.tv_config("sweep", sigma_index)
    N, W = cfg.nbranch * cfg.W, cfg.W
    zt, zd, a_ref = _upload(cfg)
    desc = lib.tv_desc(cfg.nbranch, W, cfg.V, N, "bf16", "f32")
    res = lib.specopd_e2e_tv(desc, zt, None, zd)
    torch.cuda.synchronize()
    assert lib.specopd_get_device_status() == 0

    a = to_np(res["a"]).astype(np.float64)
    assert_close_elementwise(a, a_ref, 1e-5, 1e-7, "a")
    P_ref = otv.prefix_products(a_ref.reshape(cfg.nbranch, W))
    assert_close_elementwise(to_np(res["prefix"]).reshape(cfg.nbranch, W), P_ref, 1e-5, 1e-7,
                             "prefix")
    loss_ref = otv.loss_from_overlaps(a_ref.reshape(cfg.nbranch, W), N)
    assert abs(res["loss"].item() - loss_ref) <= 1e-4 * abs(loss_ref) + 1e-7

    # identical rows overlap fully; disjoint-support rows barely overlap
    kinds = [synth.row_kind(cfg, n) for n in range(N)]
    ident = [n for n, k in enumerate(kinds) if k == "identical"]
    disj = [n for n, k in enumerate(kinds) if k == "disjoint"]
    assert ident and disj
    assert np.all(np.abs(a[ident] - 1.0) < 1e-5)
    assert np.all(a_ref[disj] < 1e-3) and np.all(a[disj] < 1e-3)
    assert_close_elementwise(a[disj], a_ref[disj], 1e-5, 1e-7, "a (disjoint rows)")
    assert_close_elementwise(a[ident], a_ref[ident], 1e-5, 1e-7, "a (identical rows)")

    # gradient rows of sampled whole branches, one of them holding an
    # identical row and one a disjoint row
    branches = sorted({0, cfg.nbranch - 1, ident[0] // W, disj[0] // W, cfg.nbranch // 2})
    g = res["grad"]
    for b in branches:
        t, d = synth.logits(cfg, positions=range(b * W, (b + 1) * W))
        ref = otv.e2e_tv(t, None, d, 1, W, norm_count=N)
        for i in range(W):
            gr = ref["grad"][i]
            got = to_np(g[b * W + i]).astype(np.float64)
            if np.max(np.abs(gr)) == 0:
                assert np.max(np.abs(got)) < 1e-12
            else:
                assert rel_err(got, gr) < 1e-3, (b, i)
