"""GPU parity: E2E-TV with the LM heads fused (specopd_e2e_tv_lmhead) against
the fp64 oracle (oracle.lmhead) on identical seeded bf16 hidden rows and
heads, through the C ABI.

Tolerances.  Given the logits, the E2E-TV tests' bounds hold (1e-5 relative
per element for overlaps and prefix products, 1e-7 floor; loss 1e-4;
gradients 1e-3 normwise per row, since a tie q_v = p_v may fall on either
side of the subgradient of min).  Here the logits themselves are formed on
the tensor cores as fp32 sums of d exact bf16 products, against the
oracle's fp64: each rounding of a running sum is at most 2^-24 of its
magnitude, so over d terms a logit moves by about sqrt(d) 2^-24 zmax (zmax:
the largest logit of the rows compared), every probability by that
relative amount and an overlap by at most twice it.  The per-element bound
for overlaps and prefix products is therefore
    1e-5 + 2 sqrt(d) 2^-24 zmax   relative (1e-7 floor),
which is about 3e-5 at d = 192 and 1e-4 at d = 4096 for these inputs.
"""

import numpy as np
import pytest
import torch

import synth
from oracle import lmhead as olm
from tests._util import assert_close_elementwise, dev_tensor, rel_err, to_np

pytestmark = pytest.mark.gpu

RTOL, ATOL = 1e-5, 1e-7


def _rtol(x, rows=None):
    """The overlap/prefix tolerance of the module docstring for these inputs
    (zmax from the oracle's fp64 logits of the rows compared)."""
    rows = np.arange(x.h_draft.shape[0]) if rows is None else np.asarray(rows)
    zt = olm.lm_logits(x.h_target[x.target_row[rows]], x.w_target)
    zd = olm.lm_logits(x.h_draft[rows], x.w_draft)
    zmax = max(float(np.max(np.abs(zt))), float(np.max(np.abs(zd))))
    d = x.w_target.shape[1]
    return RTOL + 2.0 * np.sqrt(d) * 2.0 ** -24 * zmax


def _run(lib, x, nb, W, grad_dtype="f32", compute_grad=True, norm_count=0, identity=False):
    V, d = x.w_target.shape
    rows_t = x.h_target.shape[0]
    desc = lib.lmhead_tv_desc(nb, W, V, d, rows_t, grad_dtype, compute_grad, norm_count)
    tr = None if identity else torch.tensor(x.target_row, dtype=torch.int32, device="cuda")
    res = lib.specopd_e2e_tv_lmhead(desc, dev_tensor(x.h_target, "bf16"), tr,
                                    dev_tensor(x.w_target, "bf16"), dev_tensor(x.h_draft, "bf16"),
                                    dev_tensor(x.w_draft, "bf16"))
    torch.cuda.synchronize()
    return res


def _check(res, ref, rtol, grad=True, rows=None):
    assert_close_elementwise(to_np(res["a"]), ref["a"], rtol, ATOL, "a")
    assert_close_elementwise(to_np(res["prefix"]), ref["prefix"], rtol, ATOL, "prefix")
    assert abs(res["loss"].item() - ref["loss"]) <= 1e-4 * abs(ref["loss"]) + 1e-7
    assert abs(res["numer"].item() - ref["numer"]) <= 1e-5 * abs(ref["numer"]) + 1e-7
    if grad:
        g = res["grad"]
        for n in (rows if rows is not None else ref["grad"].keys()):
            assert rel_err(to_np(g[n]), ref["grad"][n]) < 1e-3, n


# (nbranch, W, V, d, rows_target): ragged row and vocabulary tiles, a hidden
# size that is not a multiple of the 64-column stage, and a vocabulary long
# enough that every CTA runs several tiles (both accumulator buffers reused).
SHAPES = [
    (25, 8, 1000, 192, 230),
    (3, 5, 40000, 200, 15),
    (160, 8, 24000, 512, 1280),
]


@pytest.mark.parametrize("nb,W,V,d,rows_t", SHAPES)
def test_lmhead_tv_matches_oracle(lib, nb, W, V, d, rows_t):
    x = synth.lmhead_inputs(7, nb, W, V, d, rows_t)
    ref = olm.e2e_tv_lmhead(x.h_target, x.target_row, x.w_target, x.h_draft, x.w_draft, nb, W)
    res = _run(lib, x, nb, W)
    _check(res, ref, _rtol(x))
    assert lib.specopd_get_device_status() == 0


def test_lmhead_tv_bf16_grad_identity_rows_norm_count(lib):
    nb, W, V, d = 12, 4, 3000, 128
    x = synth.lmhead_inputs(8, nb, W, V, d)
    ref = olm.e2e_tv_lmhead(x.h_target, None, x.w_target, x.h_draft, x.w_draft, nb, W,
                            norm_count=500)
    res = _run(lib, x, nb, W, grad_dtype="bf16", norm_count=500, identity=True)
    x.target_row = np.arange(nb * W, dtype=np.int32)  # the identity map the call used
    assert_close_elementwise(to_np(res["a"]), ref["a"], _rtol(x), ATOL, "a")
    assert abs(res["loss"].item() - ref["loss"]) <= 1e-4 * abs(ref["loss"]) + 1e-7
    for n in range(nb * W):
        # bf16 rounding of the stored gradient: 2^-8 relative per element
        assert rel_err(to_np(res["grad"][n]), ref["grad"][n]) < 2 ** -8 + 1e-3


def test_lmhead_tv_without_grad(lib):
    nb, W, V, d = 6, 3, 5000, 64
    x = synth.lmhead_inputs(9, nb, W, V, d, 40)
    ref = olm.e2e_tv_lmhead(x.h_target, x.target_row, x.w_target, x.h_draft, x.w_draft, nb, W,
                            compute_grad=False)
    res = _run(lib, x, nb, W, compute_grad=False)
    assert res["grad"] is None
    _check(res, ref, _rtol(x), grad=False)


def test_lmhead_tv_agrees_with_logit_path(lib):
    # The fused call against specopd_e2e_tv fed the same logits formed in fp32
    # by torch: same overlaps within the fp32 rounding of two summation orders.
    nb, W, V, d = 8, 4, 4096, 256
    x = synth.lmhead_inputs(10, nb, W, V, d, 32)
    res = _run(lib, x, nb, W)
    ht = torch.tensor(x.h_target[x.target_row], device="cuda", dtype=torch.float64)
    hd = torch.tensor(x.h_draft, device="cuda", dtype=torch.float64)
    zt = (ht @ torch.tensor(x.w_target, device="cuda", dtype=torch.float64).T).float()
    zd = (hd @ torch.tensor(x.w_draft, device="cuda", dtype=torch.float64).T).float()
    desc = lib.tv_desc(nb, W, V, nb * W, "f32", "f32", True, 0)
    r2 = lib.specopd_e2e_tv(desc, zt.contiguous(), None, zd.contiguous())
    torch.cuda.synchronize()
    assert_close_elementwise(to_np(res["a"]), to_np(r2["a"]), 1e-5, 1e-7, "a vs logit path")
    for n in range(nb * W):
        assert rel_err(to_np(res["grad"][n]), to_np(r2["grad"][n])) < 1e-3


def test_lmhead_tv_target_row_out_of_range(lib):
    nb, W, V, d = 4, 3, 700, 64
    x = synth.lmhead_inputs(11, nb, W, V, d, 12)
    x.target_row[4] = 12  # branch 1, position 1: outside [0, rows_target)
    lib.specopd_get_device_status()
    res = _run(lib, x, nb, W)
    # that position's overlap, its branch's prefix products from it on, its
    # branch's gradient rows (g_n involves every overlap of the branch) and
    # the loss are NaN; everything else is finite
    a, pre, g = to_np(res["a"]), to_np(res["prefix"]), to_np(res["grad"])
    assert np.isnan(a[4]) and np.all(np.isfinite(np.delete(a, 4)))
    assert np.all(np.isnan(pre[4:6])) and np.all(np.isfinite(np.delete(pre, [4, 5])))
    assert np.all(np.isnan(g[3:6])) and np.all(np.isfinite(np.delete(g, [3, 4, 5], axis=0)))
    assert np.isnan(res["loss"].item())
    assert lib.specopd_get_device_status() & lib.DEV_ROW_RANGE


@pytest.mark.slow
def test_lmhead_tv_full_size_sampled(lib):
    # The configuration bench.py times: N = 512 (64 branches of W = 8),
    # V = 151,936, hidden size 4096 (36 vocabulary chunks of 32-33 tiles per
    # CTA).  The GPU runs every branch; the oracle recomputes a seeded sample
    # of whole branches (their overlaps, prefix products and gradient rows
    # depend on their own positions and on the global normalisation only).
    nb, W, V, d = 64, 8, 151936, 4096
    x = synth.lmhead_inputs(21, nb, W, V, d)
    res = _run(lib, x, nb, W)
    assert lib.specopd_get_device_status() == 0
    rng = np.random.default_rng(5)
    branches = sorted(set(rng.choice(nb, size=3, replace=False).tolist()) | {0, nb - 1})
    pos = np.concatenate([np.arange(b * W, (b + 1) * W) for b in branches])
    ref = olm.e2e_tv_lmhead(x.h_target, x.target_row[pos], x.w_target, x.h_draft[pos],
                            x.w_draft, len(branches), W, norm_count=nb * W)
    rtol = _rtol(x, pos)
    assert_close_elementwise(to_np(res["a"])[pos], ref["a"], rtol, ATOL, "a")
    assert_close_elementwise(to_np(res["prefix"])[pos], ref["prefix"], rtol, ATOL, "prefix")
    g = res["grad"]
    for k, n in enumerate(pos):
        assert rel_err(to_np(g[int(n)]), ref["grad"][k]) < 1e-3, int(n)
