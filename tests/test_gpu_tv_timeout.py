"""A bounded device-side wait of E2E-TV runs out, on purpose, without a GPU
fault: the library winds the call down and reports it.

The test-only hook specopd_debug_fault_injection makes the scorer of one
supervised position skip publishing its overlap, so the other positions of
its branch wait for it in vain, and shortens those branch waits to 5 ms.
Nothing else is changed: the copy ring, the consumers and every
other branch run normally.  Expected (the error contract of
include/specopd.h): the call returns, the device status word reads
SPECOPD_DEV_TIMEOUT, the affected branch's overlaps, prefix products and
gradient rows are NaN (and so is the loss, which sums every branch), every
other branch matches the fp64 oracle, and the next call without the hook is
correct again.
"""

import numpy as np
import pytest
import torch

import synth
from oracle import tv as otv
from tests._util import assert_close_elementwise, dev_tensor, rel_err, to_np

pytestmark = pytest.mark.gpu


def _inputs(nb, W, V, seed):
    rng = np.random.default_rng(seed)
    zt = (2.0 * rng.standard_normal((nb * W, V))).astype(np.float32)
    zd = (zt + rng.standard_normal((nb * W, V))).astype(np.float32)
    return synth.round_bf16(zt), synth.round_bf16(zd)


def _run(lib, zt, zd, nb, W):
    desc = lib.tv_desc(nb, W, zt.shape[1], zt.shape[0], "bf16", "f32")
    res = lib.specopd_e2e_tv(desc, dev_tensor(zt, "bf16"), None, dev_tensor(zd, "bf16"))
    torch.cuda.synchronize()
    return res


@pytest.mark.parametrize("withheld_branch,withheld_offset", [(5, 0), (117, 2)])
def test_tv_branch_wait_runs_out(lib, withheld_branch, withheld_offset):
    # 160 branches of W = 4 at a 16-byte aligned vocabulary: the whole-row
    # schedule, four or five positions per CTA, so tasks after the timed-out
    # one run on the same CTAs.
    nb, W, V = 160, 4, 8192
    zt, zd = _inputs(nb, W, V, seed=withheld_branch)
    ref = otv.e2e_tv(zt, None, zd, nb, W)
    assert lib.specopd_get_device_status() == 0
    withheld = withheld_branch * W + withheld_offset
    lib.specopd_debug_fault_injection(withheld, 5_000_000)
    try:
        res = _run(lib, zt, zd, nb, W)
        status = lib.specopd_get_device_status()
    finally:
        lib.specopd_debug_fault_injection(-1, 0)
    assert status & lib.DEV_TIMEOUT, hex(status)

    rows = slice(withheld_branch * W, (withheld_branch + 1) * W)
    a, prefix = to_np(res["a"]), to_np(res["prefix"])
    grad = to_np(res["grad"])
    assert np.all(np.isnan(a[rows])) and np.all(np.isnan(prefix[rows]))
    assert np.all(np.isnan(grad[rows]))
    assert np.isnan(res["loss"].item())
    keep = np.ones(nb * W, dtype=bool)
    keep[rows] = False
    assert np.all(np.isfinite(a[keep])) and np.all(np.isfinite(prefix[keep]))
    assert_close_elementwise(a[keep], ref["a"][keep], 1e-5, 1e-7, "a")
    assert_close_elementwise(prefix[keep], ref["prefix"][keep], 1e-5, 1e-7, "prefix")
    for n in np.flatnonzero(keep)[:: 7]:
        assert rel_err(grad[n], ref["grad"][n]) < 1e-3, n

    # the next call, without the hook, is whole again
    res2 = _run(lib, zt, zd, nb, W)
    assert lib.specopd_get_device_status() == 0
    assert_close_elementwise(to_np(res2["a"]), ref["a"], 1e-5, 1e-7, "a")
    assert abs(res2["loss"].item() - ref["loss"]) <= 1e-4 * abs(ref["loss"])
    for n in range(0, nb * W, 11):
        assert rel_err(to_np(res2["grad"][n]), ref["grad"][n]) < 1e-3, n
