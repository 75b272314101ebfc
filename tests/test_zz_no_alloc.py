"""specopd_e2e_tv_noalloc: the E2E-TV entry point for callers that cannot
allocate device memory (it uses the library's fixed scratch array instead of
a caller workspace).  Checked through the C ABI against specopd_e2e_tv, with
the tolerances of the other E2E-TV tests, on two calls in a row (the second
call reuses the array the first one left behind).  This file is collected
last, so a failure here stops a fail-fast run only after every other test.
"""

import numpy as np
import pytest
import torch

import synth
from tests._util import assert_close_elementwise, dev_tensor, rel_err, to_np
from tree_attention_specopd_b200 import api

pytestmark = pytest.mark.gpu


def _outputs(N, V, grad_dtype=torch.float32):
    dev = "cuda"
    return dict(a=torch.full((N,), float("nan"), device=dev),
                prefix=torch.full((N,), float("nan"), device=dev),
                loss=torch.full((1,), float("nan"), device=dev),
                numer=torch.full((1,), float("nan"), dtype=torch.float64, device=dev),
                grad=torch.full((N, V), float("nan"), dtype=grad_dtype, device=dev))


def _compare(got, ref):
    assert_close_elementwise(to_np(got["a"]), to_np(ref["a"]), 1e-5, 1e-7, "a")
    assert_close_elementwise(to_np(got["prefix"]), to_np(ref["prefix"]), 1e-5, 1e-7, "prefix")
    assert abs(got["loss"].item() - ref["loss"].item()) <= 1e-4 * abs(ref["loss"].item())
    assert abs(got["numer"].item() - ref["numer"].item()) <= 1e-5 * abs(ref["numer"].item())
    g, gr = to_np(got["grad"]), to_np(ref["grad"])
    for n in range(gr.shape[0]):
        assert rel_err(g[n], gr[n]) < 1e-3, n


@pytest.mark.parametrize("nb,W,V,dtype,gather", [
    (4, 4, 1024, "f32", False),
    (16, 8, 151936, "bf16", True),
])
def test_noalloc_matches_workspace_entry_point(nb, W, V, dtype, gather):
    rng = np.random.default_rng(nb * W)
    N = nb * W
    zt = (rng.standard_normal((N, V)) * 3).astype(np.float32)
    zd = (zt + rng.standard_normal((N, V))).astype(np.float32)
    if dtype == "bf16":
        zt, zd = synth.round_bf16(zt), synth.round_bf16(zd)
    if gather:
        # target rows scattered in a larger packed table, read through a row map
        rows_t = 3 * N
        perm = rng.permutation(rows_t)[:N].astype(np.int32)
        table = np.zeros((rows_t, V), np.float32)
        table[perm] = zt
        zt_dev = dev_tensor(table, dtype)
        trow = torch.tensor(perm, device="cuda")
    else:
        rows_t = N
        zt_dev = dev_tensor(zt, dtype)
        trow = None
    zd_dev = dev_tensor(zd, dtype)
    desc = api.tv_desc(nb, W, V, rows_t, dtype, "f32", True)
    ref = api.specopd_e2e_tv(desc, zt_dev, trow, zd_dev)
    torch.cuda.synchronize()
    for _ in range(2):
        out = _outputs(N, V)
        api.specopd_e2e_tv_noalloc(desc, zt_dev, trow, zd_dev, **out)
        torch.cuda.synchronize()
        _compare(out, ref)
    assert api.specopd_get_device_status() == 0


def test_noalloc_rejects_sizes_beyond_the_array():
    # A million positions need more scratch than the fixed array holds, even
    # on the schedules that need the least (about 10 bytes per position).
    desc = api.tv_desc(250_000, 4, 16, 1_000_000, "f32", "f32", True)
    assert api.specopd_e2e_tv_workspace_size(desc) > api.E2E_TV_STATIC_SCRATCH_BYTES
    dummy = torch.empty(1, device="cuda")
    with pytest.raises(api.SpecopdError) as ei:
        api.specopd_e2e_tv_noalloc(desc, dummy, None, dummy, dummy, dummy, dummy, None, dummy)
    assert ei.value.status == 3  # SPECOPD_ERR_WORKSPACE
