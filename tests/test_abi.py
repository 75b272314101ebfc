"""The C-ABI library loads and exports every symbol include/specopd.h declares.

CPU only: no compute call needs a GPU here; only host-side entry points
(status strings, workspace sizes, argument validation that fails before any
device work) are called.
"""

import ctypes

import pytest

from tree_attention_specopd_b200 import api, build


@pytest.fixture(scope="module")
def lib():
    build.build()
    return api.load()


def test_exports_every_declared_symbol(lib):
    names = api.header_functions()
    assert len(names) == 16
    for n in names:
        assert hasattr(lib, n), n
        assert ctypes.cast(getattr(lib, n), ctypes.c_void_p).value


def test_status_strings(lib):
    assert lib.specopd_status_string(0) == b"SPECOPD_OK"
    assert lib.specopd_status_string(3) == b"SPECOPD_ERR_WORKSPACE"
    assert lib.specopd_status_string(99) == b"SPECOPD_ERR_UNKNOWN"
    assert lib.specopd_version() == 10000


def test_workspace_sizes_are_host_only(lib):
    d = api.attn_desc(1, 64, 8, 32, 8, 128, "bf16")
    n = api.specopd_tree_attn_workspace_size(d, [0, 4096])
    assert n >= 448 * (32 + 8) * 128 * 2
    t = api.tv_desc(64, 8, 151936, 4544, "bf16")
    assert api.specopd_e2e_tv_workspace_size(t) >= 512 * 16
    # invalid descriptors report 0
    bad = api.attn_desc(1, 64, 8, 30, 8, 128, "bf16")  # Hq % Hkv != 0
    assert api.specopd_tree_attn_workspace_size(bad, [0, 4096]) == 0
    assert api.specopd_tree_attn_workspace_size(d, [1, 4096]) == 0  # cu[0] != 0
    assert api.specopd_e2e_tv_workspace_size(api.tv_desc(0, 8, 100, 10, "f32")) == 0
    # vocabularies beyond the slice schedule's slice count are unsupported
    assert api.specopd_e2e_tv_workspace_size(api.tv_desc(1, 1, 10_000_000, 1, "f32")) == 0


def test_invalid_arguments_rejected_before_device(lib):
    cu = (ctypes.c_int32 * 2)(0, 10)
    # S = 0
    assert lib.specopd_tree_build(0, cu, None, 1, 1, None, None, None, None) == 1
    # non-increasing cu_trunk
    bad = (ctypes.c_int32 * 2)(0, 0)
    assert lib.specopd_tree_build(1, bad, ctypes.c_void_p(16), 1, 2, ctypes.c_void_p(16),
                                  None, None, None) == 1
    # rope with odd D
    d = api.RopeDesc(7, 0, 10000.0)
    assert lib.specopd_rope_apply(ctypes.byref(d), None, None, 4, 1, None) == 1


def test_bf16_branch_span_limit(lib):
    # bf16 tree attention rotates a query tile's branch keys -- its
    # floor(128 / G) rows plus up to W - 2 earlier nodes of its first branch --
    # in three 64-key tiles; longer spans are refused before any device work.
    cu = (ctypes.c_int32 * 2)(0, 4096)
    fake = ctypes.c_void_p(256)  # never dereferenced: validation fails first
    args = [fake] * 5 + [fake, cu, fake, fake, fake, None, fake, 1 << 20, None]
    d = api.attn_desc(1, 4, 70, 8, 8, 128, "bf16")  # G = 1: 128 + 68 = 196 > 192
    assert lib.specopd_tree_attn(ctypes.byref(d), *args) == 2  # SPECOPD_ERR_UNSUPPORTED


def test_lmhead_tv_validation(lib):
    # specopd_e2e_tv_lmhead: descriptor and pointer checks come before any
    # device work.
    ok = api.lmhead_tv_desc(64, 8, 151936, 4096, 512)
    assert api.specopd_e2e_tv_lmhead_workspace_size(ok) >= 512 * 4096 * 2
    assert api.specopd_e2e_tv_lmhead_workspace_size(api.lmhead_tv_desc(0, 8, 100, 64, 8)) == 0
    fake = ctypes.c_void_p(256)  # never dereferenced: validation fails first
    ptrs = [fake, None, fake, fake, fake, fake, fake, fake, None, fake, fake, 1 << 30, None]
    bad_d = api.lmhead_tv_desc(2, 4, 1000, 100, 8)  # hidden size not a multiple of 8
    assert lib.specopd_e2e_tv_lmhead(ctypes.byref(bad_d), *ptrs) == 2  # UNSUPPORTED
    bad_w = api.lmhead_tv_desc(2, 300, 1000, 64, 600)  # W above 256
    assert lib.specopd_e2e_tv_lmhead(ctypes.byref(bad_w), *ptrs) == 2
    d = api.lmhead_tv_desc(2, 4, 1000, 64, 8)
    missing = list(ptrs)
    missing[2] = None  # no target head
    assert lib.specopd_e2e_tv_lmhead(ctypes.byref(d), *missing) == 1  # INVALID_ARG
    unaligned = list(ptrs)
    unaligned[0] = ctypes.c_void_p(264)  # h_target off a 16-byte boundary
    assert lib.specopd_e2e_tv_lmhead(ctypes.byref(d), *unaligned) == 2
    rows = api.lmhead_tv_desc(2, 4, 1000, 64, 7)  # identity rows need rows_target >= N
    assert lib.specopd_e2e_tv_lmhead(ctypes.byref(rows), *ptrs) == 1
