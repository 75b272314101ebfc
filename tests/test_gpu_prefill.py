"""GPU parity of specopd_trunk_prefill against the fp64 oracle's
trunk_prefill, through the C ABI.

The trunk prefill is the step before the branch pass (SpecOPD review
(jaehun.me) §3.2(a): the trunk is computed once and its K/V cached): causal
self-attention of every trunk row over its own sequence, with RoPE at the
row's position, and the rotated keys written back as the K cache.

Tolerances: bf16 outputs 2e-2 absolute at unit-scale activations (the
target's bound for bf16 attention) and 1e-2 of the output scale normwise, as
for the branch pass; the K cache within one bf16 rounding of the fp64
rotation plus 1e-5 absolute (the rotation is evaluated in fp32); fp32 outputs 1e-5 relative per element with a 1e-6 absolute floor
(RoPE angles are evaluated in fp32).
"""

import numpy as np
import pytest
import torch

import synth
from oracle import attention as oatt
from tests._util import assert_close_elementwise, dev_tensor, rel_err, to_np

pytestmark = pytest.mark.gpu


def _inputs(cfg, seed=0):
    rng = np.random.default_rng(seed)
    cu = np.concatenate([[0], np.cumsum(cfg.T)]).astype(np.int32)
    n = int(cu[-1])

    def draw(*shape):
        x = rng.standard_normal(size=shape, dtype=np.float32)
        return synth.round_bf16(x) if cfg.dtype == "bf16" else x
    return cu, draw(n, cfg.Hq, cfg.D), draw(n, cfg.Hkv, cfg.D), draw(n, cfg.Hkv, cfg.D)


def _run(lib, cfg, cu, q, k, v, lse=False):
    dt = cfg.dtype
    desc = lib.attn_desc(cfg.S, 1, 1, cfg.Hq, cfg.Hkv, cfg.D, dt, cfg.rope_base)
    kd = dev_tensor(k, dt)
    ls = torch.empty((q.shape[0], cfg.Hq), dtype=torch.float32, device="cuda") if lse else None
    out = lib.specopd_trunk_prefill(desc, dev_tensor(q, dt), kd, dev_tensor(v, dt),
                                    torch.tensor(cu, device="cuda"), [int(c) for c in cu], lse=ls)
    torch.cuda.synchronize()
    return to_np(out), to_np(kd), (to_np(ls) if lse else None)


def _check_bf16(got, ref, rows):
    g, r = got[rows], ref[rows]
    assert np.all(np.isfinite(g))
    assert np.max(np.abs(g - r)) < 2e-2
    assert rel_err(g, r) < 1e-2


@pytest.mark.parametrize("S,T,Hq,Hkv,D,dtype", [
    (1, (300,), 8, 2, 128, "bf16"),          # one sequence, several query tiles
    (3, (5, 200, 77), 8, 2, 128, "bf16"),    # packed, tiles spanning sequence boundaries
    (2, (130, 64), 5, 1, 64, "bf16"),        # G = 5 (padded tile rows), D = 64
    (2, (1, 97), 4, 4, 128, "bf16"),         # G = 1, a one-token sequence
    (3, (7, 40, 33), 4, 1, 64, "f32"),       # fp32: the SIMT kernel
    (1, (65,), 2, 2, 128, "f32"),
])
def test_prefill_small(lib, S, T, Hq, Hkv, D, dtype):
    cfg = synth.custom_attn_config(S, T, 1, 1, Hq, Hkv, D, dtype)
    cu, q, k, v = _inputs(cfg, seed=sum(T))
    out, kc, lse = _run(lib, cfg, cu, q, k, v, lse=True)
    ref, kref = oatt.trunk_prefill(q, k, v, cu, cfg.rope_base)
    rows = np.arange(int(cu[-1]))
    if dtype == "bf16":
        _check_bf16(out, ref, rows)
        # K cache: the fp64 rotation rounded once to bf16 (2^-8 relative), plus
        # the fp32 evaluation of the rotation (angles and products in fp32:
        # about 1e-6 absolute at unit scale, which dominates near zero)
        assert np.all(np.abs(kc - kref) <= 2.0 ** -8 * np.abs(kref) + 1e-5)
    else:
        assert_close_elementwise(out, ref, 1e-5, 1e-6, "out")
        assert_close_elementwise(kc, kref, 1e-5, 1e-6, "k cache")
    # lse of a few rows, by the definition
    for t in (0, int(cu[-1]) - 1, int(cu[-1]) // 2):
        s = int(np.searchsorted(cu, t, side="right")) - 1
        p = t - int(cu[s])
        kk = kref[cu[s]: t + 1, 0]
        qq = oatt.rope(q[t: t + 1].astype(np.float64), [p], cfg.rope_base)[0, 0]
        sc = kk @ qq / np.sqrt(D)
        want = np.log(np.sum(np.exp(sc - sc.max()))) + sc.max()
        assert abs(lse[t, 0] - want) < (2e-2 if dtype == "bf16" else 1e-5 * max(1, abs(want)))
    assert lib.specopd_get_device_status() == 0


@pytest.mark.parametrize("name,nsample", [("8b", 192), ("packed", 96)])
def test_prefill_full_size(lib, name, nsample):
    # The trunks of the 8B-shaped and packed workloads (4,096 and about
    # 55,000 tokens), every row computed on the GPU; the oracle checks a
    # seeded sample of rows (and every sequence's first and last rows).
    base = synth.attn_config(name)
    cfg = synth.custom_attn_config(base.S, base.T, 1, 1, base.Hq, base.Hkv, base.D, "bf16")
    cu, q, k, v = _inputs(cfg, seed=7)
    out, kc, _ = _run(lib, cfg, cu, q, k, v)
    assert np.all(np.isfinite(out))
    rng = np.random.default_rng(99)
    n = int(cu[-1])
    rows = set(rng.choice(n, size=nsample, replace=False).tolist())
    rows |= set(int(c) for c in cu[:-1]) | set(int(c) - 1 for c in cu[1:])
    rows = sorted(rows)
    ref, kref = oatt.trunk_prefill(q, k, v, cu, cfg.rope_base, rows=rows)
    _check_bf16(out, ref, rows)
    assert np.all(np.abs(kc - kref) <= 2.0 ** -8 * np.abs(kref) + 1e-5)
    assert lib.specopd_get_device_status() == 0


def test_prefill_feeds_the_branch_pass(lib):
    # Prefill the trunk, then score branches over the K cache it wrote: the
    # branch rows match the unrolled oracle on the raw inputs.
    cfg = synth.custom_attn_config(2, (300, 520), 6, 5, 8, 2, 128, "bf16",
                                   anchor_lo=(150, 260), anchor_hi=(295, 515))
    inp = synth.attention_inputs(cfg)
    cu = [int(c) for c in inp.cu_trunk]
    rng = np.random.default_rng(3)
    q_tr = synth.round_bf16(rng.standard_normal((inp.T_tot, cfg.Hq, cfg.D), dtype=np.float32))
    desc = lib.attn_desc(cfg.S, cfg.B, cfg.W, cfg.Hq, cfg.Hkv, cfg.D, "bf16", cfg.rope_base)
    cu_dev = torch.tensor(inp.cu_trunk, device="cuda")
    k_cache = dev_tensor(inp.k_tr, "bf16")
    v_tr = dev_tensor(inp.v_tr, "bf16")
    lib.specopd_trunk_prefill(desc, dev_tensor(q_tr, "bf16"), k_cache, v_tr, cu_dev, cu)
    anchors = torch.tensor(inp.anchors, device="cuda")
    _, sem_pos, _ = lib.specopd_tree_build(cu, anchors, cfg.B, cfg.W)
    out = lib.specopd_tree_attn(desc, dev_tensor(inp.q_br, "bf16"), dev_tensor(inp.k_br, "bf16"),
                                dev_tensor(inp.v_br, "bf16"), k_cache, v_tr, cu_dev, cu, anchors,
                                sem_pos)
    torch.cuda.synchronize()
    ref = oatt.branch_attention_unrolled_dense(inp.q_br, inp.k_br, inp.v_br, inp.k_tr, inp.v_tr,
                                               inp.cu_trunk, inp.anchors, cfg.B, cfg.W,
                                               cfg.rope_base)
    got = to_np(out)
    assert np.max(np.abs(got - ref)) < 2e-2 and rel_err(got, ref) < 1e-2
    assert lib.specopd_get_device_status() == 0
