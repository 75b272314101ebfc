"""GPU parity: tree_build, rope_apply, fp32 tree attention and E2E-TV against
the fp64 oracle on identical seeded inputs (calls go through the C ABI).

Tolerances (stated by the target of this library): integer outputs
bit-exact; fp32 outputs within 1e-5 relative; loss within 1e-4 relative;
gradients within 1e-3 relative (normwise per row, which absorbs mask flips at
exact-tie elements).
"""

import numpy as np
import pytest
import torch

import synth
from oracle import attention as oatt
from oracle import tree as otree
from oracle import tv as otv
from tests._util import assert_close_elementwise, dev_tensor, rel_err, to_np

pytestmark = pytest.mark.gpu


def _status(lib):
    return lib.specopd_get_device_status()


# ---------------------------------------------------------------- tree build

@pytest.mark.parametrize("name", ["tiny", "8b", "long", "packed"])
def test_tree_build_bit_exact(lib, name):
    cfg = synth.attn_config(name)
    rng = np.random.default_rng(cfg.seed)
    cu = np.concatenate([[0], np.cumsum(cfg.T)]).astype(np.int32)
    anchors = synth.draw_anchors(rng, cfg.S, cfg.B, cfg.anchor_lo, cfg.anchor_hi)
    par, pos, srow = lib.specopd_tree_build(cu, torch.tensor(anchors, device="cuda"), cfg.B, cfg.W)
    rp, rs, rr = otree.tree_build(cu, anchors, cfg.B, cfg.W)
    assert np.array_equal(par.cpu().numpy(), rp)
    assert np.array_equal(pos.cpu().numpy(), rs)
    assert np.array_equal(srow.cpu().numpy(), rr)
    assert _status(lib) == 0


def test_tree_build_edges(lib):
    cu = np.array([0, 1, 7, 20], dtype=np.int32)
    # a=0, a=T-1, duplicates, unsorted
    anchors = np.array([0, 0, 0, 5, 3, 3, 12, 0, 7], dtype=np.int32)
    for W in (1, 2, 5):
        par, pos, srow = lib.specopd_tree_build(cu, torch.tensor(anchors, device="cuda"), 3, W)
        rp, rs, rr = otree.tree_build(cu, anchors, 3, W)
        assert np.array_equal(par.cpu().numpy(), rp)
        assert np.array_equal(pos.cpu().numpy(), rs)
        assert np.array_equal(srow.cpu().numpy(), rr)
    assert _status(lib) == 0


def test_tree_build_anchor_out_of_range_flags(lib):
    cu = np.array([0, 10], dtype=np.int32)
    anchors = torch.tensor([3, 10], dtype=torch.int32, device="cuda")
    par, pos, srow = lib.specopd_tree_build(cu, anchors, 2, 3)
    assert _status(lib) & lib.DEV_ANCHOR_RANGE
    assert srow.cpu().tolist()[3:] == [-1, -1, -1]
    assert _status(lib) == 0  # cleared by the read


# ---------------------------------------------------------------- rope

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_rope_apply(lib, dtype):
    rng = np.random.default_rng(0)
    n, H, D = 300, 3, 128
    x = rng.standard_normal((n, H, D)).astype(np.float32)
    if dtype == "bf16":
        x = synth.round_bf16(x)
    pos = rng.integers(0, 33000, size=n).astype(np.int32)
    pos[0] = 0
    xt = dev_tensor(x, dtype)
    lib.specopd_rope_apply(xt, torch.tensor(pos, device="cuda"), 10000.0)
    ref = oatt.rope(x.astype(np.float64), pos, 10000.0)
    got = to_np(xt)
    if dtype == "f32":
        assert np.max(np.abs(got - ref)) < 3e-6
        assert np.array_equal(got[0], x[0])  # position 0 is the identity
    else:
        # one rounding to bf16: |err| <= 2^-8 |ref| (+ tiny angle error)
        assert np.all(np.abs(got - ref) <= np.abs(ref) * 2.0 ** -8 + 1e-5)


# ---------------------------------------------------------------- attention (fp32)

def _attn_run(lib, inp, rope_base=10000.0):
    cfg = inp.cfg
    dt = cfg.dtype
    cu = [int(c) for c in inp.cu_trunk]
    anchors = torch.tensor(inp.anchors, device="cuda")
    _, sem_pos, _ = lib.specopd_tree_build(cu, anchors, cfg.B, cfg.W)
    k_tr = dev_tensor(inp.k_tr, dt)
    lib.specopd_rope_apply(k_tr, sem_pos[: inp.T_tot].contiguous(), rope_base)
    desc = lib.attn_desc(cfg.S, cfg.B, cfg.W, cfg.Hq, cfg.Hkv, cfg.D, dt, rope_base)
    lse = torch.empty((inp.R, cfg.Hq), dtype=torch.float32, device="cuda")
    out = lib.specopd_tree_attn(desc, dev_tensor(inp.q_br, dt), dev_tensor(inp.k_br, dt),
                                dev_tensor(inp.v_br, dt), k_tr, dev_tensor(inp.v_tr, dt),
                                torch.tensor(inp.cu_trunk, device="cuda"), cu, anchors, sem_pos,
                                lse=lse)
    torch.cuda.synchronize()
    return to_np(out), to_np(lse)


# fp32 attention outputs: 1e-5 relative per element, plus an absolute floor
# for outputs near zero.  An output is a softmax-weighted mean of unit-scale
# values; the RoPE angles are evaluated in fp32 on the GPU (about 1e-7
# relative on the rotated q/k), so scores, and hence every output, carry an
# absolute error of order 1e-7 whatever the output's own size.
ATT32_RTOL, ATT32_ATOL = 1e-5, 1e-6


def _attn_ref(inp):
    cfg = inp.cfg
    return oatt.branch_attention_unrolled_dense(inp.q_br, inp.k_br, inp.v_br, inp.k_tr, inp.v_tr,
                                                inp.cu_trunk, inp.anchors, cfg.B, cfg.W,
                                                cfg.rope_base)


def test_attention_tiny_fp32(lib):
    inp = synth.attention_inputs(synth.attn_config("tiny"))
    out, lse = _attn_run(lib, inp)
    ref = _attn_ref(inp)
    assert out.shape == ref.shape == (12, 4, 64)
    assert rel_err(out, ref) < 1e-5
    assert_close_elementwise(out, ref, ATT32_RTOL, ATT32_ATOL, "out")
    assert _status(lib) == 0


@pytest.mark.parametrize("S,T,B,W,Hq,Hkv,D,anchors", [
    (1, (40,), 3, 2, 2, 1, 64, [0, 39, 39]),          # a = 0, a = T-1, duplicates, W = 2
    (3, (5, 64, 17), 2, 5, 8, 2, 128, [4, 0, 63, 12, 16, 1]),  # packed, unsorted, D = 128
    (1, (30,), 4, 1, 2, 2, 64, [1, 2, 3, 4]),          # W = 1: no rows
])
def test_attention_fp32_edges(lib, S, T, B, W, Hq, Hkv, D, anchors):
    cfg = synth.custom_attn_config(S, T, B, W, Hq, Hkv, D, "f32")
    inp = synth.attention_inputs(cfg, anchors=anchors)
    if inp.R == 0:
        out, _ = _attn_run(lib, inp)
        assert out.shape[0] == 0
        return
    out, _ = _attn_run(lib, inp)
    ref = _attn_ref(inp)
    assert rel_err(out, ref) < 1e-5
    assert_close_elementwise(out, ref, ATT32_RTOL, ATT32_ATOL, "out")
    assert _status(lib) == 0


def test_attention_lse_fp32(lib):
    # lse = log sum exp of the scaled scores; check against the definition on
    # one row computed from the oracle's rotated vectors.
    inp = synth.attention_inputs(synth.attn_config("tiny"))
    _, lse = _attn_run(lib, inp)
    cfg = inp.cfg
    b, i, h = 2, 3, 1
    r = b * (cfg.W - 1) + (i - 1)
    a = int(inp.anchors[b])
    pos = np.arange(a + cfg.W)
    seq_k = np.concatenate([inp.k_tr[: a + 1], inp.k_br[b * (cfg.W - 1): (b + 1) * (cfg.W - 1)]])
    k = oatt.rope(seq_k.astype(np.float64), pos, 1e4)[: a + 1 + i, h // (cfg.Hq // cfg.Hkv)]
    q = oatt.rope(inp.q_br[r: r + 1].astype(np.float64), [a + i], 1e4)[0, h]
    s = k @ q / np.sqrt(cfg.D)
    ref = np.log(np.sum(np.exp(s - s.max()))) + s.max()
    assert abs(lse[r, h] - ref) < 1e-5 * max(1, abs(ref))


def test_attention_anchor_out_of_range_nan(lib):
    cfg = synth.custom_attn_config(1, (20,), 2, 3, 2, 1, 64, "f32")
    inp = synth.attention_inputs(cfg, anchors=[5, 25])
    # tree_build flags it too; attention writes NaN for the bad branch
    out, _ = _attn_run(lib, inp)
    assert np.all(np.isnan(out[2:])) and not np.any(np.isnan(out[:2]))
    assert _status(lib) & lib.DEV_ANCHOR_RANGE


# ---------------------------------------------------------------- E2E-TV

def _tv_run(lib, zt, zd, nb, W, dtype, grad_dtype="f32", target_row=None, zt_rows=None,
            compute_grad=True, norm_count=0):
    rows_t = zt.shape[0] if zt_rows is None else zt_rows.shape[0]
    desc = lib.tv_desc(nb, W, zd.shape[1], rows_t, dtype, grad_dtype, compute_grad, norm_count)
    zt_dev = dev_tensor(zt if zt_rows is None else zt_rows, dtype)
    tr = None if target_row is None else torch.tensor(target_row, dtype=torch.int32, device="cuda")
    res = lib.specopd_e2e_tv(desc, zt_dev, tr, dev_tensor(zd, dtype))
    torch.cuda.synchronize()
    return res


# fp32 outputs: 1e-5 relative per element, with a 1e-7 floor for reference
# values at or near zero (disjoint supports, late prefix products of
# low-overlap branches).  Gradient rows are compared normwise per row: near a
# tie q_v = p_v the fp32 kernel and the fp64 oracle may take different sides
# of the subgradient of min, which moves single elements of a row.
TV_RTOL, TV_ATOL = 1e-5, 1e-7


def _check_tv(res, ref, rows=None, grad=True):
    assert_close_elementwise(to_np(res["a"]), ref["a"], TV_RTOL, TV_ATOL, "a")
    assert_close_elementwise(to_np(res["prefix"]), ref["prefix"], TV_RTOL, TV_ATOL, "prefix")
    assert abs(res["loss"].item() - ref["loss"]) <= 1e-4 * abs(ref["loss"]) + 1e-7
    assert abs(res["numer"].item() - ref["numer"]) <= 1e-5 * abs(ref["numer"]) + 1e-7
    if grad:
        g = res["grad"]
        for n in (rows if rows is not None else ref["grad"].keys()):
            gr = ref["grad"][n]
            if np.max(np.abs(gr)) == 0:
                assert np.max(np.abs(to_np(g[n]))) < 1e-12
            else:
                assert rel_err(to_np(g[n]), gr) < 1e-3, n


def test_tv_tiny_fp32(lib):
    cfg = synth.tv_config("tiny")
    zt, zd = synth.logits(cfg)
    ref = otv.e2e_tv(zt, None, zd, cfg.nbranch, cfg.W)
    res = _tv_run(lib, zt, zd, cfg.nbranch, cfg.W, "f32")
    _check_tv(res, ref)
    assert _status(lib) == 0


def test_tv_8b_bf16_through_score_rows(lib):
    # The 8B-shaped workload: target logits live in the packed node order
    # [T_tot + R, V] and are read through the tree's score-row map.
    acfg = synth.attn_config("8b")
    cfg = synth.tv_config("8b")
    rng = np.random.default_rng(acfg.seed)
    anchors = synth.draw_anchors(rng, 1, acfg.B, acfg.anchor_lo, acfg.anchor_hi)
    cu = [0, acfg.T[0]]
    _, _, score_row = otree.tree_build(cu, anchors, acfg.B, acfg.W)
    zt, zd = synth.logits(cfg)
    rows_t = acfg.T[0] + acfg.B * (acfg.W - 1)
    zt_packed = torch.zeros((rows_t, cfg.V), dtype=torch.bfloat16, device="cuda")
    zt_packed[torch.tensor(score_row, device="cuda")] = dev_tensor(zt, "bf16")
    desc = lib.tv_desc(cfg.nbranch, cfg.W, cfg.V, rows_t, "bf16", "f32")
    res = lib.specopd_e2e_tv(desc, zt_packed, torch.tensor(score_row, dtype=torch.int32, device="cuda"),
                             dev_tensor(zd, "bf16"))
    torch.cuda.synchronize()
    rows = [0, 1, 7, 100, 257, 511]
    ref = otv.e2e_tv(zt, None, zd, cfg.nbranch, cfg.W, rows=set(rows))
    _check_tv(res, ref, rows=rows)
    assert _status(lib) == 0


@pytest.mark.parametrize("V,W,nb,dtype,gdt", [
    (1001, 3, 5, "f32", "f32"),    # V not a multiple of the vector width (unaligned path)
    (1003, 2, 3, "bf16", "bf16"),  # odd row stride in bf16, bf16 grads
    (4096, 1, 7, "bf16", "f32"),   # W = 1
    (1000, 3, 4, "f32", "bf16"),   # fp32 logits, bf16 gradient (aligned path)
    (111_104, 4, 2, "bf16", "f32"),  # ragged last slice, aligned path
    (40_000, 64, 2, "bf16", "f32"),  # W*NS = 256 tasks per branch, rounds of whole branches
    (151_936, 16, 3, "bf16", "f32"),  # the long trunk's vocabulary and W (NS = 12)
    (248_320, 16, 4, "bf16", "f32"),  # the packed batch's vocabulary and W
    (4096, 160, 1, "bf16", "f32"),   # W above the SM count: the slice schedule, aligned rows
    (140_000, 4, 3, "f32", "f32"),   # fp32 rows too long for pass B's bits: pass C reads both rows
    (50_000, 4, 5, "bf16", "bf16"),  # whole-row schedule, pass-C bits, bf16 gradient rows
])
def test_tv_shapes(lib, V, W, nb, dtype, gdt):
    rng = np.random.default_rng(V + W)
    zt = (rng.standard_normal((nb * W, V)) * 2).astype(np.float32)
    zd = (zt + rng.standard_normal((nb * W, V)) * 0.7).astype(np.float32)
    if dtype == "bf16":
        zt, zd = synth.round_bf16(zt), synth.round_bf16(zd)
    ref = otv.e2e_tv(zt, None, zd, nb, W)
    res = _tv_run(lib, zt, zd, nb, W, dtype, gdt)
    if gdt == "bf16":
        # bf16 output rounding: 2^-8 relative per element on top of fp32 error
        for n in ref["grad"]:
            assert rel_err(to_np(res["grad"][n]), ref["grad"][n]) < 8e-3
        _check_tv(res, ref, grad=False)
    else:
        _check_tv(res, ref)
    assert _status(lib) == 0


def test_tv_special_rows(lib):
    # identical rows (a = 1, zero grad), disjoint supports via -inf (a = 0),
    # the worked example (a = 0.8), and a -inf entry in a normal row.
    V = 64
    rng = np.random.default_rng(3)
    zt = rng.standard_normal((8, V)).astype(np.float32)
    zd = (zt + rng.standard_normal((8, V))).astype(np.float32)
    zd[0] = zt[0]
    zt[1, 32:] = -np.inf
    zd[1, :32] = -np.inf
    zt[2] = -np.inf
    zt[2, :3] = np.log([0.4, 0.4, 0.2])
    zd[2] = -np.inf
    zd[2, :2] = 0.0
    zd[5, 7] = -np.inf
    ref = otv.e2e_tv(zt, None, zd, 2, 4)
    res = _tv_run(lib, zt, zd, 2, 4, "f32")
    a = to_np(res["a"])
    assert abs(a[0] - 1) < 1e-6 and a[1] == 0.0 and abs(a[2] - 0.8) < 1e-6
    _check_tv(res, ref)
    assert _status(lib) == 0


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_tv_row_maxima_across_chunks(lib, dtype):
    # Rows long enough for several shared-memory chunks, whose maxima appear
    # late: a first stretch 100 nats below the rest (longer than a chunk),
    # a leading run of -inf longer than a chunk, slowly and quickly rising
    # rows.
    V = 40_000
    rng = np.random.default_rng(17)
    zt = (2.0 * rng.standard_normal((8, V))).astype(np.float32)
    zd = (zt + rng.standard_normal((8, V))).astype(np.float32)
    zt[1, :15_000] -= 100.0
    zd[1, :15_000] -= 100.0
    zt[2, :20_000] = -np.inf
    zd[3, :13_000] = -np.inf
    zt[3, :15_000] -= 100.0
    zt[4] = np.linspace(-50.0, 50.0, V)
    zd[4] = zt[4] + rng.standard_normal(V).astype(np.float32)
    zd[5] = np.linspace(-200.0, 200.0, V)
    if dtype == "bf16":
        zt = synth.round_bf16(zt)
        zd = synth.round_bf16(zd)
    ref = otv.e2e_tv(zt, None, zd, 2, 4)
    res = _tv_run(lib, zt, zd, 2, 4, dtype)
    _check_tv(res, ref)
    assert _status(lib) == 0


def test_tv_all_neg_inf_row_flags(lib):
    zt = np.zeros((2, 16), np.float32)
    zd = np.zeros((2, 16), np.float32)
    zt[1] = -np.inf
    res = _tv_run(lib, zt, zd, 1, 2, "f32")
    assert np.isnan(res["a"][1].item())
    assert _status(lib) & lib.DEV_ALL_NEG_INF


def test_tv_norm_count_and_no_grad(lib):
    # Distributed normalisation: a shard with the global count reproduces the
    # unsharded gradient coefficients; compute_grad = 0 skips the gradient.
    rng = np.random.default_rng(5)
    nb, W, V = 6, 3, 500
    zt = rng.standard_normal((nb * W, V)).astype(np.float32)
    zd = (zt + rng.standard_normal((nb * W, V))).astype(np.float32)
    full = otv.e2e_tv(zt, None, zd, nb, W)
    r0 = _tv_run(lib, zt[:6], zd[:6], 2, W, "f32", norm_count=nb * W)
    r1 = _tv_run(lib, zt[6:], zd[6:], 4, W, "f32", norm_count=nb * W)
    tot = r0["numer"].item() + r1["numer"].item()
    assert abs((1 - tot / (nb * W)) - full["loss"]) < 1e-6
    for n in range(6):
        assert rel_err(to_np(r0["grad"][n]), full["grad"][n]) < 1e-3
    r2 = _tv_run(lib, zt, zd, nb, W, "f32", compute_grad=False)
    assert r2["grad"] is None
    assert abs(r2["loss"].item() - full["loss"]) < 1e-5


def test_tv_no_grad_many_tasks(lib):
    # Many positions per CTA without the gradient: the overlaps, prefix
    # products and loss are the same bits as with it, and match the oracle.
    rng = np.random.default_rng(11)
    nb, W, V = 512, 4, 2000
    zt = (2.0 * rng.standard_normal((nb * W, V))).astype(np.float32)
    zd = (zt + rng.standard_normal((nb * W, V))).astype(np.float32)
    zt = torch.from_numpy(zt).to(torch.bfloat16).float().numpy()
    zd = torch.from_numpy(zd).to(torch.bfloat16).float().numpy()
    ref = otv.e2e_tv(zt, None, zd, nb, W, compute_grad=False)
    rg = _tv_run(lib, zt, zd, nb, W, "bf16", compute_grad=True)
    rn = _tv_run(lib, zt, zd, nb, W, "bf16", compute_grad=False)
    assert rn["grad"] is None
    for k in ("a", "prefix", "loss", "numer"):
        assert torch.equal(rg[k], rn[k]), k
    assert_close_elementwise(to_np(rn["a"]), ref["a"], TV_RTOL, TV_ATOL, "a")
    assert abs(rn["loss"].item() - ref["loss"]) <= 1e-4 * abs(ref["loss"]) + 1e-7


def test_tv_deterministic(lib):
    cfg = synth.tv_config("tiny")
    zt, zd = synth.logits(cfg)
    r1 = _tv_run(lib, zt, zd, cfg.nbranch, cfg.W, "f32")
    r2 = _tv_run(lib, zt, zd, cfg.nbranch, cfg.W, "f32")
    for k in ("a", "prefix", "loss", "numer", "grad"):
        assert torch.equal(r1[k], r2[k]), k
