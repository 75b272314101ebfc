"""Pins of the oracle's branch attention (CPU only).

oracle.attention scores each branch as its own unrolled sequence.  These
tests tie it to what the pages and mathematics fix: a packed tree with an
explicit ancestor mask gives the same rows (review §3.2(a): packed scoring
yields the same supervision as per-branch scoring), masked keys cannot
influence a row, a single branch reduces to textbook causal attention
(library SDPA), GQA reduces to replicated kv heads, and RoPE matches the
complex-rotation definition and depends only on relative position.
"""

import numpy as np
import pytest
import torch

from oracle import attention as att
from oracle import tree


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def test_rope_pos0_is_identity():
    rng = np.random.default_rng(0)
    x = _rand(rng, 5, 3, 16)
    np.testing.assert_array_equal(att.rope(x, np.zeros(5, int), 10000.0), x)


def test_rope_matches_complex_rotation():
    # Independent statement of the half-split RoPE: pair (x_k, x_{k+D/2}) as the
    # complex number x_k + i x_{k+D/2}, multiplied by exp(i * pos * theta_k).
    rng = np.random.default_rng(1)
    n, H, D, base = 7, 2, 64, 10000.0
    x = _rand(rng, n, H, D)
    pos = rng.integers(0, 40000, size=n)
    half = D // 2
    theta = np.array([base ** (-(2.0 * k) / D) for k in range(half)])
    z = x[..., :half] + 1j * x[..., half:]
    zr = z * np.exp(1j * pos[:, None, None] * theta[None, None, :])
    ref = np.concatenate([zr.real, zr.imag], axis=-1)
    np.testing.assert_allclose(att.rope(x, pos, base), ref, rtol=0, atol=1e-10)  # angles up to 4e4 rad


def test_rope_2d_by_hand():
    # D = 2: theta_0 = 1, so (1, 0) at position 1 is (cos 1, sin 1).
    y = att.rope(np.array([[[1.0, 0.0]]]), np.array([1]), 10000.0)
    np.testing.assert_allclose(y[0, 0], [np.cos(1.0), np.sin(1.0)], atol=1e-15)


def test_rope_relative_position():
    rng = np.random.default_rng(2)
    q = _rand(rng, 1, 1, 32)
    k = _rand(rng, 1, 1, 32)
    d1 = float((att.rope(q, [100], 1e4) * att.rope(k, [90], 1e4)).sum())
    d2 = float((att.rope(q, [5010], 1e4) * att.rope(k, [5000], 1e4)).sum())
    assert abs(d1 - d2) < 1e-9


def _case(rng, S, T, B, W, Hq, Hkv, D, anchors=None):
    cu = np.concatenate([[0], np.cumsum(T)]).astype(int)
    if anchors is None:
        anchors = np.concatenate([rng.integers(0, t, size=B) for t in T])
    R = S * B * (W - 1)
    return dict(
        cu=cu, anchors=np.asarray(anchors), B=B, W=W,
        q=_rand(rng, R, Hq, D), kb=_rand(rng, R, Hkv, D), vb=_rand(rng, R, Hkv, D),
        kt=_rand(rng, cu[-1], Hkv, D), vt=_rand(rng, cu[-1], Hkv, D),
    )


def _unrolled(c, base=10000.0):
    return att.branch_attention_unrolled_dense(c["q"], c["kb"], c["vb"], c["kt"], c["vt"],
                                               c["cu"], c["anchors"], c["B"], c["W"], base)


@pytest.mark.parametrize("S,T,B,W,Hq,Hkv,D", [
    (1, [24], 3, 4, 2, 1, 8),
    (2, [9, 20], 4, 5, 4, 2, 16),
    (3, [1, 5, 13], 2, 3, 3, 3, 8),
])
def test_packed_tree_equals_unrolled(S, T, B, W, Hq, Hkv, D):
    # Review §3.2(a): one packed pass with the tree mask scores every branch
    # exactly as scoring the branch alone would.
    rng = np.random.default_rng(S + B + W)
    c = _case(rng, S, T, B, W, Hq, Hkv, D)
    c["anchors"][0] = 0
    c["anchors"][-1] = T[-1] - 1
    parent, sem_pos, _ = tree.tree_build(c["cu"], c["anchors"], B, W)
    packed = att.packed_tree_attention(c["q"], c["kb"], c["vb"], c["kt"], c["vt"],
                                       parent, sem_pos, int(c["cu"][-1]), 10000.0)
    np.testing.assert_allclose(packed, _unrolled(c), rtol=1e-12, atol=1e-12)


def test_masked_keys_do_not_matter():
    # Review §3.2(a): sibling branches and future reference tokens are masked.
    rng = np.random.default_rng(3)
    c = _case(rng, 1, [30], 3, 4, 2, 1, 8, anchors=[5, 12, 12])
    base = _unrolled(c)
    c2 = dict(c)
    kt, vt = c["kt"].copy(), c["vt"].copy()
    kt[6:] += 100.0          # trunk after anchor 5: invisible to branch 0
    vt[6:] -= 50.0
    c2.update(kt=kt, vt=vt)
    out2 = _unrolled(c2)
    np.testing.assert_array_equal(out2[0:3], base[0:3])
    kb = c["kb"].copy()
    kb[3:] *= -7.0           # branches 1,2 rows: invisible to branch 0
    c3 = dict(c, kb=kb)
    np.testing.assert_array_equal(_unrolled(c3)[0:3], base[0:3])
    # ...and a later branch token is invisible to an earlier row.
    kb = c["kb"].copy()
    kb[2] += 9.0
    c4 = dict(c, kb=kb)
    np.testing.assert_array_equal(_unrolled(c4)[0:2], base[0:2])
    assert not np.array_equal(_unrolled(c4)[2], base[2])


def test_single_branch_is_textbook_causal_attention():
    # One branch, Hq = Hkv = 1: the branch rows are the last W-1 rows of plain
    # causal attention over (trunk[0..a], branch), checked with torch SDPA.
    rng = np.random.default_rng(4)
    a, W, D = 10, 5, 16
    c = _case(rng, 1, [20], 1, W, 1, 1, D, anchors=[a])
    out = _unrolled(c)
    pos = np.arange(a + W)
    k = att.rope(np.concatenate([c["kt"][: a + 1], c["kb"]]), pos, 1e4)[:, 0]
    v = np.concatenate([c["vt"][: a + 1], c["vb"]])[:, 0]
    q = att.rope(c["q"], pos[a + 1:], 1e4)[:, 0]
    mask = torch.tensor(pos[None, :] <= pos[a + 1:, None])
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q)[None], torch.tensor(k)[None], torch.tensor(v)[None],
        attn_mask=mask[None])[0].numpy()
    np.testing.assert_allclose(out[:, 0], ref, rtol=1e-12, atol=1e-12)


def test_gqa_equals_replicated_kv_heads():
    rng = np.random.default_rng(5)
    c = _case(rng, 1, [16], 2, 3, 4, 2, 8)
    gqa = _unrolled(c)
    rep = dict(c, kb=np.repeat(c["kb"], 2, axis=1), vb=np.repeat(c["vb"], 2, axis=1),
               kt=np.repeat(c["kt"], 2, axis=1), vt=np.repeat(c["vt"], 2, axis=1))
    np.testing.assert_allclose(gqa, _unrolled(rep), rtol=0, atol=1e-14)


def test_width_one_has_no_rows():
    rng = np.random.default_rng(6)
    c = _case(rng, 1, [16], 3, 1, 2, 1, 8)
    assert _unrolled(c).shape == (0, 2, 8)


def test_rows_are_convex_combinations_of_visible_values():
    # softmax weights are a probability vector: with all visible V equal to a
    # constant vector, the output is that vector.
    rng = np.random.default_rng(8)
    c = _case(rng, 1, [12], 2, 4, 2, 1, 8)
    c["vt"][:] = 0.25
    c["vb"][:] = 0.25
    np.testing.assert_allclose(_unrolled(c), 0.25, rtol=0, atol=1e-14)


# ---------------------------------------------------------------- trunk prefill

def _prefill_case(rng, T, Hq, Hkv, D):
    cu = np.concatenate([[0], np.cumsum(T)]).astype(int)
    n = int(cu[-1])
    return cu, _rand(rng, n, Hq, D), _rand(rng, n, Hkv, D), _rand(rng, n, Hkv, D)


def test_prefill_single_sequence_is_textbook_causal_attention():
    # One sequence, Hq = Hkv = 1: torch SDPA with is_causal on the rotated
    # inputs (a library routine, independent of the oracle's own softmax).
    rng = np.random.default_rng(11)
    cu, q, k, v = _prefill_case(rng, [37], 1, 1, 16)
    out, kc = att.trunk_prefill(q, k, v, cu, 1e4)
    pos = np.arange(37)
    qr = att.rope(q, pos, 1e4)[:, 0]
    kr = att.rope(k, pos, 1e4)[:, 0]
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(qr)[None], torch.tensor(kr)[None], torch.tensor(v[:, 0])[None],
        is_causal=True)[0].numpy()
    np.testing.assert_allclose(out[:, 0], ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_array_equal(kc[:, 0], kr)


def test_prefill_first_row_is_its_own_value():
    # Position 0 sees only itself: its output is v_0 for every head.
    rng = np.random.default_rng(12)
    cu, q, k, v = _prefill_case(rng, [5, 9, 1], 4, 2, 8)
    out, _ = att.trunk_prefill(q, k, v, cu, 1e4)
    for s in range(3):
        r = cu[s]
        np.testing.assert_allclose(out[r], np.repeat(v[r], 2, axis=0), rtol=0, atol=1e-15)


def test_prefill_sequences_do_not_see_each_other():
    # A packed batch gives each sequence exactly its own prefill, and keys
    # after a row's position cannot move it.
    rng = np.random.default_rng(13)
    T = [6, 11, 4]
    cu, q, k, v = _prefill_case(rng, T, 2, 1, 8)
    out, kc = att.trunk_prefill(q, k, v, cu, 1e4)
    for s in range(3):
        rows = slice(cu[s], cu[s + 1])
        o1, k1 = att.trunk_prefill(q[rows], k[rows], v[rows], [0, T[s]], 1e4)
        np.testing.assert_array_equal(out[rows], o1)
        np.testing.assert_array_equal(kc[rows], k1)
    k2, v2 = k.copy(), v.copy()
    k2[cu[1] + 5:] += 50.0   # sequence 1 from position 5 on, and everything after it
    v2[cu[1] + 5:] -= 9.0
    out2, _ = att.trunk_prefill(q, k2, v2, cu, 1e4)
    np.testing.assert_array_equal(out2[: cu[1] + 5], out[: cu[1] + 5])
    assert not np.array_equal(out2[cu[1] + 5], out[cu[1] + 5])


def test_prefill_then_branch_equals_one_longer_prefill():
    # Review §3.2(a): the branch pass reuses the cached trunk.  A branch
    # scored over the prefilled cache gives the same rows as prefilling the
    # linear sequence trunk[0..a] followed by the branch tokens: its last W-1
    # rows.  The two sides use different formulations (packed tree mask
    # against per-sequence causal attention).
    rng = np.random.default_rng(14)
    T, a, W, Hq, Hkv, D = 20, 12, 4, 2, 1, 8
    c = _case(rng, 1, [T], 1, W, Hq, Hkv, D, anchors=[a])
    parent, sem_pos, _ = tree.tree_build(c["cu"], c["anchors"], 1, W)
    branch = att.packed_tree_attention(c["q"], c["kb"], c["vb"], c["kt"], c["vt"], parent,
                                       sem_pos, T, 1e4)
    q_seq = np.concatenate([_rand(rng, a + 1, Hq, D), c["q"]])
    k_seq = np.concatenate([c["kt"][: a + 1], c["kb"]])
    v_seq = np.concatenate([c["vt"][: a + 1], c["vb"]])
    out, _ = att.trunk_prefill(q_seq, k_seq, v_seq, [0, a + W], 1e4)
    np.testing.assert_allclose(out[a + 1:], branch, rtol=1e-12, atol=1e-12)


def test_prefill_sampled_rows_equal_full_rows():
    rng = np.random.default_rng(15)
    cu, q, k, v = _prefill_case(rng, [9, 30, 4], 4, 2, 8)
    full, kc = att.trunk_prefill(q, k, v, cu, 1e4)
    rows = [0, 8, 9, 25, 38, 42]
    part, kc2 = att.trunk_prefill(q, k, v, cu, 1e4, rows=rows)
    np.testing.assert_allclose(part[rows], full[rows], rtol=1e-12, atol=1e-13)  # BLAS blocking
    np.testing.assert_array_equal(kc2, kc)
    others = np.setdiff1d(np.arange(cu[-1]), rows)
    assert np.all(np.isnan(part[others]))
