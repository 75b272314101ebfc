"""Pins of the oracle's LM-head E2E-TV (CPU only).

oracle.lmhead forms the logits from hidden rows through the two LM heads
(review §3.2(a), score-row reading rule) and hands them to oracle.tv, which
its own pins tie to the pages.  These pins tie the head to facts that do not
depend on retyping its product:
  * a one-hot hidden row e_k reads out column k of the head (W e_k), which a
    transposed head would not;
  * with identity heads the call reduces to the pinned oracle.tv.e2e_tv on
    the hidden rows themselves, target-row gather included;
  * with a common non-involutory permutation head the overlaps, prefix
    products and loss are unchanged (a relabelling of the vocabulary) and
    the gradient's columns are permuted the same way;
  * a draft head 2I against a target head I is the draft at temperature 1/2,
    which swapping the two heads would break.
"""

import numpy as np

from oracle import lmhead, tv


def _rows(rng, n, d, scale=2.0):
    return rng.standard_normal((n, d)) * scale


def test_one_hot_row_reads_head_column():
    rng = np.random.default_rng(0)
    V, d = 7, 5
    w = rng.standard_normal((V, d))
    for k in range(d):
        e = np.zeros((1, d))
        e[0, k] = 1.0
        z = lmhead.lm_logits(e, w)
        assert z.shape == (1, V)
        assert np.array_equal(z[0], w[:, k])


def test_identity_head_reduces_to_tv_oracle():
    rng = np.random.default_rng(1)
    nb, W, V = 3, 4, 9
    N = nb * W
    ht = _rows(rng, N + 5, V)
    hd = _rows(rng, N, V)
    trow = rng.permutation(N + 5)[:N]
    eye = np.eye(V)
    got = lmhead.e2e_tv_lmhead(ht, trow, eye, hd, eye, nb, W, norm_count=50)
    ref = tv.e2e_tv(ht, trow, hd, nb, W, norm_count=50)
    for key in ("a", "s", "prefix", "g"):
        assert np.allclose(got[key], ref[key], rtol=1e-13, atol=1e-15), key
    assert abs(got["loss"] - ref["loss"]) < 1e-13
    assert abs(got["numer"] - ref["numer"]) < 1e-12
    for n in range(N):
        assert np.allclose(got["grad"][n], ref["grad"][n], rtol=1e-12, atol=1e-15)


def test_permutation_head_relabels_vocabulary():
    rng = np.random.default_rng(2)
    nb, W, V = 2, 3, 8
    N = nb * W
    ht = _rows(rng, N, V)
    hd = _rows(rng, N, V)
    # a cycle of length V: its own inverse only for V <= 2
    pi = np.roll(np.arange(V), 3)
    perm = np.zeros((V, V))
    perm[np.arange(V), pi] = 1.0        # (perm h)[v] = h[pi[v]]
    got = lmhead.e2e_tv_lmhead(ht, None, perm, hd, perm, nb, W)
    ref = tv.e2e_tv(ht, None, hd, nb, W)
    for key in ("a", "prefix"):
        assert np.allclose(got[key], ref[key], rtol=1e-13, atol=1e-15), key
    assert abs(got["loss"] - ref["loss"]) < 1e-13
    for n in range(N):
        assert np.allclose(got["grad"][n], ref["grad"][n][pi], rtol=1e-12, atol=1e-15)
    # the transposed head permutes the other way, and the gradient shows it
    got_t = lmhead.e2e_tv_lmhead(ht, None, perm.T, hd, perm.T, nb, W)
    assert not np.allclose(got_t["grad"][0], got["grad"][0])


def test_heads_are_not_swapped():
    rng = np.random.default_rng(3)
    nb, W, V = 2, 2, 6
    N = nb * W
    ht = _rows(rng, N, V, 1.0)
    hd = _rows(rng, N, V, 1.0)
    eye = np.eye(V)
    got = lmhead.e2e_tv_lmhead(ht, None, eye, hd, 2.0 * eye, nb, W)
    ref = tv.e2e_tv(ht, None, 2.0 * hd, nb, W)
    assert np.allclose(got["a"], ref["a"], rtol=1e-13)
    swapped = tv.e2e_tv(2.0 * ht, None, hd, nb, W)
    assert not np.allclose(got["a"], swapped["a"], rtol=1e-6)
