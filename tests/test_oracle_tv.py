"""Pins of the oracle's E2E-TV loss and gradient (CPU only).

Ties oracle.tv to: the pages' worked examples (review §3.3 overlap 0.8 with
target mass kept, review §5.1 alpha_1 = 0.2, review §1.2 acceptance lengths
3 and 5, "errs earlier => larger loss"), the exact acceptance probability of
the speculative-sampling rule by enumeration, a = 1 - TV, the prefix-product
reading by Monte Carlo, finite differences and torch autograd for the
gradient, and the distributed-normalisation identity (review §3.2).
"""

import numpy as np
import pytest
import torch

from oracle import tv


def _p(logits):
    return tv.softmax(np.log(np.asarray(logits, dtype=np.float64)))


def test_identical_rows_overlap_one():
    rng = np.random.default_rng(0)
    z = rng.standard_normal(1000) * 3
    p = tv.softmax(z)
    assert abs(tv.overlap(p, p) - 1.0) < 1e-12


def test_disjoint_supports_overlap_zero():
    zt = np.array([0.0, 1.0, -np.inf, -np.inf])
    zd = np.array([-np.inf, -np.inf, 2.0, 0.5])
    assert tv.overlap(tv.softmax(zt), tv.softmax(zd)) == 0.0


def test_worked_example_keeps_out_of_support_mass():
    # Review §3.3: q = (0.5, 0.5, 0), p = (0.4, 0.4, 0.2): TV 0.2, overlap 0.8;
    # renormalising p over {X, Y} would (wrongly) give overlap 1.
    q = np.array([0.5, 0.5, 0.0])
    p = np.array([0.4, 0.4, 0.2])
    assert abs(tv.total_variation(p, q) - 0.2) < 1e-15
    assert abs(tv.overlap(p, q) - 0.8) < 1e-15
    pr = p[:2] / p[:2].sum()
    assert abs(tv.overlap(pr, q[:2]) - 1.0) < 1e-15
    # and through the logit path, with -inf for the drafter's missing token
    a = tv.overlap(tv.softmax(np.log([0.4, 0.4, 0.2])), tv.softmax(np.array([0.0, 0.0, -np.inf])))
    assert abs(a - 0.8) < 1e-15


def test_alpha_one_example():
    # Review §5.1 (App. C.2 counterexample): q1 = (0.9, 0.1), p1 = (0.1, 0.9) -> 0.2.
    assert abs(tv.overlap([0.1, 0.9], [0.9, 0.1]) - 0.2) < 1e-15


def test_overlap_is_acceptance_probability_of_speculative_sampling():
    # Review §1.1: the acceptance probability of one drafted token under the
    # single-sample rejection rule (draw y ~ q, accept w.p. min(1, p(y)/q(y)))
    # is the overlap.  Exact enumeration over the vocabulary.
    rng = np.random.default_rng(1)
    for _ in range(20):
        V = int(rng.integers(2, 30))
        p = tv.softmax(rng.standard_normal(V) * 2)
        q = tv.softmax(rng.standard_normal(V) * 2)
        accept = sum(q[y] * min(1.0, p[y] / q[y]) for y in range(V))
        assert abs(accept - tv.overlap(p, q)) < 1e-13
        assert abs(tv.overlap(p, q) - (1.0 - tv.total_variation(p, q))) < 1e-13
        assert abs(tv.overlap(p, q) - tv.overlap(q, p)) < 1e-15
        assert 0.0 <= tv.overlap(p, q) <= 1.0


def test_acceptance_length_examples():
    # Review §1.2: accept, accept, reject -> AL 3; all four accepted -> 4 + 1 = 5.
    assert tv.expected_acceptance_length([[1, 1, 0, 1]])[0] == 3.0
    assert tv.expected_acceptance_length([[1, 1, 0, 0.3]])[0] == 3.0
    assert tv.expected_acceptance_length([[1, 1, 1, 1]])[0] == 5.0


def test_prefix_product_is_survival_probability_monte_carlo():
    # Accepting position i with probability a_i given the earlier ones were
    # accepted: E[accepted prefix] = sum_i prod_{j<=i} a_j.  Monte Carlo.
    rng = np.random.default_rng(2)
    a = np.array([0.9, 0.7, 0.8, 0.5, 0.95])
    trials = 200_000
    u = rng.random((trials, a.size))
    acc = u < a[None, :]
    prefix_len = np.argmin(np.concatenate([acc, np.zeros((trials, 1), bool)], 1), axis=1)
    est = prefix_len.mean()
    exact = tv.prefix_products(a[None])[0].sum()
    assert abs(est - exact) < 4 * prefix_len.std() / np.sqrt(trials)


def test_errs_earlier_gives_larger_loss():
    # Review §3.3 (App. C.2): same per-token error, earlier mismatch -> larger loss.
    early = tv.loss_from_overlaps([[0.5, 1.0]])
    late = tv.loss_from_overlaps([[1.0, 0.5]])
    assert abs(early - 0.5) < 1e-15 and abs(late - 0.25) < 1e-15
    assert early > late


def test_loss_bounds_and_mean_definition():
    # Summary §2.3: loss = 1 - mean over the B*W tokens of the prefix product.
    rng = np.random.default_rng(3)
    a = rng.random((6, 5))
    P = np.array([[np.prod(a[b, : i + 1]) for i in range(5)] for b in range(6)])
    assert abs(tv.loss_from_overlaps(a) - (1 - P.mean())) < 1e-15
    assert 0 <= tv.loss_from_overlaps(a) <= 1
    assert tv.loss_from_overlaps(np.ones((3, 4))) == 0.0
    assert tv.loss_from_overlaps(np.zeros((3, 4))) == 1.0


def _tiny_problem(rng, nb, W, V, ties_ok=False):
    zt = rng.standard_normal((nb * W, V)) * 1.5
    zd = zt + rng.standard_normal((nb * W, V)) * 0.8
    return zt, zd


def _loss_of(zt, zd, nb, W):
    a = np.array([tv.overlap(tv.softmax(zt[n]), tv.softmax(zd[n])) for n in range(nb * W)])
    return tv.loss_from_overlaps(a.reshape(nb, W))


def test_gradient_matches_finite_differences():
    rng = np.random.default_rng(4)
    nb, W, V = 2, 4, 12
    zt, zd = _tiny_problem(rng, nb, W, V)
    res = tv.e2e_tv(zt, None, zd, nb, W)
    h = 1e-6
    for n in range(nb * W):
        for u in range(V):
            zp = zd.copy(); zp[n, u] += h
            zm = zd.copy(); zm[n, u] -= h
            fd = (_loss_of(zt, zp, nb, W) - _loss_of(zt, zm, nb, W)) / (2 * h)
            assert abs(fd - res["grad"][n][u]) < 1e-8, (n, u)


def test_gradient_matches_torch_autograd():
    rng = np.random.default_rng(5)
    nb, W, V = 3, 5, 40
    zt, zd = _tiny_problem(rng, nb, W, V)
    res = tv.e2e_tv(zt, None, zd, nb, W)
    zd_t = torch.tensor(zd, dtype=torch.float64, requires_grad=True)
    p = torch.softmax(torch.tensor(zt, dtype=torch.float64), dim=-1)
    q = torch.softmax(zd_t, dim=-1)
    a = torch.minimum(p, q).sum(-1).reshape(nb, W)
    loss = 1 - torch.cumprod(a, dim=1).mean()
    loss.backward()
    assert abs(loss.item() - res["loss"]) < 1e-14
    g = np.stack([res["grad"][n] for n in range(nb * W)])
    np.testing.assert_allclose(g, zd_t.grad.numpy(), rtol=1e-10, atol=1e-14)


def test_gradient_invariants():
    rng = np.random.default_rng(6)
    nb, W, V = 2, 3, 50
    zt, zd = _tiny_problem(rng, nb, W, V)
    zd[1] = zt[1]  # one identical row
    res = tv.e2e_tv(zt, None, zd, nb, W)
    for n in range(nb * W):
        assert abs(res["grad"][n].sum()) < 1e-15   # softmax gradient sums to 0
    assert np.all(res["grad"][1] == 0.0)            # identical row: no gradient
    assert abs(res["a"][1] - 1.0) < 1e-12


def test_distributed_normalisation_identity():
    # Review §3.2 [numerical consistency]: numerators and counts gathered
    # separately, so a sharded run with the global count reproduces the
    # unsharded loss and gradients exactly.
    rng = np.random.default_rng(7)
    nb, W, V = 6, 3, 20
    zt, zd = _tiny_problem(rng, nb, W, V)
    full = tv.e2e_tv(zt, None, zd, nb, W)
    cut = 2 * W
    r0 = tv.e2e_tv(zt[:cut], None, zd[:cut], 2, W, norm_count=nb * W)
    r1 = tv.e2e_tv(zt[cut:], None, zd[cut:], 4, W, norm_count=nb * W)
    assert abs(1 - (r0["numer"] + r1["numer"]) / (nb * W) - full["loss"]) < 1e-15
    np.testing.assert_allclose(np.concatenate([r0["g"], r1["g"]]), full["g"], rtol=1e-15)


def test_target_row_gather():
    rng = np.random.default_rng(8)
    zt = rng.standard_normal((10, 7))
    zd = rng.standard_normal((4, 7))
    tr = np.array([9, 0, 3, 3])
    r1 = tv.e2e_tv(zt, tr, zd, 2, 2)
    r2 = tv.e2e_tv(zt[tr], None, zd, 2, 2)
    np.testing.assert_array_equal(r1["a"], r2["a"])


def test_all_neg_inf_row_is_nan():
    zt = np.array([[0.0, 1.0], [-np.inf, -np.inf]])
    zd = np.array([[0.0, 0.0], [0.0, 0.0]])
    r = tv.e2e_tv(zt, None, zd, 1, 2)
    assert np.isnan(r["a"][1]) and not np.isnan(r["a"][0])
