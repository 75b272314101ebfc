"""E2E-TV acceptance-length loss and its gradient, in fp64.

Oracle (test infrastructure only; see ``oracle/__init__.py``).

Sources:
  * SpecOPD review (jaehun.me) §1.1: under the rejection-sampling rule that
    draws one sample, the probability that a drafter token is accepted is
    the overlap of the two distributions, 1 - TV; acceptance length counts
    the accepted prefix plus one bonus token (example in §1.2: two accepted
    then a rejection gives 3; all four accepted gives 5).
  * Review §3.3: the loss is built from prefix products of the per-position
    overlaps within each branch (an early mismatch weighs on every later
    term); target mass outside the drafter's support is kept (no
    renormalisation of p); the gradient differentiates the overlaps with the
    sampled tokens and the target held fixed, with no score-function term.
  * Paper summary (rustineverything.app) §2.3: the loss is 1 minus the mean,
    over the B*W proposed tokens, of the prefix product.

Readings (design notes list each): temperature 1 and full-vocabulary
softmax for both p and q; subgradient of min at a tie q_v = p_v is taken as
the p-side ([q_v < p_v] strict); the gradient is written without dividing
by any overlap.
"""

from __future__ import annotations

import numpy as np


def softmax(z):
    """Full-vocabulary softmax of one logit row, fp64.  -inf -> probability 0.
    A row with no finite entry yields NaN (the library flags such rows)."""
    z = np.asarray(z, dtype=np.float64)
    m = np.max(z)
    if not np.isfinite(m):
        return np.full(z.shape, np.nan)
    e = np.exp(z - m)
    return e / np.sum(e)


def overlap(p, q):
    """Acceptance probability of one drafted token: sum_v min(p_v, q_v)."""
    return float(np.sum(np.minimum(p, q)))


def total_variation(p, q):
    """TV(p, q) = 1/2 sum_v |p_v - q_v|."""
    return 0.5 * float(np.sum(np.abs(np.asarray(p) - np.asarray(q))))


def prefix_products(a):
    """P[b, i] = prod_{j <= i} a[b, j] for a[nbranch, W]."""
    return np.cumprod(np.asarray(a, dtype=np.float64), axis=1)


def expected_acceptance_length(a):
    """E[AL_b] = 1 + sum_i P[b, i]  (accepted prefix plus the bonus token),
    valid when position i is accepted with probability a[b, i] given that
    the earlier positions were."""
    return 1.0 + prefix_products(a).sum(axis=1)


def loss_from_overlaps(a, norm_count=None):
    """loss = 1 - sum_{b,i} P[b,i] / norm_count   (norm_count defaults to B*W)."""
    P = prefix_products(a)
    n = P.size if norm_count is None else norm_count
    return 1.0 - P.sum() / n


def overlap_grad_coeff(a, norm_count=None):
    """g[b, j] = d loss / d a[b, j] = -(1/n) * P[b, j-1] * S[b, j],
    P[b, 0] = 1, S[b, W] = 1, S[b, j] = 1 + a[b, j+1] * S[b, j+1]
    (1-based j).  Written without any division by an overlap."""
    a = np.asarray(a, dtype=np.float64)
    nb, W = a.shape
    n = a.size if norm_count is None else norm_count
    P = prefix_products(a)
    P_prev = np.concatenate([np.ones((nb, 1)), P[:, :-1]], axis=1)
    S = np.ones((nb, W))
    for j in range(W - 2, -1, -1):
        S[:, j] = 1.0 + a[:, j + 1] * S[:, j + 1]
    return -(1.0 / n) * P_prev * S


def e2e_tv(z_target, target_row, z_draft, nbranch, W, norm_count=None,
           compute_grad=True, rows=None):
    """E2E-TV over nbranch branches of W positions.

    z_target [rows_t, V], target_row [N] (None = identity), z_draft [N, V];
    position n = b*W + (i-1).  Returns dict with a[N], s[N], prefix[N],
    loss, numer (= sum prefix), g[N] and, if compute_grad, grad[N, V].
    ``rows`` restricts the gradient to those positions (others are None);
    a, prefix and loss are always computed over every position.
    """
    N = nbranch * W
    if target_row is None:
        target_row = np.arange(N)
    a = np.empty(N)
    s = np.empty(N)
    probs = {}
    for n in range(N):
        p = softmax(z_target[int(target_row[n])])
        q = softmax(z_draft[n])
        a[n] = overlap(p, q)
        m = q < p
        s[n] = float(np.sum(q[m]))
        if compute_grad and (rows is None or n in rows):
            probs[n] = (p, q)
    A = a.reshape(nbranch, W)
    P = prefix_products(A)
    nc = N if norm_count is None else norm_count
    out = {
        "a": a,
        "s": s,
        "prefix": P.reshape(-1),
        "numer": float(P.sum()),
        "loss": 1.0 - float(P.sum()) / nc,
        "g": overlap_grad_coeff(A, nc).reshape(-1),
    }
    if compute_grad:
        g = out["g"]
        grad = {}
        for n, (p, q) in probs.items():
            m = (q < p).astype(np.float64)
            # d a_n / d z_u = q_u * (m_u - s_n)   (softmax Jacobian applied to m)
            grad[n] = g[n] * q * (m - s[n])
        out["grad"] = grad
    return out
