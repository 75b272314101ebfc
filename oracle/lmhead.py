"""E2E-TV with the LM head in front of it, in fp64.

Oracle (test infrastructure only; see ``oracle/__init__.py``).

Sources:
  * SpecOPD review (jaehun.me) §3.2(a), the score-row reading rule: the
    logits that score a position are read from the output of its predictor
    row, so the target logits of position n come from the hidden state of
    target row ``target_row[n]``.
  * Review §3.3: E2E-TV on those logits (``oracle.tv``).

The LM head is the linear map from a row's hidden state h [d] to its
vocabulary logits z = W h, W [V, d] (row v of W scores token v).  The pages
name no bias, normalisation or temperature in front of the loss, so none is
applied (a reading).  The target and the drafter each have their own head.

    z_target[n] = W_target h_target[target_row[n]]
    z_draft[n]  = W_draft  h_draft[n]

and then exactly ``oracle.tv.e2e_tv`` on those rows: the overlaps, prefix
products, loss and the gradient with respect to the draft LOGITS.
"""

from __future__ import annotations

import numpy as np

from . import tv


def lm_logits(h, w):
    """Vocabulary logits of hidden rows: out[r, v] = sum_k h[r, k] * w[v, k],
    in fp64.  h [rows, d], w [V, d] -> [rows, V]."""
    h = np.asarray(h, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    return h @ w.T


def e2e_tv_lmhead(h_target, target_row, w_target, h_draft, w_draft, nbranch, W,
                  norm_count=None, compute_grad=True, rows=None):
    """E2E-TV of nbranch branches of W positions whose logits come from hidden
    rows through the two LM heads.

    h_target [rows_t, d], target_row [N] (None = identity), w_target [V, d],
    h_draft [N, d], w_draft [V, d].  Returns what ``oracle.tv.e2e_tv``
    returns for the logits z_target = h_target[target_row] W_target^T and
    z_draft = h_draft W_draft^T (a, s, prefix, numer, loss, g and, if
    compute_grad, the gradient with respect to the draft logits for the
    positions in ``rows``, or all).
    """
    N = nbranch * W
    if target_row is None:
        target_row = np.arange(N)
    target_row = np.asarray(target_row)
    z_t = lm_logits(np.asarray(h_target)[target_row], w_target)
    z_d = lm_logits(h_draft, w_draft)
    return tv.e2e_tv(z_t, None, z_d, nbranch, W, norm_count=norm_count,
                     compute_grad=compute_grad, rows=rows)
