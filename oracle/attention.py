"""Branch scoring under full (GQA) attention, in fp64, by unrolling.

Oracle (test infrastructure only; see ``oracle/__init__.py``).

Sources:
  * SpecOPD review (jaehun.me) §3.1: the drafter's condition at branch
    position i is the reference prefix up to the anchor and the earlier
    samples of the same branch, h_{b,i} = (x_{<=a_b}, y_{b,<i}).
  * Review §3.2(a): the trunk K/V is computed once and cached; branch
    queries attach to that cache under a tree mask so that each query reads
    only itself and its ancestors; sibling branches and future reference
    tokens are masked; RoPE uses each token's logical position, not its
    packing order.

Readings where the pages are silent (each is one line of the design notes):
  * RoPE: half-split pairing (d, d+D/2), theta_k = base^(-2k/D).
  * Softmax scale 1/sqrt(D); q head h uses kv head h // (Hq/Hkv).
  * The anchor's own trunk token is visible (x_{<=a}); a branch row sees
    itself.  Branch token i sits at position a+i.

Every branch is scored as its own linear sequence, trunk[0..a] followed by
the branch tokens, with textbook causal attention; no tiling, packing or
online softmax.  ``packed_tree_attention`` is a second formulation (one
packed sequence with an explicit dense tree mask) used only to pin
packed == unrolled.

``trunk_prefill`` is the step before the branch pass: the shared prefix
computed once (review §3.2(a): the trunk K/V is computed once and cached;
the aimodeling.com page: the trunk is prefilled once and its branches reuse
it).  Every trunk position of every sequence is a query of plain causal
attention over its own sequence, with RoPE at the trunk position, and the
rotated trunk keys are the K cache the branch pass reads.
"""

from __future__ import annotations

import numpy as np


def rope(x, pos, base: float):
    """Rotate x[n, H, D] (fp64) at positions pos[n]; half-split pairing."""
    x = np.asarray(x, dtype=np.float64)
    D = x.shape[-1]
    half = D // 2
    theta = float(base) ** (-2.0 * np.arange(half, dtype=np.float64) / D)
    ang = np.asarray(pos, dtype=np.float64)[:, None] * theta[None, :]  # [n, half]
    cos = np.cos(ang)[:, None, :]
    sin = np.sin(ang)[:, None, :]
    x1 = x[..., :half]
    x2 = x[..., half:]
    return np.concatenate([x1 * cos - x2 * sin, x2 * cos + x1 * sin], axis=-1)


def softmax_rows(s):
    """exp(s - max) / sum, row-wise, fp64; -inf entries get probability 0."""
    m = np.max(s, axis=-1, keepdims=True)
    e = np.exp(s - m)
    return e / np.sum(e, axis=-1, keepdims=True)


def causal_attention(q, k, v, q_pos, k_pos, scale):
    """Naive causal attention: query at position p sees keys at positions <= p.

    q [nq, D], k [nk, D], v [nk, Dv] (fp64) for one head.
    """
    s = (q @ k.T) * scale
    visible = np.asarray(k_pos)[None, :] <= np.asarray(q_pos)[:, None]
    s = np.where(visible, s, -np.inf)
    return softmax_rows(s) @ v


def branch_attention_unrolled(
    q_br, k_br, v_br, k_tr_raw, v_tr, cu_trunk, anchors, B, W, base,
    scale=None, branches=None,
):
    """Outputs of the branch rows, one unrolled sequence per branch.

    Shapes (any float dtype, computed in fp64):
      q_br [R, Hq, D], k_br/v_br [R, Hkv, D]  (branch rows, not rotated)
      k_tr_raw/v_tr [T_tot, Hkv, D]           (trunk, K NOT rotated)
    Row layout: branch (s,b) owns rows (s*B+b)*(W-1) .. +W-2 (tokens 1..W-1).
    ``branches``: iterable of flat branch ids s*B+b to compute (default all).
    Returns dict {branch_id: out[W-1, Hq, D] fp64}.
    """
    q_br = np.asarray(q_br, dtype=np.float64)
    k_br = np.asarray(k_br, dtype=np.float64)
    v_br = np.asarray(v_br, dtype=np.float64)
    k_tr_raw = np.asarray(k_tr_raw, dtype=np.float64)
    v_tr = np.asarray(v_tr, dtype=np.float64)
    cu = [int(c) for c in cu_trunk]
    S = len(cu) - 1
    Hq, D = q_br.shape[1], q_br.shape[2]
    Hkv = k_br.shape[1]
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    if branches is None:
        branches = range(S * B)
    out = {}
    for bid in branches:
        s, b = divmod(int(bid), B)
        a = int(anchors[bid])
        rows = slice(bid * (W - 1), (bid + 1) * (W - 1))
        # The branch's own linear sequence: x_0..x_a, then y_1..y_{W-1}.
        seq_k = np.concatenate([k_tr_raw[cu[s]: cu[s] + a + 1], k_br[rows]], axis=0)
        seq_v = np.concatenate([v_tr[cu[s]: cu[s] + a + 1], v_br[rows]], axis=0)
        pos = np.arange(a + W, dtype=np.int64)  # logical positions 0..a+W-1
        k_rot = rope(seq_k, pos, base)
        q_pos = pos[a + 1:]                      # branch tokens sit at a+1..a+W-1
        q_rot = rope(q_br[rows], q_pos, base)
        o = np.empty((W - 1, Hq, D), dtype=np.float64)
        for h in range(Hq):
            g = h // G
            o[:, h, :] = causal_attention(q_rot[:, h], k_rot[:, g], seq_v[:, g],
                                          q_pos, pos, scale)
        out[int(bid)] = o
    return out


def branch_attention_unrolled_dense(q_br, k_br, v_br, k_tr_raw, v_tr, cu_trunk,
                                    anchors, B, W, base, scale=None):
    """All branch rows as one array out[R, Hq, D] (fp64)."""
    cu = [int(c) for c in cu_trunk]
    S = len(cu) - 1
    per = branch_attention_unrolled(q_br, k_br, v_br, k_tr_raw, v_tr, cu,
                                    anchors, B, W, base, scale)
    Hq, D = np.shape(q_br)[1], np.shape(q_br)[2]
    out = np.empty((S * B * (W - 1), Hq, D), dtype=np.float64)
    for bid, o in per.items():
        out[bid * (W - 1): (bid + 1) * (W - 1)] = o
    return out


def packed_tree_attention(q_br, k_br, v_br, k_tr_raw, v_tr, parent, sem_pos,
                          T_tot, base, scale=None):
    """Packed formulation: one sequence of T_tot + R nodes with a dense tree
    mask built from the parent map (node m visible to node n iff m is an
    ancestor of n or n itself), RoPE at sem_pos.  Returns out[R, Hq, D] for
    the branch nodes.  Used only to pin packed == unrolled on small inputs.
    """
    q_br = np.asarray(q_br, dtype=np.float64)
    k_all = np.concatenate([np.asarray(k_tr_raw, np.float64),
                            np.asarray(k_br, np.float64)], axis=0)
    v_all = np.concatenate([np.asarray(v_tr, np.float64),
                            np.asarray(v_br, np.float64)], axis=0)
    n_nodes = k_all.shape[0]
    R = q_br.shape[0]
    Hq, D = q_br.shape[1], q_br.shape[2]
    Hkv = k_all.shape[1]
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    mask = np.zeros((R, n_nodes), dtype=bool)
    for r in range(R):
        n = T_tot + r
        while n >= 0:
            mask[r, n] = True
            n = int(parent[n])
    k_rot = rope(k_all, sem_pos, base)
    q_rot = rope(q_br, np.asarray(sem_pos)[T_tot:], base)
    out = np.empty((R, Hq, D), dtype=np.float64)
    for h in range(Hq):
        g = h // G
        s = (q_rot[:, h] @ k_rot[:, g].T) * scale
        s = np.where(mask, s, -np.inf)
        out[:, h, :] = softmax_rows(s) @ v_all[:, g]
    return out


def trunk_prefill(q_tr, k_tr_raw, v_tr, cu_trunk, base, scale=None, rows=None):
    """Causal self-attention over each trunk sequence, with RoPE.

    q_tr [T_tot, Hq, D], k_tr_raw / v_tr [T_tot, Hkv, D] (any float dtype,
    computed in fp64; K not rotated).  Sequence s owns rows
    cu_trunk[s] .. cu_trunk[s+1]-1 at positions 0 .. T_s-1; a query at
    position t sees the keys of its own sequence at positions <= t.
    Returns (out [T_tot, Hq, D], k_cache [T_tot, Hkv, D]), both fp64, where
    k_cache is K rotated at the trunk positions.  With ``rows`` (packed row
    indices), only those rows of ``out`` are computed (the others are NaN),
    each with the same formula over its own visible keys.
    """
    q_tr = np.asarray(q_tr, dtype=np.float64)
    k_tr_raw = np.asarray(k_tr_raw, dtype=np.float64)
    v_tr = np.asarray(v_tr, dtype=np.float64)
    cu = [int(c) for c in cu_trunk]
    Hq, D = q_tr.shape[1], q_tr.shape[2]
    Hkv = k_tr_raw.shape[1]
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    out = np.full_like(q_tr, np.nan)
    k_cache = np.empty_like(k_tr_raw)
    want = None if rows is None else np.asarray(sorted(set(int(r) for r in rows)), dtype=np.int64)
    for s in range(len(cu) - 1):
        seq = slice(cu[s], cu[s + 1])
        pos = np.arange(cu[s + 1] - cu[s], dtype=np.int64)
        k_rot = rope(k_tr_raw[seq], pos, base)
        k_cache[seq] = k_rot
        if want is None:
            sel = pos
        else:
            sel = want[(want >= cu[s]) & (want < cu[s + 1])] - cu[s]
            if sel.size == 0:
                continue
        q_rot = rope(q_tr[seq][sel], sel, base)
        for h in range(Hq):
            g = h // G
            out[cu[s] + sel, h, :] = causal_attention(q_rot[:, h], k_rot[:, g], v_tr[seq, g], sel,
                                                      pos, scale)
    return out, k_cache
