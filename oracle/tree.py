"""Proposal-tree construction, written out from the definitions.

Oracle (test infrastructure only; see ``oracle/__init__.py``).

Sources:
  * SpecOPD review (jaehun.me) §3.1: the trunk is the reference (prompt plus
    response); anchors are positions of the response; a branch is the W
    tokens the drafter continues with after an anchor; branches are attached
    to their anchors to form a tree.
  * Paper summary (rustineverything.app) §2.1: the first branch token's
    parent is the anchor token, each later token's parent is the previously
    sampled token; the semantic position is the anchor position plus the
    offset.
  * Review §3.2(a) and §3.4, summary §2.2: the anchor row scores the first
    branch token and each branch row scores the next token; the last sample
    gets no row, so B branches add B(W-1) rows after the shared trunk.

Packed node order (a layout choice of this library, the pages fix none):
trunk nodes ``cu_trunk[s] + j``; branch node (s, b, i), i = 1..W-1, at
``T_tot + (s*B + b)*(W-1) + (i-1)``.  Supervised position (s, b, i),
i = 1..W, at ``(s*B + b)*W + (i-1)``.
"""

from __future__ import annotations

import numpy as np


def counts(S: int, B: int, W: int) -> tuple[int, int]:
    """(R, N): new scoring rows R = S*B*(W-1) and supervised positions N = S*B*W."""
    return S * B * (W - 1), S * B * W


def tree_build(cu_trunk, anchors, B: int, W: int):
    """Parent map, semantic positions and score-row map of the packed tree.

    cu_trunk: int[S+1] prefix sums of trunk lengths; anchors: int[S*B] local
    positions.  Returns int64 arrays (parent[T_tot+R], sem_pos[T_tot+R],
    score_row[S*B*W]).  Raises ValueError for an anchor outside its trunk.
    """
    cu = [int(x) for x in cu_trunk]
    anchors = [int(x) for x in anchors]
    S = len(cu) - 1
    T_tot = cu[-1]
    R, N = counts(S, B, W)
    if len(anchors) != S * B:
        raise ValueError("anchors must have S*B entries")
    parent = np.full(T_tot + R, -2, dtype=np.int64)
    sem_pos = np.full(T_tot + R, -2, dtype=np.int64)
    score_row = np.full(N, -2, dtype=np.int64)

    # Trunk: a plain causal chain per sequence.
    for s in range(S):
        for j in range(cu[s + 1] - cu[s]):
            n = cu[s] + j
            parent[n] = n - 1 if j > 0 else -1
            sem_pos[n] = j

    # Branches: one chain per anchor, hanging off the anchor's trunk node.
    for s in range(S):
        T_s = cu[s + 1] - cu[s]
        for b in range(B):
            a = anchors[s * B + b]
            if not (0 <= a < T_s):
                raise ValueError(f"anchor {a} outside trunk of length {T_s}")
            anchor_node = cu[s] + a
            first = T_tot + (s * B + b) * (W - 1)  # node of branch token i=1
            for i in range(1, W):
                node = first + (i - 1)
                parent[node] = anchor_node if i == 1 else node - 1
                sem_pos[node] = a + i
            for i in range(1, W + 1):
                # Token i is scored by the output of its predecessor's row.
                score_row[(s * B + b) * W + (i - 1)] = (
                    anchor_node if i == 1 else first + (i - 2)
                )
    return parent, sem_pos, score_row


def ancestors(parent, node: int) -> list[int]:
    """Nodes on the path root -> node (inclusive), by walking the parent map."""
    path = []
    n = int(node)
    while n >= 0:
        path.append(n)
        n = int(parent[n])
    return path[::-1]


def shared_rows(L: int, K: int, W: int) -> int:
    """Rows a shared-prefix pass computes: the trunk once plus K(W-1) branch rows.

    Review §3.4 (with P = W-1 new score rows per branch).
    """
    return L + K * (W - 1)


def cacheless_rows(anchors, W: int) -> int:
    """Rows independent cacheless scoring computes: each branch re-runs its
    prefix x_{<=a} plus its W-1 scored branch rows, i.e. (a+1) + (W-1) = a+W.

    Review §3.4 (the cacheless side of the row-count comparison).
    """
    return int(sum(int(a) + W for a in anchors))
