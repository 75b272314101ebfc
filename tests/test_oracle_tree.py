"""Pins of the oracle's proposal-tree construction (CPU only).

Each test ties oracle.tree to a fact the pages fix: the worked example's
structure (hand-derived fixture), the B(W-1) row count, the analytical row
model's printed figures, and the parent-walk definition of a branch's
history.
"""

import os

import numpy as np
import pytest

from oracle import tree

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_fixture(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *rest = line.split()
            vals[key] = [int(x) for x in rest]
    return vals


def test_worked_example_fixture():
    # Review §3.1 worked example: a six-token reference, anchors at tokens 1 and 3.
    fx = _read_fixture("tree_enjoy_example.txt")
    parent, sem_pos, score_row = tree.tree_build(fx["cu_trunk"], fx["anchors"],
                                                 fx["B"][0], fx["W"][0])
    assert parent.tolist() == fx["parent"]
    assert sem_pos.tolist() == fx["sem_pos"]
    assert score_row.tolist() == fx["score_row"]
    assert tree.counts(fx["S"][0], fx["B"][0], fx["W"][0]) == (fx["R"][0], fx["N"][0])


@pytest.mark.parametrize("S,B,W", [(1, 4, 4), (1, 64, 8), (8, 128, 16), (3, 5, 1), (2, 7, 2)])
def test_b_times_w_minus_1_new_rows(S, B, W):
    # Review §3.2(a) / summary §2.2: B branches add exactly B(W-1) rows.
    rng = np.random.default_rng(S * 100 + B + W)
    T = [int(x) for x in rng.integers(20, 60, size=S)]
    cu = np.concatenate([[0], np.cumsum(T)])
    anchors = np.concatenate([rng.integers(0, t, size=B) for t in T])
    parent, sem_pos, score_row = tree.tree_build(cu, anchors, B, W)
    assert len(parent) - cu[-1] == S * B * (W - 1)
    assert len(score_row) == S * B * W
    # Every supervised position reads a distinct row and no row reads the
    # token it scores: the row scoring token i is the node of token i-1.
    assert np.all(score_row >= 0)


def test_analytical_row_model_printed_figures():
    # Review §3.4: L=2048, W=7, K=512 -> 5,120 shared rows and 529,664
    # cacheless rows (ratio 103.45x) for a uniform batch of anchors.
    assert tree.shared_rows(2048, 512, 7) == 5120
    # Uniform anchors on [8, 2047] (mean 1027.5), rounded in symmetric pairs so
    # the mean stays exact.
    x = np.linspace(8, 2047, 512)
    a = np.floor(x[:256] + 0.5).astype(np.int64)
    anchors = np.concatenate([a, (2055 - a)[::-1]])
    assert anchors.min() >= 8 and anchors.max() <= 2047
    assert tree.cacheless_rows(anchors, 7) == 529664
    assert round(529664 / 5120, 2) == 103.45


def _branch_history_by_definition(cu, anchors, B, W, s, b, i):
    """Review §3.1: h_{b,i} = (x_{<=a_b}, y_{b,<=i}) as packed node ids."""
    T_tot = cu[-1]
    a = anchors[s * B + b]
    trunk = list(range(cu[s], cu[s] + a + 1))
    first = T_tot + (s * B + b) * (W - 1)
    return trunk + [first + k for k in range(i)]


def test_parent_walk_is_branch_history():
    # Summary §2.1: walking parents from branch node (s,b,i) visits exactly the
    # trunk up to the anchor and the branch's earlier tokens.
    rng = np.random.default_rng(7)
    S, B, W = 3, 5, 5
    T = [17, 1, 30]
    cu = [0] + list(np.cumsum(T))
    anchors = [int(rng.integers(0, t)) for t in T for _ in range(B)]
    anchors[0] = 0
    anchors[B * 2 + 1] = T[2] - 1  # anchor at the last trunk token
    anchors[B * 2 + 2] = anchors[B * 2 + 3]  # duplicate anchors
    parent, sem_pos, _ = tree.tree_build(cu, anchors, B, W)
    for s in range(S):
        for b in range(B):
            for i in range(1, W):
                node = cu[-1] + (s * B + b) * (W - 1) + (i - 1)
                assert tree.ancestors(parent, node) == _branch_history_by_definition(
                    cu, anchors, B, W, s, b, i)
                # semantic position = anchor position + offset
                assert sem_pos[node] == anchors[s * B + b] + i


def test_single_token_branch_adds_no_rows():
    parent, sem_pos, score_row = tree.tree_build([0, 10], [3, 9], 2, 1)
    assert len(parent) == 10
    assert score_row.tolist() == [3, 9]  # token 1 is scored by the anchor row


def test_anchor_out_of_range_rejected():
    with pytest.raises(ValueError):
        tree.tree_build([0, 10], [10], 1, 3)
