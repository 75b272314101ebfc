"""Plain, slow, fp64 CPU oracle of the SpecOPD branch-scoring pass.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import or run it.  It shares no
code with the CUDA path (no kernels, headers, helpers or tables); both sides
only consume the same seeded inputs from ``synth``.

What it computes, and from which passage (pages on arXiv 2611.02846):

* ``oracle.tree``       -- proposal tree: parent map, semantic positions and
  the score-row map.  SpecOPD review (jaehun.me) §3.1 and §3.2(a) "score-row
  reading rule"; paper summary (rustineverything.app) §2.1 and §2.2.
* ``oracle.attention``  -- branch scoring under full (GQA) attention.  Each
  branch is UNROLLED into its own linear sequence (reference prefix up to the
  anchor, then the branch tokens) and run through naive causal softmax
  attention with RoPE at logical positions.  Review §3.1 (the condition of
  position i), §3.2(a) (tree mask: each query reads itself and its
  ancestors; RoPE uses logical positions).  A second, independent packed
  formulation with an explicit dense tree mask is provided for the
  packed == unrolled pin.
* ``oracle.tv``         -- E2E-TV: overlap a = sum min(p, q) = 1 - TV,
  prefix products, loss 1 - mean prefix product, closed-form gradient with
  respect to the draft logits.  Review §1.1 and §3.3; summary §2.3.
* ``oracle.lmhead``     -- the same E2E-TV with the logits formed from hidden
  rows through the target's and the drafter's LM heads (z = W h), target
  rows gathered by the score-row map.  Review §3.2(a) (score-row reading
  rule) and §3.3.

Parity pins (tests/test_oracle_*.py, run with ``-m "not gpu"``) tie every
function to facts the pages or mathematics fix; see those tests.  Parity
unpinned: none of the functions here (the only unpinned figure of the pages,
the 69.2x attention-pair ratio, is not computed by the oracle).
"""

from . import attention, lmhead, tree, tv  # noqa: F401

__all__ = ["attention", "lmhead", "tree", "tv"]
