"""Independent per-pair visibility enumerator (oracle cross-check).

TEST INFRASTRUCTURE ONLY.  Decides each (query i, key j) with an if-chain over
the pages' wording instead of the cumsum rule, so that agreement with
``attention.prefill_mask`` on every small ar pattern pins the rule's direction,
its <= and its segment term.

Sources (page title, section):

* "VLA 代码精读 - OpenPI & StarVLA", 1.2 "Prefix-Suffix 注意力掩码": a True
  ar_mask entry is a causal boundary -- the tokens before it cannot see it (nor,
  since it starts a new block, anything after it); False tokens share
  attention with the tokens before them.
* "π0.5 vs MM-DiT joint attention", permission table: expert queries never read
  FAST keys; every other row follows the block structure.
* Padding (negative segment id): a padding token is neither read nor reads.
"""

from __future__ import annotations

from .attention import EXPERT, FAST


def visible(i, j, ar, seg=None):
    """True iff key j is visible to query i, by walking the boundaries.

    A key at or before the query is always readable (a block sees every earlier
    block and itself).  A key after the query is readable only if no causal
    boundary (a True ar entry) lies in (i, j]: the key is then in the query's
    own bidirectional block.
    """
    if seg is not None and (seg[i] < 0 or seg[j] < 0):
        return False
    if seg is not None and seg[i] == EXPERT and seg[j] == FAST:
        return False
    if j <= i:
        return True
    for t in range(i + 1, j + 1):
        if ar[t]:
            return False
    return True


def mask(ar, seg=None):
    """S x S list-of-lists mask built pair by pair with ``visible``."""
    S = len(ar)
    return [[visible(i, j, ar, seg) for j in range(S)] for i in range(S)]


def attention_row(q_row, keys, values, vis, scale=1.0):
    """One query head's output by explicit loops (tiny inputs only).

    q_row [d], keys/values [Sk][d] as nested sequences, vis [Sk] booleans.
    Uses math.exp over the visible scores after subtracting their maximum.
    """
    import math

    scores = []
    for j, kj in enumerate(keys):
        if vis[j]:
            scores.append((j, scale * sum(a * b for a, b in zip(q_row, kj))))
    if not scores:                 # a padding query: no visible key
        return [0.0] * len(q_row)
    mx = max(s for _, s in scores)
    w = [(j, math.exp(s - mx)) for j, s in scores]
    den = sum(x for _, x in w)
    d = len(q_row)
    return [sum(x * values[j][c] for j, x in w) / den for c in range(d)]
