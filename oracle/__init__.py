"""CPU oracle for the pi0 / pi0.5 joint (prefix-LM) attention.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
(and its ``--impl reference`` arm) may call it.  It shares no code with the CUDA
library under ``vla_prefix_lm_b200/csrc`` and imports nothing from the product
package.

Everything is plain numpy in float64: the visibility mask is built explicitly
as a boolean matrix from the pages' rule, the scores are a plain matrix
product, and the softmax is the textbook definition.  See ``attention.py`` for
the joint prefill / suffix-pass attention, ``brute.py`` for an independent
per-pair visibility enumerator, and ``counts.py`` for the attention-pair
counting convention.

Parity status per function (what pins it; tests live in tests/test_oracle.py):

* ``prefill_mask`` / ``suffix_mask`` -- pinned: the Pi0-FAST mask picture
  (golden file), the pi0.5 five-row permission table (golden file), the
  all-False / all-True special cases, and exhaustive agreement with the
  independent ``brute.visible`` if-chain on every ar pattern up to S = 10.
* ``attention`` / ``prefill`` / ``suffix`` -- pinned: closed forms (q = 0 gives
  the mean of the visible values; a single visible key returns its value row),
  invariances (duplicated heads, key permutation inside a bidirectional
  block), equality with torch's scaled_dot_product_attention in float64, the
  log-sum-exp against scipy, and suffix-pass == prefill suffix rows.
* ``backward.prefill_backward`` -- pinned: central finite differences of
  ``prefill`` on tiny inputs (every element of dq, dk, dv), torch autograd
  through float64 scaled_dot_product_attention with the oracle's mask, and the
  closed forms sum_j dK_j = 0 (softmax is shift-invariant in the keys) and
  sum_j dV_j = sum of dO over the rows that see a key.
* ``prepost.positions`` / ``rope`` / ``euler_step`` -- pinned: a worked
  positions example with padding and a padded prefix, RoPE's closed forms
  (identity at 0, pair norms kept, a stated turn of pairs 0 and 4), the
  relative-position property, and the Euler loop against the exact solution.
* ``counts.full_pairs`` / ``visible_pairs`` -- pinned: the pages' worked
  counts (480^2 = 230,400 fused scores, 32 x 448 cross scores, 28 x 4250^2
  MM-DiT pairs) and the number of True entries of the explicit masks.
"""

from .attention import (  # noqa: F401
    EXPERT,
    FAST,
    OTHER,
    ar_cumsum,
    attention,
    prefill,
    prefill_mask,
    softmax_probs,
    suffix,
    suffix_mask,
)
from . import backward, brute, counts, prepost  # noqa: F401
