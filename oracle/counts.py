"""Attention-pair counting (oracle side).

TEST INFRASTRUCTURE ONLY.  Two conventions:

* ``full_pairs(S)`` -- every query scores every key: S * S.  This is how
  "08-vla-architectures", section 7 架构量级手算 (例 3) counts a fused
  480-token sequence (480^2 = 230,400 scores) and how "π0.5 vs MM-DiT joint
  attention", section 对照与代价, counts 28 MM-DiT steps over 4096 + 154 tokens.
* ``visible_pairs(M)`` -- the number of True entries of an explicit mask; the
  unit in which the library reports throughput (unmasked pairs per second),
  per (batch, query head).
"""

from __future__ import annotations

import numpy as np


def full_pairs(Sq, Sk=None):
    return int(Sq) * int(Sq if Sk is None else Sk)


def visible_pairs(M):
    return int(np.count_nonzero(np.asarray(M)))

