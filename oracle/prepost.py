"""Plain float64 definitions of the steps on either side of the attention
(oracle).  TEST INFRASTRUCTURE ONLY -- see the package docstring.

Sources (page title, section):

* "VLA 代码精读 - OpenPI & StarVLA", 1.6 Pi0.sample_actions: the prefix tokens
  get positions cumsum(prefix_mask) - 1; each Euler step's suffix tokens get
  sum(prefix_mask) + cumsum(suffix_mask) - 1 (their positions continue after
  the valid prefix tokens); the step is x <- x + dt * v with dt = -1 / steps,
  from t = 1 (noise) to t = 0.  The same page's 1.5 Pi0.compute_loss gives the
  joint positions cumsum(input_mask) - 1.
* same page, comparison table ("位置编码"): pi0 uses the LLM's built-in RoPE.

Reading taken (the pages give no RoPE formula): the standard rotary embedding
on pairs (i, i + d/2) of each head vector, angle pos * base^(-2i/d) with base
10000 -- for x1 = x[:d/2], x2 = x[d/2:]:
    out = [x1 cos - x2 sin, x2 cos + x1 sin].
"""

from __future__ import annotations

import numpy as np


def positions(token_mask, prefix_mask=None):
    """[B, S] int64 positions: cumsum(token_mask) - 1, offset by the number of
    valid prefix tokens when ``prefix_mask`` ([B, P]) is given."""
    m = np.asarray(token_mask) != 0
    pos = np.cumsum(m, axis=-1, dtype=np.int64) - 1
    if prefix_mask is not None:
        pos = pos + (np.asarray(prefix_mask) != 0).sum(axis=-1, dtype=np.int64)[:, None]
    return pos


def rope(x, pos, base=10000.0):
    """Rotary embedding of x [B, S, H, d] at positions pos [B, S], in float64."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    half = d // 2
    inv = base ** (-2.0 * np.arange(half, dtype=np.float64) / d)        # [d/2]
    ang = np.asarray(pos, dtype=np.float64)[:, :, None, None] * inv     # [B, S, 1, d/2]
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def euler_step(x, v, dt):
    """One Euler step of the flow-matching ODE: x + dt * v (float64)."""
    return np.asarray(x, dtype=np.float64) + dt * np.asarray(v, dtype=np.float64)
