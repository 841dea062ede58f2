"""Gradient of the joint masked attention (oracle).  TEST INFRASTRUCTURE ONLY
-- see the package docstring.

Source (page title, section): "VLA 代码精读 - OpenPI & StarVLA", 1.5
Pi0.compute_loss -- the training step runs the joint forward (the mask built
from the concatenated ar_mask, one attention over the shared KV pool) under
gradient, so training needs the derivative of ``attention.prefill`` with
respect to q, k and v.  The pages print no backward; this is the plain
derivative of the forward, written per (batch element, query head h) with g
the key/value head h reads:

    S  = scale * Q K_g^T,  P = softmax of S over the visible keys of each row
         (a row with no visible key: P = 0),  O = P V_g
    dV_g += P^T dO          dP = dO V_g^T
    dS  = P * (dP - rowsum(P * dP))
    dQ  = scale * dS K_g    dK_g += scale * dS^T Q

(the sums over h run over the query heads that share key/value head g).
"""

from __future__ import annotations

import numpy as np

from .attention import prefill_mask, softmax_probs


def prefill_backward(q, k, v, ar, dout, seg=None, scale=1.0):
    """(dq, dk, dv) in float64 for the joint prefill.

    q, dout [B, S, Hq, d]; k, v [B, S, Hkv, d]; ar [S] or [B, S]; seg as in
    ``attention.prefill`` (negative = padding)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    dout = np.asarray(dout, dtype=np.float64)
    B, S, Hq, d = q.shape
    Hkv = k.shape[2]
    group = Hq // Hkv
    M = prefill_mask(ar, seg=seg, B=B)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(B):
        for h in range(Hq):
            g = h // group
            s = scale * (q[b, :, h] @ k[b, :, g].T)              # [S, S]
            P = softmax_probs(s, M[b])
            dP = dout[b, :, h] @ v[b, :, g].T
            dS = P * (dP - (P * dP).sum(axis=1, keepdims=True))
            dq[b, :, h] = scale * (dS @ k[b, :, g])
            dk[b, :, g] += scale * (dS.T @ q[b, :, h])
            dv[b, :, g] += P.T @ dout[b, :, h]
    return dq, dk, dv
