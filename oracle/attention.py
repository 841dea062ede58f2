"""Plain float64 definition of the pi0 / pi0.5 joint attention (oracle).

TEST INFRASTRUCTURE ONLY -- see the package docstring.  No blocking, no
online softmax, no fusion: the mask is an explicit boolean matrix and every
row's softmax is computed from its full score vector.

Sources (page title, section):

* "VLA 代码精读 - OpenPI & StarVLA", 1.2 原理与公式, "Prefix-Suffix 注意力掩码":
  ar_mask False means a token shares attention with the tokens before it;
  True means the tokens before it cannot see it.
* "π0.5 vs MM-DiT joint attention", section "π0.5:三段,两处看不到": make_attn_mask
  is the one-line rule cumsum(ar)_j <= cumsum(ar)_i, and the permission table,
  whose last row forbids expert queries from reading FAST keys.
* same page, "joint attention 只管算子,mask 才管权限": per-expert q, k, v are
  concatenated along the token axis into one pool and one softmax runs over it;
  8 query heads share 1 KV head, head_dim 256.
* "VLA 代码精读 - OpenPI & StarVLA", 1.6 Pi0.sample_actions: the suffix-only pass
  concatenates a key mask that shows every prefix key to every suffix query with
  make_attn_mask over the suffix alone; the prefix KV cache is read, not
  appended.

Conventions (readings the pages leave open):

* Row index i is the query, column index j is the key.
* q is [B, Sq, Hq, d]; k, v are [B, Sk, Hkv, d]; query head h reads KV head
  h // (Hq // Hkv).
* ``scale`` multiplies the dot product before the softmax (the pages never state
  it; the workloads fold 1/sqrt(d) into q and k and use scale = 1).
* ``lse`` is the natural-log log-sum-exp of the scaled, visible scores.
* Padding (not in the pages' workloads; openpi and Pi0-FAST AND a per-token
  validity mask into the attention mask): a negative segment id marks a
  padding token.  A padding key is visible to no query and a padding query
  sees no key.  A query row with no visible key outputs 0 with lse = -inf.
  In the suffix pass a per-batch ``cache_valid`` mask hides padded prefix keys.
"""

from __future__ import annotations

import numpy as np

# segment ids: the tag of each token for pi0.5's extra rule.
OTHER = 0   # prefix (image patches, text, discrete state) or anything else
FAST = 1    # FAST discrete action tokens
EXPERT = 2  # the action expert's continuous chunk
PAD = -1    # any negative id: a padding token


def _as_batched(x, B, name):
    x = np.asarray(x)
    if x.ndim == 1:
        x = np.broadcast_to(x, (B, x.shape[0]))
    if x.ndim != 2 or x.shape[0] != B:
        raise ValueError(f"{name} must be [S] or [B, S], got {x.shape}")
    return x


def ar_cumsum(ar):
    """cumsum over the token axis of the boolean ar_mask, as int64.

    "π0.5 vs MM-DiT joint attention", "π0.5:三段,两处看不到": the block index
    of a token is the running count of True entries up to and including it.
    """
    ar = np.asarray(ar)
    return np.cumsum(ar != 0, axis=-1, dtype=np.int64)


def prefill_mask(ar, seg=None, B=None, rows=None):
    """Explicit [B, S, S] boolean visibility matrix of the joint prefill.

    M[b, i, j] = cumsum(ar)[j] <= cumsum(ar)[i]            (the cumsum rule)
                 and not (seg[i] == EXPERT and seg[j] == FAST)
                                                   (pi0.5's 'expert <- FAST' row)

    ``ar`` and ``seg`` are [S] (shared by the batch) or [B, S].  ``B`` sets the
    batch when both are 1-D (default 1).  ``rows`` (a list of query indices)
    returns only those rows, [B, len(rows), S], for sequences too long to hold
    the full matrix.
    """
    ar = np.asarray(ar)
    if B is None:
        B = ar.shape[0] if ar.ndim == 2 else 1
    ar = _as_batched(ar, B, "ar")
    cs = ar_cumsum(ar)                                   # [B, S]
    qi = np.arange(cs.shape[1]) if rows is None else np.asarray(rows)
    M = cs[:, None, :] <= cs[:, qi, None]                # [B, i, j]
    if seg is not None:
        seg = _as_batched(seg, B, "seg")
        forbid = (seg[:, qi, None] == EXPERT) & (seg[:, None, :] == FAST)
        M = M & ~forbid
        valid = seg >= 0                                 # padding: negative ids
        M = M & valid[:, qi, None] & valid[:, None, :]
    return M


def suffix_mask(ar_suf, P, B=None, seg_suf=None, cache_valid=None):
    """[B, Sq, P + Sq] visibility of the suffix-only pass against a P-token cache.

    "VLA 代码精读 - OpenPI & StarVLA", 1.6: every suffix query sees every (valid)
    prefix key -- the prefix mask repeated over the suffix rows -- concatenated
    on the key axis with make_attn_mask over the suffix tokens alone.
    ``cache_valid`` ([P] or [B, P], nonzero = valid) hides padded prefix keys;
    ``seg_suf`` tags the suffix tokens as in ``prefill_mask`` (negative =
    padding).
    """
    ar_suf = np.asarray(ar_suf)
    if B is None:
        B = ar_suf.shape[0] if ar_suf.ndim == 2 else 1
    Msuf = prefill_mask(ar_suf, seg_suf, B=B)            # [B, Sq, Sq]
    Sq = Msuf.shape[1]
    pre = np.ones((B, Sq, P), dtype=bool)
    if cache_valid is not None:
        cv = _as_batched(np.asarray(cache_valid) != 0, B, "cache_valid")
        pre = pre & cv[:, None, :]
    if seg_suf is not None:
        vq = _as_batched(seg_suf, B, "seg_suf") >= 0
        pre = pre & vq[:, :, None]
    return np.concatenate([pre, Msuf], axis=2)


def softmax_probs(s, M):
    """Row softmax of the scores ``s`` restricted to the visible entries ``M``.

    Masked entries get probability exactly 0.  A row with no visible entry (a
    padding query) has all probabilities 0.
    """
    s = np.where(M, s, -np.inf)
    m = s.max(axis=-1, keepdims=True)
    empty = ~np.isfinite(m)
    e = np.exp(s - np.where(empty, 0.0, m))
    den = e.sum(axis=-1, keepdims=True)
    return np.where(empty, 0.0, e / np.where(empty, 1.0, den))


def attention(q, k, v, M, scale=1.0, rows=None):
    """Masked grouped-query attention over one shared KV pool.

    q [B, Sq, Hq, d], k/v [B, Sk, Hkv, d], M [B, Sq, Sk] bool.
    Returns (out [B, Sq, Hq, d], lse [B, Sq, Hq]) in float64.

    ``rows`` optionally restricts the computation to a list of (b, i) query
    rows; the returned arrays then hold only those rows in that order
    (out [R, Hq, d], lse [R, Hq]).  Each row's result is the same per-row
    definition either way.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, Sq, Hq, d = q.shape
    Hkv = k.shape[2]
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    group = Hq // Hkv

    def one_row(b, i):
        o = np.empty((Hq, d))
        lse = np.empty(Hq)
        for h in range(Hq):
            kv = h // group
            s = scale * (k[b, :, kv, :] @ q[b, i, h, :])           # [Sk]
            p = softmax_probs(s[None, :], M[b, i][None, :])[0]
            o[h] = p @ v[b, :, kv, :]
            vis = s[M[b, i]]
            if vis.size == 0:
                lse[h] = -np.inf
                continue
            mx = vis.max()
            lse[h] = mx + np.log(np.exp(vis - mx).sum())
        return o, lse

    if rows is not None:
        outs, lses = zip(*(one_row(b, i) for (b, i) in rows)) if len(rows) else ((), ())
        return (np.array(outs).reshape(len(rows), Hq, d),
                np.array(lses).reshape(len(rows), Hq))

    out = np.empty((B, Sq, Hq, d))
    lse = np.empty((B, Sq, Hq))
    for b in range(B):
        for h in range(Hq):
            kv = h // group
            s = scale * (q[b, :, h, :] @ k[b, :, kv, :].T)          # [Sq, Sk]
            p = softmax_probs(s, M[b])
            out[b, :, h, :] = p @ v[b, :, kv, :]
            sm = np.where(M[b], s, -np.inf)
            mx = sm.max(axis=-1, keepdims=True)
            empty = ~np.isfinite(mx)
            mxf = np.where(empty, 0.0, mx)
            with np.errstate(divide="ignore"):
                lse_b = mxf + np.log(np.exp(sm - mxf).sum(axis=-1, keepdims=True))
            lse[b, :, h] = np.where(empty, -np.inf, lse_b)[:, 0]
    return out, lse


def prefill(q, k, v, ar, seg=None, scale=1.0, rows=None):
    """Joint prefill over [prefix, suffix] with the explicit prefix-LM mask.

    "VLA 代码精读 - OpenPI & StarVLA", 1.5 Pi0.compute_loss (one forward over the
    concatenated tokens with make_attn_mask), masked as in ``prefill_mask``.
    """
    B = q.shape[0]
    M = prefill_mask(ar, seg, B=B)
    return attention(q, k, v, M, scale, rows)


def suffix(q_suf, k_suf, v_suf, k_cache, v_cache, ar_suf, scale=1.0, rows=None,
           seg_suf=None, cache_valid=None):
    """Suffix-only pass: suffix queries against [prefix cache, suffix] keys.

    "VLA 代码精读 - OpenPI & StarVLA", 1.6 Pi0.sample_actions: the keys are the
    cached prefix keys followed by this step's suffix keys; the cache is not
    extended.  ``seg_suf`` / ``cache_valid`` add padding as in ``suffix_mask``.
    """
    B = q_suf.shape[0]
    P = np.asarray(k_cache).shape[1]
    M = suffix_mask(ar_suf, P, B=B, seg_suf=seg_suf, cache_valid=cache_valid)
    k = np.concatenate([np.asarray(k_cache, np.float64), np.asarray(k_suf, np.float64)], axis=1)
    v = np.concatenate([np.asarray(v_cache, np.float64), np.asarray(v_suf, np.float64)], axis=1)
    return attention(q_suf, k, v, M, scale, rows)
