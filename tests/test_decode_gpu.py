"""Single-token decode against a growing cache.

"Pi0-FAST 模型架构", 4.1 KV 缓存推理: after the prefix, FAST action tokens are
decoded one at a time, each attending to the whole cache plus itself, and the
cache grows by one token per step.  This is the suffix-only call with Sq = 1
(one query token, its own key and value, ar_mask = [True]) against a cache of
P tokens; the caller appends the token's K/V to the cache between steps.
Checked against the oracle at every step of a short growing-cache loop, and
at single-token shapes that span several 128-key tiles with ragged tails.
"""

import numpy as np
import pytest
import torch

import oracle
from vla_prefix_lm_b200 import workloads as W

pytestmark = pytest.mark.gpu

TOL_BF16 = 2e-2


def _b():
    from vla_prefix_lm_b200 import binding
    return binding


@pytest.mark.parametrize("B,P", [(1, 1), (1, 127), (1, 128), (4, 1000), (2, 2047), (16, 300)])
def test_bf16_single_token_decode(B, P):
    Hq, d = 8, 256
    ar = np.array([1], np.uint8)
    q, q64 = W.draw((B, 1, Hq, d), 501, d, "bf16")
    k, k64 = W.draw((B, 1, 1, d), 502, d, "bf16")
    v, v64 = W.draw((B, 1, 1, d), 503, d, "bf16")
    kc, kc64 = W.draw((B, P, 1, d), 504, d, "bf16")
    vc, vc64 = W.draw((B, P, 1, d), 505, d, "bf16")
    out = _b().pi_attn_suffix(q.cuda(), k.cuda(), v.cuda(), kc.cuda(), vc.cuda(),
                              torch.from_numpy(ar).cuda())
    ref, _ = oracle.suffix(q64, k64, v64, kc64, vc64, ar)
    err = float(np.abs(out.float().cpu().numpy() - ref).max())
    assert err <= TOL_BF16, err
    assert _b().pi_attn_read_status() == _b().PI_OK


def test_bf16_decode_growing_cache():
    """Five decode steps; each appends the step's K/V to the cache."""
    B, P0, Hq, d = 2, 200, 8, 256
    ar = torch.ones(1, dtype=torch.uint8, device="cuda")
    kc, kc64 = W.draw((B, P0, 1, d), 511, d, "bf16")
    vc, vc64 = W.draw((B, P0, 1, d), 512, d, "bf16")
    kc, vc = kc.cuda(), vc.cuda()
    for step in range(5):
        q, q64 = W.draw((B, 1, Hq, d), 520 + 3 * step, d, "bf16")
        k, k64 = W.draw((B, 1, 1, d), 521 + 3 * step, d, "bf16")
        v, v64 = W.draw((B, 1, 1, d), 522 + 3 * step, d, "bf16")
        out = _b().pi_attn_suffix(q.cuda(), k.cuda(), v.cuda(), kc, vc, ar)
        ref, _ = oracle.suffix(q64, k64, v64, kc64, vc64, np.array([1], np.uint8))
        err = float(np.abs(out.float().cpu().numpy() - ref).max())
        assert err <= TOL_BF16, (step, err)
        kc = torch.cat([kc, k.cuda()], dim=1).contiguous()
        vc = torch.cat([vc, v.cuda()], dim=1).contiguous()
        kc64 = np.concatenate([kc64, k64], axis=1)
        vc64 = np.concatenate([vc64, v64], axis=1)
