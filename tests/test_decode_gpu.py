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


def test_bf16_decode_bench_shape_full():
    """The bench's decode step in full: B=32, one token x 8 heads against an
    880-token cache (every row compared), with a garbage-filled workspace."""
    B, P, Hq, d = 32, 880, 8, 256
    ar = np.array([1], np.uint8)
    q, q64 = W.draw((B, 1, Hq, d), 531, d, "bf16")
    k, k64 = W.draw((B, 1, 1, d), 532, d, "bf16")
    v, v64 = W.draw((B, 1, 1, d), 533, d, "bf16")
    kc, kc64 = W.draw((B, P, 1, d), 534, d, "bf16")
    vc, vc64 = W.draw((B, P, 1, d), 535, d, "bf16")
    b = _b()
    args = (q.cuda(), k.cuda(), v.cuda(), kc.cuda(), vc.cuda(), torch.from_numpy(ar).cuda())
    need = b.pi_attn_suffix_workspace_bytes(args[0], args[1], args[3], args[5])
    ws = torch.full((need,), 255, dtype=torch.uint8, device="cuda")
    out = b.pi_attn_suffix(*args, workspace=ws)
    ref, _ = oracle.suffix(q64, k64, v64, kc64, vc64, ar)
    err = float(np.abs(out.float().cpu().numpy() - ref).max())
    print(f"decode B=32 P=880 max-abs err {err:.3e}")
    assert err <= TOL_BF16, err


@pytest.mark.parametrize("Sq,Hq,P", [(2, 4, 130), (4, 2, 64), (8, 1, 700), (1, 4, 0), (3, 2, 65)])
def test_bf16_few_rows_suffix_with_block_mask(Sq, Hq, P):
    """Suffixes of up to 8 query rows (Sq x Hq): the cached keys are visible to
    every row, the suffix keys by the block-index rule over the suffix alone."""
    B, d = 3, 256
    rng = np.random.default_rng(Sq * 10 + Hq + P)
    ar = (rng.random(Sq) < 0.5).astype(np.uint8)
    ar[0] = 1
    q, q64 = W.draw((B, Sq, Hq, d), 541, d, "bf16")
    k, k64 = W.draw((B, Sq, 1, d), 542, d, "bf16")
    v, v64 = W.draw((B, Sq, 1, d), 543, d, "bf16")
    kc, kc64 = W.draw((B, P, 1, d), 544, d, "bf16")
    vc, vc64 = W.draw((B, P, 1, d), 545, d, "bf16")
    out = _b().pi_attn_suffix(q.cuda(), k.cuda(), v.cuda(), kc.cuda() if P else None,
                              vc.cuda() if P else None, torch.from_numpy(ar).cuda(),
                              softmax_scale=0.8)
    ref, _ = oracle.suffix(q64, k64, v64, kc64, vc64, ar, scale=0.8)
    err = float(np.abs(out.float().cpu().numpy() - ref).max())
    assert err <= TOL_BF16, err


@pytest.mark.parametrize("Sq,Hq", [(1, 8), (2, 4)])
def test_bf16_decode_padding_and_segments(Sq, Hq):
    """Few-row suffix with a per-batch cache validity mask (one element with no
    valid cached key) and suffix segment ids (FAST / expert tags, a padded
    token): padded rows write 0."""
    B, P, d = 4, 333, 256
    rng = np.random.default_rng(Sq + 70)
    ar = np.ones(Sq, np.uint8)
    q, q64 = W.draw((B, Sq, Hq, d), 551, d, "bf16")
    k, k64 = W.draw((B, Sq, 1, d), 552, d, "bf16")
    v, v64 = W.draw((B, Sq, 1, d), 553, d, "bf16")
    kc, kc64 = W.draw((B, P, 1, d), 554, d, "bf16")
    vc, vc64 = W.draw((B, P, 1, d), 555, d, "bf16")
    valid = (rng.random((B, P)) < 0.6).astype(np.uint8)
    valid[1, :] = 0
    seg = np.zeros((B, Sq), np.int32)
    seg[:, 0] = 1                     # FAST
    if Sq > 1:
        seg[:, 1] = 2                 # expert: hides the FAST key
        seg[2, 1] = -1                # a padded token
    out = _b().pi_attn_suffix(q.cuda(), k.cuda(), v.cuda(), kc.cuda(), vc.cuda(),
                              torch.from_numpy(np.tile(ar, (B, 1))).cuda(),
                              segment_ids=torch.from_numpy(seg).cuda(),
                              cache_valid=torch.from_numpy(valid).cuda())
    ref, _ = oracle.suffix(q64, k64, v64, kc64, vc64, np.tile(ar, (B, 1)), seg_suf=seg,
                           cache_valid=valid)
    got = out.float().cpu().numpy()
    err = float(np.abs(got - ref).max())
    assert err <= TOL_BF16, err
    assert np.all(got[seg < 0] == 0)
