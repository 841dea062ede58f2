"""The largest sizes the library accepts, against the oracle.

The prefill takes at most 16383 tokens (the 16-bit per-token mask codes); the
suffix pass takes any cache length.  At these sizes the oracle computes a
sample of rows exactly (its ``rows`` argument), chosen so that every part of
the key range and both CTAs of a pair tile are represented.
"""

import numpy as np
import pytest
import torch

import oracle
from vla_prefix_lm_b200 import workloads as W

pytestmark = pytest.mark.gpu

TOL_BF16 = 2e-2
MAX_TOKENS = 16383


def _b():
    from vla_prefix_lm_b200 import binding
    return binding


def _err(got, want):
    return float(np.abs(got.detach().float().cpu().numpy().astype(np.float64) - want).max())


def test_prefill_at_the_token_limit_sampled_rows():
    """S = 16383 (the limit) with a prefix-LM layout: a bidirectional prefix of
    15000 tokens, then a state token and 1382 causal action tokens.  One token
    of every eighth 256-row tile, plus the first and last tokens, all 8 heads."""
    S, Hq, d = MAX_TOKENS, 8, 256
    ar = np.concatenate([np.zeros(15000, np.uint8), W.pi0_suffix_ar(S - 15001)])
    assert ar.shape[0] == S
    q, q64 = W.draw((1, S, Hq, d), 9501, d, "bf16")
    k, k64 = W.draw((1, S, 1, d), 9502, d, "bf16")
    v, v64 = W.draw((1, S, 1, d), 9503, d, "bf16")
    lse = torch.empty((1, S, Hq), dtype=torch.float32, device="cuda")
    out = _b().pi_attn_prefill(q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(ar).cuda(),
                               lse=lse)
    torch.cuda.synchronize()
    assert _b().pi_attn_read_status() == _b().PI_OK
    tok_per_tile = 256 // Hq
    toks = sorted({0, S - 1} | {min(t * tok_per_tile + (11 * t) % tok_per_tile, S - 1)
                                for t in range(0, (S + tok_per_tile - 1) // tok_per_tile, 8)})
    rows = [(0, i) for i in toks]
    ref, ref_lse = oracle.prefill(q64, k64, v64, ar, rows=rows)
    got = torch.stack([out[0, i] for i in toks])
    got_lse = torch.stack([lse[0, i] for i in toks])
    e, el = _err(got, ref), _err(got_lse, ref_lse)
    print(f"S = {S}: {len(toks)} tokens x {Hq} heads, max-abs err out {e:.3e}, lse {el:.3e}")
    assert e <= TOL_BF16
    assert el <= TOL_BF16


@pytest.mark.parametrize("B,P,Sq", [(2, 16000, 1), (1, 16000, 51)])
def test_suffix_against_a_long_cache(B, P, Sq):
    """A cache of 16000 keys: the decode kernel (one token x 8 heads; 1001
    16-key tiles over a cluster of 8 CTAs) and the split-K suffix pass (51
    tokens; the cache split over many SM pairs), every row checked."""
    Hq, d = 8, 256
    ar = W.pi0_suffix_ar(Sq - 1) if Sq > 1 else np.ones(1, np.uint8)
    qs, q64 = W.draw((B, Sq, Hq, d), 9601 + Sq, d, "bf16")
    ks, k64 = W.draw((B, Sq, 1, d), 9602 + Sq, d, "bf16")
    vs, v64 = W.draw((B, Sq, 1, d), 9603 + Sq, d, "bf16")
    kc, kc64 = W.draw((B, P, 1, d), 9604 + Sq, d, "bf16")
    vc, vc64 = W.draw((B, P, 1, d), 9605 + Sq, d, "bf16")
    out = _b().pi_attn_suffix(qs.cuda(), ks.cuda(), vs.cuda(), kc.cuda(), vc.cuda(),
                              torch.from_numpy(ar).cuda())
    torch.cuda.synchronize()
    assert _b().pi_attn_read_status() == _b().PI_OK
    ref, _ = oracle.suffix(q64, k64, v64, kc64, vc64, ar)
    e = _err(out, ref)
    print(f"B = {B}, cache {P}, Sq = {Sq}: max-abs err {e:.3e}")
    assert e <= TOL_BF16
