"""Padding (a negative segment id; a per-batch validity mask for cached prefix
keys) on the GPU path vs the oracle, element by element.

The oracle's padding semantics are pinned in test_oracle.py (a padded token
behaves as if absent; a row that sees no key is 0 with lse = -inf).  Here the
CUDA kernels must match it: bf16 within 2e-2, fp32 within 1e-4, padding rows
exactly 0, and the debug mask bit for bit.
"""

import numpy as np
import pytest
import torch

import oracle
from vla_prefix_lm_b200 import workloads as W

pytestmark = pytest.mark.gpu

TOL_BF16 = 2e-2
TOL_F32 = 1e-4


def _b():
    from vla_prefix_lm_b200 import binding
    return binding


def _inputs(B, S, Hq, d, dtype, seed, P=0):
    q, q64 = W.draw((B, S, Hq, d), seed, d, dtype)
    k, k64 = W.draw((B, S, 1, d), seed + 1, d, dtype)
    v, v64 = W.draw((B, S, 1, d), seed + 2, d, dtype)
    return q, q64, k, k64, v, v64


def _layout(rng, B, S, shared, with_fast=False):
    ar = (rng.random(S) < 0.08).astype(np.uint8)
    if with_fast:
        seg = rng.choice([0, 1, 2], size=(B, S), p=[0.6, 0.2, 0.2])
    else:
        seg = np.zeros((B, S), np.int32)
    pad = rng.random((B, S)) < 0.2
    seg = np.where(pad, -1, seg).astype(np.int32)
    if shared:
        seg = seg[:1].copy()
    return ar, seg


def _check(out, ref, seg, tol):
    o = out.float().cpu().numpy().astype(np.float64)
    err = float(np.abs(o - ref).max())
    assert err <= tol, err
    padrows = np.broadcast_to(seg < 0, o.shape[:2])
    assert np.all(o[padrows] == 0.0)


@pytest.mark.parametrize("shared", [True, False])
@pytest.mark.parametrize("with_fast", [False, True])
def test_bf16_prefill_padding(shared, with_fast):
    rng = np.random.default_rng(100 + 2 * shared + with_fast)
    B, S, Hq, d = 3, 300, 8, 256
    ar, seg = _layout(rng, B, S, shared, with_fast)
    q, q64, k, k64, v, v64 = _inputs(B, S, Hq, d, "bf16", 400)
    ar_t = torch.from_numpy(ar if shared else np.tile(ar, (B, 1))).cuda()
    seg_t = torch.from_numpy(seg if shared else seg).cuda()
    if shared:
        ar_t, seg_t = ar_t.contiguous(), seg_t[0].contiguous()
    lse = torch.empty((B, S, Hq), dtype=torch.float32, device="cuda")
    out = _b().pi_attn_prefill(q.cuda(), k.cuda(), v.cuda(), ar_t, seg_t, lse=lse)
    ref, ref_lse = oracle.prefill(q64, k64, v64, np.broadcast_to(ar, (B, S)),
                                  np.broadcast_to(seg, (B, S)))
    _check(out, ref, np.broadcast_to(seg, (B, S)), TOL_BF16)
    l = lse.cpu().numpy().astype(np.float64)
    padrows = np.broadcast_to(seg < 0, (B, S))
    assert np.all(np.isneginf(l[padrows]))
    np.testing.assert_allclose(l[~padrows], ref_lse[~padrows], atol=2e-2)


def test_bf16_prefill_fully_padded_batch_element():
    rng = np.random.default_rng(7)
    B, S, Hq, d = 2, 200, 8, 256
    ar = (rng.random(S) < 0.1).astype(np.uint8)
    seg = np.zeros((B, S), np.int32)
    seg[1, :] = -1                       # every token of element 1 is padding
    seg[0, 150:] = -1                    # element 0 right-padded
    q, q64, k, k64, v, v64 = _inputs(B, S, Hq, d, "bf16", 410)
    out = _b().pi_attn_prefill(q.cuda(), k.cuda(), v.cuda(),
                               torch.from_numpy(np.tile(ar, (B, 1))).cuda(),
                               torch.from_numpy(seg).cuda())
    ref, _ = oracle.prefill(q64, k64, v64, np.tile(ar, (B, 1)), seg)
    _check(out, ref, seg, TOL_BF16)


def test_f32_prefill_padding():
    rng = np.random.default_rng(8)
    B, S, Hq, d = 2, 49, 2, 64
    ar, seg = _layout(rng, B, S, shared=False, with_fast=True)
    q, q64, k, k64, v, v64 = _inputs(B, S, Hq, d, "f32", 420)
    out = _b().pi_attn_prefill(q.cuda(), k.cuda(), v.cuda(),
                               torch.from_numpy(np.tile(ar, (B, 1))).cuda(),
                               torch.from_numpy(seg).cuda())
    ref, _ = oracle.prefill(q64, k64, v64, np.tile(ar, (B, 1)), seg)
    _check(out, ref, seg, TOL_F32)


def test_debug_mask_with_padding_bit_exact():
    rng = np.random.default_rng(9)
    B, S = 3, 257
    ar, seg = _layout(rng, B, S, shared=False, with_fast=True)
    m = _b().pi_attn_debug_mask(torch.from_numpy(np.tile(ar, (B, 1))).cuda(),
                                torch.from_numpy(seg).cuda(), B=B, mode=0)
    want = oracle.prefill_mask(np.tile(ar, (B, 1)), seg)
    assert np.array_equal(m.cpu().numpy().astype(bool), want)


@pytest.mark.parametrize("B", [32, 2])          # one split; split-K over the cache
def test_bf16_suffix_cache_and_token_padding(B):
    rng = np.random.default_rng(10 + B)
    P, Sq, Hq, d = 816, 51, 8, 256
    ar = W.pi0_suffix_ar(Sq - 1)
    qs, q64 = W.draw((B, Sq, Hq, d), 431, d, "bf16")
    ks, k64 = W.draw((B, Sq, 1, d), 432, d, "bf16")
    vs, v64 = W.draw((B, Sq, 1, d), 433, d, "bf16")
    kc, kc64 = W.draw((B, P, 1, d), 434, d, "bf16")
    vc, vc64 = W.draw((B, P, 1, d), 435, d, "bf16")
    valid = (rng.random((B, P)) < 0.7).astype(np.uint8)
    valid[0, :] = 0                      # element 0 sees no cached key
    valid[1 % B, 700:] = 0               # right-padded prefix
    seg = np.zeros(Sq, np.int32)
    seg[[5, 17, 50]] = -1                # a few padded suffix tokens (shared)
    out = _b().pi_attn_suffix(qs.cuda(), ks.cuda(), vs.cuda(), kc.cuda(), vc.cuda(),
                              torch.from_numpy(ar).cuda(),
                              segment_ids=torch.from_numpy(seg).cuda(),
                              cache_valid=torch.from_numpy(valid).cuda())
    n = min(B, 4)
    ref, _ = oracle.suffix(q64[:n], k64[:n], v64[:n], kc64[:n], vc64[:n], ar, seg_suf=seg,
                           cache_valid=valid[:n])
    _check(out[:n], ref, np.broadcast_to(seg, (n, Sq)), TOL_BF16)
    assert _b().pi_attn_read_status() == _b().PI_OK


def test_f32_suffix_cache_padding():
    rng = np.random.default_rng(12)
    B, P, Sq, Hq, d = 2, 40, 9, 2, 64
    ar = W.pi0_suffix_ar(Sq - 1)
    qs, q64 = W.draw((B, Sq, Hq, d), 441, d, "f32")
    ks, k64 = W.draw((B, Sq, 1, d), 442, d, "f32")
    vs, v64 = W.draw((B, Sq, 1, d), 443, d, "f32")
    kc, kc64 = W.draw((B, P, 1, d), 444, d, "f32")
    vc, vc64 = W.draw((B, P, 1, d), 445, d, "f32")
    valid = (rng.random((B, P)) < 0.5).astype(np.uint8)
    out = _b().pi_attn_suffix(qs.cuda(), ks.cuda(), vs.cuda(), kc.cuda(), vc.cuda(),
                              torch.from_numpy(ar).cuda(),
                              cache_valid=torch.from_numpy(valid).cuda())
    ref, _ = oracle.suffix(q64, k64, v64, kc64, vc64, ar, cache_valid=valid)
    _check(out, ref, np.zeros((B, Sq), np.int32), TOL_F32)
