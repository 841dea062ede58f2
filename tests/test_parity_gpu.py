"""CUDA path vs the CPU oracle, element by element, through the C ABI.

Tolerances: max-abs 2e-2 for bf16 inputs with fp32 accumulation, 1e-4 for the
fp32 path (the bounds the library's specification states).  Inputs are the
seeded workload draws; the oracle receives the same rounded values in float64.
Sizes span several 128-row query tiles and 128-key tiles with ragged tails;
the full-size workloads are checked in full (the largest, MM-DiT, on one whole
call plus one row of every work unit of another).
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


def _cuda(t):
    return None if t is None else t.cuda()


def _err(got, want):
    return float(np.abs(got.detach().float().cpu().numpy().astype(np.float64) - want).max())


def _prefill_case(B, ar, seg, Hq, d, dtype, seed, scale=1.0, lse=False, std=None):
    S = np.asarray(ar).shape[-1]
    s = d ** -0.25 if std is None else std
    q, q64 = W.draw((B, S, Hq, d), seed * 4, d, dtype, s)
    k, k64 = W.draw((B, S, 1, d), seed * 4 + 1, d, dtype, s)
    v, v64 = W.draw((B, S, 1, d), seed * 4 + 2, d, dtype, s)
    tar = torch.tensor(np.asarray(ar), dtype=torch.uint8).cuda()
    tseg = None if seg is None else torch.tensor(np.asarray(seg), dtype=torch.int32).cuda()
    tl = torch.empty((B, S, Hq), dtype=torch.float32, device="cuda") if lse else None
    out = _b().pi_attn_prefill(q.cuda(), k.cuda(), v.cuda(), tar, tseg, lse=tl,
                               softmax_scale=scale)
    torch.cuda.synchronize()
    ref, ref_lse = oracle.prefill(q64, k64, v64, np.asarray(ar), seg, scale=scale)
    return out, ref, tl, ref_lse


# ----------------------------------------------------------------- fp32 path


def test_tiny_f32_workload():
    w = W.workload(1)
    x = W.prefill_inputs(w, W.seed_for(1))
    tl = torch.empty((w.B, w.Sq, w.Hq), dtype=torch.float32, device="cuda")
    out = _b().pi_attn_prefill(x.q.cuda(), x.k.cuda(), x.v.cuda(), x.ar.cuda(), None, lse=tl)
    ref, ref_lse = oracle.prefill(x.q64, x.k64, x.v64, np.array(w.ar))
    assert _err(out, ref) <= TOL_F32
    assert _err(tl, ref_lse) <= TOL_F32


@pytest.mark.parametrize("d,Hq,Hkv", [(64, 2, 1), (128, 4, 2), (256, 8, 1), (32, 3, 3)])
def test_f32_prefill_shapes(d, Hq, Hkv):
    rng = np.random.default_rng(d + Hq)
    S = 77
    ar, seg = W.random_layout(S, rng, with_seg=True)
    q, q64 = W.draw((2, S, Hq, d), 11, d, "f32")
    k, k64 = W.draw((2, S, Hkv, d), 12, d, "f32")
    v, v64 = W.draw((2, S, Hkv, d), 13, d, "f32")
    out = _b().pi_attn_prefill(q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(ar).cuda(),
                               torch.from_numpy(seg).cuda(), softmax_scale=0.7)
    ref, _ = oracle.prefill(q64, k64, v64, ar, seg, scale=0.7)
    assert _err(out, ref) <= TOL_F32


def test_f32_suffix():
    B, P, Sq, Hq, d = 2, 40, 9, 2, 64
    ar = W.pi0_suffix_ar(Sq - 1)
    qs, q64 = W.draw((B, Sq, Hq, d), 21, d, "f32")
    ks, k64 = W.draw((B, Sq, 1, d), 22, d, "f32")
    vs, v64 = W.draw((B, Sq, 1, d), 23, d, "f32")
    kc, kc64 = W.draw((B, P, 1, d), 24, d, "f32")
    vc, vc64 = W.draw((B, P, 1, d), 25, d, "f32")
    out = _b().pi_attn_suffix(qs.cuda(), ks.cuda(), vs.cuda(), kc.cuda(), vc.cuda(),
                              torch.from_numpy(ar).cuda())
    ref, _ = oracle.suffix(q64, k64, v64, kc64, vc64, ar)
    assert _err(out, ref) <= TOL_F32


# ----------------------------------------------------------------- bf16 path


def test_bf16_pi0_small_multi_tile():
    """B=2, pi0 layout with a 200-token prefix: 13 query tiles, ragged last key tile."""
    ar = np.concatenate([np.zeros(200, np.uint8), W.pi0_suffix_ar(50)])
    out, ref, tl, rl = _prefill_case(2, ar, None, 8, 256, "bf16", 101, lse=True)
    assert _err(out, ref) <= TOL_BF16
    assert _err(tl, rl) <= TOL_BF16


def test_bf16_pi0_workload():
    w = W.workload(2)
    x = W.prefill_inputs(w, W.seed_for(2))
    tl = torch.empty((w.B, w.Sq, w.Hq), dtype=torch.float32, device="cuda")
    out = _b().pi_attn_prefill(x.q.cuda(), x.k.cuda(), x.v.cuda(), x.ar.cuda(), None, lse=tl)
    ref, ref_lse = oracle.prefill(x.q64, x.k64, x.v64, np.array(w.ar))
    e = _err(out, ref)
    print(f"pi0 prefill max-abs err {e:.3e}")
    assert e <= TOL_BF16
    assert _err(tl, ref_lse) <= TOL_BF16


def test_bf16_pi05_workload():
    w = W.workload(4)
    x = W.prefill_inputs(w, W.seed_for(4))
    out = _b().pi_attn_prefill(x.q.cuda(), x.k.cuda(), x.v.cuda(), x.ar.cuda(), x.seg.cuda())
    ref, _ = oracle.prefill(x.q64, x.k64, x.v64, np.array(w.ar), np.array(w.seg))
    e = _err(out, ref)
    print(f"pi0.5 prefill max-abs err {e:.3e}")
    assert e <= TOL_BF16


def test_bf16_mmdit_full_call():
    """MM-DiT (B=4, S=4250, all False), the first of its 28 calls compared in
    full: every (batch, token, head) row of out and lse against the oracle."""
    w = W.workload(5)
    x = W.prefill_inputs(w, W.seed_for(5, 0))
    tl = torch.empty((w.B, w.Sq, w.Hq), dtype=torch.float32, device="cuda")
    out = _b().pi_attn_prefill(x.q.cuda(), x.k.cuda(), x.v.cuda(), x.ar.cuda(), None, lse=tl)
    torch.cuda.synchronize()
    ref, ref_lse = oracle.prefill(x.q64, x.k64, x.v64, np.array(w.ar))
    e, el = _err(out, ref), _err(tl, ref_lse)
    print(f"MM-DiT call 0, all {w.B * w.Sq * w.Hq} rows: max-abs err out {e:.3e}, lse {el:.3e}")
    assert e <= TOL_BF16
    assert el <= TOL_BF16


def test_bf16_mmdit_every_pair_tile_last_call():
    """MM-DiT, the last of the 28 calls: one query token (all 8 heads) from
    every 256-row pair tile (32 tokens) of every batch element, so that every
    work unit the persistent scheduler walks is compared with the oracle.  The
    token's offset inside its tile varies, covering both CTAs of the pair."""
    w = W.workload(5)
    x = W.prefill_inputs(w, W.seed_for(5, w.calls - 1))
    out = _b().pi_attn_prefill(x.q.cuda(), x.k.cuda(), x.v.cuda(), x.ar.cuda(), None)
    torch.cuda.synchronize()
    tok_per_tile = 256 // w.Hq
    n_tiles = (w.Sq + tok_per_tile - 1) // tok_per_tile
    rows = []
    for b in range(w.B):
        for t in range(n_tiles):
            i = min(t * tok_per_tile + (7 * t + 5 * b) % tok_per_tile, w.Sq - 1)
            rows.append((b, i))
    ref, _ = oracle.prefill(x.q64, x.k64, x.v64, np.array(w.ar), rows=rows)
    got = torch.stack([out[b, i] for b, i in rows])
    e = _err(got, ref)
    print(f"MM-DiT call {w.calls - 1}, {len(rows)} rows (one per pair tile): max-abs err {e:.3e}")
    assert e <= TOL_BF16


@pytest.mark.parametrize("Hq", [1, 2, 4, 16])
def test_bf16_head_counts(Hq):
    rng = np.random.default_rng(Hq)
    ar, seg = W.random_layout(150, rng, with_seg=True)
    out, ref, _, _ = _prefill_case(2, ar, seg, Hq, 256, "bf16", 200 + Hq)
    assert _err(out, ref) <= TOL_BF16


@pytest.mark.parametrize("S", [1, 7, 16, 17, 129, 256, 257])
def test_bf16_ragged_lengths(S):
    rng = np.random.default_rng(S)
    ar, seg = W.random_layout(S, rng, with_seg=True)
    out, ref, tl, rl = _prefill_case(3, ar, seg, 8, 256, "bf16", 300 + S, lse=True)
    assert _err(out, ref) <= TOL_BF16
    assert _err(tl, rl) <= TOL_BF16


def test_bf16_causal_and_bidirectional():
    S = 300
    for ar in (np.ones(S, np.uint8), np.zeros(S, np.uint8)):
        out, ref, _, _ = _prefill_case(2, ar, None, 8, 256, "bf16", 400 + int(ar[0]))
        assert _err(out, ref) <= TOL_BF16


def test_bf16_per_batch_masks_and_scale():
    rng = np.random.default_rng(9)
    B, S = 3, 190
    ar = np.stack([W.random_layout(S, rng, False)[0] for _ in range(B)])
    seg = rng.integers(0, 3, (B, S)).astype(np.int32)
    out, ref, _, _ = _prefill_case(B, ar, seg, 8, 256, "bf16", 500, scale=0.0625)
    assert _err(out, ref) <= TOL_BF16


def test_bf16_unscaled_stress():
    """N(0,1) values without the d^-0.25 factor: logits of std 16 stress the rescaling."""
    ar = np.concatenate([np.zeros(100, np.uint8), W.pi0_suffix_ar(50)])
    out, ref, _, _ = _prefill_case(2, ar, None, 8, 256, "bf16", 600, std=1.0, scale=1 / 16)
    assert _err(out, ref) <= TOL_BF16


# ------------------------------------------------------------------ suffix


def _suffix_case(w, B, step, std=None):
    c = W.cache_inputs(w, W.seed_for(3, 999), B=B)
    x = W.suffix_inputs(w, W.seed_for(3, step), B=B, std_scale=std)
    out = _b().pi_attn_suffix(x.q.cuda(), x.k.cuda(), x.v.cuda(), c.k.cuda(), c.v.cuda(),
                              x.ar.cuda())
    torch.cuda.synchronize()
    ref, _ = oracle.suffix(x.q64, x.k64, x.v64, c.k64, c.v64, np.array(w.ar))
    return out, ref


def test_bf16_suffix_workload_steps():
    w = W.workload(3)
    for step in (0, 9):
        out, ref = _suffix_case(w, w.B, step)
        e = _err(out, ref)
        print(f"suffix step {step} max-abs err {e:.3e}")
        assert e <= TOL_BF16


def test_bf16_suffix_unscaled_stress():
    w = W.workload(3)
    out, ref = _suffix_case(w, 2, 3, std=1.0)
    # unit-variance q/k with scale 1 gives logits of std 16: still within tolerance
    assert _err(out, ref) <= TOL_BF16


@pytest.mark.parametrize("P,Sq", [(0, 51), (1, 5), (127, 3), (128, 130), (300, 1)])
def test_bf16_suffix_edge_sizes(P, Sq):
    B, Hq, d = 2, 8, 256
    ar = W.pi0_suffix_ar(max(Sq - 1, 1))[:Sq]
    qs, q64 = W.draw((B, Sq, Hq, d), 31, d, "bf16")
    ks, k64 = W.draw((B, Sq, 1, d), 32, d, "bf16")
    vs, v64 = W.draw((B, Sq, 1, d), 33, d, "bf16")
    kc, kc64 = W.draw((B, P, 1, d), 34, d, "bf16")
    vc, vc64 = W.draw((B, P, 1, d), 35, d, "bf16")
    out = _b().pi_attn_suffix(qs.cuda(), ks.cuda(), vs.cuda(),
                              kc.cuda() if P else None, vc.cuda() if P else None,
                              torch.from_numpy(ar).cuda())
    ref, _ = oracle.suffix(q64, k64, v64, kc64, vc64, ar)
    assert _err(out, ref) <= TOL_BF16


@pytest.mark.parametrize("B,P", [(1, 816), (2, 816), (4, 2000), (1, 3000)])
def test_bf16_suffix_split_k(B, P):
    """Small-batch suffix passes split the key tiles over several CTA pairs
    (caller-provided workspace, partials merged by the combine kernel)."""
    Sq, Hq, d = 51, 8, 256
    ar = W.pi0_suffix_ar(Sq - 1)
    qs, q64 = W.draw((B, Sq, Hq, d), 61, d, "bf16")
    ks, k64 = W.draw((B, Sq, 1, d), 62, d, "bf16")
    vs, v64 = W.draw((B, Sq, 1, d), 63, d, "bf16")
    kc, kc64 = W.draw((B, P, 1, d), 64, d, "bf16")
    vc, vc64 = W.draw((B, P, 1, d), 65, d, "bf16")
    args = (qs.cuda(), ks.cuda(), vs.cuda(), kc.cuda(), vc.cuda(), torch.from_numpy(ar).cuda())
    need = _b().pi_attn_suffix_workspace_bytes(args[0], args[1], args[3], args[5])
    assert need > 0
    ws = torch.full((need,), 0xAB, dtype=torch.uint8, device="cuda")  # garbage in: no init needed
    out = _b().pi_attn_suffix(*args, workspace=ws)
    ref, _ = oracle.suffix(q64, k64, v64, kc64, vc64, ar)
    assert _err(out, ref) <= TOL_BF16
    with pytest.raises(Exception):
        _b().pi_attn_suffix(*args, workspace=ws[: need - 16])


def test_suffix_equals_prefill_suffix_rows_on_gpu():
    """Suffix pass == rows [P:] of a joint prefill over [prefix, suffix] (any prefix q)."""
    B, P, Sq, Hq, d = 2, 260, 51, 8, 256
    ar_suf = W.pi0_suffix_ar(Sq - 1)
    q, _ = W.draw((B, P + Sq, Hq, d), 41, d, "bf16")
    k, _ = W.draw((B, P + Sq, 1, d), 42, d, "bf16")
    v, _ = W.draw((B, P + Sq, 1, d), 43, d, "bf16")
    q, k, v = q.cuda(), k.cuda(), v.cuda()
    ar = torch.from_numpy(np.concatenate([np.zeros(P, np.uint8), ar_suf])).cuda()
    full = _b().pi_attn_prefill(q, k, v, ar)
    suf = _b().pi_attn_suffix(q[:, P:].contiguous(), k[:, P:].contiguous(),
                              v[:, P:].contiguous(), k[:, :P].contiguous(),
                              v[:, :P].contiguous(), torch.from_numpy(ar_suf).cuda())
    assert (full[:, P:].float() - suf.float()).abs().max().item() <= 4e-3


def test_repeated_calls_identical():
    """Deterministic: two calls on the same inputs give identical bytes."""
    w = W.workload(2)
    x = W.prefill_inputs(w, 77, B=2)
    a = _b().pi_attn_prefill(x.q.cuda(), x.k.cuda(), x.v.cuda(), x.ar.cuda())
    b = _b().pi_attn_prefill(x.q.cuda(), x.k.cuda(), x.v.cuda(), x.ar.cuda())
    assert torch.equal(a, b)


def test_output_guard_band_untouched():
    """Nothing is written outside the output tensor (canary bands on both sides)."""
    B, S, Hq, d = 2, 77, 8, 256
    ar = np.concatenate([np.zeros(26, np.uint8), W.pi0_suffix_ar(50)])
    q, _ = W.draw((B, S, Hq, d), 51, d, "bf16")
    k, _ = W.draw((B, S, 1, d), 52, d, "bf16")
    v, _ = W.draw((B, S, 1, d), 53, d, "bf16")
    n = B * S * Hq * d
    guard = 4096
    buf = torch.full((n + 2 * guard,), 7.0, dtype=torch.bfloat16, device="cuda")
    out = buf[guard:guard + n].view(B, S, Hq, d)
    _b().pi_attn_prefill(q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(ar).cuda(), out=out)
    torch.cuda.synchronize()
    assert (buf[:guard] == 7.0).all() and (buf[guard + n:] == 7.0).all()


def test_status_clean_and_wait_timeout_reported():
    """Normal calls leave the status word clean; a wait that nothing satisfies
    runs out after the (short) limit and is reported as PI_ERR_TIMEOUT, and the
    GPU stays usable afterwards."""
    b = _b()
    assert b.pi_attn_read_status() == b.PI_OK
    prev = b.pi_attn_set_wait_limit(2_000_000)   # ~1 ms of SM cycles
    try:
        assert b.pi_attn_selftest_wait() == b.PI_OK
        assert b.pi_attn_read_status() == b.PI_ERR_TIMEOUT
        assert b.pi_attn_read_status() == b.PI_OK  # cleared by the read
    finally:
        b.pi_attn_set_wait_limit(prev)
    w = W.workload(1)
    x = W.prefill_inputs(w, 1)
    out = b.pi_attn_prefill(x.q.cuda(), x.k.cuda(), x.v.cuda(), x.ar.cuda())
    ref, _ = oracle.prefill(x.q64, x.k64, x.v64, np.array(w.ar))
    assert _err(out, ref) <= TOL_F32
    assert b.pi_attn_read_status() == b.PI_OK
