"""Gradient of the joint prefill (dq, dk, dv) on the GPU vs the oracle's
plain derivative, element by element.

The training step of "VLA 代码精读 - OpenPI & StarVLA", 1.5 runs the joint
forward under gradient.  The CUDA backward takes the forward's own out and lse
(as a training step would) and writes fp32 gradients; the oracle differentiates
the float64 forward of the same rounded inputs.  Tolerance: the forward's
bound (bf16 2e-2, fp32 1e-4) relative to the gradient's scale,
max|got - ref| <= tol * max(1, max|ref|), since the key/value gradients sum
over up to S query rows and can exceed 1.
"""

import numpy as np
import pytest
import torch

from oracle import backward as obwd
from vla_prefix_lm_b200 import workloads as W

pytestmark = pytest.mark.gpu

TOL = {"bf16": 2e-2, "f32": 1e-4}


def _b():
    from vla_prefix_lm_b200 import binding
    return binding


def _check(got, ref, tol, name):
    got = got.cpu().numpy().astype(np.float64)
    err = float(np.abs(got - ref).max())
    scale = max(1.0, float(np.abs(ref).max()))
    bound = tol * scale
    print(f"{name}: max-abs err {err:.3e}, max|ref| {float(np.abs(ref).max()):.3e}, "
          f"scaled err {err / scale:.3e} (bound {tol:.0e})")
    assert err <= bound, f"{name}: max err {err:.3e} > {bound:.3e}"


def _run(q, k, v, ar, seg, dtype, seed, scale=1.0):
    """Forward + backward on the GPU; returns the three fp32 gradients and the
    rounded float64 inputs for the oracle."""
    b = _b()
    dev = "cuda"
    dout, dout64 = W.draw(tuple(q.shape), seed, q.shape[-1], dtype, 0.5)
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, dout))
    ard = ar.to(dev)
    segd = None if seg is None else seg.to(dev)
    B, S, Hq, _ = q.shape
    lse = torch.empty((B, S, Hq), dtype=torch.float32, device=dev)
    out = b.pi_attn_prefill(qd, kd, vd, ard, segment_ids=segd, lse=lse, softmax_scale=scale)
    need = b.pi_attn_prefill_backward_workspace_bytes(qd, kd, ard, scale)
    ws = torch.full((need,), 255, dtype=torch.uint8, device=dev)   # garbage-filled scratch
    grads = b.pi_attn_prefill_backward(qd, kd, vd, ard, out, lse, dod, segment_ids=segd,
                                       workspace=ws, softmax_scale=scale)
    torch.cuda.synchronize()
    assert b.pi_attn_read_status() == b.PI_OK
    return grads, dout64


def _oracle(q, k, v, ar, seg, dout64, scale=1.0):
    to64 = lambda t: t.to(torch.float64).numpy()
    return obwd.prefill_backward(to64(q), to64(k), to64(v), ar.numpy(), dout64,
                                 seg=None if seg is None else seg.numpy(), scale=scale)


@pytest.mark.parametrize("config", [2, 4])
def test_backward_matches_oracle_on_the_workloads(config):
    """At the workloads' full sizes, in the bench's launch configuration: pi0
    prefill (B=8, S=611) and pi0.5 (B=16, S=938, FAST/expert segments,
    expert <- FAST hole) in bf16."""
    w = W.workload(config)
    x = W.prefill_inputs(w, W.seed_for(config, 77), B=w.B)
    (dq, dk, dv), dout64 = _run(x.q, x.k, x.v, x.ar, x.seg, w.dtype, 801 + config)
    rq, rk, rv = _oracle(x.q, x.k, x.v, x.ar, x.seg, dout64)
    _check(dq, rq, TOL[w.dtype], "dq")
    _check(dk, rk, TOL[w.dtype], "dk")
    _check(dv, rv, TOL[w.dtype], "dv")


@pytest.mark.parametrize("S", [1, 17, 257])
def test_backward_ragged_lengths_bf16(S):
    rng = np.random.default_rng(90 + S)
    ar, _ = W.random_layout(S, rng, with_seg=False)
    q, _ = W.draw((2, S, 8, 256), 910 + S, 256, "bf16")
    k, _ = W.draw((2, S, 1, 256), 911 + S, 256, "bf16")
    v, _ = W.draw((2, S, 1, 256), 912 + S, 256, "bf16")
    art = torch.from_numpy(ar)
    (dq, dk, dv), dout64 = _run(q, k, v, art, None, "bf16", 913 + S, scale=0.8)
    rq, rk, rv = _oracle(q, k, v, art, None, dout64, scale=0.8)
    for got, ref, n in ((dq, rq, "dq"), (dk, rk, "dk"), (dv, rv, "dv")):
        _check(got, ref, TOL["bf16"], n)


def test_backward_f32_grouped_heads_per_batch_masks_and_padding():
    """fp32, Hq=4 over Hkv=2, d=64, a per-batch ar_mask and segment ids with
    FAST / expert tags and padded tokens; padded tokens get exact zeros."""
    rng = np.random.default_rng(95)
    B, S, Hq, Hkv, d = 2, 97, 4, 2, 64
    ar = (rng.random((B, S)) < 0.1).astype(np.uint8)
    seg = rng.choice([0, 1, 2], size=(B, S), p=[0.6, 0.2, 0.2]).astype(np.int32)
    seg[0, 40:47] = -1
    seg[1, -5:] = -1
    q, _ = W.draw((B, S, Hq, d), 951, d, "f32")
    k, _ = W.draw((B, S, Hkv, d), 952, d, "f32")
    v, _ = W.draw((B, S, Hkv, d), 953, d, "f32")
    art, segt = torch.from_numpy(ar), torch.from_numpy(seg)
    (dq, dk, dv), dout64 = _run(q, k, v, art, segt, "f32", 954, scale=0.6)
    rq, rk, rv = _oracle(q, k, v, art, segt, dout64, scale=0.6)
    for got, ref, n in ((dq, rq, "dq"), (dk, rk, "dk"), (dv, rv, "dv")):
        _check(got, ref, TOL["f32"], n)
    pad = torch.from_numpy(seg < 0)
    assert torch.all(dq.cpu()[pad] == 0) and torch.all(dk.cpu()[pad] == 0)
    assert torch.all(dv.cpu()[pad] == 0)


@pytest.mark.parametrize("Hq", [1, 2, 16])
def test_backward_bf16_head_counts(Hq):
    """The tensor-core backward at the other head counts it supports: row
    tiles of 256 / Hq tokens, a ragged last tile and a causal block."""
    rng = np.random.default_rng(40 + Hq)
    S = 150
    ar = np.concatenate([np.zeros(90, np.uint8), (rng.random(S - 90) < 0.5).astype(np.uint8)])
    q, _ = W.draw((2, S, Hq, 256), 960 + Hq, 256, "bf16")
    k, _ = W.draw((2, S, 1, 256), 961 + Hq, 256, "bf16")
    v, _ = W.draw((2, S, 1, 256), 962 + Hq, 256, "bf16")
    art = torch.from_numpy(ar)
    (dq, dk, dv), dout64 = _run(q, k, v, art, None, "bf16", 963 + Hq, scale=0.9)
    rq, rk, rv = _oracle(q, k, v, art, None, dout64, scale=0.9)
    for got, ref, n in ((dq, rq, "dq"), (dk, rk, "dk"), (dv, rv, "dv")):
        _check(got, ref, TOL["bf16"], n)


def test_backward_bf16_per_batch_masks_segments_and_padding():
    """bf16 on tensor cores: a per-batch ar_mask, FAST / expert tags (the
    expert <- FAST hole), padded tokens (exact zero gradients) and a length
    spanning several 256-key groups."""
    rng = np.random.default_rng(97)
    B, S, Hq = 3, 530, 8
    ar = (rng.random((B, S)) < 0.05).astype(np.uint8)
    seg = rng.choice([0, 1, 2], size=(B, S), p=[0.6, 0.2, 0.2]).astype(np.int32)
    seg[0, 100:140] = -1
    seg[1, -30:] = -1
    seg[2, :5] = -1
    q, _ = W.draw((B, S, Hq, 256), 971, 256, "bf16")
    k, _ = W.draw((B, S, 1, 256), 972, 256, "bf16")
    v, _ = W.draw((B, S, 1, 256), 973, 256, "bf16")
    art, segt = torch.from_numpy(ar), torch.from_numpy(seg)
    (dq, dk, dv), dout64 = _run(q, k, v, art, segt, "bf16", 974, scale=0.75)
    rq, rk, rv = _oracle(q, k, v, art, segt, dout64, scale=0.75)
    for got, ref, n in ((dq, rq, "dq"), (dk, rk, "dk"), (dv, rv, "dv")):
        _check(got, ref, TOL["bf16"], n)
    pad = torch.from_numpy(seg < 0)
    assert torch.all(dq.cpu()[pad] == 0) and torch.all(dk.cpu()[pad] == 0)
    assert torch.all(dv.cpu()[pad] == 0)


def test_backward_is_deterministic():
    w = W.workload(2)
    x = W.prefill_inputs(w, W.seed_for(2, 78), B=1)
    g1, _ = _run(x.q, x.k, x.v, x.ar, x.seg, w.dtype, 820)
    g2, _ = _run(x.q, x.k, x.v, x.ar, x.seg, w.dtype, 820)
    for a, c in zip(g1, g2):
        assert torch.equal(a, c)
