"""RoPE at the pages' positions and the Euler update on the GPU vs the oracle,
and the 10-step sampling loop's attention-side steps captured as one CUDA
graph.

Positions: cumsum(mask) - 1, continued after the valid prefix tokens in the
suffix pass ("VLA 代码精读 - OpenPI & StarVLA", 1.5 and 1.6).  Tolerances:
bf16 2e-2 (one bf16 rounding of values of order 1), fp32 1e-4; positions
bit-exact.
"""

import numpy as np
import pytest
import torch

import oracle
from oracle import prepost
from vla_prefix_lm_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _b():
    from vla_prefix_lm_b200 import binding
    return binding


def _err(t, ref):
    return float(np.abs(t.float().cpu().numpy().astype(np.float64) - ref).max())


@pytest.mark.parametrize("dtype,B,S,Hq,Hkv,d,tol", [("bf16", 8, 611, 8, 1, 256, 2e-2),
                                                     ("f32", 2, 4250, 8, 1, 256, 1e-4),
                                                     ("bf16", 2, 97, 4, 2, 64, 2e-2),
                                                     ("f32", 2, 131, 11, 1, 48, 1e-4)])
def test_rope_prefill_positions(dtype, B, S, Hq, Hkv, d, tol):
    """The first case is the pi0 prefill at full size (the bench's RoPE leg)."""
    rng = np.random.default_rng(31)
    mask = (rng.random((B, S)) < 0.9).astype(np.uint8)        # some padded tokens
    q, q64 = W.draw((B, S, Hq, d), 601, d, dtype)
    k, k64 = W.draw((B, S, Hkv, d), 602, d, dtype)
    qd, kd = q.cuda(), k.cuda()
    pos = _b().pi_rope_inplace(qd, kd, torch.from_numpy(mask).cuda(), positions=True)
    want_pos = prepost.positions(mask)
    assert np.array_equal(pos.cpu().numpy(), want_pos)
    assert _err(qd, prepost.rope(q64, want_pos)) <= tol
    assert _err(kd, prepost.rope(k64, want_pos)) <= tol


def test_rope_suffix_positions_continue_after_prefix():
    """One pi0 Euler step's suffix q/k at full size (B=32, 816 prefix tokens)."""
    rng = np.random.default_rng(32)
    B, P, Sq, Hq, d = 32, 816, 51, 8, 256
    pmask = (rng.random((B, P)) < 0.8).astype(np.uint8)
    smask = np.ones((B, Sq), np.uint8)
    q, q64 = W.draw((B, Sq, Hq, d), 611, d, "bf16")
    k, k64 = W.draw((B, Sq, 1, d), 612, d, "bf16")
    qd, kd = q.cuda(), k.cuda()
    pos = _b().pi_rope_inplace(qd, kd, torch.from_numpy(smask).cuda(),
                               prefix_mask=torch.from_numpy(pmask).cuda(), positions=True)
    want_pos = prepost.positions(smask, pmask)
    assert np.array_equal(pos.cpu().numpy(), want_pos)
    assert _err(qd, prepost.rope(q64, want_pos)) <= 2e-2
    assert _err(kd, prepost.rope(k64, want_pos)) <= 2e-2


@pytest.mark.parametrize("vdtype", ["bf16", "f32"])
def test_euler_update(vdtype):
    rng = np.random.default_rng(33)
    n = 32 * 50 * 32 + 3                                     # ragged tail
    x = torch.from_numpy(rng.standard_normal(n).astype(np.float32)).cuda()
    x64 = x.cpu().numpy().astype(np.float64)
    v, v64 = W.draw((n,), 621, 1, vdtype, 1.0)
    _b().pi_euler_update(x, v.cuda(), -0.1)
    np.testing.assert_allclose(x.cpu().numpy(), prepost.euler_step(x64, v64, -0.1), atol=1e-6)


def test_ten_step_loop_as_one_cuda_graph():
    """Per step: RoPE of this step's suffix q/k at the continued positions,
    the suffix pass against the (already rotated) prefix cache, and the Euler
    update with the step's velocity; the whole 10-step loop is one CUDA graph.
    (The action expert that maps the attention output to a velocity is
    outside this path, so each step's velocity is a given input here.)"""
    B, P, Sq, Hq, d, A, D = 4, 816, 51, 8, 256, 50, 32
    steps, dt = 10, -0.1
    rng = np.random.default_rng(34)
    pmask = np.ones((B, P), np.uint8)
    pmask[1, 700:] = 0
    smask = np.ones((B, Sq), np.uint8)
    ar = W.pi0_suffix_ar(Sq - 1)
    kc, kc64 = W.draw((B, P, 1, d), 631, d, "bf16")
    vc, vc64 = W.draw((B, P, 1, d), 632, d, "bf16")
    qs = [W.draw((B, Sq, Hq, d), 640 + 3 * s, d, "bf16") for s in range(steps)]
    ks = [W.draw((B, Sq, 1, d), 641 + 3 * s, d, "bf16") for s in range(steps)]
    vs = [W.draw((B, Sq, 1, d), 642 + 3 * s, d, "bf16") for s in range(steps)]
    vel = [W.draw((B, A, D), 700 + s, 1, "f32", 1.0) for s in range(steps)]
    x0 = rng.standard_normal((B, A, D)).astype(np.float32)

    dev = "cuda"
    src_q = [t[0].to(dev) for t in qs]
    src_k = [t[0].to(dev) for t in ks]
    vsd = [t[0].to(dev) for t in vs]
    veld = [t[0].to(dev) for t in vel]
    wq = [torch.empty_like(t) for t in src_q]
    wk = [torch.empty_like(t) for t in src_k]
    outs = [torch.empty_like(t) for t in src_q]
    kcd, vcd = kc.to(dev), vc.to(dev)
    pm, sm_, ard = (torch.from_numpy(a).to(dev) for a in (pmask, smask, ar))
    cv = pm.clone()
    x = torch.from_numpy(x0).to(dev)
    need = _b().pi_attn_suffix_workspace_bytes(src_q[0], src_k[0], kcd, ard)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    st = torch.cuda.Stream()

    def loop():
        for s in range(steps):
            wq[s].copy_(src_q[s])
            wk[s].copy_(src_k[s])
            _b().pi_rope_inplace(wq[s], wk[s], sm_, prefix_mask=pm, stream=st)
            _b().pi_attn_suffix(wq[s], wk[s], vsd[s], kcd, vcd, ard, out=outs[s], workspace=ws,
                                stream=st, cache_valid=cv)
            _b().pi_euler_update(x, veld[s], dt, stream=st)

    with torch.cuda.stream(st):
        loop()                                   # warm-up outside the capture
    torch.cuda.synchronize()
    x.copy_(torch.from_numpy(x0))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=st):
        loop()
    x.copy_(torch.from_numpy(x0))
    torch.cuda.synchronize()
    with torch.cuda.stream(st):
        g.replay()
    torch.cuda.synchronize()
    assert _b().pi_attn_read_status() == _b().PI_OK

    want_x = x0.astype(np.float64)
    pos = prepost.positions(smask, pmask)
    for s in range(steps):
        want_x = prepost.euler_step(want_x, vel[s][1], dt)
    np.testing.assert_allclose(x.cpu().numpy(), want_x, atol=1e-5)
    for s in (0, steps - 1):
        assert _err(wq[s], prepost.rope(qs[s][1], pos)) <= 2e-2
        assert _err(wk[s], prepost.rope(ks[s][1], pos)) <= 2e-2
        # the attention reads the bf16-rounded rotated values
        q_rot = wq[s].float().cpu().numpy().astype(np.float64)
        k_rot = wk[s].float().cpu().numpy().astype(np.float64)
        ref, _ = oracle.suffix(q_rot, k_rot, vs[s][1], kc64, vc64, ar, cache_valid=pmask)
        assert _err(outs[s], ref) <= 2e-2
