"""Nothing is written outside the caller's buffers.

Every output (and lse, gradient) tensor is a view into a larger buffer whose
bands on both sides hold a canary value, and every caller-provided workspace
is handed over with canary bytes past its required size.  Each kernel family
is covered in the configuration that reaches its own writes: the suffix pass
split over several SM pairs (partials in the workspace, merged by the combine
kernel), the few-row decode kernel (output written by each CTA of a cluster),
the prefill whose last round is split (fp32 pieces in the workspace, merged by
the tail kernel), and the backward (P / dS / D / partial sums in the
workspace, fp32 gradients).  The guarded call's results must also equal an
unguarded call's, bit for bit.
"""

import numpy as np
import pytest
import torch

from vla_prefix_lm_b200 import workloads as W

pytestmark = pytest.mark.gpu

GUARD = 4096          # elements (or bytes for workspaces) on each side
CANARY = 7.0          # exact in bf16 and fp32
WS_CANARY = 0x5A


def _b():
    from vla_prefix_lm_b200 import binding
    return binding


def _guarded(shape, dtype):
    """A contiguous tensor of `shape` inside a canary-filled buffer."""
    n = int(np.prod(shape))
    buf = torch.full((n + 2 * GUARD,), CANARY, dtype=dtype, device="cuda")
    return buf, buf[GUARD:GUARD + n].view(*shape)


def _bands_clean(buf):
    return bool((buf[:GUARD] == CANARY).all()) and bool((buf[-GUARD:] == CANARY).all())


def _workspace(need):
    """`need` bytes of garbage workspace followed by GUARD canary bytes."""
    ws = torch.full((need + GUARD,), WS_CANARY, dtype=torch.uint8, device="cuda")
    ws[:need].fill_(0xA5)
    return ws


def _ws_tail_clean(ws, need):
    return bool((ws[need:] == WS_CANARY).all())


def test_suffix_split_k_writes_only_out_and_its_workspace():
    """B = 1 against a 3000-key cache: the key tiles are split over several SM
    pairs, the partials go to the workspace and the combine kernel writes out."""
    b = _b()
    B, P, Sq, Hq, d = 1, 3000, 51, 8, 256
    ar = torch.from_numpy(W.pi0_suffix_ar(Sq - 1)).cuda()
    qs, _ = W.draw((B, Sq, Hq, d), 901, d, "bf16")
    ks, _ = W.draw((B, Sq, 1, d), 902, d, "bf16")
    vs, _ = W.draw((B, Sq, 1, d), 903, d, "bf16")
    kc, _ = W.draw((B, P, 1, d), 904, d, "bf16")
    vc, _ = W.draw((B, P, 1, d), 905, d, "bf16")
    args = tuple(t.cuda() for t in (qs, ks, vs, kc, vc)) + (ar,)
    need = b.pi_attn_suffix_workspace_bytes(args[0], args[1], args[3], args[5])
    assert need > 0
    ws = _workspace(need)
    buf, out = _guarded((B, Sq, Hq, d), torch.bfloat16)
    b.pi_attn_suffix(*args, out=out, workspace=ws)
    ref = b.pi_attn_suffix(*args)
    torch.cuda.synchronize()
    assert b.pi_attn_read_status() == b.PI_OK
    assert _bands_clean(buf)
    assert _ws_tail_clean(ws, need)
    assert torch.equal(out, ref)


def test_decode_writes_only_out():
    """Single-token decode (Sq x Hq = 8 rows): one cluster of CTAs per batch
    element, each CTA writing its own 32 columns of every row."""
    b = _b()
    B, P, Hq, d = 4, 880, 8, 256
    ar = torch.ones(1, dtype=torch.uint8, device="cuda")
    q, _ = W.draw((B, 1, Hq, d), 911, d, "bf16")
    k, _ = W.draw((B, 1, 1, d), 912, d, "bf16")
    v, _ = W.draw((B, 1, 1, d), 913, d, "bf16")
    kc, _ = W.draw((B, P, 1, d), 914, d, "bf16")
    vc, _ = W.draw((B, P, 1, d), 915, d, "bf16")
    args = tuple(t.cuda() for t in (q, k, v, kc, vc)) + (ar,)
    buf, out = _guarded((B, 1, Hq, d), torch.bfloat16)
    b.pi_attn_suffix(*args, out=out)
    ref = b.pi_attn_suffix(*args)
    torch.cuda.synchronize()
    assert b.pi_attn_read_status() == b.PI_OK
    assert _bands_clean(buf)
    assert torch.equal(out, ref)


def test_prefill_split_last_round_writes_only_out_lse_and_its_workspace():
    """A layout whose sparse last round is split into pieces: fp32 pieces in
    the workspace, merged by the tail kernel into out and lse."""
    b = _b()
    B, S, Hq, d = 2, 2400, 8, 256
    ar = torch.zeros(S, dtype=torch.uint8)
    q, _ = W.draw((B, S, Hq, d), 921, d, "bf16")
    k, _ = W.draw((B, S, 1, d), 922, d, "bf16")
    v, _ = W.draw((B, S, 1, d), 923, d, "bf16")
    qd, kd, vd, ard = q.cuda(), k.cuda(), v.cuda(), ar.cuda()
    assert b.pi_attn_prefill_tail_splits(qd, kd, ard) > 1
    need = b.pi_attn_prefill_workspace_bytes(qd, kd, ard)
    ws = _workspace(need)
    obuf, out = _guarded((B, S, Hq, d), torch.bfloat16)
    lbuf, lse = _guarded((B, S, Hq), torch.float32)
    b.pi_attn_prefill(qd, kd, vd, ard, out=out, lse=lse, workspace=ws)
    lse_ref = torch.empty((B, S, Hq), dtype=torch.float32, device="cuda")
    ref = b.pi_attn_prefill(qd, kd, vd, ard, lse=lse_ref)
    torch.cuda.synchronize()
    assert b.pi_attn_read_status() == b.PI_OK
    assert _bands_clean(obuf) and _bands_clean(lbuf)
    assert _ws_tail_clean(ws, need)
    # the split pieces and a whole unit sum the keys in different orders: the
    # two agree to the bf16 parity bound
    assert float((out.float() - ref.float()).abs().max()) <= 2e-2


def test_backward_writes_only_the_gradients_and_its_workspace():
    """Tensor-core backward (bf16, one KV head, d = 256): P / dS / D and the
    dK / dV partial sums in the workspace, fp32 gradients."""
    b = _b()
    B, S, Hq, d = 2, 300, 8, 256
    ar = torch.from_numpy(np.concatenate([np.zeros(249, np.uint8),
                                          W.pi0_suffix_ar(50)])).cuda()
    q, _ = W.draw((B, S, Hq, d), 931, d, "bf16")
    k, _ = W.draw((B, S, 1, d), 932, d, "bf16")
    v, _ = W.draw((B, S, 1, d), 933, d, "bf16")
    dout, _ = W.draw((B, S, Hq, d), 934, d, "bf16", 0.5)
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), dout.cuda()
    lse = torch.empty((B, S, Hq), dtype=torch.float32, device="cuda")
    out = b.pi_attn_prefill(qd, kd, vd, ar, lse=lse)
    need = b.pi_attn_prefill_backward_workspace_bytes(qd, kd, ar)
    ws = _workspace(need)
    bq, dq = _guarded((B, S, Hq, d), torch.float32)
    bk, dk = _guarded((B, S, 1, d), torch.float32)
    bv, dv = _guarded((B, S, 1, d), torch.float32)
    b.pi_attn_prefill_backward(qd, kd, vd, ar, out, lse, dod, dq=dq, dk=dk, dv=dv, workspace=ws)
    rq, rk, rv = b.pi_attn_prefill_backward(qd, kd, vd, ar, out, lse, dod)
    torch.cuda.synchronize()
    assert b.pi_attn_read_status() == b.PI_OK
    assert _bands_clean(bq) and _bands_clean(bk) and _bands_clean(bv)
    assert _ws_tail_clean(ws, need)
    assert torch.equal(dq, rq) and torch.equal(dk, rk) and torch.equal(dv, rv)
