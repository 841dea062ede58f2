"""The prefill's split last round (pi_attn_prefill with a workspace): full rounds
of 256-row query tiles run whole on the SM pairs, and when the last round would
leave at least half of them idle and the sequence is long enough for pieces of
6 key tiles, each remaining tile is split over several pairs by key tiles and
merged from fp32 partials.  Compared with the oracle on the MM-DiT workload
(14 tail tiles x 5 pieces) and the pi0 / pi0.5 workloads (short: left whole) in
full, and on random layouts with segments and padding split 2, 3 and 6 ways;
the workspace content never matters."""

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


def _err(got, want):
    """Max-abs difference; equal entries (padding rows' lse = -inf on both
    sides) count as 0."""
    g = got.detach().float().cpu().numpy().astype(np.float64)
    with np.errstate(invalid="ignore"):
        d = np.where(g == want, 0.0, np.abs(g - want))
    return float(d.max())


def _ws(q, k, ar, fill=None):
    n = _b().pi_attn_prefill_workspace_bytes(q, k, ar)
    assert n > 0
    if fill is None:
        return torch.empty(n, dtype=torch.uint8, device="cuda")
    return torch.full((n,), fill, dtype=torch.uint8, device="cuda")


def _run(q, k, v, ar, seg, ws):
    B, S, Hq, _ = q.shape
    tl = torch.empty((B, S, Hq), dtype=torch.float32, device="cuda")
    out = _b().pi_attn_prefill(q, k, v, ar, seg, lse=tl, workspace=ws)
    assert _b().pi_attn_read_status() == _b().PI_OK
    return out, tl


@pytest.mark.parametrize("cfg", [2, 4, 5])
def test_tail_split_workload_full_call(cfg):
    """pi0 (B=8, S=611), pi0.5 (B=16, S=938, segments and padding) and MM-DiT
    (B=4, S=4250): every row of out and lse, with a garbage-filled workspace."""
    w = W.workload(cfg)
    x = W.prefill_inputs(w, W.seed_for(cfg, 1))
    q, k, v, ar = x.q.cuda(), x.k.cuda(), x.v.cuda(), x.ar.cuda()
    seg = None if w.seg is None else torch.tensor(np.array(w.seg), dtype=torch.int32).cuda()
    out, tl = _run(q, k, v, ar, seg, _ws(q, k, ar, fill=0xA5))
    ref, ref_lse = oracle.prefill(x.q64, x.k64, x.v64, np.array(w.ar),
                                  None if w.seg is None else np.array(w.seg))
    assert _err(out, ref) <= TOL_BF16
    assert _err(tl, ref_lse) <= TOL_BF16


def _tail_splits(B, S, Hq, n_slots):
    """The split the host picks: full rounds of n_slots query tiles run whole;
    a last round under half full splits each tile s = min(n_slots / rem, 8,
    (S / 128) / 6) ways (pieces of at least 6 key tiles); else no split."""
    units = B * ((S * Hq + 255) // 256)
    full, rem = divmod(units, n_slots)
    s = min(n_slots // rem, 8, ((S + 127) // 128) // 6) if rem else 0
    return s if full >= 1 and s >= 2 else 1


@pytest.mark.parametrize("B,S,Hq,want", [(5, 2100, 8, 2), (2, 2400, 8, 3), (1, 4800, 8, 6),
                                         (8, 300, 8, 1), (16, 938, 8, 1)])
def test_tail_split_random_layouts(B, S, Hq, want):
    """Tail tiles split 2, 3 and 6 ways (and two short controls left whole),
    random block layouts with FAST / expert tags and scattered padding."""
    n_slots = torch.cuda.get_device_properties(0).multi_processor_count // 2
    if n_slots == 74:
        assert _tail_splits(B, S, Hq, n_slots) == want
    rng = np.random.default_rng(5000 + S + Hq + B)
    dummy = torch.empty((B, S, Hq, 256), dtype=torch.bfloat16, device="cuda")
    assert _b().pi_attn_prefill_tail_splits(dummy, dummy[:, :, :1], torch.ones(
        S, dtype=torch.uint8, device="cuda")) == _tail_splits(B, S, Hq, n_slots)
    ar, seg = W.random_layout(S, rng, with_seg=True)
    seg[rng.random(S) < 0.05] = -1
    s = 256 ** -0.25
    q, q64 = W.draw((B, S, Hq, 256), 900 + S, 256, "bf16", s)
    k, k64 = W.draw((B, S, 1, 256), 901 + S, 256, "bf16", s)
    v, v64 = W.draw((B, S, 1, 256), 902 + S, 256, "bf16", s)
    tar = torch.from_numpy(np.asarray(ar, np.uint8)).cuda()
    tseg = torch.from_numpy(np.asarray(seg, np.int32)).cuda()
    out, tl = _run(q.cuda(), k.cuda(), v.cuda(), tar, tseg, _ws(q.cuda(), k.cuda(), tar))
    ref, ref_lse = oracle.prefill(q64, k64, v64, ar, seg)
    assert _err(out, ref) <= TOL_BF16
    assert _err(tl, ref_lse) <= TOL_BF16


def test_tail_split_matches_whole_rounds():
    """The same call with and without the workspace agree to fp32 rounding of
    the merge (bf16 outputs within one ulp-scale step)."""
    w = W.workload(2)
    x = W.prefill_inputs(w, W.seed_for(2, 2))
    q, k, v, ar = x.q.cuda(), x.k.cuda(), x.v.cuda(), x.ar.cuda()
    a = _b().pi_attn_prefill(q, k, v, ar)
    b, _ = _run(q, k, v, ar, None, _ws(q, k, ar))
    assert float((a.float() - b.float()).abs().max()) <= 1e-2


def test_tail_split_workspace_errors():
    w = W.workload(2)
    x = W.prefill_inputs(w, W.seed_for(2, 3))
    q, k, v, ar = x.q.cuda(), x.k.cuda(), x.v.cuda(), x.ar.cuda()
    n = _b().pi_attn_prefill_workspace_bytes(q, k, ar)
    with pytest.raises(_b().PiAttnError):
        _b().pi_attn_prefill(q, k, v, ar, workspace=torch.empty(n - 16, dtype=torch.uint8,
                                                                device="cuda"))
    # per-batch masks take no scratch (size 0) and ignore one
    arb = ar.expand(w.B, -1).contiguous()
    assert _b().pi_attn_prefill_workspace_bytes(q, k, arb) == 0
