"""The kernels' visibility predicate, exported by pi_attn_debug_mask, equals
the oracle's explicitly built mask bit for bit: on every workload layout and on
randomised ar_mask / segment-id fuzz (batched rows included)."""

import numpy as np
import pytest
import torch

import oracle
from vla_prefix_lm_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _b():
    from vla_prefix_lm_b200 import binding
    return binding


@pytest.mark.parametrize("cfg", [1, 2, 4, 5])
def test_prefill_mask_workloads(cfg):
    w = W.workload(cfg)
    ar = torch.tensor(w.ar, dtype=torch.uint8, device="cuda")
    seg = None if w.seg is None else torch.tensor(w.seg, dtype=torch.int32, device="cuda")
    got = _b().pi_attn_debug_mask(ar, seg, B=2).cpu().numpy().astype(bool)
    want = oracle.prefill_mask(np.array(w.ar), None if w.seg is None else np.array(w.seg), B=2)
    assert np.array_equal(got, want)


def test_suffix_mask_workload():
    w = W.workload(3)
    ar = torch.tensor(w.ar, dtype=torch.uint8, device="cuda")
    got = _b().pi_attn_debug_mask(ar, None, B=3, P=w.P, mode=1).cpu().numpy().astype(bool)
    want = oracle.suffix_mask(np.array(w.ar), w.P, B=3)
    assert np.array_equal(got, want)


def test_mask_fuzz():
    rng = np.random.default_rng(0)
    for seed in range(200):
        S = int(rng.integers(1, 300))
        ar, seg = W.random_layout(S, rng, with_seg=bool(seed % 2))
        B = int(rng.integers(1, 4))
        if seed % 3 == 0:  # per-batch rows
            ar = np.stack([W.random_layout(S, rng, False)[0] for _ in range(B)])
            if seg is not None:
                seg = np.stack([rng.integers(0, 3, S).astype(np.int32) for _ in range(B)])
        tar = torch.from_numpy(ar).cuda()
        tseg = None if seg is None else torch.from_numpy(seg).cuda()
        got = _b().pi_attn_debug_mask(tar, tseg, B=B).cpu().numpy().astype(bool)
        want = oracle.prefill_mask(ar, seg, B=B)
        assert np.array_equal(got, want), seed


def test_suffix_mask_fuzz():
    rng = np.random.default_rng(1)
    for seed in range(50):
        Sq = int(rng.integers(1, 120))
        P = int(rng.integers(0, 300))
        ar, _ = W.random_layout(Sq, rng, False)
        got = _b().pi_attn_debug_mask(torch.from_numpy(ar).cuda(), None, B=2, P=P,
                                      mode=1).cpu().numpy().astype(bool)
        assert np.array_equal(got, oracle.suffix_mask(ar, P, B=2)), seed


def test_max_tokens_mask():
    S = 16383
    ar = np.zeros(S, np.uint8)
    ar[::97] = 1
    seg = np.zeros(S, np.int32)
    seg[8000:9000] = 1
    seg[9000:] = 2
    got = _b().pi_attn_debug_mask(torch.from_numpy(ar).cuda(), torch.from_numpy(seg).cuda(),
                                  B=1).cpu().numpy()
    rows = [0, 1, 96, 97, 5000, 8500, 9001, S - 1]   # sampled rows of the explicit mask
    want = oracle.prefill_mask(ar, seg, rows=rows)[0]
    assert np.array_equal(got[0, rows].astype(bool), want)
