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


def _brute_tile_classes(M, Hq, seg=None):
    """From an explicit [B, S, S] mask: per (batch, 256-row tile, 128-key
    tile) whether no pair is visible (0), every pair is (1, complete tiles
    only) or neither (2).  Padding query rows are left out: the kernel masks a
    padding row whole, whatever the class of the tile."""
    B, S, _ = M.shape
    tok = 256 // Hq
    n_pairs, n_kt = (S * Hq + 255) // 256, (S + 127) // 128
    live = np.ones((B, S), bool)
    if seg is not None:
        live = np.broadcast_to(np.asarray(seg) >= 0, (B, S))
    out = np.zeros((B, n_pairs, n_kt), np.uint8)
    for b in range(B):
        for p in range(n_pairs):
            r0, r1 = p * tok, min(p * tok + tok, S)
            rows = M[b, r0:r1][live[b, r0:r1]]
            for t in range(n_kt):
                blk = rows[:, 128 * t:128 * t + 128]
                if not blk.any():
                    out[b, p, t] = 0
                elif blk.all() and 128 * t + 128 <= S:
                    out[b, p, t] = 1
                else:
                    out[b, p, t] = 2
    return out


@pytest.mark.parametrize("cfg", [2, 4, 5])
def test_tile_classes_on_the_workloads(cfg):
    """The prefill kernel's skip / full / partial classes against a brute-force
    scan of the oracle's explicit mask, on the pi0, pi0.5 and MM-DiT layouts.
    Without padding the classes are exact; with the pi0.5 segments a tile
    the kernel skips has no visible pair and a tile it calls full has every
    pair visible."""
    w = W.workload(cfg)
    ar = np.array(w.ar, np.uint8)
    seg = None if w.seg is None else np.array(w.seg, np.int32)
    got = _b().pi_attn_debug_tiles(torch.from_numpy(ar).cuda(),
                                   None if seg is None else torch.from_numpy(seg).cuda(),
                                   B=1, Hq=w.Hq).cpu().numpy()
    want = _brute_tile_classes(oracle.prefill_mask(ar, seg), w.Hq, seg)
    if seg is None:
        assert np.array_equal(got, want)
    else:
        assert np.all(want[got == 0] == 0)
        assert np.all(want[got == 1] == 1)
        assert np.all(got[want != 0] != 0)
    print(f"config {cfg}: {int((got == 0).sum())} skipped, {int((got == 1).sum())} full, "
          f"{int((got == 2).sum())} partial tiles")


def test_tile_classes_fuzz():
    """Random layouts (per-batch ar_mask, FAST / expert tags, padding), every
    head count: a skipped tile has no visible pair, a full tile every pair,
    and no tile with a visible pair is skipped; without tags or padding the
    classes equal the brute-force scan exactly."""
    rng = np.random.default_rng(77)
    for it in range(60):
        B = int(rng.integers(1, 4))
        S = int(rng.integers(1, 700))
        Hq = int(rng.choice([1, 2, 4, 8, 16]))
        ar = np.stack([W.random_layout(S, rng, False)[0] for _ in range(B)])
        use_seg = it % 2 == 1
        seg = None
        if use_seg:
            seg = rng.choice([0, 1, 2], size=(B, S), p=[0.5, 0.25, 0.25]).astype(np.int32)
            seg[rng.random((B, S)) < 0.05] = -1
        got = _b().pi_attn_debug_tiles(torch.from_numpy(ar).cuda(),
                                       None if seg is None else torch.from_numpy(seg).cuda(),
                                       B=B, Hq=Hq).cpu().numpy()
        want = _brute_tile_classes(oracle.prefill_mask(ar, seg), Hq, seg)
        if seg is None:
            assert np.array_equal(got, want), (B, S, Hq)
        else:
            assert np.all(want[got == 0] == 0), (B, S, Hq)
            assert np.all(want[got == 1] == 1), (B, S, Hq)
            assert np.all(got[want != 0] != 0), (B, S, Hq)
