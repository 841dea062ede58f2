"""Pins for the CPU oracle against what the pages and the mathematics fix.

None of these checks re-types the oracle's formula: the masks are compared to
the pages' own pictures and tables (tests/golden, each file cites its page),
to an independent boundary-walking enumerator over all small ar patterns, and
the attention values to closed forms, invariances, torch's float64
scaled_dot_product_attention and scipy's logsumexp.
"""

import itertools
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle
from oracle import brute, counts
from oracle.attention import EXPERT, FAST, OTHER

from conftest import GOLDEN


def _load_rows(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


# ------------------------------------------------------------------ masks


def test_fast_mask_picture():
    """Pi0-FAST 模型架构 2.3: 3 image + 2 language + 3 action tokens."""
    ar = [0, 0, 0, 0, 0, 1, 1, 1]
    M = oracle.prefill_mask(ar)[0]
    seen = set()
    for label, toks, bits in _load_rows("fast_mask_picture.txt"):
        want = np.array([c == "1" for c in bits])
        for t in map(int, toks.split(",")):
            np.testing.assert_array_equal(M[t], want, err_msg=label)
            seen.add(t)
    assert seen == set(range(8))


def test_causal_tril_all_true():
    """VLA论文阅读 Part 3: an all-True ar_mask is the causal (lower-triangular) mask."""
    want = np.array([[c == "1" for c in r[0]] for r in _load_rows("causal_verify_tril.txt")])
    np.testing.assert_array_equal(oracle.prefill_mask([1, 1, 1, 1])[0], want)
    for S in (1, 7, 33):
        np.testing.assert_array_equal(oracle.prefill_mask(np.ones(S))[0],
                                      np.tril(np.ones((S, S), bool)))


def test_all_false_is_bidirectional():
    """MM-DiT is fully bidirectional: all-False ar_mask sees every key."""
    for S in (1, 5, 154):
        assert oracle.prefill_mask(np.zeros(S))[0].all()


def test_pi0_prefix_never_sees_suffix():
    """OpenPI 1.2: prefix <-> prefix, suffix -> prefix, prefix -/-> suffix."""
    n_pre = 20
    ar = [0] * n_pre + [1, 1] + [0] * 9
    M = oracle.prefill_mask(ar)[0]
    assert M[:n_pre, :n_pre].all()
    assert not M[:n_pre, n_pre:].any()
    assert M[n_pre:, :n_pre].all()
    # state row sees prefix + itself only; action rows see state and all actions
    assert M[n_pre, : n_pre + 1].all() and not M[n_pre, n_pre + 1:].any()
    assert M[n_pre + 1:, :].all()


_SEG_NAME = {OTHER: "prefix", FAST: "FAST", EXPERT: "expert"}


def _check_permission_table(n_pre, n_fast, n_exp):
    ar = [0] * n_pre + [1] * n_fast + [1] + [0] * (n_exp - 1)
    seg = [OTHER] * n_pre + [FAST] * n_fast + [EXPERT] * n_exp
    M = oracle.prefill_mask(ar, seg)[0]
    spans = {"prefix": slice(0, n_pre), "FAST": slice(n_pre, n_pre + n_fast),
             "expert": slice(n_pre + n_fast, n_pre + n_fast + n_exp)}
    rows = _load_rows("pi05_permission_table.txt")
    assert len(rows) == 9
    for qname, kname, rel in rows:
        blk = M[spans[qname], spans[kname]]
        if rel == "all":
            assert blk.all(), (qname, kname)
        elif rel == "none":
            assert not blk.any(), (qname, kname)
        elif rel == "causal":
            assert blk.shape[0] == blk.shape[1]
            np.testing.assert_array_equal(blk, np.tril(np.ones(blk.shape, bool)))
        else:
            raise AssertionError(rel)
    return ar, seg


def test_pi05_permission_table_small():
    _check_permission_table(6, 4, 5)


def test_pi05_permission_table_full_layout():
    """The pi0.5 layout of the three-segment workload: 824 | 64 | 50."""
    ar, seg = _check_permission_table(824, 64, 50)
    # the cumsum rule alone would let expert queries read FAST keys: the
    # segment term is what enforces the table's last row
    M_nosg = oracle.prefill_mask(ar)[0]
    assert M_nosg[824 + 64:, 824:824 + 64].all()


def test_brute_force_all_patterns():
    """cumsum rule == boundary-walking if-chain on every ar pattern, S <= 10."""
    for S in range(1, 11):
        for bits in itertools.product((0, 1), repeat=S):
            M = oracle.prefill_mask(list(bits))[0]
            np.testing.assert_array_equal(M, np.array(brute.mask(list(bits))), err_msg=str(bits))


def test_brute_force_random_segments():
    rng = np.random.default_rng(7)
    for _ in range(400):
        S = int(rng.integers(1, 13))
        ar = rng.integers(0, 2, S)
        seg = rng.integers(0, 3, S)
        M = oracle.prefill_mask(ar, seg)[0]
        np.testing.assert_array_equal(M, np.array(brute.mask(list(ar), list(seg))))


def test_batched_ar_and_seg():
    """[B, S] ar / seg give per-batch masks; 1-D ones broadcast."""
    ar = np.array([[0, 0, 1, 0], [1, 1, 1, 1]])
    seg = np.array([[0, 1, 2, 2], [0, 0, 0, 0]])
    M = oracle.prefill_mask(ar, seg)
    for b in range(2):
        np.testing.assert_array_equal(M[b], np.array(brute.mask(list(ar[b]), list(seg[b]))))
    assert oracle.prefill_mask([0, 1], B=3).shape == (3, 2, 2)


def test_suffix_mask_construction():
    """OpenPI 1.6: every suffix row sees every prefix key, then make_attn_mask over the suffix."""
    ar_suf = [1, 1, 0, 0]
    M = oracle.suffix_mask(ar_suf, P=5)[0]
    assert M.shape == (4, 9)
    assert M[:, :5].all()
    np.testing.assert_array_equal(M[:, 5:], np.array(brute.mask(ar_suf)))


# ------------------------------------------------------------ attention values


def _rand(shape, rng, s=1.0):
    return rng.standard_normal(shape) * s


def test_softmax_rows_sum_to_one_and_masked_zero():
    rng = np.random.default_rng(1)
    S = 40
    ar = (rng.random(S) < 0.2).astype(int)
    M = oracle.prefill_mask(ar)[0]
    p = oracle.softmax_probs(_rand((S, S), rng, 3.0), M)
    np.testing.assert_allclose(p.sum(-1), 1.0, rtol=0, atol=1e-12)
    assert (p[~M] == 0).all()
    assert (p[M] > 0).all()


def test_q_zero_gives_mean_of_visible_values():
    rng = np.random.default_rng(2)
    B, S, Hq, d = 2, 17, 4, 8
    ar = [0] * 6 + [1, 0, 0, 1, 1, 0, 0, 0, 1, 0, 0]
    q = np.zeros((B, S, Hq, d))
    k = _rand((B, S, 1, d), rng)
    v = _rand((B, S, 1, d), rng)
    out, lse = oracle.prefill(q, k, v, ar)
    M = np.array(brute.mask(ar))
    for b in range(B):
        for i in range(S):
            want = v[b, M[i], 0, :].mean(0)
            for h in range(Hq):
                np.testing.assert_allclose(out[b, i, h], want, atol=1e-13)
                # all visible logits are 0: lse = log(#visible)
                assert abs(lse[b, i, h] - np.log(M[i].sum())) < 1e-13


def test_single_visible_key_returns_its_value():
    rng = np.random.default_rng(3)
    B, S, Hq, d = 1, 9, 2, 16
    q = _rand((B, S, Hq, d), rng)
    k = _rand((B, S, 1, d), rng)
    v = _rand((B, S, 1, d), rng)
    out, _ = oracle.prefill(q, k, v, [1] * S)
    for h in range(Hq):
        np.testing.assert_allclose(out[0, 0, h], v[0, 0, 0], atol=1e-14)


def test_duplicated_heads_identical():
    rng = np.random.default_rng(4)
    B, S, Hq, d = 2, 21, 8, 32
    q = _rand((B, S, Hq, d), rng)
    q[:, :, 5] = q[:, :, 2]
    k = _rand((B, S, 1, d), rng)
    v = _rand((B, S, 1, d), rng)
    ar = [0] * 10 + [1, 1] + [0] * 9
    out, _ = oracle.prefill(q, k, v, ar)
    np.testing.assert_array_equal(out[:, :, 5], out[:, :, 2])


def test_key_permutation_inside_bidirectional_block():
    """Keys of one bidirectional block are a set: permuting them (with V) changes nothing."""
    rng = np.random.default_rng(5)
    B, S, Hq, d = 1, 30, 4, 16
    ar = [0] * 20 + [1] + [0] * 9
    q = _rand((B, S, Hq, d), rng)
    k = _rand((B, S, 1, d), rng)
    v = _rand((B, S, 1, d), rng)
    out, lse = oracle.prefill(q, k, v, ar)
    perm = np.arange(S)
    perm[:20] = rng.permutation(20)
    out2, lse2 = oracle.prefill(q, k[:, perm], v[:, perm], ar)
    np.testing.assert_allclose(out2, out, atol=1e-13)
    np.testing.assert_allclose(lse2, lse, atol=1e-13)


@pytest.mark.parametrize("Hq,Hkv,scale", [(8, 1, 1.0), (4, 2, 0.37), (2, 1, 1 / 8.0)])
def test_equals_torch_sdpa_float64(Hq, Hkv, scale):
    """Library special case: torch SDPA (float64, CPU) with the explicit bool mask."""
    rng = np.random.default_rng(6)
    B, S, d = 2, 37, 16
    ar = [0] * 15 + [1] * 8 + [1] + [0] * 13
    seg = [OTHER] * 15 + [FAST] * 8 + [EXPERT] * 14
    q = _rand((B, S, Hq, d), rng)
    k = _rand((B, S, Hkv, d), rng)
    v = _rand((B, S, Hkv, d), rng)
    out, _ = oracle.prefill(q, k, v, ar, seg, scale=scale)
    M = torch.from_numpy(np.array(brute.mask(ar, seg)))
    tq, tk, tv = (torch.from_numpy(x).permute(0, 2, 1, 3) for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(
        tq, tk, tv, attn_mask=M, scale=scale, enable_gqa=True)
    np.testing.assert_allclose(out, ref.permute(0, 2, 1, 3).numpy(), atol=1e-12)


def test_lse_matches_scipy_logsumexp():
    rng = np.random.default_rng(8)
    B, S, Hq, d = 1, 25, 2, 8
    ar = [0] * 12 + [1] + [0] * 12
    q = _rand((B, S, Hq, d), rng)
    k = _rand((B, S, 1, d), rng)
    v = _rand((B, S, 1, d), rng)
    _, lse = oracle.prefill(q, k, v, ar, scale=0.5)
    M = np.array(brute.mask(ar))
    for i in range(S):
        for h in range(Hq):
            s = 0.5 * (k[0, :, 0] @ q[0, i, h])
            assert abs(lse[0, i, h] - scipy.special.logsumexp(s[M[i]])) < 1e-12


def test_pure_python_brute_attention():
    """Pure-Python loops (math.exp) over brute.visible agree with the oracle."""
    rng = np.random.default_rng(9)
    B, S, Hq, d = 1, 11, 2, 4
    ar = [0, 0, 0, 1, 1, 0, 1, 0, 0, 1, 1]
    seg = [0, 0, 0, 1, 1, 1, 2, 2, 2, 0, 1]
    q = _rand((B, S, Hq, d), rng)
    k = _rand((B, S, 1, d), rng)
    v = _rand((B, S, 1, d), rng)
    out, _ = oracle.prefill(q, k, v, ar, seg, scale=0.8)
    for i in range(S):
        vis = [brute.visible(i, j, ar, seg) for j in range(S)]
        for h in range(Hq):
            want = brute.attention_row(list(q[0, i, h]), k[0, :, 0].tolist(),
                                       v[0, :, 0].tolist(), vis, scale=0.8)
            np.testing.assert_allclose(out[0, i, h], want, atol=1e-13)


def test_suffix_pass_equals_prefill_suffix_rows():
    """Suffix-only pass == rows [P:] of the joint prefill, for any prefix queries."""
    rng = np.random.default_rng(10)
    B, P, Sq, Hq, d = 2, 13, 9, 4, 8
    ar_suf = [1, 1] + [0] * (Sq - 2)
    k_c, v_c = _rand((B, P, 1, d), rng), _rand((B, P, 1, d), rng)
    qs, ks, vs = _rand((B, Sq, Hq, d), rng), _rand((B, Sq, 1, d), rng), _rand((B, Sq, 1, d), rng)
    out_s, lse_s = oracle.suffix(qs, ks, vs, k_c, v_c, ar_suf, scale=0.7)
    for trial in range(2):
        q_pre = _rand((B, P, Hq, d), rng)
        q = np.concatenate([q_pre, qs], 1)
        k = np.concatenate([k_c, ks], 1)
        v = np.concatenate([v_c, vs], 1)
        out_p, lse_p = oracle.prefill(q, k, v, [0] * P + ar_suf, scale=0.7)
        np.testing.assert_allclose(out_s, out_p[:, P:], atol=1e-13)
        np.testing.assert_allclose(lse_s, lse_p[:, P:], atol=1e-13)


def test_rows_subset_matches_full():
    rng = np.random.default_rng(11)
    B, S, Hq, d = 2, 19, 4, 8
    ar = [0] * 9 + [1] * 4 + [1] + [0] * 5
    seg = [0] * 9 + [1] * 4 + [2] * 6
    q, k, v = _rand((B, S, Hq, d), rng), _rand((B, S, 1, d), rng), _rand((B, S, 1, d), rng)
    out, lse = oracle.prefill(q, k, v, ar, seg)
    rows = [(1, 18), (0, 0), (1, 10), (0, 14)]
    o2, l2 = oracle.prefill(q, k, v, ar, seg, rows=rows)
    for r, (b, i) in enumerate(rows):
        np.testing.assert_allclose(o2[r], out[b, i], atol=1e-14)
        np.testing.assert_allclose(l2[r], lse[b, i], atol=1e-14)


# ------------------------------------------------------------------ counts


def test_pair_counts():
    vals = {r[0]: float(r[1]) for r in _load_rows("pair_counts.txt")}
    assert counts.full_pairs(392 + 48 + 8 + 32) == vals["fused_480_scores"]
    assert counts.full_pairs(32, 448) == vals["cross_32x448_scores"]
    mmdit = 28 * counts.full_pairs(4096 + 154)
    assert float(f"{mmdit:.0e}") == vals["mmdit_28_steps_about"]
    assert counts.visible_pairs(oracle.prefill_mask(np.zeros(480))) == 230400


# ----------------------------------------------------------- planted mistakes


def _pins_pass(mask_fn):
    """Run the mask pins against a candidate mask builder; True if all hold."""
    try:
        M = mask_fn([0, 0, 0, 0, 0, 1, 1, 1], None)
        for label, toks, bits in _load_rows("fast_mask_picture.txt"):
            for t in map(int, toks.split(",")):
                if not (M[t] == np.array([c == "1" for c in bits])).all():
                    return False
        ar = [0] * 6 + [1] * 4 + [1] + [0] * 4
        seg = [0] * 6 + [1] * 4 + [2] * 5
        M = mask_fn(ar, seg)
        if not (M == np.array(brute.mask(ar, seg))).all():
            return False
        for S in range(1, 7):
            for bits in itertools.product((0, 1), repeat=S):
                if not (mask_fn(list(bits), None) == np.array(brute.mask(list(bits)))).all():
                    return False
        return True
    except Exception:
        return False


def test_planted_mask_mistakes_are_caught():
    def good(ar, seg):
        return oracle.prefill_mask(ar, seg)[0]

    def transposed(ar, seg):
        return oracle.prefill_mask(ar, seg)[0].T

    def strict(ar, seg):
        cs = oracle.ar_cumsum(np.asarray(ar))
        return cs[None, :] < cs[:, None]

    def no_seg_rule(ar, seg):
        return oracle.prefill_mask(ar, None)[0]

    def seg_rule_reversed(ar, seg):
        M = oracle.prefill_mask(ar, None)[0]
        if seg is not None:
            s = np.asarray(seg)
            M &= ~((s[:, None] == FAST) & (s[None, :] == EXPERT))
        return M

    def exclusive_cumsum(ar, seg):
        a = (np.asarray(ar) != 0).astype(int)
        cs = np.cumsum(a) - a
        return cs[None, :] <= cs[:, None]

    assert _pins_pass(good)
    for bad in (transposed, strict, no_seg_rule, seg_rule_reversed, exclusive_cumsum):
        assert not _pins_pass(bad), bad.__name__


def test_planted_value_mistakes_are_caught():
    """Dropping the scale, swapping q/k roles or mis-grouping heads breaks the SDPA pin."""
    rng = np.random.default_rng(12)
    B, S, Hq, Hkv, d = 1, 12, 4, 2, 8
    ar = [0] * 6 + [1] + [0] * 5
    q, k, v = _rand((B, S, Hq, d), rng), _rand((B, S, Hkv, d), rng), _rand((B, S, Hkv, d), rng)
    M = oracle.prefill_mask(ar, B=B)
    tq, tk, tv = (torch.from_numpy(x).permute(0, 2, 1, 3) for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(
        tq, tk, tv, attn_mask=torch.from_numpy(M[0]), scale=0.5, enable_gqa=True
    ).permute(0, 2, 1, 3).numpy()

    good, _ = oracle.attention(q, k, v, M, 0.5)
    assert np.abs(good - ref).max() < 1e-12
    no_scale, _ = oracle.attention(q, k, v, M, 1.0)
    assert np.abs(no_scale - ref).max() > 1e-3
    # modulo head grouping instead of contiguous groups
    q_regroup = q[:, :, [0, 2, 1, 3], :]
    bad_group, _ = oracle.attention(q_regroup, k, v, M, 0.5)
    assert np.abs(bad_group[:, :, [0, 2, 1, 3]] - ref).max() > 1e-3
    # transposed mask
    bad_t, _ = oracle.attention(q, k, v, np.swapaxes(M, 1, 2), 0.5)
    assert np.abs(bad_t - ref).max() > 1e-3


# ---------------------------------------------------------------- padding
# A negative segment id marks a padding token (openpi and Pi0-FAST AND a
# per-token validity mask into the attention mask; the workloads have none).
# The pins below tie the padded oracle to what padding must mean: a padding
# token behaves exactly as if it were absent, and a query row that sees no
# key outputs 0 with lse = -inf.

def _rand_qkv(rng, B, S, Hq=2, d=8):
    q = rng.standard_normal((B, S, Hq, d))
    k = rng.standard_normal((B, S, 1, d))
    v = rng.standard_normal((B, S, 1, d))
    return q, k, v


def test_padding_brute_force_all_patterns():
    """Exhaustive: every ar pattern (S <= 7) with random pad / FAST / EXPERT tags."""
    rng = np.random.default_rng(11)
    for S in range(1, 8):
        for bits in itertools.product([0, 1], repeat=S):
            ar = np.array(bits, dtype=np.uint8)
            seg = rng.integers(-1, 3, size=S)
            got = oracle.prefill_mask(ar, seg)[0]
            want = np.array(brute.mask(ar, seg))
            assert np.array_equal(got, want), (ar, seg)


def test_padding_equals_removing_the_tokens():
    """Pad tokens with ar = False anywhere in the sequence: every valid row's
    output equals the oracle on the sequence with the pad tokens deleted, and
    pad rows are 0 with lse = -inf."""
    rng = np.random.default_rng(12)
    for trial in range(20):
        S = int(rng.integers(2, 40))
        ar = (rng.random(S) < 0.25).astype(np.uint8)
        seg = rng.choice([OTHER, FAST, EXPERT], size=S)
        pad = rng.random(S) < 0.3
        ar[pad] = 0
        seg_p = np.where(pad, -1, seg)
        q, k, v = _rand_qkv(rng, 1, S)
        out, lse = oracle.prefill(q, k, v, ar, seg_p, scale=0.7)
        keep = ~pad
        if keep.any():
            o2, l2 = oracle.prefill(q[:, keep], k[:, keep], v[:, keep], ar[keep], seg[keep],
                                    scale=0.7)
            np.testing.assert_allclose(out[:, keep], o2, atol=1e-12)
            np.testing.assert_allclose(lse[:, keep], l2, atol=1e-12)
        assert np.all(out[:, pad] == 0.0)
        assert np.all(np.isneginf(lse[:, pad]))


def test_padding_matches_torch_sdpa_on_valid_rows():
    rng = np.random.default_rng(13)
    B, S, Hq, d = 2, 30, 4, 16
    ar = (rng.random((B, S)) < 0.2).astype(np.uint8)
    seg = np.where(rng.random((B, S)) < 0.25, -1, 0)
    q, k, v = _rand_qkv(rng, B, S, Hq, d)
    out, _ = oracle.prefill(q, k, v, ar, seg)
    M = oracle.prefill_mask(ar, seg)
    for b in range(B):
        rows = np.nonzero(M[b].any(axis=1))[0]
        qt = torch.from_numpy(q[b].transpose(1, 0, 2)[:, rows])          # [Hq, R, d]
        kt = torch.from_numpy(np.repeat(k[b].transpose(1, 0, 2), Hq, 0))  # [Hq, S, d]
        vt = torch.from_numpy(np.repeat(v[b].transpose(1, 0, 2), Hq, 0))
        mt = torch.from_numpy(M[b][rows])
        ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mt,
                                                               scale=1.0)
        np.testing.assert_allclose(out[b, rows].transpose(1, 0, 2), ref.numpy(), atol=1e-12)


def test_suffix_cache_padding_equals_removing_cache_rows():
    rng = np.random.default_rng(14)
    B, P, Sq, Hq, d = 3, 37, 9, 2, 8
    ar = np.zeros(Sq, np.uint8); ar[0] = 1; ar[1] = 1
    q = rng.standard_normal((B, Sq, Hq, d))
    ks = rng.standard_normal((B, Sq, 1, d)); vs = rng.standard_normal((B, Sq, 1, d))
    kc = rng.standard_normal((B, P, 1, d)); vc = rng.standard_normal((B, P, 1, d))
    valid = rng.random((B, P)) < 0.6
    valid[2] = False                         # a batch element whose cache is all padding
    out, lse = oracle.suffix(q, ks, vs, kc, vc, ar, cache_valid=valid)
    for b in range(B):
        keep = valid[b]
        o2, l2 = oracle.suffix(q[b:b + 1], ks[b:b + 1], vs[b:b + 1], kc[b:b + 1, keep],
                               vc[b:b + 1, keep], ar)
        np.testing.assert_allclose(out[b:b + 1], o2, atol=1e-12)
        np.testing.assert_allclose(lse[b:b + 1], l2, atol=1e-12)


def test_suffix_token_padding_rows_are_zero():
    rng = np.random.default_rng(15)
    B, P, Sq, Hq, d = 1, 12, 6, 2, 8
    ar = np.array([1, 1, 0, 0, 0, 0], np.uint8)
    seg = np.array([0, 0, 0, -1, 0, -1])
    q = rng.standard_normal((B, Sq, Hq, d))
    ks = rng.standard_normal((B, Sq, 1, d)); vs = rng.standard_normal((B, Sq, 1, d))
    kc = rng.standard_normal((B, P, 1, d)); vc = rng.standard_normal((B, P, 1, d))
    out, lse = oracle.suffix(q, ks, vs, kc, vc, ar, seg_suf=seg)
    assert np.all(out[:, seg < 0] == 0.0) and np.all(np.isneginf(lse[:, seg < 0]))
    keep = seg >= 0
    o2, _ = oracle.suffix(q[:, keep], ks[:, keep], vs[:, keep], kc, vc, ar[keep])
    np.testing.assert_allclose(out[:, keep], o2, atol=1e-12)


def test_planted_padding_mistakes_are_caught():
    """A padding term that forgets the query side, or the key side, fails."""
    rng = np.random.default_rng(16)
    S = 12
    ar = (rng.random(S) < 0.3).astype(np.uint8)
    seg = np.where(rng.random(S) < 0.3, -1, 0)
    seg[0] = -1
    seg[5] = -1
    good = oracle.prefill_mask(ar, seg)[0]
    base = oracle.prefill_mask(ar, None)[0]
    valid = seg >= 0
    keys_only = base & valid[None, :]
    rows_only = base & valid[:, None]
    brute_m = np.array(brute.mask(ar, seg))
    assert np.array_equal(good, brute_m)
    assert not np.array_equal(keys_only, brute_m)
    assert not np.array_equal(rows_only, brute_m)


# ---------------------------------------------------- pre/post steps (f3)
from oracle import prepost  # noqa: E402


def test_positions_follow_the_pages():
    """Prefix positions are cumsum(mask) - 1; suffix positions continue after
    the valid prefix tokens ('VLA 代码精读 - OpenPI & StarVLA', 1.6)."""
    pm = np.array([[1, 1, 1, 0, 0], [1, 0, 1, 1, 1]])
    assert prepost.positions(pm).tolist() == [[0, 1, 2, 2, 2], [0, 0, 1, 2, 3]]
    sm = np.ones((2, 3), np.uint8)
    assert prepost.positions(sm, pm).tolist() == [[3, 4, 5], [4, 5, 6]]


def _rope_pins_pass(rope):
    """The RoPE pins as one predicate of a rope function (x, pos) -> x'."""
    try:
        rng = np.random.default_rng(21)
        x = rng.standard_normal((2, 5, 3, 16))
        # position 0 is the identity
        assert np.allclose(rope(x, np.zeros((2, 5))), x, atol=0)
        # each (i, i + d/2) pair is rotated: the pair's norm is kept
        y = rope(x, rng.integers(0, 1000, (2, 5)))
        n_x = x[..., :8] ** 2 + x[..., 8:] ** 2
        n_y = y[..., :8] ** 2 + y[..., 8:] ** 2
        np.testing.assert_allclose(n_y, n_x, rtol=1e-12)
        # pair 0 turns by exactly pos radians (frequency base^0 = 1), counter-clockwise
        e = np.zeros((1, 1, 1, 16)); e[..., 0] = 1.0
        z = rope(e, np.array([[np.pi / 2]]))
        np.testing.assert_allclose(z[0, 0, 0, [0, 8]], [0.0, 1.0], atol=1e-15)
        # pair 4 of d = 16 has frequency 10000^(-8/16) = 1/100: position 50*pi
        # turns it by a quarter turn, while pair 0 turns by 50*pi (25 whole
        # turns: unchanged).
        e4 = np.zeros((1, 1, 1, 16)); e4[..., 4] = 1.0; e4[..., 0] = 1.0
        z4 = rope(e4, np.array([[50 * np.pi]]))
        np.testing.assert_allclose(z4[0, 0, 0, [4, 12]], [0.0, 1.0], atol=1e-12)
        np.testing.assert_allclose(z4[0, 0, 0, [0, 8]], [1.0, 0.0], atol=1e-12)
        # <rope(q, m), rope(k, n)> is a function of m - n, and not symmetric
        q = rng.standard_normal((1, 1, 1, 32))
        k = rng.standard_normal((1, 1, 1, 32))

        def score(m, n):
            return float(np.sum(rope(q, np.array([[m]])) * rope(k, np.array([[n]]))))
        for m, n in [(5, 2), (105, 102), (7, 7), (1000, 997)]:
            np.testing.assert_allclose(score(m, n), score(m - n, 0), atol=1e-9)
        assert abs(score(5, 2) - score(2, 5)) > 1e-3
    except AssertionError:
        return False
    return True


def test_rope_pins_hold_for_the_oracle():
    assert _rope_pins_pass(prepost.rope)


def _rope_variant(mistake):
    """prepost.rope with one planted mistake."""
    def rope(x, pos, base=10000.0):
        x = np.asarray(x, dtype=np.float64)
        d = x.shape[-1]
        half = d // 2
        i = np.arange(half, dtype=np.float64)
        inv = base ** ((-1.0 if mistake == "exponent" else -2.0) * i / d)
        if mistake == "growing":
            inv = base ** (2.0 * i / d)
        ang = np.asarray(pos, dtype=np.float64)[:, :, None, None] * inv
        c, s = np.cos(ang), np.sin(ang)
        if mistake == "cos_sin":
            c, s = s, c
        if mistake == "interleaved":
            x1, x2 = x[..., 0::2], x[..., 1::2]
            out = np.empty_like(x)
            out[..., 0::2], out[..., 1::2] = x1 * c - x2 * s, x2 * c + x1 * s
            return out
        x1, x2 = x[..., :half], x[..., half:]
        if mistake == "direction":
            return np.concatenate([x1 * c + x2 * s, x2 * c - x1 * s], axis=-1)
        return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)
    return rope


@pytest.mark.parametrize("mistake", ["direction", "exponent", "growing", "cos_sin",
                                     "interleaved"])
def test_rope_pins_catch_planted_mistakes(mistake):
    assert _rope_variant("none")(np.ones((1, 1, 1, 8)), np.array([[3]])).shape == (1, 1, 1, 8)
    assert _rope_pins_pass(_rope_variant("none"))
    assert not _rope_pins_pass(_rope_variant(mistake))


def test_positions_pin_catches_planted_mistakes():
    """An exclusive cumsum, a missing -1, or a prefix offset that counts the
    padded prefix tokens each break the worked example."""
    pm = np.array([[1, 1, 1, 0, 0], [1, 0, 1, 1, 1]])
    sm = np.ones((2, 3), np.uint8)
    want_pre = [[0, 1, 2, 2, 2], [0, 0, 1, 2, 3]]
    want_suf = [[3, 4, 5], [4, 5, 6]]
    exclusive = np.cumsum(pm, axis=-1) - pm
    assert exclusive.tolist() != want_pre
    assert np.cumsum(pm, axis=-1).tolist() != want_pre
    padded_count = np.cumsum(sm, axis=-1) - 1 + pm.shape[1]
    assert padded_count.tolist() != want_suf
    assert prepost.positions(pm).tolist() == want_pre
    assert prepost.positions(sm, pm).tolist() == want_suf


def test_euler_step_reaches_the_ode_solution():
    """dx/dt = v constant: ten steps of dt = -1/10 from t = 1 land on x - v."""
    rng = np.random.default_rng(23)
    x = rng.standard_normal((4, 50, 32))
    v = rng.standard_normal((4, 50, 32))
    y = x.copy()
    for _ in range(10):
        y = prepost.euler_step(y, v, -0.1)
    np.testing.assert_allclose(y, x - v, atol=1e-12)


# --------------------------------------------------------------- backward (f2)

from oracle import backward  # noqa: E402


def _fd_grads(q, k, v, ar, seg, dout, scale, eps=1e-6):
    """Central differences of L = sum(dout * prefill(q, k, v)) -- uses only the
    forward, so it is independent of the backward's formulas."""
    def loss(q_, k_, v_):
        out, _ = oracle.prefill(q_, k_, v_, ar, seg, scale=scale)
        return float(np.sum(dout * out))
    grads = []
    for which in range(3):
        xs = [q.copy(), k.copy(), v.copy()]
        g = np.zeros_like(xs[which])
        it = np.nditer(xs[which], flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            x0 = xs[which][idx]
            xs[which][idx] = x0 + eps
            lp = loss(*xs)
            xs[which][idx] = x0 - eps
            lm = loss(*xs)
            xs[which][idx] = x0
            g[idx] = (lp - lm) / (2 * eps)
        grads.append(g)
    return grads


def _tiny_case(seed=40):
    rng = np.random.default_rng(seed)
    B, S, Hq, Hkv, d = 2, 7, 4, 2, 3
    ar = [0, 0, 1, 1, 0, 1, 0]
    seg = [OTHER, OTHER, FAST, FAST, EXPERT, EXPERT, -1]        # a padded token at the end
    q = _rand((B, S, Hq, d), rng)
    k = _rand((B, S, Hkv, d), rng)
    v = _rand((B, S, Hkv, d), rng)
    dout = _rand((B, S, Hq, d), rng)
    return q, k, v, ar, seg, dout


def test_backward_equals_finite_differences():
    """Every element of dq, dk, dv against central differences of the forward,
    on a layout with a bidirectional prefix, a causal block, the expert <- FAST
    hole and a padded token."""
    q, k, v, ar, seg, dout = _tiny_case()
    dq, dk, dv = backward.prefill_backward(q, k, v, ar, dout, seg=seg, scale=0.7)
    fq, fk, fv = _fd_grads(q, k, v, ar, seg, dout, 0.7)
    np.testing.assert_allclose(dq, fq, atol=1e-8)
    np.testing.assert_allclose(dk, fk, atol=1e-8)
    np.testing.assert_allclose(dv, fv, atol=1e-8)
    # the padded token neither receives nor passes gradient
    assert np.all(dq[:, -1] == 0) and np.all(dk[:, -1] == 0) and np.all(dv[:, -1] == 0)


def test_backward_planted_transposed_mask_fails_finite_differences(monkeypatch):
    q, k, v, ar, seg, dout = _tiny_case()
    fq, fk, fv = _fd_grads(q, k, v, ar, seg, dout, 0.7)
    good = backward.prefill_mask
    monkeypatch.setattr(backward, "prefill_mask",
                        lambda *a, **kw: np.swapaxes(good(*a, **kw), 1, 2))
    dq, dk, dv = backward.prefill_backward(q, k, v, ar, dout, seg=seg, scale=0.7)
    assert np.abs(dq - fq).max() > 1e-3 or np.abs(dk - fk).max() > 1e-3


@pytest.mark.parametrize("Hq,Hkv,scale", [(8, 1, 1.0), (4, 2, 0.37)])
def test_backward_equals_torch_autograd_float64(Hq, Hkv, scale):
    """Library special case: autograd through float64 torch SDPA with the
    explicit mask, on a pi0-like layout (bidirectional prefix, state, actions)."""
    rng = np.random.default_rng(41)
    B, S, d = 2, 40, 16
    ar = [0] * 30 + [1] + [1] + [0] * 8
    q = _rand((B, S, Hq, d), rng)
    k = _rand((B, S, Hkv, d), rng)
    v = _rand((B, S, Hkv, d), rng)
    dout = _rand((B, S, Hq, d), rng)
    dq, dk, dv = backward.prefill_backward(q, k, v, ar, dout, scale=scale)
    M = torch.from_numpy(np.array(brute.mask(ar)))
    tq, tk, tv = (torch.from_numpy(x).permute(0, 2, 1, 3).clone().requires_grad_(True)
                  for x in (q, k, v))
    out = torch.nn.functional.scaled_dot_product_attention(
        tq, tk, tv, attn_mask=M, scale=scale, enable_gqa=True)
    out.backward(torch.from_numpy(dout).permute(0, 2, 1, 3))
    for mine, t in ((dq, tq), (dk, tk), (dv, tv)):
        np.testing.assert_allclose(mine, t.grad.permute(0, 2, 1, 3).numpy(), atol=1e-11)


def test_backward_closed_forms():
    """Softmax is invariant to adding one vector to every key a row sees, so
    the key gradients of each (batch, kv head) sum to zero; the value
    gradients sum to the sum of dO over the rows that see any key."""
    rng = np.random.default_rng(42)
    B, S, Hq, Hkv, d = 2, 23, 4, 1, 8
    ar = [0] * 10 + [1] * 5 + [1] + [0] * 7
    seg = [OTHER] * 10 + [FAST] * 5 + [EXPERT] * 7 + [-1]
    q = _rand((B, S, Hq, d), rng)
    k = _rand((B, S, Hkv, d), rng)
    v = _rand((B, S, Hkv, d), rng)
    dout = _rand((B, S, Hq, d), rng)
    dq, dk, dv = backward.prefill_backward(q, k, v, ar, dout, seg=seg, scale=0.5)
    np.testing.assert_allclose(dk.sum(axis=1), 0.0, atol=1e-12)
    live = np.array([s >= 0 for s in seg])
    np.testing.assert_allclose(dv.sum(axis=1)[:, 0], dout[:, live].sum(axis=(1, 2)), atol=1e-12)


def _backward_variant(mistake):
    """oracle.backward.prefill_backward with one planted mistake."""
    def bwd(q, k, v, ar, dout, seg=None, scale=1.0):
        B, S, Hq, d = q.shape
        group = Hq // k.shape[2]
        M = oracle.prefill_mask(ar, seg=seg, B=B)
        dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
        for b in range(B):
            for h in range(Hq):
                g = h // group
                s = scale * (q[b, :, h] @ k[b, :, g].T)
                P = oracle.softmax_probs(s, M[b])
                dP = dout[b, :, h] @ v[b, :, g].T
                D = 0.0 if mistake == "no_D" else (P * dP).sum(axis=1, keepdims=True)
                dS = P * (dP - D)
                dq[b, :, h] = (1.0 if mistake == "dq_scale" else scale) * (dS @ k[b, :, g])
                dk[b, :, g] += scale * ((dS if mistake == "dk_untransposed" else dS.T) @ q[b, :, h])
                dv[b, :, g] += (P if mistake == "dv_untransposed" else P.T) @ dout[b, :, h]
        return dq, dk, dv
    return bwd


@pytest.mark.parametrize("mistake", ["no_D", "dq_scale", "dk_untransposed", "dv_untransposed"])
def test_backward_pins_catch_planted_mistakes(mistake):
    """A dropped rowsum term, a missing scale, or an untransposed dS / P each
    disagree with the finite differences of the forward."""
    q, k, v, ar, seg, dout = _tiny_case()
    fd = _fd_grads(q, k, v, ar, seg, dout, 0.7)
    good = _backward_variant("none")(q, k, v, ar, dout, seg=seg, scale=0.7)
    for mine, ref in zip(good, fd):
        np.testing.assert_allclose(mine, ref, atol=1e-8)
    bad = _backward_variant(mistake)(q, k, v, ar, dout, seg=seg, scale=0.7)
    assert max(float(np.abs(m - r).max()) for m, r in zip(bad, fd)) > 1e-3
