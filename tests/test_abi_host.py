"""Host-side checks of the C ABI: the library loads, exports every symbol the
header declares, and rejects bad arguments before touching the GPU.

Nothing here launches a kernel; each call below fails validation (or is a
B == 0 no-op) before any CUDA runtime call is made, or is a host-only size
query (which at most asks the runtime for the device's SM count).
"""

import ctypes
import os
import re

import pytest

from conftest import ROOT


def _lib():
    from vla_prefix_lm_b200 import binding, build
    build.build()
    return binding, binding.lib()


def _declared():
    src = open(os.path.join(ROOT, "include", "pi_attn.h")).read()
    return sorted(set(re.findall(r"\b(pi_(?:attn|rope|euler)\w*)\s*\(", src)))


def test_header_declares_the_two_calls():
    names = _declared()
    assert "pi_attn_prefill" in names and "pi_attn_suffix" in names


def test_library_exports_every_declared_symbol():
    binding, L = _lib()
    for name in _declared():
        assert hasattr(L, name), name
    assert set(binding.EXPORTED) <= set(_declared())


def _desc(binding, **kw):
    d = dict(B=2, Sq=16, P=0, Hq=8, Hkv=1, d=256, dtype=binding.PI_BF16, softmax_scale=1.0,
             mask_batch_stride=0)
    d.update(kw)
    return binding.PiAttnDesc(**d)


FAKE = ctypes.c_void_p(0x10000)      # 16-byte aligned, never dereferenced
FAKE_MIS = ctypes.c_void_p(0x10008)  # misaligned


def _prefill(L, desc, q=FAKE, k=FAKE, v=FAKE, ar=FAKE, seg=None, out=FAKE, lse=None):
    return L.pi_attn_prefill(ctypes.byref(desc) if desc is not None else None,
                             q, k, v, ar, seg, out, lse, None)


def test_prefill_argument_errors():
    b, L = _lib()
    assert _prefill(L, None) == b.PI_ERR_ARG
    assert _prefill(L, _desc(b, Hq=0)) == b.PI_ERR_ARG
    assert _prefill(L, _desc(b, P=3)) == b.PI_ERR_ARG          # prefill has no cache
    assert _prefill(L, _desc(b, Hq=6, Hkv=4)) == b.PI_ERR_ARG
    assert _prefill(L, _desc(b, softmax_scale=float("nan"))) == b.PI_ERR_ARG
    assert _prefill(L, _desc(b, softmax_scale=0.0)) == b.PI_ERR_ARG
    assert _prefill(L, _desc(b, softmax_scale=-1.0)) == b.PI_ERR_ARG
    assert _prefill(L, _desc(b, mask_batch_stride=5)) == b.PI_ERR_ARG
    assert _prefill(L, _desc(b), q=None) == b.PI_ERR_ARG
    assert _prefill(L, _desc(b), ar=None) == b.PI_ERR_ARG
    assert _prefill(L, _desc(b), k=FAKE_MIS) == b.PI_ERR_ALIGN
    assert _prefill(L, _desc(b), out=FAKE_MIS) == b.PI_ERR_ALIGN


def test_prefill_unsupported_geometry():
    b, L = _lib()
    assert _prefill(L, _desc(b, d=128)) == b.PI_ERR_UNSUPPORTED
    assert _prefill(L, _desc(b, Hkv=2)) == b.PI_ERR_UNSUPPORTED
    assert _prefill(L, _desc(b, Hq=3, Hkv=1)) == b.PI_ERR_UNSUPPORTED
    assert _prefill(L, _desc(b, dtype=7)) == b.PI_ERR_UNSUPPORTED
    assert _prefill(L, _desc(b, Sq=16384)) == b.PI_ERR_UNSUPPORTED
    assert _prefill(L, _desc(b, dtype=b.PI_F32, d=48)) == b.PI_ERR_UNSUPPORTED


def test_empty_inputs_are_noops():
    b, L = _lib()
    assert _prefill(L, _desc(b, B=0), q=None, k=None, v=None, ar=None, out=None) == b.PI_OK
    assert _prefill(L, _desc(b, Sq=0), q=None, k=None, v=None, ar=None, out=None) == b.PI_OK
    d = _desc(b, Sq=0, P=10)
    assert L.pi_attn_suffix(ctypes.byref(d), None, None, None, None, None, None, None, None, 0,
                            None) == b.PI_OK


def test_suffix_argument_errors():
    b, L = _lib()
    d = _desc(b, P=816, Sq=51)
    args = [FAKE] * 7
    rc = L.pi_attn_suffix(ctypes.byref(d), *args[:3], None, None, args[5], args[6], None, 0,
                          None)
    assert rc == b.PI_ERR_ARG                                   # P > 0 needs a cache
    rc = L.pi_attn_suffix(ctypes.byref(d), *args[:3], FAKE_MIS, FAKE, FAKE, FAKE, None, 0, None)
    assert rc == b.PI_ERR_ALIGN
    d2 = _desc(b, P=-1)
    rc = L.pi_attn_suffix(ctypes.byref(d2), *args, None, 0, None)
    assert rc == b.PI_ERR_ARG


def test_workspace_query_is_host_only():
    b, L = _lib()
    d = _desc(b, B=32, Sq=51, P=816)
    n = L.pi_attn_suffix_workspace_bytes(ctypes.byref(d))
    assert n >= 0
    assert L.pi_attn_suffix_workspace_bytes(ctypes.byref(_desc(b, Hq=0))) == 0
    assert L.pi_attn_suffix_workspace_bytes(None) == 0


def _sm_count():
    """The SM count the library plans with: the device's, or 148 (a B200) with
    no device, as the library assumes when the runtime finds none."""
    import torch
    if torch.cuda.is_available():
        return torch.cuda.get_device_properties(0).multi_processor_count
    return 148


@pytest.mark.parametrize("B,S", [(8, 611), (16, 938), (2, 300), (1, 17), (3, 2000)])
def test_backward_workspace_follows_its_layout(B, S):
    """The bf16 backward's workspace is D (fp32 per row), P and dS (bf16
    [B, rows, Skp], Skp = S rounded up to 64), each 256-byte aligned, plus the
    dK / dV partials of 2 <= n_chunks <= (256-row tiles) row chunks when the
    rows are split: 2 * n_chunks * B * (256-key groups) * 256 * 256 fp32."""
    b, L = _lib()
    Hq = 8
    n = L.pi_attn_prefill_backward_workspace_bytes(ctypes.byref(_desc(b, B=B, Sq=S, Hq=Hq)))
    up = lambda x: (x + 255) // 256 * 256
    rows = S * Hq
    skp = (S + 63) // 64 * 64
    base = up(B * rows * 4) + 2 * up(B * rows * skp * 2)
    assert n >= base
    chunk = 2 * B * ((S + 255) // 256) * 256 * 256 * 4
    extra = n - base
    assert extra % chunk == 0, (n, base, chunk)
    n_chunks = extra // chunk
    assert n_chunks == 0 or 2 <= n_chunks <= (rows + 255) // 256
    if (B, S) == (8, 611):
        assert n == 138_011_392        # the pi0 figure the bench reports


def test_prefill_split_workspace_and_plan():
    """pi_attn_prefill_ws: one round of fp32 pieces (256 rows x (256 + 2)
    floats each) per SM pair for bf16 with a batch-shared mask, nothing
    otherwise; MM-DiT (532 units on 74 SM pairs: 14 in the last round) splits
    5 ways, pi0 and pi0.5 stay whole."""
    b, L = _lib()
    pairs = _sm_count() // 2
    q = lambda **kw: ctypes.byref(_desc(b, **kw))
    assert L.pi_attn_prefill_workspace_bytes(q(B=4, Sq=4250)) == pairs * 256 * 258 * 4
    assert L.pi_attn_prefill_workspace_bytes(q(B=4, Sq=4250, dtype=b.PI_F32)) == 0
    assert L.pi_attn_prefill_workspace_bytes(q(B=4, Sq=4250, mask_batch_stride=4250)) == 0
    assert L.pi_attn_prefill_tail_splits(q(B=8, Sq=611)) == 1
    assert L.pi_attn_prefill_tail_splits(q(B=16, Sq=938)) == 1
    if pairs == 74:
        assert L.pi_attn_prefill_tail_splits(q(B=4, Sq=4250)) == 5


def test_suffix_workspace_and_noalloc_capacity():
    """Split-K suffix scratch is a whole number s of partial sets (B x Sq*Hq
    rows of 256 + 2 fp32), 2 <= s <= 8, and s x (CTA pairs per element) x B
    never exceeds the SM pairs; none when the batch fills the SMs (the pi0
    suffix step, B = 32) or for a few-row suffix (the decode kernel).  At the
    pi0 suffix shape every batch size and cache length fits the no-alloc
    buffer."""
    b, L = _lib()
    pairs = _sm_count() // 2
    cap = L.pi_attn_suffix_noalloc_capacity()
    assert cap == 16 << 20
    q = lambda **kw: ctypes.byref(_desc(b, **kw))
    assert L.pi_attn_suffix_workspace_bytes(q(B=1, Sq=1, P=3000)) == 0
    if pairs == 74:
        assert L.pi_attn_suffix_workspace_bytes(q(B=32, Sq=51, P=816)) == 0
    for Bn in list(range(1, 40)) + [64, 128]:
        for P in (1, 128, 816, 3000, 16000):
            n = L.pi_attn_suffix_workspace_bytes(q(B=Bn, Sq=51, P=P))
            part = Bn * 51 * 8 * 258 * 4
            assert n % part == 0
            s = n // part
            assert s == 0 or 2 <= s <= 8
            assert s * 2 * Bn <= pairs          # two CTA pairs per element (408 rows)
            assert n <= cap, (Bn, P, n)


def test_split_prefill_and_noalloc_argument_errors():
    """Host-side rejections, before anything is enqueued: a split-prefill
    workspace smaller than the query's size (PI_ERR_ARG) or misaligned
    (PI_ERR_ALIGN); a no-alloc suffix whose split-K scratch would exceed the
    fixed buffer (PI_ERR_UNSUPPORTED: B = 1, 512 tokens x 8 heads against a
    3000-key cache needs 4 splits x 4096 rows x 1032 B = 16.1 MiB)."""
    b, L = _lib()
    d = _desc(b, B=4, Sq=4250)
    need = L.pi_attn_prefill_workspace_bytes(ctypes.byref(d))
    assert need > 0
    args = (FAKE, FAKE, FAKE, FAKE, None, FAKE, None)
    rc = L.pi_attn_prefill_ws(ctypes.byref(d), *args, FAKE, ctypes.c_size_t(need - 16), None)
    assert rc == b.PI_ERR_ARG
    rc = L.pi_attn_prefill_ws(ctypes.byref(d), *args, FAKE_MIS, ctypes.c_size_t(need), None)
    assert rc == b.PI_ERR_ALIGN
    big = _desc(b, B=1, Sq=512, P=3000)
    if _sm_count() != 148:
        return                      # the split count (and so the size) follows the SM count
    assert L.pi_attn_suffix_workspace_bytes(ctypes.byref(big)) > L.pi_attn_suffix_noalloc_capacity()
    rc = L.pi_attn_suffix_noalloc(ctypes.byref(big), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                  None)
    assert rc == b.PI_ERR_UNSUPPORTED


def test_status_strings_and_wait_limit():
    b, L = _lib()
    for code in range(6):
        assert b.status_string(code).startswith("PI_")
    prev = b.pi_attn_set_wait_limit(12345)
    assert b.pi_attn_set_wait_limit(0) == 12345
    assert b.pi_attn_set_wait_limit(prev) == 1 << 31


@pytest.mark.parametrize("value,expect", [("777", 777), ("abc", 1 << 31), ("0", 1 << 31)])
def test_watchdog_env_sets_the_initial_wait_limit(value, expect):
    """PIATTN_WATCHDOG_CYCLES (a positive integer) is the wait bound in force
    when the library loads; anything else leaves the default."""
    import subprocess
    import sys
    _lib()   # built
    code = ("import sys; sys.path.insert(0, %r)\n"
            "from vla_prefix_lm_b200 import binding\n"
            "print(binding.pi_attn_set_wait_limit(5))\n" % ROOT)
    env = dict(os.environ, PIATTN_WATCHDOG_CYCLES=value)
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr
    assert int(r.stdout.strip().splitlines()[-1]) == expect


def test_debug_mask_argument_errors():
    b, L = _lib()
    d = _desc(b)
    assert L.pi_attn_debug_mask(ctypes.byref(d), 2, FAKE, None, FAKE, None) == b.PI_ERR_ARG
    assert L.pi_attn_debug_mask(ctypes.byref(d), 0, None, None, FAKE, None) == b.PI_ERR_ARG
    d1 = _desc(b, P=4)
    assert L.pi_attn_debug_mask(ctypes.byref(d1), 1, FAKE, FAKE, FAKE, None) == b.PI_ERR_ARG


def test_product_path_has_no_oracle_import():
    """The package never imports the oracle (test infrastructure only)."""
    pkg = os.path.join(ROOT, "vla_prefix_lm_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                txt = open(os.path.join(dirpath, f), encoding="utf-8").read()
                assert "import oracle" not in txt and "from oracle" not in txt, f


def _rope_desc(binding, **kw):
    d = dict(B=2, S=16, P=0, Hq=8, Hkv=1, d=256, dtype=binding.PI_BF16, base=10000.0,
             mask_batch_stride=0, prefix_batch_stride=0)
    d.update(kw)
    return binding.PiRopeDesc(**d)


def test_rope_and_euler_argument_errors():
    b, L = _lib()
    rope = lambda desc, q=FAKE, k=FAKE, tm=FAKE, pm=None: L.pi_rope_inplace(
        ctypes.byref(desc) if desc is not None else None, q, k, tm, pm, None, None)
    assert rope(None) == b.PI_ERR_ARG
    assert rope(_rope_desc(b, d=250)) == b.PI_ERR_UNSUPPORTED
    assert rope(_rope_desc(b, d=512)) == b.PI_ERR_UNSUPPORTED
    assert rope(_rope_desc(b, base=1.0)) == b.PI_ERR_ARG
    assert rope(_rope_desc(b, P=4)) == b.PI_ERR_ARG            # a prefix needs its mask
    assert rope(_rope_desc(b), q=FAKE_MIS) == b.PI_ERR_ALIGN
    assert rope(_rope_desc(b), tm=None) == b.PI_ERR_ARG
    assert rope(_rope_desc(b, B=0), q=None, tm=None) == b.PI_OK
    eu = L.pi_euler_update
    assert eu(FAKE, FAKE, 7, ctypes.c_float(0.1), 16, None) == b.PI_ERR_UNSUPPORTED
    assert eu(FAKE, FAKE, b.PI_F32, ctypes.c_float(float("nan")), 16, None) == b.PI_ERR_ARG
    assert eu(FAKE_MIS, FAKE, b.PI_F32, ctypes.c_float(0.1), 16, None) == b.PI_ERR_ALIGN
    assert eu(None, None, b.PI_F32, ctypes.c_float(0.1), 0, None) == b.PI_OK


def test_rope_rejects_heads_beyond_shared_memory():
    b, L = _lib()
    desc = _rope_desc(b, Hq=200, d=256, dtype=b.PI_F32)   # 201 KB per token
    assert L.pi_rope_inplace(ctypes.byref(desc), FAKE, FAKE, FAKE, None, None, None) == \
        b.PI_ERR_UNSUPPORTED


def test_backward_argument_errors():
    """Every host-side check of pi_attn_prefill_backward, before any launch."""
    b, L = _lib()
    ws = L.pi_attn_prefill_backward_workspace_bytes
    need = ws(ctypes.byref(_desc(b)))
    # bf16 / one KV head / d = 256 runs on tensor cores: D (B x rows fp32) and the
    # bf16 P and dS tiles (B x rows x S rounded up to 64 keys); one row tile, so the
    # dK/dV pass needs no partial sums.
    rows = 16 * 8
    assert need == 2 * rows * 4 + 2 * (2 * rows * 64 * 2)
    # the SIMT path (fp32): codes (rounded to 256) + D
    assert ws(ctypes.byref(_desc(b, dtype=b.PI_F32))) == 256 + 2 * rows * 4

    def bwd(desc, ws_bytes=need, ptrs=None, seg=None, lse=FAKE):
        p = dict(q=FAKE, k=FAKE, v=FAKE, ar=FAKE, out=FAKE, dout=FAKE, dq=FAKE, dk=FAKE,
                 dv=FAKE, w=FAKE)
        p.update(ptrs or {})
        return L.pi_attn_prefill_backward(
            ctypes.byref(desc) if desc is not None else None, p["q"], p["k"], p["v"], p["ar"],
            seg, p["out"], lse, p["dout"], p["dq"], p["dk"], p["dv"], p["w"], ws_bytes, None)

    assert bwd(None) == b.PI_ERR_ARG
    assert bwd(_desc(b, P=3)) == b.PI_ERR_ARG
    assert bwd(_desc(b, Hq=6, Hkv=4)) == b.PI_ERR_ARG
    assert bwd(_desc(b, softmax_scale=0.0)) == b.PI_ERR_ARG
    assert bwd(_desc(b, mask_batch_stride=3)) == b.PI_ERR_ARG
    assert bwd(_desc(b, d=48)) == b.PI_ERR_UNSUPPORTED
    assert bwd(_desc(b, d=512)) == b.PI_ERR_UNSUPPORTED
    assert bwd(_desc(b, dtype=7)) == b.PI_ERR_UNSUPPORTED
    assert bwd(_desc(b, Sq=16384)) == b.PI_ERR_UNSUPPORTED
    assert bwd(_desc(b), lse=None) == b.PI_ERR_ARG
    assert bwd(_desc(b), ws_bytes=need - 1) == b.PI_ERR_ARG
    for name in ("q", "dout", "dq", "dk", "dv", "w"):
        assert bwd(_desc(b), ptrs={name: FAKE_MIS}) == b.PI_ERR_ALIGN, name
        assert bwd(_desc(b), ptrs={name: None}) == b.PI_ERR_ARG, name
    assert bwd(_desc(b), seg=ctypes.c_void_p(0x10002)) == b.PI_ERR_ALIGN
    assert bwd(_desc(b, B=0), ptrs={"q": None}) == b.PI_OK
    # fp32 and grouped heads are in range of the backward (unlike the bf16 forward)
    assert ws(ctypes.byref(_desc(b, dtype=b.PI_F32, Hq=4, Hkv=2, d=64))) > 0


def test_plain_c_client_compiles_links_and_runs():
    """The header is plain C (C11, -Wall -Wextra -Werror) and the library links
    without torch or C++: a small C client of the host-side paths runs clean."""
    import shutil
    import subprocess
    _lib()                                              # builds the library
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    out_dir = os.path.join(ROOT, "_build")
    os.makedirs(out_dir, exist_ok=True)
    exe = os.path.join(out_dir, "abi_check")
    libdir = os.path.join(ROOT, "vla_prefix_lm_b200")
    subprocess.run([gcc, "-std=c11", "-Wall", "-Wextra", "-Werror",
                    "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c_abi", "abi_check.c"),
                    "-L", libdir, "-lpiattn", f"-Wl,-rpath,{libdir}", "-o", exe], check=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    assert "c abi ok" in r.stdout
