"""pi_attn_suffix_noalloc: the suffix pass with its split-K scratch in the
library's fixed device buffer.  It must give the same result as
pi_attn_suffix with a caller workspace (within the bf16 tolerance), on two
calls in a row, and reject a shape whose scratch exceeds the buffer before
launching anything.  Collected last on purpose: it must pass after every
other GPU test has run in the same process, as well as alone.
"""

import ctypes

import numpy as np
import pytest
import torch

from vla_prefix_lm_b200 import workloads as W

TOL_BF16 = 2e-2


def _b():
    from vla_prefix_lm_b200 import binding
    return binding


def test_noalloc_rejects_oversize_on_the_host():
    from vla_prefix_lm_b200 import build
    build.build()
    b = _b()
    L = b.lib()
    cap = int(L.pi_attn_suffix_noalloc_capacity())
    assert cap == 16 << 20
    fake = ctypes.c_void_p(0x10000)       # never dereferenced: rejected before any launch
    # 18 batches x 32 tokens x 8 heads against a 2000-key cache: 36 CTAs, 4
    # splits, 4 x 4608 rows x 1032 B = 19.0 MB of partials > 16 MiB.
    d = b.PiAttnDesc(18, 32, 2000, 8, 1, 256, b.PI_BF16, 1.0, 0)
    assert L.pi_attn_suffix_workspace_bytes(ctypes.byref(d)) > cap
    rc = L.pi_attn_suffix_noalloc(ctypes.byref(d), fake, fake, fake, fake, fake, fake, fake,
                                  None)
    assert rc == b.PI_ERR_UNSUPPORTED
    assert L.pi_attn_suffix_noalloc(None, fake, fake, fake, fake, fake, fake, fake,
                                    None) == b.PI_ERR_ARG
    d0 = b.PiAttnDesc(0, 51, 816, 8, 1, 256, b.PI_BF16, 1.0, 0)
    assert L.pi_attn_suffix_noalloc(ctypes.byref(d0), None, None, None, None, None, None, None,
                                    None) == b.PI_OK


@pytest.mark.gpu
# (18, 816) needs the most scratch of the pi0 suffix shapes (two splits over
# 72 CTAs, about 15 MB of the 16 MiB); (32, 816) needs none (one split).
@pytest.mark.parametrize("B,P", [(2, 816), (1, 3000), (8, 816), (18, 816), (32, 816)])
def test_noalloc_matches_workspace_entry_point(B, P):
    b = _b()
    Sq, Hq, d = 51, 8, 256
    ar = torch.from_numpy(W.pi0_suffix_ar(Sq - 1)).cuda()
    qs, _ = W.draw((B, Sq, Hq, d), 71, d, "bf16")
    ks, _ = W.draw((B, Sq, 1, d), 72, d, "bf16")
    vs, _ = W.draw((B, Sq, 1, d), 73, d, "bf16")
    kc, _ = W.draw((B, P, 1, d), 74, d, "bf16")
    vc, _ = W.draw((B, P, 1, d), 75, d, "bf16")
    args = (qs.cuda(), ks.cuda(), vs.cuda(), kc.cuda(), vc.cuda(), ar)
    need = b.pi_attn_suffix_workspace_bytes(args[0], args[1], args[3], args[5])
    assert need <= int(b.lib().pi_attn_suffix_noalloc_capacity())
    ref = b.pi_attn_suffix(*args).float()
    outs = [torch.full_like(args[0], float("nan")) for _ in range(2)]
    for o in outs:                       # two calls in a row on the same buffer
        b.pi_attn_suffix_noalloc(*args, out=o)
    torch.cuda.synchronize()
    assert b.pi_attn_read_status() == b.PI_OK
    for o in outs:
        err = float((o.float() - ref).abs().max())
        assert np.isfinite(err) and err <= TOL_BF16, err
