"""Host-side logic outside the kernels: the bench's pair counter, the
multi-rank timing plumbing (2 gloo ranks on CPU), and the launcher checks."""

import os
import socket
import subprocess
import sys

import numpy as np
import pytest

import oracle
from oracle import counts
from vla_prefix_lm_b200 import dist
from vla_prefix_lm_b200 import workloads as W

from conftest import ROOT

sys.path.insert(0, ROOT)
import bench  # noqa: E402


@pytest.mark.parametrize("cfg", [1, 2, 4])
def test_pair_counter_matches_oracle_mask(cfg):
    w = W.workload(cfg)
    seg = None if w.seg is None else np.array(w.seg)
    M = oracle.prefill_mask(np.array(w.ar), seg)
    assert bench.visible_pairs_per_bh(w.ar, seg) == counts.visible_pairs(M)


def test_pair_counter_suffix_matches_oracle_mask():
    w = W.workload(3)
    M = oracle.suffix_mask(np.array(w.ar), w.P)
    assert bench.visible_pairs_per_bh(w.ar, P=w.P) == counts.visible_pairs(M)


def test_pair_counter_fuzz():
    rng = np.random.default_rng(3)
    for _ in range(100):
        S = int(rng.integers(1, 200))
        ar, seg = W.random_layout(S, rng, with_seg=True)
        assert bench.visible_pairs_per_bh(ar, seg) == counts.visible_pairs(
            oracle.prefill_mask(ar, seg))


def test_workload_work_figures():
    """Unmasked pairs per call of the pi0 / pi0.5 / MM-DiT / suffix workloads."""
    per_call = {}
    for cfg in (2, 3, 4, 5):
        w = W.workload(cfg)
        per_call[cfg] = bench.visible_pairs_per_bh(w.ar, None if w.seg is None else w.seg,
                                                   P=w.P) * w.B * w.Hq
    assert per_call[2] == 22_061_504
    assert per_call[3] == 11_306_752
    assert per_call[4] == 99_518_976
    assert per_call[5] == 578_000_000


_WORKER = r"""
import os, sys
sys.path.insert(0, {root!r})
from vla_prefix_lm_b200 import dist
rank, ws, _ = dist.world()
assert dist.init(backend="gloo", timeout_s=60)
dist.barrier()
m = dist.max_over_ranks(10.0 + rank)
s = dist.sum_over_ranks(1.0)
tot = dist.sum_over_ranks(8)
dist.shutdown()
print("RESULT", rank, m, s, tot, flush=True)
"""


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_rank_gloo_plumbing():
    port = _free_port()
    procs = []
    for r in range(2):
        env = dict(os.environ, RANK=str(r), WORLD_SIZE="2", LOCAL_RANK=str(r),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, "-c", _WORKER.format(root=ROOT)], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = [p.communicate(timeout=120) for p in procs]
    for p, (o, e) in zip(procs, outs):
        assert p.returncode == 0, e
    res = sorted(line.split()[1:] for o, _ in outs for line in o.splitlines()
                 if line.startswith("RESULT"))
    assert [r[0] for r in res] == ["0", "1"]
    for r in res:
        assert float(r[1]) == 11.0      # max over ranks
        assert float(r[2]) == 2.0       # sum over ranks
        assert float(r[3]) == 16.0      # each rank's 8 batch elements, summed


def test_reference_arm_runs_on_cpu():
    """bench.py --impl reference: the oracle leg alone, one JSON line."""
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "2", "--warmup", "1"], capture_output=True, text=True,
                       timeout=300, env=dict(os.environ, CUDA_VISIBLE_DEVICES=""))
    assert r.returncode == 0, r.stderr
    import json
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_reference_arm_nonzero_rank_exits_quietly():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "0"], capture_output=True,
                       text=True, timeout=120,
                       env=dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1"))
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_bench_two_rank_plumbing_end_to_end():
    """bench.py under torch.distributed.run with 2 gloo ranks on CPU: the same
    barrier / max-over-ranks / whole-job value arithmetic as the GPU arm; rank
    0 alone prints one line, with n_gpus == 2 and the slower rank's time."""
    import json
    port = _free_port()
    r = subprocess.run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
                        "--nproc-per-node=2", "--master-addr", "127.0.0.1", "--master-port",
                        str(port), os.path.join(ROOT, "bench.py"), "--plumbing-check",
                        "--gpus", "2", "--steps", "4", "--warmup", "3"],
                       capture_output=True, text=True, timeout=300,
                       env=dict(os.environ, CUDA_VISIBLE_DEVICES=""))
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["n_gpus"] == 2 and line["steps"] == 4
    assert line["max_rank_ms"] >= line["rank_ms"]          # rank 1 is slower by design
    assert abs(line["value"] - 2 * 1000 * 4 / (line["max_rank_ms"] / 1e3)) < 1e-6 * line["value"]


def test_bench_gpus_mismatch_is_an_error():
    """--gpus N with a launcher that started a different number of ranks."""
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "4",
                        "--steps", "1", "--warmup", "3"], capture_output=True, text=True,
                       timeout=120, env=dict(os.environ, RANK="0", WORLD_SIZE="2",
                                             LOCAL_RANK="0", CUDA_VISIBLE_DEVICES=""))
    assert r.returncode != 0 and "WORLD_SIZE=2" in r.stderr


def test_bench_case_names_cover_profiles():
    """Every --case a profile summary names exists in bench.py."""
    import glob
    import re
    for f in glob.glob(os.path.join(ROOT, "profiles", "*.md")):
        for m in re.findall(r"--case (\w+)", open(f).read()):
            assert m in bench.CASES, (f, m)
