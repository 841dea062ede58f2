"""Seeded synthetic inputs for the joint-attention workloads.

This module holds no attention arithmetic: it only spells out the token
layouts (ar_mask / segment-id patterns) of each workload and draws the q, k, v
tensors.  Both the CUDA path and the CPU oracle consume what it returns, so it
imports neither.

Token layouts follow the pages:

* pi0 prefix = images + text, ar_mask all False; suffix = 1 state token (True)
  then the action tokens, the first True and the rest False
  ("VLA 代码精读 - OpenPI & StarVLA", 1.2, Prefix-Suffix 注意力掩码).
* pi0.5 = [prefix (3 x 256 patches + 48 text + 8 discrete-state tokens, False) |
  FAST (64 tokens, all True) | expert chunk (50 tokens: True, then False)] with
  segment ids 0 / 1 / 2 ("π0.5 vs MM-DiT joint attention", π0.5:三段).
* MM-DiT = 4096 patches + 154 text, all False ("π0.5 vs MM-DiT joint
  attention", 对照与代价).

Values: q, k, v are iid N(0, 1) * d**-0.25 drawn in float64 from numpy's
PCG64 and then rounded to the workload's dtype (bf16 round-to-nearest-even
via torch, or fp32); the float64 copy handed to the oracle is the rounded
value, upcast.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

OTHER, FAST, EXPERT = 0, 1, 2


def pi0_suffix_ar(n_actions: int) -> np.ndarray:
    """state (True), actions[0] (True), actions[1:] (False)."""
    return np.array([1, 1] + [0] * (n_actions - 1), dtype=np.uint8)


@dataclass(frozen=True)
class Workload:
    name: str
    mode: str            # "prefill" or "suffix"
    B: int
    Hq: int
    Hkv: int
    d: int
    dtype: str           # "bf16" or "f32"
    ar: tuple            # prefill: the full ar_mask; suffix: the suffix ar_mask
    seg: tuple | None = None
    P: int = 0           # suffix mode: cached prefix length
    calls: int = 1       # repeated calls (suffix: Euler steps; MM-DiT: 28 steps)
    scale: float = 1.0
    note: str = ""
    extra: dict = field(default_factory=dict)

    @property
    def Sq(self) -> int:
        return len(self.ar)

    @property
    def Sk(self) -> int:
        return self.P + len(self.ar) if self.mode == "suffix" else len(self.ar)


def _ar(parts):
    return tuple(int(x) for x in np.concatenate([np.asarray(p, np.uint8) for p in parts]))


def tiny_f32() -> Workload:
    ar = _ar([np.zeros(32 + 8), pi0_suffix_ar(8)])
    return Workload("tiny_joint_prefill_f32", "prefill", B=1, Hq=2, Hkv=1, d=64,
                    dtype="f32", ar=ar,
                    note="32 image + 8 text (False); state True; 8 actions (True, False x7); S=49")


def pi0_prefill() -> Workload:
    ar = _ar([np.zeros(2 * 256 + 48), pi0_suffix_ar(50)])
    return Workload("pi0_joint_prefill", "prefill", B=8, Hq=8, Hkv=1, d=256,
                    dtype="bf16", ar=ar,
                    note="2 cameras x 256 patches + 48 text (False); state True; 50 actions; S=611")


def pi0_suffix() -> Workload:
    return Workload("pi0_euler_suffix", "suffix", B=32, Hq=8, Hkv=1, d=256,
                    dtype="bf16", ar=tuple(int(x) for x in pi0_suffix_ar(50)), P=3 * 256 + 48,
                    calls=10,
                    note="prefix KV cache 816 tokens; 10 Euler steps x 51 suffix tokens")


def pi05_prefill() -> Workload:
    n_pre, n_fast, n_exp = 3 * 256 + 48 + 8, 64, 50
    ar = _ar([np.zeros(n_pre), np.ones(n_fast), [1], np.zeros(n_exp - 1)])
    seg = tuple([OTHER] * n_pre + [FAST] * n_fast + [EXPERT] * n_exp)
    return Workload("pi05_three_segment_prefill", "prefill", B=16, Hq=8, Hkv=1, d=256,
                    dtype="bf16", ar=ar, seg=seg,
                    note="824 prefix (False) | 64 FAST (True) | 50 expert (True, False x49); S=938")


def mmdit() -> Workload:
    ar = tuple([0] * (4096 + 154))
    return Workload("mmdit_full_bidirectional", "prefill", B=4, Hq=8, Hkv=1, d=256,
                    dtype="bf16", ar=ar, calls=28,
                    note="4096 patches + 154 text, all False; 28 calls with fresh inputs")


WORKLOADS = {1: tiny_f32, 2: pi0_prefill, 3: pi0_suffix, 4: pi05_prefill, 5: mmdit}


def workload(i: int) -> Workload:
    return WORKLOADS[i]()


# ---------------------------------------------------------------- sampling

def seed_for(config: int, call: int = 0) -> int:
    """1000 * config + call; the suffix workload's prefix cache uses 1000 * config + 999."""
    return 1000 * config + call


def _round(x64: np.ndarray, dtype: str):
    """Round float64 draws to the workload dtype; return (device-ready tensor, float64 copy)."""
    t = torch.from_numpy(np.ascontiguousarray(x64))
    if dtype == "bf16":
        t = t.to(torch.bfloat16)
    elif dtype == "f32":
        t = t.to(torch.float32)
    else:
        raise ValueError(dtype)
    return t, t.to(torch.float64).numpy()


def draw(shape, seed: int, d: int, dtype: str, std_scale: float | None = None):
    """iid N(0,1) * d**-0.25 (or * std_scale), rounded to ``dtype``."""
    rng = np.random.Generator(np.random.PCG64(seed))
    s = d ** -0.25 if std_scale is None else std_scale
    return _round(rng.standard_normal(shape) * s, dtype)


def device_draw(shape, seed: int, d: int, dtype: str, device, std_scale: float | None = None):
    """iid N(0,1) * d**-0.25 (or * std_scale) drawn on ``device`` from a seeded
    torch generator and rounded to ``dtype``.  For timing runs that need many
    fresh input sets quickly; parity tests use ``draw``, whose float64 values
    the oracle also receives."""
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    s = d ** -0.25 if std_scale is None else std_scale
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32) * s
    return x.to(torch.bfloat16 if dtype == "bf16" else torch.float32)


@dataclass
class PrefillInputs:
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    ar: torch.Tensor          # uint8 [S]
    seg: torch.Tensor | None  # int32 [S]
    q64: np.ndarray
    k64: np.ndarray
    v64: np.ndarray


def prefill_inputs(w: Workload, seed: int, B: int | None = None) -> PrefillInputs:
    """q [B,S,Hq,d], k/v [B,S,Hkv,d] drawn from three consecutive streams of ``seed``."""
    B = w.B if B is None else B
    S = w.Sq
    q, q64 = draw((B, S, w.Hq, w.d), seed * 4 + 0, w.d, w.dtype)
    k, k64 = draw((B, S, w.Hkv, w.d), seed * 4 + 1, w.d, w.dtype)
    v, v64 = draw((B, S, w.Hkv, w.d), seed * 4 + 2, w.d, w.dtype)
    ar = torch.tensor(w.ar, dtype=torch.uint8)
    seg = None if w.seg is None else torch.tensor(w.seg, dtype=torch.int32)
    return PrefillInputs(q, k, v, ar, seg, q64, k64, v64)


@dataclass
class SuffixInputs:
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    ar: torch.Tensor          # uint8 [Sq]
    q64: np.ndarray
    k64: np.ndarray
    v64: np.ndarray


@dataclass
class CacheInputs:
    k: torch.Tensor
    v: torch.Tensor
    k64: np.ndarray
    v64: np.ndarray


def cache_inputs(w: Workload, seed: int, B: int | None = None) -> CacheInputs:
    """The prefix KV cache [B, P, Hkv, d] (computed once per control step)."""
    B = w.B if B is None else B
    k, k64 = draw((B, w.P, w.Hkv, w.d), seed * 4 + 0, w.d, w.dtype)
    v, v64 = draw((B, w.P, w.Hkv, w.d), seed * 4 + 1, w.d, w.dtype)
    return CacheInputs(k, v, k64, v64)


def suffix_inputs(w: Workload, seed: int, B: int | None = None,
                  std_scale: float | None = None) -> SuffixInputs:
    """One Euler step's fresh suffix q [B,Sq,Hq,d] and k/v [B,Sq,Hkv,d]."""
    B = w.B if B is None else B
    Sq = w.Sq
    q, q64 = draw((B, Sq, w.Hq, w.d), seed * 4 + 0, w.d, w.dtype, std_scale)
    k, k64 = draw((B, Sq, w.Hkv, w.d), seed * 4 + 1, w.d, w.dtype, std_scale)
    v, v64 = draw((B, Sq, w.Hkv, w.d), seed * 4 + 2, w.d, w.dtype, std_scale)
    ar = torch.tensor(w.ar, dtype=torch.uint8)
    return SuffixInputs(q, k, v, ar, q64, k64, v64)


def random_layout(S: int, rng: np.random.Generator, with_seg: bool):
    """A random ar_mask (and segment ids) for fuzzing: runs of False broken by Trues."""
    ar = (rng.random(S) < rng.choice([0.02, 0.1, 0.3, 0.7])).astype(np.uint8)
    seg = None
    if with_seg:
        seg = rng.integers(0, 3, size=S).astype(np.int32)
    return ar, seg
