"""Seeded synthetic inputs for split-KV (replicated prefix + suffix) attention.

This module is shared by the tests, the benchmark and the CPU oracle checks.
It holds no attention arithmetic: it only draws tensors, describes the
workload shapes and overwrites padding regions with poison values.

Recipe (one per workload): a CPU ``torch.Generator`` seeded with the
workload's seed draws, in this fixed order, ``q``, ``k_prefix``, ``v_prefix``,
``k_suffix``, ``v_suffix`` with ``torch.randn`` in fp32; each draw is
multiplied by its standard deviation and rounded to bf16 (round to nearest
even).  Layout is BSND: ``[batch, seq, heads, head_dim]``.  Tail padding is
whatever the generator drew there (N(0,1) garbage) unless ``poison_pad``
overwrites it.

The shapes follow the joint/cross attention workloads the pages describe:
replicated text prefix (333 or 512 tokens) plus image/video suffix, sequence-
parallel tail padding from the even-shard plan (4429 -> 4432), GQA with
4 query heads per KV head, and a short-KV cross-attention case.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional, Sequence

import torch

__all__ = [
    "Workload",
    "WORKLOADS",
    "get",
    "make_inputs",
    "poison_pad",
    "random_workload",
    "PackedWorkload",
    "PACKED",
    "make_packed",
]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    D: int
    Sq: int
    Sp: int
    Ss: int
    real_len: Optional[tuple]  # per batch row; None => all Sp+Ss keys valid
    seed: int
    qk_std: float = 1.0
    v_std: float = 1.0
    description: str = ""

    @property
    def Skv(self) -> int:
        return self.Sp + self.Ss

    def real_lens(self) -> List[int]:
        if self.real_len is None:
            return [self.Skv] * self.B
        return list(self.real_len)


WORKLOADS: Dict[str, Workload] = {
    w.name: w
    for w in [
        Workload(
            "tiny", B=1, Hq=2, Hkv=2, D=64, Sq=64, Sp=16, Ss=64, real_len=None,
            seed=0, description="tiny parity case: 16 prefix + 64 suffix keys, no pad",
        ),
        Workload(
            "cosmos_self", B=1, Hq=16, Hkv=16, D=128, Sq=4096, Sp=512, Ss=4096,
            real_len=None, seed=1, qk_std=1.0 / math.sqrt(2.0), v_std=1.0,
            description="Cosmos-like self attention: 512 replicated text keys + 4096 video keys",
        ),
        Workload(
            "tail_padded_joint", B=2, Hq=24, Hkv=24, D=128, Sq=4432, Sp=0, Ss=4432,
            real_len=(4429, 4429), seed=2,
            description="joint attention, 333 text + 4096 image tokens padded to 4432 (3 pad at tail)",
        ),
        Workload(
            "cross_short_kv", B=1, Hq=16, Hkv=16, D=128, Sq=32760, Sp=512, Ss=512,
            real_len=None, seed=3,
            description="cross attention: 32760 video queries over 512 + 512 keys",
        ),
        Workload(
            "long_gqa", B=1, Hq=32, Hkv=8, D=128, Sq=25088, Sp=512, Ss=24576,
            real_len=(25048,), seed=4,
            description="long GQA self attention: 512 + 24576 keys, last 40 suffix tokens are pad",
        ),
        Workload(
            "pad_heavy", B=1, Hq=16, Hkv=16, D=128, Sq=8192, Sp=512, Ss=8192,
            real_len=(4608,), seed=6,
            description="pad-exclusion evidence: the last 4096 of 8192 suffix keys are tail pad "
                        "(DRAM reads must be Q + the valid K/V only)",
        ),
    ]
}

# The order in which workloads are listed (index 0 = tiny, 1 = cosmos_self ...).
ORDER = list(WORKLOADS.keys())


def get(name_or_index) -> Workload:
    if isinstance(name_or_index, int):
        return WORKLOADS[ORDER[name_or_index]]
    return WORKLOADS[name_or_index]


def _draw(gen: torch.Generator, shape: Sequence[int], std: float) -> torch.Tensor:
    x = torch.randn(*shape, generator=gen, dtype=torch.float32)
    if std != 1.0:
        x = x * std
    return x.to(torch.bfloat16)


def make_inputs(w: Workload, seed: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """Draw q, k_prefix, v_prefix, k_suffix, v_suffix on the CPU as bf16."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(w.seed if seed is None else seed)
    out = {}
    out["q"] = _draw(gen, (w.B, w.Sq, w.Hq, w.D), w.qk_std)
    out["k_prefix"] = _draw(gen, (w.B, w.Sp, w.Hkv, w.D), w.qk_std)
    out["v_prefix"] = _draw(gen, (w.B, w.Sp, w.Hkv, w.D), w.v_std)
    out["k_suffix"] = _draw(gen, (w.B, w.Ss, w.Hkv, w.D), w.qk_std)
    out["v_suffix"] = _draw(gen, (w.B, w.Ss, w.Hkv, w.D), w.v_std)
    return out


def poison_pad(
    t: Dict[str, torch.Tensor],
    Sp: int,
    real_len: Sequence[int],
    q_valid: Optional[Sequence[int]],
    value: float,
) -> Dict[str, torch.Tensor]:
    """Return copies whose tail-pad keys/values (and pad query rows) hold ``value``.

    Key position j (in prefix-then-suffix order) is pad when j >= real_len[b];
    query row i is pad when i >= q_valid[b].
    """
    out = {k: v.clone() for k, v in t.items()}
    for b, n in enumerate(real_len):
        if n < Sp:
            out["k_prefix"][b, n:] = value
            out["v_prefix"][b, n:] = value
            out["k_suffix"][b, :] = value
            out["v_suffix"][b, :] = value
        else:
            out["k_suffix"][b, n - Sp:] = value
            out["v_suffix"][b, n - Sp:] = value
        if q_valid is not None:
            out["q"][b, q_valid[b]:] = value
    return out


def random_workload(
    gen: torch.Generator,
    D: int,
    max_sq: int = 300,
    max_skv: int = 400,
    allow_gqa: bool = True,
    name: str = "random",
) -> Workload:
    """A small random workload shape (for property sweeps), drawn from ``gen``."""

    def ri(lo, hi):
        return int(torch.randint(lo, hi + 1, (1,), generator=gen).item())

    B = ri(1, 3)
    Hkv = ri(1, 3)
    g = ri(1, 3) if allow_gqa else 1
    Hq = Hkv * g
    Sq = ri(1, max_sq)
    Sp = ri(0, max_skv // 2)
    Ss = ri(0 if Sp > 0 else 1, max_skv - Sp)
    Skv = Sp + Ss
    real_len = tuple(ri(0, Skv) for _ in range(B))
    seed = ri(0, 2**31 - 1)
    return Workload(name, B=B, Hq=Hq, Hkv=Hkv, D=D, Sq=Sq, Sp=Sp, Ss=Ss,
                    real_len=real_len, seed=seed)


@dataclasses.dataclass(frozen=True)
class PackedWorkload:
    """Packed variable-length self-attention: ``n_seg`` independent samples of
    lengths drawn uniformly from [min_len, max_len] (a CPU generator seeded
    with ``seed``), concatenated on one token axis (cu_seqlens)."""

    name: str
    n_seg: int
    min_len: int
    max_len: int
    Hq: int
    Hkv: int
    D: int
    seed: int
    description: str = ""


PACKED: Dict[str, PackedWorkload] = {
    w.name: w
    for w in [
        PackedWorkload(
            "packed", n_seg=64, min_len=256, max_len=4096, Hq=16, Hkv=16, D=128, seed=7,
            description="64 packed samples of 256-4096 tokens (image/video latents of mixed "
                        "resolutions in one batch), self-attention within each sample",
        ),
    ]
}


def make_packed(w: PackedWorkload) -> Dict[str, object]:
    """Draw the segment lengths, then q [T, Hq, D], k and v [T, Hkv, D] (bf16,
    N(0,1)) in that order from one generator; cu_seqlens shared by q and k."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(w.seed)
    lens = torch.randint(w.min_len, w.max_len + 1, (w.n_seg,), generator=gen).tolist()
    cu = [0]
    for n in lens:
        cu.append(cu[-1] + int(n))
    T = cu[-1]
    return {
        "q": _draw(gen, (T, w.Hq, w.D), 1.0),
        "k": _draw(gen, (T, w.Hkv, w.D), 1.0),
        "v": _draw(gen, (T, w.Hkv, w.D), 1.0),
        "cu_seqlens": cu,
        "lens": [int(n) for n in lens],
    }
