"""Sequence-parallel shard helpers: even tail-padded shards and the attention
metadata they imply ("sglang PR 30107", unified SP shard utils).

Layout invariant (same page): a sequence of ``orig_len`` tokens is split into
``sp_size`` equal chunks of ``local_len = ceil(orig_len / sp_size)`` tokens;
the ``num_pad = local_len * sp_size - orig_len`` pad tokens all sit at the end
of the LAST rank's chunk, so the gathered sequence carries one contiguous pad
block at its global tail.  That is exactly the layout ``attn_fwd_split_kv``
excludes for free through ``real_len``: after the sequence is gathered (or
after a Ulysses all-to-all), every rank passes ``real_len = orig_len`` (times
any per-token row multiplier) and no pad key enters the softmax.

Host-side plumbing only (shape math, ``F.pad``/``narrow``/``cat`` and
``torch.distributed`` gathers); nothing here is on the attention hot path.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Optional, Sequence, Tuple

import torch
import torch.nn.functional as F

__all__ = [
    "SpShard",
    "build_shard_plan",
    "tail_attn_meta",
    "attn_real_len",
    "shard_like",
    "shard_seq",
    "gather_seq",
    "join_seqs",
    "split_seqs",
    "should_shard_text",
]


@dataclass(frozen=True)
class SpShard:
    """An even split of one token stream over ``sp_size`` ranks, as seen by
    ``sp_rank``.  Hidden states, rotary tables and every other tensor of the
    stream are cut with the same plan, so their chunks line up.

    Fields: ``orig_len`` is the count of real tokens in the whole stream;
    ``local_len`` the chunk length, identical on all ranks; ``num_pad`` the
    count of filler tokens placed after the last real token (so they end up
    at the tail of the last chunk); ``sp_size``/``sp_rank`` the group size and
    this rank's index in it.
    """

    orig_len: int
    local_len: int
    num_pad: int
    sp_size: int
    sp_rank: int

    @property
    def local_pad(self) -> int:
        """Filler rows inside this rank's chunk: those of its rows whose global
        position is at or past ``orig_len``.  While the filler fits in one chunk
        (``num_pad <= local_len``, i.e. all but tiny streams over many ranks)
        only the last rank has any, and it has all ``num_pad`` of them.  With
        more filler than a chunk holds (1 token over 4 ranks: chunks of 1, 3
        filler rows) the filler reaches into earlier chunks and this still
        counts the rows that are really there, never a negative real count."""
        end = (self.sp_rank + 1) * self.local_len
        return max(0, min(self.local_len, end - self.orig_len))

    @property
    def local_real_len(self) -> int:
        """Rows of this rank's chunk that hold real tokens."""
        return self.local_len - self.local_pad

    @property
    def padded_len(self) -> int:
        """Rows of the stream once gathered, filler included."""
        return self.local_len * self.sp_size


def _group_size_rank(group) -> Tuple[int, int]:
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()):
        return 1, 0
    return dist.get_world_size(group), dist.get_rank(group)


def build_shard_plan(seq_len: int, sp_size: Optional[int] = None, sp_rank: Optional[int] = None,
                     group=None) -> SpShard:
    """Plan the split of a ``seq_len``-token stream; touches no tensor
    ("sglang PR 30107", ``build_shard_plan``).  Each chunk gets the stream
    length divided by the group size, rounded up, and the filler is whatever
    that rounding adds to the total.  One rank (``sp_size == 1``) keeps the
    stream whole with no filler.

    ``sp_size``/``sp_rank`` default to the size and rank of ``group`` (the
    default process group), or to (1, 0) when torch.distributed is not
    initialised.
    """
    if sp_size is None or sp_rank is None:
        gs, gr = _group_size_rank(group)
        sp_size = gs if sp_size is None else sp_size
        sp_rank = gr if sp_rank is None else sp_rank
    if seq_len < 0:
        raise ValueError(f"seq_len must be >= 0, got {seq_len}")
    if sp_size < 1 or not (0 <= sp_rank < sp_size):
        raise ValueError(f"bad sp_size/sp_rank: {sp_size}/{sp_rank}")
    whole, rest = divmod(seq_len, sp_size)
    chunk = whole + (1 if rest else 0)
    return SpShard(orig_len=seq_len, local_len=chunk, num_pad=chunk * sp_size - seq_len,
                   sp_size=sp_size, sp_rank=sp_rank if sp_size > 1 else 0)


def tail_attn_meta(shard: SpShard, seqlen_multiplier: int = 1) -> Optional[dict]:
    """Attention metadata for this rank's chunk when the stream carries filler
    ("sglang PR 30107", ``tail_attn_meta``), or None when it carries none.
    ``valid_len`` counts the attention rows of the chunk's real tokens (each
    token spans ``seqlen_multiplier`` rows).  ``max_seqlen_tail`` is the longer
    of that and the filler count: a varlen kernel sized by it then also covers
    the filler segment, which the page's review found could be the longer of
    the two."""
    pad = shard.num_pad
    if pad <= 0:
        return None
    valid = shard.local_real_len * seqlen_multiplier
    meta = dict(tail=True, valid_len=valid)
    meta["max_seqlen_tail"] = valid if valid >= pad else pad
    return meta


def attn_real_len(shard: SpShard, seqlen_multiplier: int = 1, batch: int = 1) -> List[int]:
    """``real_len`` for ``attn_fwd_split_kv`` over the gathered sequence (pad at
    the global tail): the valid key count ``orig_len * multiplier`` for each of
    ``batch`` rows.  The kernel takes no ``max_seqlen``, so the page's
    ``max_seqlen_tail`` has no counterpart here."""
    return [shard.orig_len * seqlen_multiplier] * batch


def shard_like(x: torch.Tensor, shard: SpShard, dim: int = 1, pad_mode: str = "zeros") -> torch.Tensor:
    """Apply a planned shard to one tensor ("sglang PR 30107", ``shard_like``):
    pad the tail of ``dim`` with ``num_pad`` rows (zeros, or copies of the last
    row with ``pad_mode="repeat_last"``), then take this rank's ``local_len``
    rows.  Tensors of one stream (hidden states, RoPE tables, ...) sharded
    with the same plan stay aligned chunk for chunk.

    A chunk without pad is returned as a view of ``x`` (no copy).  A chunk
    holding pad is built in one pass: on CUDA with ``dim == 1`` and
    16-byte rows by the library's copy kernel (``sk_shard_pad_copy``), which
    reads only the chunk's real rows; otherwise with torch ops."""
    if x.shape[dim] != shard.orig_len:
        raise ValueError(f"dim {dim} has {x.shape[dim]} rows, plan expects {shard.orig_len}")
    if pad_mode not in ("zeros", "repeat_last"):
        raise ValueError(f"unknown pad_mode {pad_mode!r}")
    if shard.sp_size <= 1:
        return x
    start = shard.sp_rank * shard.local_len
    if start + shard.local_len <= shard.orig_len:
        return x.narrow(dim, start, shard.local_len)
    if pad_mode == "repeat_last" and shard.orig_len == 0:
        raise ValueError("repeat_last needs at least one row")
    nd = dim % x.dim()
    row_bytes = x.element_size()
    for d in x.shape[nd + 1:]:
        row_bytes *= d
    if x.is_cuda and nd == 1 and x.dim() >= 2 and row_bytes % 16 == 0 and x[0, 0].is_contiguous():
        from . import sk_shard_pad_copy

        shape = list(x.shape)
        shape[1] = shard.local_len
        out = torch.empty(shape, dtype=x.dtype, device=x.device)
        return sk_shard_pad_copy(x, out, start, pad_mode)
    real = x.narrow(dim, min(start, shard.orig_len), max(0, shard.orig_len - start))
    npad = shard.local_len - real.shape[dim]
    if pad_mode == "repeat_last":
        last = x.narrow(dim, shard.orig_len - 1, 1)
        pad = last.expand(*[npad if i == nd else -1 for i in range(x.dim())])
    else:
        pad_shape = list(x.shape)
        pad_shape[nd] = npad
        pad = torch.zeros(pad_shape, dtype=x.dtype, device=x.device)
    return torch.cat([real, pad], dim=dim)


def shard_seq(x: torch.Tensor, shard: SpShard, dim: int = 1, pad_mode: str = "zeros") -> torch.Tensor:
    """This rank's chunk of a full sequence (``shard_like`` under the stream's plan)."""
    return shard_like(x, shard, dim=dim, pad_mode=pad_mode)


def gather_seq(x_local: torch.Tensor, shard: SpShard, dim: int = 1, group=None) -> torch.Tensor:
    """Inverse of ``shard_seq`` over a process group: all-gather the ranks'
    chunks along ``dim`` (rank order) and trim the tail pad back to
    ``orig_len`` rows."""
    import torch.distributed as dist

    if x_local.shape[dim] != shard.local_len:
        raise ValueError(f"chunk has {x_local.shape[dim]} rows, plan expects {shard.local_len}")
    if shard.sp_size <= 1:
        return x_local
    xs = x_local.contiguous()
    parts = [torch.empty_like(xs) for _ in range(shard.sp_size)]
    dist.all_gather(parts, xs, group=group)
    return torch.cat(parts, dim=dim).narrow(dim, 0, shard.orig_len)


def join_seqs(firsts: Sequence[torch.Tensor], seconds: Sequence[torch.Tensor], local_pad: int,
              dim: int = 1) -> List[torch.Tensor]:
    """Joint sequences with the first stream's local pad moved to the joint
    tail: ``cat([first[:-pad], second, first[-pad:]])`` per tensor pair (e.g.
    text then image tokens, for q, k and v alike).  The page names this helper
    and states only that it keeps the pad at the tail; this is that layout."""
    if len(firsts) != len(seconds):
        raise ValueError("join_seqs needs tensor pairs")
    out = []
    for a, b in zip(firsts, seconds):
        la = a.shape[dim]
        if not 0 <= local_pad <= la:
            raise ValueError(f"local_pad {local_pad} outside [0, {la}]")
        valid = a.narrow(dim, 0, la - local_pad)
        pad = a.narrow(dim, la - local_pad, local_pad)
        out.append(torch.cat([valid, b, pad], dim=dim))
    return out


def split_seqs(joints: Sequence[torch.Tensor], first_len: int, local_pad: int,
               dim: int = 1) -> List[Tuple[torch.Tensor, torch.Tensor]]:
    """Inverse of ``join_seqs``: from ``[first valid | second | first pad]``
    return ``(first, second)`` with the first stream's pad back at its own
    tail; ``first_len`` counts the first stream's rows including the pad."""
    out = []
    for j in joints:
        n = j.shape[dim]
        valid = first_len - local_pad
        second_len = n - first_len
        if valid < 0 or second_len < 0:
            raise ValueError("first_len/local_pad do not fit the joint sequence")
        first = torch.cat([j.narrow(dim, 0, valid), j.narrow(dim, n - local_pad, local_pad)], dim=dim)
        out.append((first, j.narrow(dim, valid, second_len)))
    return out


def should_shard_text(seq_len: int, sp_size: int, min_len: int = 0) -> bool:
    """Policy gate: shard a stream across ``sp_size`` ranks unless it is
    shorter than ``min_len`` tokens (the page's default is to always shard,
    with an escape hatch for a minimum length)."""
    return sp_size > 1 and seq_len >= max(min_len, 1)
