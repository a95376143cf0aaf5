"""Ulysses sequence parallelism around the split-KV kernel ("sglang PR 26973",
``_forward_with_replicated_kv_prefix_split``; "vLLM-Omni performance
patterns", Ulysses transport and GQA head padding).

Each rank holds one sequence chunk of Q and of the K/V suffix (the tail-padded
shard of ``sp_shard``) and the whole replicated K/V prefix.  One call:

1. all-to-all of Q and of the K/V suffix from sequence shards to head shards
   (this rank gets every token of ``H / sp`` heads, chunks in rank order, so the
   shard pad lands at the global tail);
2. the replicated prefix is sliced to this rank's KV heads, with no
   communication (a strided view: the kernel reads it in place);
3. ``attn_fwd_split_kv`` on the local heads with ``real_len = Sp + orig_len``
   (prefix first, then the valid suffix tokens), so the pad is never read and
   the prefix/suffix concatenation is never built;
4. all-to-all of the output from head shards back to sequence shards.

GQA: when ``num_kv_heads`` is not a multiple of ``sp``, K/V heads are padded
with zero heads up to the next multiple and Q heads up to the same group
ratio (contiguous groups keep every real head's KV mapping); padded heads'
outputs are dropped.  A warning is issued once when the padding inflates the
Q heads by more than 1.5x.

The collectives are ``torch.distributed.all_to_all_single`` (NCCL over
NVLink/NVSwitch on GPUs); the attention itself is the CUDA kernel unless a
``local_attn`` callable with the same signature is supplied.

``ulysses_attn_fwd_split_kv_fused`` fuses step 4 into the kernel: its
epilogue stores every output row straight into the receive buffer of the rank
that owns the row's sequence chunk (``attn_fwd_split_kv_scatter``: plain
stores to buffers mapped from the other GPUs, e.g. torch symmetric memory),
so the exchange overlaps the attention of later tiles; a barrier across the
group then orders the readers after every rank's stores.
"""
from __future__ import annotations

import warnings
from typing import Callable, Optional, Sequence

import torch
import torch.nn.functional as F

from .sp_shard import SpShard

__all__ = ["seq_to_head", "head_to_seq", "gqa_head_padding", "ulysses_attn_fwd_split_kv",
           "ulysses_attn_fwd_split_kv_fused"]

_warned_inflation = False


def seq_to_head(x: torch.Tensor, sp: int, group=None) -> torch.Tensor:
    """[B, S_local, H, D] sequence chunk -> [B, sp * S_local, H / sp, D]: every
    token (chunks in rank order) of this rank's ``H / sp`` heads."""
    import torch.distributed as dist

    B, S, H, D = x.shape
    if H % sp:
        raise ValueError(f"{H} heads do not split over {sp} ranks")
    if sp == 1:
        return x
    send = x.reshape(B, S, sp, H // sp, D).permute(2, 0, 1, 3, 4).contiguous()
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    return recv.permute(1, 0, 2, 3, 4).reshape(B, sp * S, H // sp, D)


def head_to_seq(y: torch.Tensor, sp: int, group=None) -> torch.Tensor:
    """Inverse of ``seq_to_head``: [B, sp * S_local, H / sp, D] -> [B, S_local, H, D]."""
    import torch.distributed as dist

    B, S_full, Hl, D = y.shape
    if S_full % sp:
        raise ValueError("sequence length is not a multiple of sp")
    if sp == 1:
        return y
    S = S_full // sp
    send = y.reshape(B, sp, S, Hl, D).permute(1, 0, 2, 3, 4).contiguous()
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    return recv.permute(1, 2, 0, 3, 4).reshape(B, S, sp * Hl, D)


def gqa_head_padding(num_q_heads: int, num_kv_heads: int, sp: int):
    """(padded Q heads, padded KV heads): KV heads up to a multiple of ``sp``,
    Q heads by the original group ratio."""
    if num_q_heads % num_kv_heads:
        raise ValueError("num_q_heads must be a multiple of num_kv_heads")
    g = num_q_heads // num_kv_heads
    hkv = -(-num_kv_heads // sp) * sp
    return hkv * g, hkv


def _pad_heads(x: torch.Tensor, h: int) -> torch.Tensor:
    return x if x.shape[2] == h else F.pad(x, (0, 0, 0, h - x.shape[2]))


def ulysses_attn_fwd_split_kv(q, k_prefix, v_prefix, k_suffix, v_suffix, shard: SpShard,
                              group=None, softmax_scale: Optional[float] = None,
                              suffix_real_len: Optional[Sequence[int]] = None,
                              local_attn: Optional[Callable] = None) -> torch.Tensor:
    """Split-KV attention under Ulysses sequence parallelism.

    q [B, S_local, Hq, D], k/v_suffix [B, S_local, Hkv, D]: this rank's chunk
    of a stream planned by ``shard`` (``sp_shard.build_shard_plan``);
    k/v_prefix [B, Sp, Hkv, D]: replicated on every rank.
    suffix_real_len: valid suffix tokens per batch row in the gathered order
    (default ``shard.orig_len``).  Returns this rank's output chunk
    [B, S_local, Hq, D]; its pad rows are zeros.
    """
    sp = shard.sp_size
    Hq, D = q.shape[2], q.shape[3]
    if local_attn is None:
        from . import attn_fwd_split_kv as local_attn
    # q_valid: the query stream is the suffix stream, so its tail pad rows are pad too
    qh, kp, vp, ksh, vsh, real_len, q_valid, _ = _head_shard_inputs(
        q, k_prefix, v_prefix, k_suffix, v_suffix, shard, group, suffix_real_len)
    if softmax_scale is None:
        softmax_scale = D ** -0.5
    oh = local_attn(qh, kp, vp, ksh, vsh, real_len=real_len, q_valid=q_valid, softmax_scale=softmax_scale)
    out = head_to_seq(oh, sp, group)
    return out[:, :, :Hq]


def _head_shard_inputs(q, k_prefix, v_prefix, k_suffix, v_suffix, shard, group, suffix_real_len):
    """Steps 1-3 of the split path: exchanged Q / K/V suffix on this rank's
    heads, the prefix head slice, and the per-row lengths."""
    sp = shard.sp_size
    B, S_loc, Hq, D = q.shape
    Hkv = k_suffix.shape[2]
    if S_loc != shard.local_len or k_suffix.shape[1] != S_loc or v_suffix.shape[1] != S_loc:
        raise ValueError("q / k_suffix / v_suffix are not this rank's chunk of the plan")
    Hq_p, Hkv_p = gqa_head_padding(Hq, Hkv, sp)
    global _warned_inflation
    if Hq_p > 1.5 * Hq and not _warned_inflation:
        warnings.warn(f"GQA head padding inflates {Hq} query heads to {Hq_p} over {sp} ranks; "
                      "a sequence-parallel degree dividing the KV head count avoids it")
        _warned_inflation = True
    qh = seq_to_head(_pad_heads(q, Hq_p), sp, group)
    ksh = seq_to_head(_pad_heads(k_suffix, Hkv_p), sp, group)
    vsh = seq_to_head(_pad_heads(v_suffix, Hkv_p), sp, group)
    hkv_loc = Hkv_p // sp
    h0 = shard.sp_rank * hkv_loc
    kp = _pad_heads(k_prefix, Hkv_p)[:, :, h0:h0 + hkv_loc]
    vp = _pad_heads(v_prefix, Hkv_p)[:, :, h0:h0 + hkv_loc]
    Sp = k_prefix.shape[1]
    srl = [shard.orig_len] * B if suffix_real_len is None else [int(x) for x in suffix_real_len]
    return qh, kp, vp, ksh, vsh, [Sp + n for n in srl], srl, Hq_p


def ulysses_attn_fwd_split_kv_fused(q, k_prefix, v_prefix, k_suffix, v_suffix, shard: SpShard,
                                    recv_buffers: Sequence, group=None,
                                    softmax_scale: Optional[float] = None,
                                    suffix_real_len: Optional[Sequence[int]] = None,
                                    local_attn_scatter: Optional[Callable] = None):
    """``ulysses_attn_fwd_split_kv`` with the output all-to-all fused into the
    attention kernel's stores.

    recv_buffers: ``sp`` tensors [B, S_local, Hq_p, D] (Hq_p = the padded query
    head count of ``gqa_head_padding``); entry r is rank r's receive buffer as
    mapped into this process (another GPU's memory, e.g. a torch symmetric
    memory buffer; entry ``sp_rank`` is this rank's own).  This rank's heads
    land at head slot ``sp_rank * Hq_p / sp`` of every buffer.  After the
    kernel a barrier over ``group`` orders this rank's read of its own buffer
    after every rank's stores.  Returns this rank's output chunk [B, S_local,
    Hq, D] (a view of its receive buffer; pad rows are zeros).

    The returned view is valid only until the next call that uses the same
    ``recv_buffers``: that call's kernels on the other ranks overwrite the
    buffer with plain stores as soon as they run.  Every consumer of the
    result must therefore be enqueued on the calling stream before that next
    call (the exchange in front of it then orders them), or copy the result
    out; a consumer on another stream, or a view kept across calls, can see
    other ranks' newer rows.  Alternating between two buffer sets on
    consecutive calls gives each result one extra call of lifetime.
    """
    import torch.distributed as dist

    sp = shard.sp_size
    if len(recv_buffers) != sp:
        raise ValueError(f"{len(recv_buffers)} receive buffers for {sp} ranks")
    if local_attn_scatter is None:
        from . import attn_fwd_split_kv_scatter as local_attn_scatter
    Hq, D = q.shape[2], q.shape[3]
    qh, kp, vp, ksh, vsh, real_len, q_valid, Hq_p = _head_shard_inputs(
        q, k_prefix, v_prefix, k_suffix, v_suffix, shard, group, suffix_real_len)
    if softmax_scale is None:
        softmax_scale = D ** -0.5
    local_attn_scatter(qh, kp, vp, ksh, vsh, list(recv_buffers), head_offset=shard.sp_rank * (Hq_p // sp),
                       real_len=real_len, q_valid=q_valid, softmax_scale=softmax_scale)
    if sp > 1:
        dist.barrier(group=group)
    return recv_buffers[shard.sp_rank][:, :, :Hq]
