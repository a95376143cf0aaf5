"""CPU oracle (fp64) for split-KV tail-padded attention and the Q/K RMSNorm+RoPE prologue.

TEST INFRASTRUCTURE ONLY: tests/, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg are the only callers.  The product path never
imports this package, and this package never imports the product package.

The arithmetic lives in ``splitkv_oracle.c`` (plain C loops, fp64); this
module only builds it with gcc, marshals numpy/torch CPU arrays and applies
the query-row validity rule.

Pins (tests/test_oracle_pins.py) tie each function to something other than
itself: torch's scaled-dot-product attention on an explicit concatenation
with a boolean key mask, closed forms (scale 0 -> mean of valid value rows,
uniform V -> 1, one valid key -> that value row), invariants (split point,
tail pad of any content, joint key permutation, GQA head mapping), worked
examples under tests/golden/, and planted mistakes that must fail a pin.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "splitkv_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "liboracle.so")
_lock = threading.Lock()
_lib = None

# Planted-mistake codes understood by the C oracle (0 = the definition).
MUTATIONS = {
    "gqa_modulo": 1,
    "one_pad_key": 2,
    "v_from_k": 3,
    "drop_last_in_sum": 4,
    "negated_scores": 5,
    "scale_ignored": 6,
    "drop_last_dim": 7,
    "q_from_kv_head": 8,
}


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP, no fast-math, no FP contraction)."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + ".tmp%d" % os.getpid()
    cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
           "-fPIC", "-shared", "-std=c11", "-Wall", "-o", tmp, _SRC, "-lm"]
    subprocess.check_call(cmd)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            i32 = ctypes.c_int
            lib.oracle_attn_split_kv.argtypes = [P, P, P, P, P] + [i32] * 7 + [
                P, P, ctypes.c_double, P, i32, P, i32]
            lib.oracle_attn_split_kv.restype = i32
            lib.oracle_qk_rmsnorm_rope.argtypes = [P, i32, i32, i32, P, i32, P, P, i32, i32,
                                                   ctypes.c_double, P]
            lib.oracle_qk_rmsnorm_rope.restype = i32
            lib.oracle_num_threads.argtypes = []
            lib.oracle_num_threads.restype = i32
            lib.oracle_round_bf16.argtypes = [ctypes.c_double]
            lib.oracle_round_bf16.restype = ctypes.c_uint16
            _lib = lib
    return _lib


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def _bf16_bits(x) -> np.ndarray:
    """Contiguous uint16 view of a bf16 tensor (torch CPU) or a uint16 array."""
    if isinstance(x, np.ndarray):
        if x.dtype != np.uint16:
            raise TypeError("numpy inputs must be uint16 bf16 bit patterns")
        return np.ascontiguousarray(x)
    import torch  # local: torch is only needed to accept tensors

    if x.dtype != torch.bfloat16:
        raise TypeError("expected a bf16 tensor")
    return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def q_valid_rule(Sq: int, Skv: int, real_len: Sequence[int]) -> list:
    """Query rows that are not pad.

    In joint self-attention (Sq == Skv) queries and keys are the same padded
    token stream, so the tail pad covers query rows too and q_valid = real_len.
    Otherwise (cross attention, or generated-token queries over a longer joint
    K/V) every query row is real: q_valid = Sq.
    """
    if Sq == Skv:
        return [int(n) for n in real_len]
    return [Sq] * len(real_len)


def attn_split_kv(q, k_prefix, v_prefix, k_suffix, v_suffix,
                  real_len: Optional[Sequence[int]] = None,
                  q_valid: Optional[Sequence[int]] = None,
                  softmax_scale: Optional[float] = None,
                  rows: Optional[Sequence[int]] = None,
                  mutate: int = 0) -> np.ndarray:
    """Attention over cat(prefix, suffix)[:real_len[b]] per batch row, fp64.

    q [B,Sq,Hq,D], k/v_prefix [B,Sp,Hkv,D], k/v_suffix [B,Ss,Hkv,D] (bf16).
    Returns float64 [B, len(rows) or Sq, Hq, D].
    """
    lib = _load()
    qb, kpb, vpb, ksb, vsb = (_bf16_bits(t) for t in (q, k_prefix, v_prefix, k_suffix, v_suffix))
    B, Sq, Hq, D = qb.shape
    Sp, Hkv = kpb.shape[1], kpb.shape[2]
    Ss = ksb.shape[1]
    for a, S in ((kpb, Sp), (vpb, Sp), (ksb, Ss), (vsb, Ss)):
        if a.shape != (B, S, Hkv, D):
            raise ValueError("inconsistent K/V shapes")
    Skv = Sp + Ss
    rl = [Skv] * B if real_len is None else [int(x) for x in real_len]
    qv = q_valid_rule(Sq, Skv, rl) if q_valid is None else [int(x) for x in q_valid]
    rl_a = np.asarray(rl, dtype=np.int32)
    qv_a = np.asarray(qv, dtype=np.int32)
    if softmax_scale is None:
        softmax_scale = D ** -0.5
    if rows is None:
        rows_a = None
        nr = Sq
    else:
        rows_a = np.asarray(rows, dtype=np.int32)
        nr = int(rows_a.shape[0])
    out = np.empty((B, nr, Hq, D), dtype=np.float64)
    rc = lib.oracle_attn_split_kv(
        _ptr(qb), _ptr(kpb), _ptr(vpb), _ptr(ksb), _ptr(vsb),
        B, Sq, Sp, Ss, Hq, Hkv, D, _ptr(rl_a), _ptr(qv_a), float(softmax_scale),
        _ptr(rows_a) if rows_a is not None else None, nr, _ptr(out), int(mutate))
    if rc != 0:
        raise ValueError("oracle_attn_split_kv rejected its arguments")
    return out


def attn_varlen(q, k, v, cu_seqlens_q: Sequence[int], cu_seqlens_k: Sequence[int],
                seqused_q: Optional[Sequence[int]] = None,
                seqused_k: Optional[Sequence[int]] = None,
                softmax_scale: Optional[float] = None,
                rows: Optional[Sequence[int]] = None) -> np.ndarray:
    """Packed variable-length attention, fp64 ("vLLM-Omni performance
    patterns": packed samples described by cu_seqlens; "sglang PR 30107":
    varlen attention over [valid | pad] segments).  The definition is a
    block-diagonal mask: query row t of segment i attends to the first
    seqused_k[i] keys of segment i only, i.e. it is single-sequence attention
    applied to each segment's slices.  Rows past seqused_q[i] inside a segment,
    and segments without a valid key, give zeros; rows outside every segment
    are returned as zeros too.

    q [Tq, Hq, D] (or [1, Tq, Hq, D]), k/v [Tk, Hkv, D]; returns float64 [Tq, Hq, D],
    or with ``rows`` only those query rows (sorted, duplicates dropped):
    [len(rows), Hq, D].
    """
    import torch

    def as3(t):
        return t[0] if t.dim() == 4 else t

    q3, k3, v3 = as3(q), as3(k), as3(v)
    Tq, Hq, D = q3.shape
    n = len(cu_seqlens_q) - 1
    want = None if rows is None else np.asarray(sorted(set(int(r) for r in rows)), dtype=np.int64)
    out = np.zeros((Tq if want is None else len(want), Hq, D), dtype=np.float64)
    empty = k3[:0].unsqueeze(0)
    for i in range(n):
        q0, q1 = int(cu_seqlens_q[i]), int(cu_seqlens_q[i + 1])
        k0, k1 = int(cu_seqlens_k[i]), int(cu_seqlens_k[i + 1])
        if q1 == q0:
            continue
        nk = (k1 - k0) if seqused_k is None else int(seqused_k[i])
        nq = (q1 - q0) if seqused_q is None else int(seqused_q[i])
        if want is None:
            local, dst = None, slice(q0, q1)
        else:
            sel = np.nonzero((want >= q0) & (want < q1))[0]
            if sel.size == 0:
                continue
            local, dst = [int(r) - q0 for r in want[sel]], sel
        seg = attn_split_kv(q3[q0:q1].unsqueeze(0), empty, empty,
                            k3[k0:k1].unsqueeze(0), v3[k0:k1].unsqueeze(0),
                            real_len=[nk], q_valid=[nq], softmax_scale=softmax_scale, rows=local)
        out[dst] = seg[0]
    return out


def shard_chunk(x, orig_len: int, sp_size: int, sp_rank: int, pad_mode: str = "zeros",
                mutate: str = "") -> np.ndarray:
    """One rank's chunk of an even, tail-padded sequence shard, along axis 1.

    Definition ("sglang PR 30107", sp_shard_utils.py: build_shard_plan's
    shard math and shard_like's pad-then-narrow): a stream of ``orig_len``
    rows is cut into ``sp_size`` chunks of ``local_len = ceil(orig_len /
    sp_size)`` rows; the ``local_len * sp_size - orig_len`` missing rows are
    appended after the last real row, as zeros or (``pad_mode="repeat_last"``)
    as copies of the last real row; rank ``r`` holds padded rows
    ``[r * local_len, (r + 1) * local_len)``.  Written row by row: padded row
    t is source row t when t < orig_len, else the pad row.

    x: [B, orig_len, ...] bf16 tensor (compared as bit patterns) or any numpy
    array.  Returns a numpy array [B, local_len, ...] (uint16 bits for bf16).
    ``mutate`` plants a mistake for the pin tests: "floor_len" (local_len
    rounded down), "pad_first" (pad rows at the chunk head), "repeat_first"
    (pad repeats row 0).
    """
    if hasattr(x, "dtype") and not isinstance(x, np.ndarray):
        import torch

        a = _bf16_bits(x) if x.dtype == torch.bfloat16 else x.detach().cpu().numpy()
    else:
        a = np.asarray(x)
    if a.shape[1] != orig_len:
        raise ValueError("axis 1 must hold orig_len rows")
    if sp_size < 1 or not 0 <= sp_rank < sp_size:
        raise ValueError("bad sp_size / sp_rank")
    if pad_mode not in ("zeros", "repeat_last"):
        raise ValueError("pad_mode")
    local_len = -(-orig_len // sp_size) if mutate != "floor_len" else orig_len // sp_size
    num_pad = local_len * sp_size - orig_len
    out = np.zeros((a.shape[0], local_len) + a.shape[2:], dtype=a.dtype)
    for r in range(local_len):
        t = sp_rank * local_len + r
        if mutate == "pad_first" and sp_rank == sp_size - 1 and num_pad > 0:
            t = t - num_pad if r >= num_pad else orig_len  # pad rows moved to the chunk head
        if t < orig_len:
            out[:, r] = a[:, t]
        elif pad_mode == "repeat_last":
            if orig_len == 0:
                raise ValueError("repeat_last needs a real row")
            out[:, r] = a[:, 0] if mutate == "repeat_first" else a[:, orig_len - 1]
    return out


def qk_rmsnorm_rope(x, w, table, pos=None, rot_dim: Optional[int] = None,
                    interleaved: bool = False, eps: float = 1e-6) -> np.ndarray:
    """RMSNorm over head_dim then RoPE for x [..., H, D] (bf16); returns bf16 bits (uint16).

    table: float32 [rows, rot_dim] holding [cos | sin]; pos[t] picks the row of
    token t (tokens are the flattened leading dims); default pos = token index
    modulo the sequence length when x is [B, S, H, D].
    """
    lib = _load()
    xb = _bf16_bits(x)
    wb = _bf16_bits(w)
    shape = xb.shape
    H, D = shape[-2], shape[-1]
    T = int(np.prod(shape[:-2])) if len(shape) > 2 else 1
    tab = np.ascontiguousarray(np.asarray(table, dtype=np.float32))
    if rot_dim is None:
        rot_dim = tab.shape[1]
    if pos is None:
        S = shape[-3] if len(shape) >= 3 else 1
        pos = np.arange(T, dtype=np.int32) % S
    pos_a = np.ascontiguousarray(np.asarray(pos, dtype=np.int32))
    y = np.empty_like(xb)
    rc = lib.oracle_qk_rmsnorm_rope(_ptr(xb), T, H, D, _ptr(pos_a), int(tab.shape[0]),
                                    _ptr(wb), _ptr(tab), int(rot_dim), int(bool(interleaved)),
                                    float(eps), _ptr(y))
    if rc != 0:
        raise ValueError("oracle_qk_rmsnorm_rope rejected its arguments")
    return y.reshape(shape)


def round_bf16(x: float) -> int:
    """The oracle's fp64 -> bf16 rounding (nearest, ties to even), as bits."""
    return int(_load().oracle_round_bf16(float(x)))
