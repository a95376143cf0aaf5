"""Python binding of libsplitkv_attn (split-KV tail-padded attention for B200).

Argument marshalling only: every step of the computation runs in the CUDA
kernels of ``libsplitkv_attn.so`` behind the C ABI declared in
``include/splitkv_attn.h``.  PyTorch supplies device memory and the current
stream.  There is no fallback: if the library is missing or a call is
rejected, ``SplitKVError`` is raised.

Entry points (same names as the C ABI):
  attn_fwd_split_kv(q, k_prefix, v_prefix, k_suffix, v_suffix, real_len=None,
                    softmax_scale=None, out=None, q_valid=None)
  attn_fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, seqused_q=None, seqused_k=None,
                  softmax_scale=None, out=None)
  qk_rmsnorm_rope(q, k, w_q, w_k, rope_table, rot_dim=None, interleaved=False, eps=1e-6)
  sk_device_status(device=None, clear=True), sk_set_wait_timeout_ms(ms), sk_abi_version()
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional, Sequence

__all__ = [
    "SplitKVError",
    "SkTensor",
    "lib",
    "attn_fwd_split_kv",
    "attn_fwd_split_kv_scatter",
    "attn_fwd_varlen",
    "sk_shard_pad_copy",
    "qk_rmsnorm_rope",
    "sk_device_status",
    "sk_set_wait_timeout_ms",
    "sk_test_stall_mma",
    "sk_abi_version",
    "tensor_desc",
    "LIB_PATH",
    "STATUS",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsplitkv_attn.so")

STATUS = {0: "SK_OK", 1: "SK_ERR_INVALID_ARG", 2: "SK_ERR_UNSUPPORTED", 3: "SK_ERR_CUDA",
          4: "SK_ERR_DEVICE_TIMEOUT"}


class SplitKVError(RuntimeError):
    def __init__(self, status: int, message: str):
        self.status = int(status)
        self.message = message
        super().__init__(f"{STATUS.get(self.status, self.status)}: {message}")


class SkTensor(ctypes.Structure):
    _fields_ = [
        ("ptr", ctypes.c_void_p),
        ("stride_b", ctypes.c_int64),
        ("stride_s", ctypes.c_int64),
        ("stride_h", ctypes.c_int64),
        ("len_s", ctypes.c_int32),
    ]


_lock = threading.Lock()
_lib = None


def lib() -> ctypes.CDLL:
    """The loaded C library (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(
                    f"{LIB_PATH} is missing: build it with "
                    "`python -m varlen_flash_attention_b200.build` (nvcc, sm_100a)")
            L = ctypes.CDLL(LIB_PATH)
            P = ctypes.POINTER(SkTensor)
            i32, vp = ctypes.c_int32, ctypes.c_void_p
            L.attn_fwd_split_kv.argtypes = [P, P, P, P, P, vp, i32, i32, ctypes.c_float, P, i32, i32, vp]
            L.attn_fwd_split_kv.restype = i32
            L.attn_fwd_split_kv_ex.argtypes = [P, P, P, P, P, vp, i32, i32, ctypes.c_float, P, i32, i32,
                                               vp, vp]
            L.attn_fwd_split_kv_ex.restype = i32
            L.attn_fwd_split_kv_scatter.argtypes = [P, P, P, P, P, vp, vp, i32, i32, ctypes.c_float, vp, i32,
                                                    P, i32, i32, i32, vp]
            L.attn_fwd_split_kv_scatter.restype = i32
            i64 = ctypes.c_int64
            L.sk_shard_pad_copy.argtypes = [vp, i64, i64, i32, vp, i64, i64, i32, i32, i32, i32, i32, vp]
            L.sk_shard_pad_copy.restype = i32
            L.attn_fwd_varlen.argtypes = [P, P, P, vp, vp, vp, vp, i32, i32, i32, ctypes.c_float, P, i32, vp]
            L.attn_fwd_varlen.restype = i32
            L.qk_rmsnorm_rope.argtypes = [P, P, vp, vp, vp, i32, i32, i32, ctypes.c_float, i32, i32,
                                          i32, i32, i32, vp]
            L.qk_rmsnorm_rope.restype = i32
            L.sk_last_error.argtypes = []
            L.sk_last_error.restype = ctypes.c_char_p
            L.sk_device_status.argtypes = [i32, ctypes.POINTER(i32), i32]
            L.sk_device_status.restype = i32
            L.sk_set_wait_timeout_ms.argtypes = [i32]
            L.sk_set_wait_timeout_ms.restype = i32
            L.sk_test_stall_mma.argtypes = [i32]
            L.sk_test_stall_mma.restype = i32
            L.sk_abi_version.argtypes = []
            L.sk_abi_version.restype = i32
            _lib = L
    return _lib


_fast = None


def _fastcall():
    """The compiled marshalling module for attn_fwd_split_kv (built in-tree by
    build.build_binding; raises if it cannot be built or loaded)."""
    global _fast
    if _fast is None:
        with _lock:
            if _fast is None:
                if not os.path.exists(LIB_PATH):
                    raise ImportError(
                        f"{LIB_PATH} is missing: build it with "
                        "`python -m varlen_flash_attention_b200.build` (nvcc, sm_100a)")
                from . import build as _build

                m = _build.build_binding()
                m.bind_library(LIB_PATH)
                _fast = m
    return _fast


def _check(status: int) -> None:
    if status != 0:
        msg = lib().sk_last_error()
        raise SplitKVError(status, msg.decode() if msg else "")


def tensor_desc(t) -> SkTensor:
    """sk_tensor_t for a 4-D BSND bf16 CUDA tensor (head_dim contiguous)."""
    import torch

    shape = t.shape
    if len(shape) != 4:
        raise ValueError("expected a 4-D [batch, seq, heads, head_dim] tensor")
    if t.dtype != torch.bfloat16:
        raise TypeError("expected bf16")
    st = t.stride()
    if shape[3] > 1 and st[3] != 1:
        raise ValueError("head_dim must be contiguous (stride 1)")
    if shape[0] and shape[1] and shape[2] and shape[3]:
        if not t.is_cuda:
            raise ValueError("expected a CUDA tensor")
        return SkTensor(t.data_ptr(), st[0], st[1], st[2], shape[1])
    return SkTensor(None, st[0], st[1], st[2], shape[1])


def _stream_ptr(stream, device=None) -> Optional[int]:
    """Raw cudaStream_t of ``stream``, or of ``device``'s current stream."""
    import torch

    if stream is None:
        idx = torch.cuda.current_device() if device is None else device.index
        return torch._C._cuda_getCurrentRawStream(idx)
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _same_device(dev, named) -> None:
    """Every non-empty tensor must live on ``dev`` (the library launches on
    that device; a pointer into another GPU's memory must not reach a
    kernel as if it were local)."""
    for name, t in named:
        if t is not None and t.numel() > 0 and t.device != dev:
            raise ValueError(f"{name} is on {t.device}, expected {dev} (the device of q)")


def _check_attn_shapes(q, kv, out=None) -> int:
    """Shapes of q [B, Sq, Hq, D] against the four K/V tensors
    [B, S*, Hkv, D] and out [B, Sq, Hq, D]; returns Hkv.  Raises ValueError
    before anything reaches the library."""
    if q.dim() != 4:
        raise ValueError("q must be [batch, seq, heads, head_dim]")
    B, Sq, Hq, D = q.shape
    Hkv = None
    for name, t in kv:
        if t.dim() != 4:
            raise ValueError(f"{name} must be [batch, seq, kv_heads, head_dim]")
        if t.shape[0] != B or t.shape[3] != D:
            raise ValueError(f"{name} {tuple(t.shape)}: batch and head_dim must match q {tuple(q.shape)}")
        if Hkv is None:
            Hkv = t.shape[2]
        elif t.shape[2] != Hkv:
            raise ValueError(f"{name} has {t.shape[2]} heads, the other K/V tensors {Hkv}")
    if kv[0][1].shape[1] != kv[1][1].shape[1] or kv[2][1].shape[1] != kv[3][1].shape[1]:
        raise ValueError("k and v of the prefix (and of the suffix) must have the same length")
    if out is not None and tuple(out.shape) != tuple(q.shape):
        raise ValueError(f"out {tuple(out.shape)} must have q's shape {tuple(q.shape)}")
    return Hkv


class _OnDevice:
    """Make ``dev`` current for the duration of a call (a no-op when it
    already is, which is the common case and costs one query)."""

    __slots__ = ("idx", "prev")

    def __init__(self, dev):
        self.idx = dev.index

    def __enter__(self):
        import torch

        self.prev = torch.cuda.current_device()
        if self.prev != self.idx:
            torch.cuda.set_device(self.idx)
        return self

    def __exit__(self, *exc):
        import torch

        if self.prev != self.idx:
            torch.cuda.set_device(self.prev)
        return False


def _raise_if_device_timeout(device) -> None:
    st = sk_device_status(device.index, clear=True)
    if st != 0:
        raise SplitKVError(st, "a kernel gave up a bounded wait; its outputs are undefined")


def _int32_array(vals: Optional[Sequence[int]], n: int):
    if vals is None:
        return None
    vals = [int(v) for v in vals]
    if len(vals) != n:
        raise ValueError(f"expected {n} values, got {len(vals)}")
    return (ctypes.c_int32 * n)(*vals)


def attn_fwd_split_kv(q, k_prefix, v_prefix, k_suffix, v_suffix,
                      real_len: Optional[Sequence[int]] = None,
                      softmax_scale: Optional[float] = None,
                      out=None, q_valid: Optional[Sequence[int]] = None, stream=None,
                      check_status: bool = False):
    """Attention over cat(prefix, suffix)[:real_len[b]] without the concatenation.

    q [B, Sq, Hq, D]; k/v_prefix [B, Sp, Hkv, D]; k/v_suffix [B, Ss, Hkv, D];
    bf16 CUDA tensors on one device (strided views allowed, head_dim
    contiguous).  real_len: host sequence of B ints (default: all Sp + Ss keys
    valid).  Runs on q's device, on ``stream`` or that device's current stream.
    check_status: synchronise after the call and raise SplitKVError if a
    kernel gave up a bounded wait (otherwise such a failure is only visible
    through sk_device_status).  Returns ``out`` ([B, Sq, Hq, D] bf16,
    allocated if not given).

    The checks and the descriptors are built by a small compiled module
    (argument marshalling only), which keeps the host cost of a call close to
    the C ABI's own.
    """
    import torch

    if out is None:
        if q.dim() != 4:
            raise ValueError("q must be [batch, seq, heads, head_dim]")
        out = torch.empty(tuple(q.shape), dtype=q.dtype, device=q.device)
    if softmax_scale is None:
        softmax_scale = q.shape[-1] ** -0.5
    sp = 0 if stream is None else (stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))
    st = _fastcall().attn_fwd_split_kv(
        q, k_prefix, v_prefix, k_suffix, v_suffix, out,
        None if real_len is None else [int(v) for v in real_len],
        None if q_valid is None else [int(v) for v in q_valid], float(softmax_scale), sp)
    if st:
        _check(st)
    if check_status:
        _raise_if_device_timeout(q.device)
    return out


def attn_fwd_split_kv_scatter(q, k_prefix, v_prefix, k_suffix, v_suffix, dst: Sequence,
                              head_offset: int = 0, real_len: Optional[Sequence[int]] = None,
                              softmax_scale: Optional[float] = None,
                              q_valid: Optional[Sequence[int]] = None, stream=None,
                              check_status: bool = False) -> None:
    """``attn_fwd_split_kv`` with the output all-to-all fused into the store.

    The query stream is the gathered sequence of ``len(dst)`` equal chunks;
    output row s goes to ``dst[s // L][:, s % L, head_offset:head_offset + Hq]``
    with L = ``dst[r].shape[1]``.  ``dst``: 1..8 bf16 tensors of one shape and
    one stride set ([B, L, H_total, D]), e.g. the ranks' receive buffers mapped
    into this process (peer memory: such tensors may report another device).
    The caller orders their readers after this call (a barrier across ranks).
    """
    import torch

    kv = (("k_prefix", k_prefix), ("v_prefix", v_prefix), ("k_suffix", k_suffix), ("v_suffix", v_suffix))
    Hkv = _check_attn_shapes(q, kv)
    B, Sq, Hq, D = q.shape
    dev = q.device
    _same_device(dev, kv)
    dst = list(dst)
    if not 1 <= len(dst) <= 8:
        raise ValueError("1 to 8 destinations")
    shape, strides = tuple(dst[0].shape), dst[0].stride()
    for t in dst[1:]:
        if tuple(t.shape) != shape or t.stride() != strides:
            raise ValueError("destinations differ in shape or strides")
    if len(shape) != 4 or shape[0] != B or shape[3] != D or shape[1] * len(dst) != Sq:
        raise ValueError(f"destinations {shape} x {len(dst)} do not hold [B={B}, Sq={Sq}, *, D={D}]")
    if head_offset < 0 or head_offset + Hq > shape[2]:
        raise ValueError(f"heads {head_offset}..{head_offset + Hq - 1} outside the destination's {shape[2]}")
    if softmax_scale is None:
        softmax_scale = D ** -0.5
    descs = [tensor_desc(t) for t in (q, k_prefix, v_prefix, k_suffix, v_suffix)]
    layout = tensor_desc(dst[0])
    ptrs = (ctypes.c_void_p * len(dst))(*[t.data_ptr() for t in dst])
    rl = _int32_array(real_len, B)
    qv = _int32_array(q_valid, B)
    L = lib()
    with _OnDevice(dev):
        st = L.attn_fwd_split_kv_scatter(
            *[ctypes.byref(d) for d in descs],
            ctypes.cast(rl, ctypes.c_void_p) if rl is not None else None,
            ctypes.cast(qv, ctypes.c_void_p) if qv is not None else None,
            Hq, Hkv, float(softmax_scale), ctypes.cast(ptrs, ctypes.c_void_p), len(dst), ctypes.byref(layout),
            int(head_offset), B, D, _stream_ptr(stream, dev))
        _check(st)
        if check_status:
            _raise_if_device_timeout(dev)


def attn_fwd_varlen(q, k, v, cu_seqlens_q: Sequence[int], cu_seqlens_k: Sequence[int],
                    seqused_q: Optional[Sequence[int]] = None,
                    seqused_k: Optional[Sequence[int]] = None,
                    softmax_scale: Optional[float] = None, out=None, stream=None,
                    check_status: bool = False):
    """Packed variable-length attention: segment i's query rows
    [cu_q[i], cu_q[i+1]) attend only to key rows [cu_k[i], cu_k[i+1]).

    q [Tq, Hq, D] or [1, Tq, Hq, D]; k, v [Tk, Hkv, D] or [1, Tk, Hkv, D]
    (bf16 CUDA on one device, head_dim contiguous).  cu_seqlens_*: host
    sequences of num_segments + 1 ints (computed once when the batch is
    packed, no device sync).  seqused_*: optional host sequences of valid rows
    per segment (the rest is pad).  Returns ``out`` shaped like ``q``
    (allocated if not given; rows outside every segment are left as they were).
    """
    import torch

    def as4(t):
        return t.unsqueeze(0) if t.dim() == 3 else t

    q4, k4, v4 = as4(q), as4(k), as4(v)
    if q4.dim() != 4 or k4.dim() != 4 or v4.dim() != 4:
        raise ValueError("q, k, v must be [T, heads, head_dim] or [1, T, heads, head_dim]")
    if q4.shape[0] != 1 or k4.shape[0] != 1 or v4.shape[0] != 1:
        raise ValueError("packed tensors have a single batch row")
    _, Tq, Hq, D = q4.shape
    Hkv = k4.shape[2]
    if tuple(v4.shape) != tuple(k4.shape):
        raise ValueError(f"v {tuple(v.shape)} must have k's shape {tuple(k.shape)}")
    if k4.shape[3] != D:
        raise ValueError("k/v head_dim must match q's")
    dev = q.device
    _same_device(dev, (("k", k), ("v", v), ("out", out)))
    if out is None:
        out = torch.zeros_like(q)
    elif tuple(out.shape) != tuple(q.shape):
        raise ValueError(f"out {tuple(out.shape)} must have q's shape {tuple(q.shape)}")
    o4 = as4(out)
    if softmax_scale is None:
        softmax_scale = D ** -0.5
    n = len(cu_seqlens_q) - 1
    if n < 0 or len(cu_seqlens_k) != n + 1:
        raise ValueError("cu_seqlens_q and cu_seqlens_k need num_segments + 1 entries each")
    cq, ck = _int32_array(cu_seqlens_q, n + 1), _int32_array(cu_seqlens_k, n + 1)
    uq, uk = _int32_array(seqused_q, n), _int32_array(seqused_k, n)
    descs = [tensor_desc(t) for t in (q4, k4, v4, o4)]
    cp = lambda a: ctypes.cast(a, ctypes.c_void_p) if a is not None else None
    with _OnDevice(dev):
        st = lib().attn_fwd_varlen(ctypes.byref(descs[0]), ctypes.byref(descs[1]), ctypes.byref(descs[2]),
                                   cp(cq), cp(ck), cp(uq), cp(uk), n, Hq, Hkv, float(softmax_scale),
                                   ctypes.byref(descs[3]), D, _stream_ptr(stream, dev))
        _check(st)
        if check_status:
            _raise_if_device_timeout(dev)
    return out


def sk_shard_pad_copy(src, dst, first_row: int, pad_mode: str = "zeros", stream=None):
    """dst[:, r] = src[:, first_row + r] while that row exists, else zeros
    (``pad_mode="zeros"``) or src's last row (``"repeat_last"``): one rank's
    chunk of a tail-padded shard in one pass.  src [B, S, ...], dst
    [B, L, ...] CUDA tensors of one dtype on one device, with contiguous rows
    (dims >= 2)."""
    import torch

    if src.dtype != dst.dtype or src.shape[0] != dst.shape[0] or src.shape[2:] != dst.shape[2:]:
        raise ValueError("src and dst must share dtype, batch and row shape")
    row_elems = 1
    for d in src.shape[2:]:
        row_elems *= d
    es = src.element_size()
    for t in (src, dst):
        if t.numel() and (not t.is_cuda or t[:1, :1].reshape(-1).numel() != row_elems or
                          not t[0, 0].is_contiguous()):
            raise ValueError("expected CUDA tensors with contiguous rows")
    _same_device(dst.device, (("src", src),))
    mode = {"zeros": 0, "repeat_last": 1}[pad_mode]
    with _OnDevice(dst.device):
        st = lib().sk_shard_pad_copy(src.data_ptr() if src.numel() else None, src.stride(0) * es,
                                     src.stride(1) * es, src.shape[1], dst.data_ptr(), dst.stride(0) * es,
                                     dst.stride(1) * es, dst.shape[1], int(first_row), row_elems * es,
                                     src.shape[0], mode, _stream_ptr(stream, dst.device))
        _check(st)
    return dst


def qk_rmsnorm_rope(q, k, w_q, w_k, rope_table, rot_dim: Optional[int] = None,
                    interleaved: bool = False, eps: float = 1e-6, stream=None, exact: bool = False):
    """In-place fused RMSNorm(head_dim) + RoPE on q [B,S,Hq,D] and k [B,S,Hkv,D] (bf16, CUDA).

    rope_table: fp32 CUDA [rows >= S, rot_dim] holding [cos | sin] (its width
    is rot_dim); w_q, w_k: bf16 [D].  Every tensor on q's device.
    exact: False (default) evaluates in fp32 (memory-bound, within one bf16
    ulp of the exact result at the magnitude of the rotation's terms); True
    returns the exact result's bits (slower).
    """
    import torch

    if q.dim() != 4 or k.dim() != 4:
        raise ValueError("q and k must be [batch, seq, heads, head_dim]")
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    if k.shape[0] != B or k.shape[1] != S or k.shape[3] != D:
        raise ValueError(f"k {tuple(k.shape)}: batch, seq and head_dim must match q {tuple(q.shape)}")
    if rope_table.dim() != 2:
        raise ValueError("rope_table must be [rows, rot_dim]")
    if rot_dim is None:
        rot_dim = rope_table.shape[1]
    if rot_dim > 0 and rope_table.shape[1] != rot_dim:
        raise ValueError(f"rope_table has {rope_table.shape[1]} columns, rot_dim is {rot_dim}")
    for w in (w_q, w_k):
        if w.dtype != torch.bfloat16 or not w.is_contiguous() or w.numel() != D:
            raise ValueError("weights must be contiguous bf16 [head_dim]")
    if rope_table.dtype != torch.float32 or not rope_table.is_contiguous():
        raise ValueError("rope_table must be contiguous fp32")
    dev = q.device
    for name, t in (("w_q", w_q), ("w_k", w_k), ("rope_table", rope_table)):
        if not t.is_cuda or t.device != dev:
            raise ValueError(f"{name} must be a CUDA tensor on {dev}")
    _same_device(dev, (("k", k),))
    dq, dk = tensor_desc(q), tensor_desc(k)
    with _OnDevice(dev):
        st = lib().qk_rmsnorm_rope(ctypes.byref(dq), ctypes.byref(dk), w_q.data_ptr(), w_k.data_ptr(),
                                   rope_table.data_ptr() if rope_table.numel() else None,
                                   rope_table.shape[0], int(rot_dim), int(bool(interleaved)), float(eps),
                                   Hq, Hkv, B, D, int(bool(exact)), _stream_ptr(stream, dev))
        _check(st)
    return q, k


def sk_device_status(device: Optional[int] = None, clear: bool = True) -> int:
    """Synchronise the device and return its status word (0 = no kernel gave up a wait)."""
    import torch

    if device is None:
        device = torch.cuda.current_device()
    v = ctypes.c_int32(0)
    _check(lib().sk_device_status(int(device), ctypes.byref(v), int(bool(clear))))
    return v.value


def sk_set_wait_timeout_ms(ms: int) -> None:
    _check(lib().sk_set_wait_timeout_ms(int(ms)))


def sk_test_stall_mma(on: bool) -> None:
    """Test hook: make every in-kernel wait run out (see include/splitkv_attn.h)."""
    _check(lib().sk_test_stall_mma(int(bool(on))))


def sk_abi_version() -> int:
    return int(lib().sk_abi_version())
