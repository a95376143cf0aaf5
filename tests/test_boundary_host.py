"""Host-side checks of the C ABI: the library loads without a GPU, exports every
symbol include/splitkv_attn.h declares, and rejects bad arguments before any
CUDA call (so these run on CPU-only machines).  Every call here uses invalid
arguments, so nothing is ever launched, on any machine."""
import ctypes
import os
import re

import pytest
import torch

import varlen_flash_attention_b200 as sk
from varlen_flash_attention_b200 import SkTensor, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "splitkv_attn.h")
FAKE = 0x7F0000000000  # 16-byte aligned, never dereferenced: every call below fails validation


@pytest.fixture(scope="module")
def L():
    build.build()
    return sk.lib()


def _declared_symbols():
    text = open(HEADER).read()
    return re.findall(r"SK_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)


def test_header_declares_the_entry_points():
    names = set(_declared_symbols())
    assert {"attn_fwd_split_kv", "attn_fwd_split_kv_ex", "attn_fwd_varlen", "qk_rmsnorm_rope", "sk_last_error",
            "sk_device_status", "sk_set_wait_timeout_ms", "sk_abi_version"} <= names


def test_library_exports_every_declared_symbol(L):
    for name in _declared_symbols():
        assert hasattr(L, name), name


def test_abi_version(L):
    assert sk.sk_abi_version() == 2


def _t(len_s, sb, ss, sh, ptr=FAKE):
    return SkTensor(ptr, sb, ss, sh, len_s)


def _call(L, q, kp, vp, ks, vs, out, Hq=2, Hkv=2, D=64, B=1, scale=0.125, real_len=None, q_valid=None):
    rl = (ctypes.c_int32 * B)(*real_len) if real_len is not None else None
    args = [ctypes.byref(x) for x in (q, kp, vp, ks, vs)] + [
        ctypes.cast(rl, ctypes.c_void_p) if rl is not None else None, Hq, Hkv, scale,
        ctypes.byref(out), B, D]
    if q_valid is None:
        return L.attn_fwd_split_kv(*args, None)
    qv = (ctypes.c_int32 * B)(*q_valid)
    return L.attn_fwd_split_kv_ex(*args, ctypes.cast(qv, ctypes.c_void_p), None)


def _good(D=64, H=2, Sq=64, Sp=16, Ss=64):
    """Descriptors of a valid contiguous problem on fake, disjoint addresses."""
    q = _t(Sq, Sq * H * D, H * D, D, FAKE)
    kp = _t(Sp, Sp * H * D, H * D, D, FAKE + (1 << 24))
    vp = _t(Sp, Sp * H * D, H * D, D, FAKE + (2 << 24))
    ks = _t(Ss, Ss * H * D, H * D, D, FAKE + (3 << 24))
    vs = _t(Ss, Ss * H * D, H * D, D, FAKE + (4 << 24))
    out = _t(Sq, Sq * H * D, H * D, D, FAKE + (5 << 24))
    return [q, kp, vp, ks, vs, out]


INVALID, UNSUPPORTED = 1, 2


def _expect(L, status, *args, **kw):
    st = _call(L, *args, **kw)
    assert st == status, (st, L.sk_last_error())
    assert L.sk_last_error()


def test_rejects_gqa_indivisible(L):
    _expect(L, INVALID, *_good(), Hq=3, Hkv=2)


def test_rejects_unsupported_head_dim(L):
    _expect(L, UNSUPPORTED, *_good(D=96), D=96)


def test_rejects_misaligned_pointer(L):
    g = _good()
    g[0] = _t(64, 64 * 128, 128, 64, FAKE + 2)
    _expect(L, INVALID, *g)


def test_rejects_stride_not_multiple_of_8(L):
    g = _good()
    g[3] = _t(64, 64 * 128, 124, 64, FAKE + (3 << 24))
    _expect(L, INVALID, *g)


def test_rejects_real_len_out_of_range(L):
    _expect(L, INVALID, *_good(), real_len=[81])
    _expect(L, INVALID, *_good(), real_len=[-1])


def test_rejects_q_valid_out_of_range(L):
    _expect(L, INVALID, *_good(), q_valid=[65])


def test_rejects_len_mismatch(L):
    g = _good()
    g[2] = _t(15, 15 * 128, 128, 64, FAKE + (2 << 24))  # v_prefix shorter than k_prefix
    _expect(L, INVALID, *g)
    g = _good()
    g[5] = _t(63, 63 * 128, 128, 64, FAKE + (5 << 24))  # out shorter than q
    _expect(L, INVALID, *g)


def test_rejects_out_aliasing_an_input(L):
    g = _good()
    g[5] = _t(64, 64 * 128, 128, 64, FAKE + (3 << 24) + 1024)  # inside k_suffix
    _expect(L, INVALID, *g)


def test_rejects_self_overlapping_out(L):
    g = _good()
    g[5] = _t(64, 64 * 128, 64, 64, FAKE + (5 << 24))  # stride_s < heads * head_dim
    _expect(L, INVALID, *g)


def test_rejects_bad_scale(L):
    _expect(L, INVALID, *_good(), scale=float("nan"))
    _expect(L, INVALID, *_good(), scale=-1.0)


def test_rejects_null_pointer(L):
    g = _good()
    g[1] = _t(16, 16 * 128, 128, 64, None)
    _expect(L, INVALID, *g)


def test_wait_timeout_setter(L):
    assert L.sk_set_wait_timeout_ms(0) == INVALID
    assert L.sk_set_wait_timeout_ms(2000) == 0


def test_prologue_rejects_bad_args(L):
    q = _t(8, 8 * 256, 256, 128, FAKE)
    k = _t(8, 8 * 128, 128, 128, FAKE + (1 << 24))
    w = FAKE + (2 << 24)
    tab = FAKE + (3 << 24)
    # odd rot_dim
    assert L.qk_rmsnorm_rope(ctypes.byref(q), ctypes.byref(k), w, w, tab, 8, 95, 0, 1e-6, 2, 1, 1, 128, 0, None) == INVALID
    # unsupported head_dim
    assert L.qk_rmsnorm_rope(ctypes.byref(q), ctypes.byref(k), w, w, tab, 8, 64, 0, 1e-6, 2, 1, 1, 96, 0, None) == UNSUPPORTED
    # table shorter than the sequence
    assert L.qk_rmsnorm_rope(ctypes.byref(q), ctypes.byref(k), w, w, tab, 7, 96, 0, 1e-6, 2, 1, 1, 128, 0, None) == INVALID
    # half-split rotary width not a multiple of 16
    assert L.qk_rmsnorm_rope(ctypes.byref(q), ctypes.byref(k), w, w, tab, 8, 72, 0, 1e-6, 2, 1, 1, 128, 0, None) == UNSUPPORTED


def test_python_binding_raises_on_missing_library(monkeypatch, tmp_path):
    monkeypatch.setattr(sk, "_lib", None)
    monkeypatch.setattr(sk, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        sk.lib()


# ---------------------------------------------------------------- packed varlen


def _varlen_call(L, cq, ck, uq=None, uk=None, Tq=64, Tk=80, Hq=2, Hkv=2, D=64, scale=0.125,
                 out_ptr=None, nseg=None):
    q = _t(Tq, 0, Hq * D, D, FAKE)
    k = _t(Tk, 0, Hkv * D, D, FAKE + (1 << 24))
    v = _t(Tk, 0, Hkv * D, D, FAKE + (2 << 24))
    out = _t(Tq, 0, Hq * D, D, FAKE + (3 << 24) if out_ptr is None else out_ptr)
    n = len(cq) - 1 if nseg is None else nseg
    arr = lambda a: ctypes.cast((ctypes.c_int32 * len(a))(*a), ctypes.c_void_p) if a is not None else None
    return L.attn_fwd_varlen(ctypes.byref(q), ctypes.byref(k), ctypes.byref(v), arr(cq), arr(ck), arr(uq),
                             arr(uk), n, Hq, Hkv, scale, ctypes.byref(out), D, None)


@pytest.mark.parametrize("kw", [
    dict(cq=[0, 40, 30], ck=[0, 40, 80]),                     # cu_q decreases
    dict(cq=[0, 30, 64], ck=[0, 50, 81]),                     # cu_k past k.len_s
    dict(cq=[0, 30, 65], ck=[0, 50, 80]),                     # cu_q past q.len_s
    dict(cq=[-1, 30, 64], ck=[0, 50, 80]),                    # negative start
    dict(cq=[0, 30, 64], ck=[0, 50, 80], uq=[31, 34]),        # seqused_q > segment
    dict(cq=[0, 30, 64], ck=[0, 50, 80], uk=[50, 31]),        # seqused_k > segment
    dict(cq=[0, 30, 64], ck=[0, 50, 80], uk=[-1, 3]),
    dict(cq=[0, 30, 64], ck=[0, 50, 80], scale=-1.0),
    dict(cq=[0, 30, 64], ck=[0, 50, 80], Hq=3, Hkv=2),
    dict(cq=[0, 30, 64], ck=[0, 50, 80], out_ptr=FAKE + 4096),  # out overlaps q
    dict(cq=[0, 64], ck=[0, 80], nseg=-1),
])
def test_varlen_rejects_bad_arguments(L, kw):
    st = _varlen_call(L, **kw)
    assert st == INVALID, (st, L.sk_last_error())
    assert L.sk_last_error()


def test_varlen_rejects_unsupported_head_dim(L):
    assert _varlen_call(L, [0, 64], [0, 80], D=96) == UNSUPPORTED


def test_varlen_null_cu_arrays_rejected(L):
    q = _t(64, 0, 128, 64, FAKE)
    k = _t(80, 0, 128, 64, FAKE + (1 << 24))
    out = _t(64, 0, 128, 64, FAKE + (3 << 24))
    st = L.attn_fwd_varlen(ctypes.byref(q), ctypes.byref(k), ctypes.byref(k), None, None, None, None, 2, 2, 2,
                           0.125, ctypes.byref(out), 64, None)
    assert st == INVALID


# ---------------------------------------------------------------- shard pad copy


@pytest.mark.parametrize("kw", [
    dict(row_bytes=24),                   # not a multiple of 16
    dict(row_bytes=0),
    dict(src_ss=100),                     # stride not a multiple of 16
    dict(pad_mode=2),
    dict(dst_rows=-1),
    dict(src_rows=0, pad_mode=1),         # repeat_last without a source row
    dict(dst=FAKE + 8),                   # misaligned
    dict(dst=FAKE + 64),                  # overlaps src
    dict(dst_ss=16, row_bytes=32),        # destination rows overlap
])
def test_shard_pad_copy_rejects_bad_arguments(L, kw):
    a = dict(src=FAKE, src_sb=1 << 20, src_ss=256, src_rows=100, dst=FAKE + (1 << 24), dst_sb=1 << 16,
             dst_ss=256, dst_rows=13, first_row=91, row_bytes=256, batch=2, pad_mode=0)
    a.update(kw)
    st = L.sk_shard_pad_copy(a["src"], a["src_sb"], a["src_ss"], a["src_rows"], a["dst"], a["dst_sb"],
                             a["dst_ss"], a["dst_rows"], a["first_row"], a["row_bytes"], a["batch"],
                             a["pad_mode"], None)
    assert st == INVALID, (st, L.sk_last_error())


def _scatter(L, n=2, chunk=32, ptrs=None, head_offset=0, layout=None, Hq=2, D=64, Sq=64):
    g = _good(D=D, H=Hq, Sq=Sq)
    if ptrs is None:
        ptrs = [FAKE + ((6 + r) << 24) for r in range(n)]
    arr = (ctypes.c_void_p * max(1, len(ptrs)))(*ptrs) if ptrs else None
    if layout is None:
        layout = _t(chunk, chunk * 4 * Hq * D, 4 * Hq * D, D, None)
    return L.attn_fwd_split_kv_scatter(
        *[ctypes.byref(x) for x in g[:5]], None, None, Hq, Hq, 0.125,
        ctypes.cast(arr, ctypes.c_void_p) if arr is not None else None, n, ctypes.byref(layout),
        head_offset, 1, D, None)


@pytest.mark.parametrize("kw", [
    {"n": 0}, {"n": 9, "chunk": 8},                       # 1..8 destinations
    {"n": 2, "chunk": 31},                                # 2 x 31 != 64 query rows
    {"ptrs": [FAKE + (6 << 24), None]},                   # NULL destination
    {"ptrs": [FAKE + (6 << 24), FAKE + (7 << 24) + 8]},   # misaligned destination
    {"head_offset": -1},
    {"layout": _t(32, 32 * 512, 508, 64, None)},          # stride_s not a multiple of 8
    {"layout": _t(32, 32 * 512, 64, 64, None)},           # rows of 2 heads overlap
])
def test_scatter_rejects_bad_arguments(L, kw):
    st = _scatter(L, **kw)
    assert st == INVALID, (st, L.sk_last_error())
    assert L.sk_last_error()


def test_scatter_rejects_null_destination_array(L):
    g = _good()
    layout = _t(32, 32 * 512, 512, 64, None)
    st = L.attn_fwd_split_kv_scatter(*[ctypes.byref(x) for x in g[:5]], None, None, 2, 2, 0.125, None, 2,
                                     ctypes.byref(layout), 0, 1, 64, None)
    assert st == INVALID


def test_scatter_binding_checks_shapes_before_the_library():
    q = torch.zeros(1, 64, 2, 64, dtype=torch.bfloat16)
    kv = torch.zeros(1, 16, 2, 64, dtype=torch.bfloat16)
    good = [torch.zeros(1, 32, 4, 64, dtype=torch.bfloat16) for _ in range(2)]
    with pytest.raises(ValueError):
        sk.attn_fwd_split_kv_scatter(q, kv, kv, kv, kv, [])                      # no destination
    with pytest.raises(ValueError):
        sk.attn_fwd_split_kv_scatter(q, kv, kv, kv, kv, good * 5)                # 10 destinations
    with pytest.raises(ValueError):
        sk.attn_fwd_split_kv_scatter(q, kv, kv, kv, kv, [good[0], good[1][:, :16]])  # shapes differ
    with pytest.raises(ValueError):
        sk.attn_fwd_split_kv_scatter(q, kv, kv, kv, kv, good[:1])                # 1 x 32 rows != 64
    with pytest.raises(ValueError):
        sk.attn_fwd_split_kv_scatter(q, kv, kv, kv, kv, good, head_offset=3)     # heads 3..4 of 4


def test_scatter_empty_batch_is_a_no_op(L):
    """batch 0 succeeds without touching the device, like the plain entry
    (an empty query stream is rejected instead: destinations have >= 1 row)."""
    g = _good()
    layout = _t(32, 32 * 256, 256, 64, None)
    arr = (ctypes.c_void_p * 2)(FAKE + (6 << 24), FAKE + (7 << 24))
    st = L.attn_fwd_split_kv_scatter(*[ctypes.byref(x) for x in g[:5]], None, None, 2, 2, 0.125,
                                     ctypes.cast(arr, ctypes.c_void_p), 2, ctypes.byref(layout), 0, 0, 64, None)
    assert st == 0, L.sk_last_error()
    g = _good(Sq=0)
    layout = _t(0, 0, 256, 64, None)
    st = L.attn_fwd_split_kv_scatter(*[ctypes.byref(x) for x in g[:5]], None, None, 2, 2, 0.125,
                                     ctypes.cast(arr, ctypes.c_void_p), 2, ctypes.byref(layout), 0, 1, 64, None)
    assert st == 1


# ---------------------------------------------------------------- binding shape and device checks
# Each mismatch must raise ValueError from the binding's own checks (the
# message names the problem), before any tensor reaches the library.

def _bf(*shape):
    return torch.zeros(*shape, dtype=torch.bfloat16)


def _attn_args(B=2, Sq=64, Hq=4, Hkv=2, D=64, Sp=16, Ss=48):
    return dict(q=_bf(B, Sq, Hq, D), k_prefix=_bf(B, Sp, Hkv, D), v_prefix=_bf(B, Sp, Hkv, D),
                k_suffix=_bf(B, Ss, Hkv, D), v_suffix=_bf(B, Ss, Hkv, D))


@pytest.mark.parametrize("name, shape, msg", [
    ("k_prefix", (1, 16, 2, 64), "batch and head_dim"),
    ("v_suffix", (2, 48, 2, 32), "batch and head_dim"),
    ("k_suffix", (2, 48, 1, 64), "heads"),
    ("v_prefix", (2, 16, 4, 64), "heads"),
    ("v_prefix", (2, 15, 2, 64), "same length"),
    ("out", (2, 64, 2, 64), "q's shape"),
    ("out", (1, 64, 4, 64), "q's shape"),
])
def test_binding_rejects_shape_mismatch(name, shape, msg, monkeypatch):
    def no_lib():
        raise AssertionError("the library must not be reached")

    monkeypatch.setattr(sk, "lib", no_lib)
    a = _attn_args()
    a[name] = _bf(*shape)
    with pytest.raises(ValueError, match=msg):
        sk.attn_fwd_split_kv(**a)


def test_binding_rejects_cpu_weights_and_table_for_prologue(monkeypatch):
    monkeypatch.setattr(sk, "lib", lambda: (_ for _ in ()).throw(AssertionError("no library call")))
    q, k = _bf(1, 8, 2, 64), _bf(1, 8, 1, 64)
    w = _bf(64)
    tab = torch.zeros(8, 64)
    with pytest.raises(ValueError, match="CUDA tensor"):
        sk.qk_rmsnorm_rope(q, k, w, w, tab)
    with pytest.raises(ValueError, match="columns"):
        sk.qk_rmsnorm_rope(q, k, w, w, tab, rot_dim=32)
    with pytest.raises(ValueError, match="batch, seq and head_dim"):
        sk.qk_rmsnorm_rope(q, _bf(1, 7, 1, 64), w, w, tab)
    with pytest.raises(ValueError, match="batch, seq and head_dim"):
        sk.qk_rmsnorm_rope(q, _bf(2, 8, 1, 64), w, w, tab)


def test_prologue_rejects_q_k_sharing_tokens(L):
    """k placed inside q's token rows (fused layout shifted by one token, or
    head ranges that spill into the next token) is rejected: the in-place
    kernel would read and write the same elements from different threads."""
    D, Hq, Hkv, S = 64, 4, 2, 8
    ss = (Hq + 2 * Hkv) * D   # fused [B, S, Hq + 2 Hkv, D] row
    w = FAKE
    def call(k_off_elems, stride_s=ss):
        q = _t(S, S * stride_s, stride_s, D)
        k = _t(S, S * stride_s, stride_s, D, ptr=FAKE + 2 * k_off_elems)
        return L.qk_rmsnorm_rope(ctypes.byref(q), ctypes.byref(k), w, w, FAKE, S, 64, 0,
                                 ctypes.c_float(1e-6), Hq, Hkv, 1, D, 0, None)
    assert call(ss) == 1                  # k = q shifted by one token
    assert call(Hq * D, stride_s=(Hq + 1) * D) == 1  # k's heads spill into q's next token
    assert b"overlap" in L.sk_last_error()
