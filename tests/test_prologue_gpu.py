"""Parity of the fused Q/K RMSNorm + RoPE prologue kernels with the fp64 oracle.

Exact instance (exact=True).  Bar: every output element within 1 bf16 ulp of
the oracle and at least 99.99% bit-identical on the ordinary cases, where the
ulp allowance covers a sum-of-squares reduction order that differs from the
oracle's sequential one (it only matters when the row's squares span more
than fp64's precision).  The special-value, multi-block and large cases
demand every bit: the kernel decides each bf16 rounding either from an fp32
value whose error bound keeps it off the rounding midpoint or by recomputing
the element in fp64.

Default fp32 instance (exact=False): the same formula and rounding points in
fp32.  Bound, derived from the arithmetic: y = bf16(x * r * w) is computed
from an fp32 value within a few fp32 ulps of the exact one, so it equals the
oracle's y or sits one bf16 ulp away (when the exact value is that close to a
rounding midpoint); one bf16 ulp is at most 2^-7 of the value.  A rotated
output z = y * c + y' * s' (c the cosine, s' the signed sine, y' the pair's
other element) then moves by at most 2^-7 (|y c| + |y' s'|) = 2^-7 m <=
2 ulp_bf16(m), m = |y c| + |y' s'| (the magnitude of its own two terms), and
each side rounds once more (half an ulp of z <= half an ulp of m each):
|z_gpu - z_ref| <= 3 ulp_bf16(m).  Dims past rot_dim are y itself: within
1 ulp of |y|.  The tests also require at least 99.9% of the elements to be
bit-identical.
"""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sk():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    from varlen_flash_attention_b200 import build

    build.build()
    import varlen_flash_attention_b200 as m

    return m


def _table(S, rot_dim, theta=10000.0):
    pos = np.arange(S, dtype=np.float64)[:, None]
    inv = theta ** (-np.arange(0, rot_dim, 2, dtype=np.float64) / rot_dim)
    ang = pos * inv[None, :]
    return torch.from_numpy(np.concatenate([np.cos(ang), np.sin(ang)], 1).astype(np.float32))


def _ulp_check(got_bits, ref_bits):
    a = got_bits.astype(np.int32)
    b = ref_bits.astype(np.int32)
    # bf16 bit patterns are sign-magnitude; map to a monotone integer line
    a = np.where(a & 0x8000, -(a & 0x7FFF), a)
    b = np.where(b & 0x8000, -(b & 0x7FFF), b)
    d = np.abs(a - b)
    assert d.max() <= 1, d.max()
    assert (d == 0).mean() >= 0.9999, (d == 0).mean()


@pytest.mark.parametrize("D,rot,inter", [(128, 96, False), (128, 128, False), (128, 96, True),
                                          (64, 64, False), (64, 32, True), (256, 128, False),
                                          (128, 0, False)])
def test_prologue_matches_oracle(sk, D, rot, inter):
    gen = torch.Generator().manual_seed(D + rot + int(inter))
    B, S, Hq, Hkv = 2, 77, 6, 2
    q = (torch.randn(B, S, Hq, D, generator=gen) * 2).to(torch.bfloat16)
    k = (torch.randn(B, S, Hkv, D, generator=gen) * 2).to(torch.bfloat16)
    wq = (1 + 0.1 * torch.randn(D, generator=gen)).to(torch.bfloat16)
    wk = (1 + 0.1 * torch.randn(D, generator=gen)).to(torch.bfloat16)
    tab = _table(S + 5, rot) if rot else torch.zeros(S, 0)
    eps = float(np.float32(1e-6))  # the C ABI takes eps as fp32
    ref_q = oracle.qk_rmsnorm_rope(q, wq, tab.numpy() if rot else np.zeros((S, 0), np.float32),
                                   rot_dim=rot, interleaved=inter, eps=eps)
    ref_k = oracle.qk_rmsnorm_rope(k, wk, tab.numpy() if rot else np.zeros((S, 0), np.float32),
                                   rot_dim=rot, interleaved=inter, eps=eps)
    qd, kd = q.cuda(), k.cuda()
    tabd = tab.cuda() if rot else torch.zeros(S, 8, device="cuda")
    sk.qk_rmsnorm_rope(qd, kd, wq.cuda(), wk.cuda(), tabd, rot_dim=rot, interleaved=inter, eps=1e-6, exact=True)
    torch.cuda.synchronize()
    _ulp_check(qd.cpu().view(torch.int16).numpy().view(np.uint16), ref_q)
    _ulp_check(kd.cpu().view(torch.int16).numpy().view(np.uint16), ref_k)


def test_prologue_in_place_on_fused_qkv_view(sk):
    gen = torch.Generator().manual_seed(1)
    B, S, Hq, Hkv, D = 1, 300, 8, 2, 128
    qkv = torch.randn(B, S, Hq + 2 * Hkv, D, generator=gen).to(torch.bfloat16)
    wq = torch.randn(D, generator=gen).to(torch.bfloat16)
    wk = torch.randn(D, generator=gen).to(torch.bfloat16)
    tab = _table(S, 96)
    d = qkv.cuda()
    sk.qk_rmsnorm_rope(d[:, :, :Hq], d[:, :, Hq:Hq + Hkv], wq.cuda(), wk.cuda(), tab.cuda(), eps=1e-5,
                       exact=True)
    torch.cuda.synchronize()
    got = d.cpu()
    assert torch.equal(got[:, :, Hq + Hkv:], qkv[:, :, Hq + Hkv:])  # v untouched
    eps = float(np.float32(1e-5))
    ref_q = oracle.qk_rmsnorm_rope(qkv[:, :, :Hq].contiguous(), wq, tab.numpy(), eps=eps)
    ref_k = oracle.qk_rmsnorm_rope(qkv[:, :, Hq:Hq + Hkv].contiguous(), wk, tab.numpy(), eps=eps)
    _ulp_check(got[:, :, :Hq].contiguous().view(torch.int16).numpy().view(np.uint16), ref_q)
    _ulp_check(got[:, :, Hq:Hq + Hkv].contiguous().view(torch.int16).numpy().view(np.uint16), ref_k)


def _bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _run_both(sk, q, k, wq, wk, tab, rot, inter, eps, exact=True):
    S = q.shape[1]
    eps32 = float(np.float32(eps))
    ref_q = oracle.qk_rmsnorm_rope(q, wq, tab.numpy(), rot_dim=rot, interleaved=inter, eps=eps32)
    ref_k = oracle.qk_rmsnorm_rope(k, wk, tab.numpy(), rot_dim=rot, interleaved=inter, eps=eps32)
    qd, kd = q.cuda(), k.cuda()
    tabd = tab.cuda() if rot else torch.zeros(S, 8, device="cuda")
    sk.qk_rmsnorm_rope(qd, kd, wq.cuda(), wk.cuda(), tabd, rot_dim=rot, interleaved=inter, eps=eps, exact=exact)
    torch.cuda.synchronize()
    return _bits(qd.cpu()), ref_q, _bits(kd.cpu()), ref_k


@pytest.mark.parametrize("inter", [False, True])
def test_prologue_special_values_bit_exact(sk, inter):
    """Rows that leave the kernel's fast path (bf16 subnormals, zero rows with
    eps = 0, inf/NaN inputs, weights and table entries near the top of the
    range) mixed with ordinary rows: every output bit equals the oracle's."""
    gen = torch.Generator().manual_seed(11 + int(inter))
    B, S, Hq, Hkv, D, rot = 1, 40, 5, 3, 128, 96
    q = torch.randn(B, S, Hq, D, generator=gen)
    k = torch.randn(B, S, Hkv, D, generator=gen)
    q[0, 1, 2] = 0.0                                   # zero row: r = 1/sqrt(eps)
    q[0, 2, 0, :] *= 1e-38                             # bf16 subnormal inputs
    q[0, 3, 1, 5] = 3e38                               # one huge value dwarfs the rest
    q[0, 4, 4, 7] = float("inf")
    k[0, 5, 1, 9] = float("nan")
    k[0, 6, 2, :64] = 0.0                              # half-zero row
    k[0, 7, 0, 3] = 1e-40                              # subnormal next to normal values
    k[0, 3, 0, :] = -0.0                               # negative-zero row
    q[0, 9, 1, 100:110] = -0.0                         # negative zeros past rot_dim
    q[0, 11, 3, 10:40] = -0.0                          # negative zeros in rotated dims
    q, k = q.to(torch.bfloat16), k.to(torch.bfloat16)
    wq = (1 + 0.1 * torch.randn(D, generator=gen)).to(torch.bfloat16)
    wk = (1 + 0.1 * torch.randn(D, generator=gen)).to(torch.bfloat16)
    wk[17] = 1e-39                                     # y of that dim in bf16's subnormal range
    tab = _table(S, rot)
    tab[9, 3] = 1e38                                   # huge cos: overflowing rotation
    tab[10, rot // 2 + 1] = -3e38
    for eps in (1e-6, 0.0):
        q0 = q.clone()
        q0[0, 8, 3] = 0.0 if eps == 0.0 else q0[0, 8, 3]
        gq, rq, gk, rk = _run_both(sk, q0, k, wq, wk, tab, rot, inter, eps)
        assert np.array_equal(gq, rq), np.argwhere(gq != rq)[:5]
        assert np.array_equal(gk, rk), np.argwhere(gk != rk)[:5]


def test_prologue_huge_weight_bit_exact(sk):
    """A weight near bf16's maximum overflows y to inf on some rows; the
    rotation then spreads inf/NaN to the partner dims exactly as in the
    oracle."""
    gen = torch.Generator().manual_seed(5)
    B, S, Hq, Hkv, D, rot = 2, 9, 4, 2, 64, 64
    q = torch.randn(B, S, Hq, D, generator=gen).to(torch.bfloat16)
    k = torch.randn(B, S, Hkv, D, generator=gen).to(torch.bfloat16)
    wq = torch.ones(D).to(torch.bfloat16)
    wq[4] = 3e38
    wk = torch.ones(D).to(torch.bfloat16)
    tab = _table(S, rot)
    gq, rq, gk, rk = _run_both(sk, q, k, wq, wk, tab, rot, False, 1e-6)
    assert np.array_equal(gq, rq)
    assert np.array_equal(gk, rk)


@pytest.mark.parametrize("D,rot,inter", [(128, 128, False), (256, 256, True), (64, 0, False)])
def test_prologue_many_tokens_bit_exact(sk, D, rot, inter):
    """Several blocks of tokens and a ragged last block (tokens not a multiple
    of the tokens per block), ordinary values: bit-identical to the oracle."""
    gen = torch.Generator().manual_seed(D + rot)
    B, S, Hq, Hkv = 3, 171, 7, 1
    q = (torch.randn(B, S, Hq, D, generator=gen) * 3).to(torch.bfloat16)
    k = (torch.randn(B, S, Hkv, D, generator=gen) * 0.2).to(torch.bfloat16)
    wq = (1 + 0.2 * torch.randn(D, generator=gen)).to(torch.bfloat16)
    wk = (0.5 + 0.2 * torch.randn(D, generator=gen)).to(torch.bfloat16)
    tab = _table(S, rot) if rot else torch.zeros(S, 0)
    gq, rq, gk, rk = _run_both(sk, q, k, wq, wk, tab, rot, inter, 1e-5)
    assert np.array_equal(gq, rq)
    assert np.array_equal(gk, rk)


@pytest.mark.parametrize("inter,scale", [(False, 1.0), (True, 1e-3), (False, 300.0)])
def test_prologue_large_bit_exact(sk, inter, scale):
    """About 5M elements per call: enough that a few thousand elements land
    near a bf16 midpoint and take the kernel's fp64 fix-up; every output bit
    equals the oracle's."""
    gen = torch.Generator().manual_seed(int(scale * 7) + int(inter))
    B, S, Hq, Hkv, D, rot = 1, 4096, 8, 2, 128, 128
    q = (torch.randn(B, S, Hq, D, generator=gen) * scale).to(torch.bfloat16)
    k = (torch.randn(B, S, Hkv, D, generator=gen) * scale).to(torch.bfloat16)
    wq = (1 + 0.3 * torch.randn(D, generator=gen)).to(torch.bfloat16)
    wk = (0.7 + 0.3 * torch.randn(D, generator=gen)).to(torch.bfloat16)
    tab = _table(S, rot, theta=1e6)
    gq, rq, gk, rk = _run_both(sk, q, k, wq, wk, tab, rot, inter, 1e-6)
    assert np.array_equal(gq, rq), np.argwhere(gq != rq)[:5]
    assert np.array_equal(gk, rk), np.argwhere(gk != rk)[:5]


@pytest.mark.parametrize("D,inter", [(128, False), (64, True)])
def test_prologue_many_heads_bit_exact(sk, D, inter):
    """32 heads per token (20 q + 12 k) walked by one lane group, two rows
    at a time across the q/k boundary, ragged last block; every output bit
    equals the oracle's."""
    gen = torch.Generator().manual_seed(40 + D)
    B, S, Hq, Hkv, rot = 2, 100, 20, 12, D
    q = torch.randn(B, S, Hq, D, generator=gen).to(torch.bfloat16)
    k = torch.randn(B, S, Hkv, D, generator=gen).to(torch.bfloat16)
    wq = (1 + 0.2 * torch.randn(D, generator=gen)).to(torch.bfloat16)
    wk = (1 + 0.2 * torch.randn(D, generator=gen)).to(torch.bfloat16)
    tab = _table(S, rot)
    gq, rq, gk, rk = _run_both(sk, q, k, wq, wk, tab, rot, inter, 1e-6)
    assert np.array_equal(gq, rq), np.argwhere(gq != rq)[:5]
    assert np.array_equal(gk, rk), np.argwhere(gk != rk)[:5]


@pytest.mark.parametrize("Hq,Hkv,D", [(3, 2, 128), (2, 1, 64), (5, 4, 256)])
def test_prologue_odd_head_count_bit_exact(sk, Hq, Hkv, D):
    """An odd number of rows per token: the last batch of two holds one row."""
    gen = torch.Generator().manual_seed(Hq * 10 + Hkv + D)
    B, S, rot = 2, 37, D // 2 if D != 64 else 64
    q = torch.randn(B, S, Hq, D, generator=gen).to(torch.bfloat16)
    k = torch.randn(B, S, Hkv, D, generator=gen).to(torch.bfloat16)
    wq = (1 + 0.2 * torch.randn(D, generator=gen)).to(torch.bfloat16)
    wk = (1 + 0.2 * torch.randn(D, generator=gen)).to(torch.bfloat16)
    tab = _table(S, rot)
    gq, rq, gk, rk = _run_both(sk, q, k, wq, wk, tab, rot, False, 1e-6)
    assert np.array_equal(gq, rq), np.argwhere(gq != rq)[:5]
    assert np.array_equal(gk, rk), np.argwhere(gk != rk)[:5]


# ---------------------------------------------------------------- default fp32 instance


def _f64(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _ulp_bf16(m):
    """bf16 ulp at magnitude m (0 for m == 0): 2^(floor(log2 m) - 7)."""
    m = np.asarray(m, dtype=np.float64)
    e = np.floor(np.log2(np.where(m > 0, m, 1.0)))
    return np.where(m > 0, np.exp2(e - 7), 0.0)


def _fast_check(got_bits, x, w, tab, rot, inter, eps32, min_identical=0.999):
    """The default instance against the oracle: |z_gpu - z_ref| <= 3 ulp_bf16(m)
    on rotated dims, m the magnitude of the output's own two terms (|y_a c| +
    |y_p s| for the first element of a pair, |y_p c| + |y_a s| for the
    second; y = the oracle's normalised value, c / s the pair's table
    entries), within 1 ulp of |y| past rot_dim; and at least min_identical of
    the elements bit-identical."""
    ref = oracle.qk_rmsnorm_rope(x, w, tab.numpy(), rot_dim=rot, interleaved=inter, eps=eps32)
    y = _f64(oracle.qk_rmsnorm_rope(x, w, np.zeros((tab.shape[0], 0), np.float32), rot_dim=0, eps=eps32))
    B, S, H, D = y.shape
    m = np.abs(y).copy()
    allow = _ulp_bf16(m)
    if rot:
        t = tab.numpy().astype(np.float64)[:S]
        half = rot // 2
        i = np.arange(half)
        if inter:
            a_idx, p_idx = 2 * i, 2 * i + 1
        else:
            a_idx, p_idx = i, i + half
        c = t[:, i][None, :, None, :]
        sn = t[:, half + i][None, :, None, :]
        ya, yp = y[..., a_idx], y[..., p_idx]
        m[..., a_idx] = np.abs(ya * c) + np.abs(yp * sn)
        m[..., p_idx] = np.abs(yp * c) + np.abs(ya * sn)
        allow = _ulp_bf16(m)
        allow[..., a_idx] *= 3
        allow[..., p_idx] *= 3
    g, r = _f64(got_bits), _f64(ref)
    both_nan = np.isnan(g) & np.isnan(r)
    same_inf = np.isinf(g) & (g == r)
    diff = np.where(both_nan | same_inf, 0.0, np.abs(g - r))
    assert not np.any(np.isnan(diff)), "NaN where the oracle has a number (or the reverse)"
    bad = diff > allow
    assert not bad.any(), (np.argwhere(bad)[:5], diff[bad][:5], allow[bad][:5])
    ident = float((got_bits == ref).mean())
    assert ident >= min_identical, ident
    return ident


@pytest.mark.parametrize("D,rot,inter", [(128, 96, False), (128, 128, False), (128, 96, True),
                                          (64, 64, False), (64, 32, True), (256, 128, False),
                                          (128, 0, False)])
def test_fast_prologue_within_bound(sk, D, rot, inter):
    gen = torch.Generator().manual_seed(100 + D + rot + int(inter))
    B, S, Hq, Hkv = 2, 333, 6, 2
    q = (torch.randn(B, S, Hq, D, generator=gen) * 2).to(torch.bfloat16)
    k = (torch.randn(B, S, Hkv, D, generator=gen) * 0.5).to(torch.bfloat16)
    wq = (1 + 0.1 * torch.randn(D, generator=gen)).to(torch.bfloat16)
    wk = (1 + 0.1 * torch.randn(D, generator=gen)).to(torch.bfloat16)
    tab = _table(S + 5, rot) if rot else torch.zeros(S, 0)
    gq, _, gk, _ = _run_both(sk, q, k, wq, wk, tab, rot, inter, 1e-6, exact=False)
    eps32 = float(np.float32(1e-6))
    _fast_check(gq, q, wq, tab, rot, inter, eps32)
    _fast_check(gk, k, wk, tab, rot, inter, eps32)


@pytest.mark.parametrize("inter", [False, True])
def test_fast_prologue_large_and_special_values(sk, inter):
    """About 5M elements per call, plus zero, inf and NaN rows (eps > 0): the
    fp32 instance stays within the bound and propagates inf/NaN as the oracle
    does.  (With eps = 0, a row whose squares all underflow fp32 differs: its
    fp32 sum is 0; the exact instance covers that case.)"""
    gen = torch.Generator().manual_seed(7 + int(inter))
    B, S, Hq, Hkv, D, rot = 1, 4096, 8, 2, 128, 128
    q = torch.randn(B, S, Hq, D, generator=gen)
    k = torch.randn(B, S, Hkv, D, generator=gen) * 30
    q[0, 1, 2] = 0.0
    q[0, 4, 4, 7] = float("inf")
    k[0, 5, 1, 9] = float("nan")
    k[0, 3, 0, :] = -0.0
    q, k = q.to(torch.bfloat16), k.to(torch.bfloat16)
    wq = (1 + 0.3 * torch.randn(D, generator=gen)).to(torch.bfloat16)
    wk = (0.7 + 0.3 * torch.randn(D, generator=gen)).to(torch.bfloat16)
    tab = _table(S, rot, theta=1e6)
    gq, _, gk, _ = _run_both(sk, q, k, wq, wk, tab, rot, inter, 1e-6, exact=False)
    eps32 = float(np.float32(1e-6))
    _fast_check(gq, q, wq, tab, rot, inter, eps32)
    _fast_check(gk, k, wk, tab, rot, inter, eps32)


def test_fast_prologue_fused_view_leaves_v_untouched(sk):
    gen = torch.Generator().manual_seed(2)
    B, S, Hq, Hkv, D = 1, 300, 8, 2, 128
    qkv = torch.randn(B, S, Hq + 2 * Hkv, D, generator=gen).to(torch.bfloat16)
    wq = torch.randn(D, generator=gen).to(torch.bfloat16)
    wk = torch.randn(D, generator=gen).to(torch.bfloat16)
    tab = _table(S, 96)
    d = qkv.cuda()
    sk.qk_rmsnorm_rope(d[:, :, :Hq], d[:, :, Hq:Hq + Hkv], wq.cuda(), wk.cuda(), tab.cuda(), eps=1e-5)
    torch.cuda.synchronize()
    got = d.cpu()
    assert torch.equal(got[:, :, Hq + Hkv:], qkv[:, :, Hq + Hkv:])
    eps = float(np.float32(1e-5))
    _fast_check(_bits(got[:, :, :Hq]), qkv[:, :, :Hq].contiguous(), wq, tab, 96, False, eps)
    _fast_check(_bits(got[:, :, Hq:Hq + Hkv]), qkv[:, :, Hq:Hq + Hkv].contiguous(), wk, tab, 96, False, eps)


@pytest.mark.parametrize("B,S,Hq,Hkv,D,rot,inter", [
    (2, 333, 6, 2, 128, 96, False),      # fewer tokens than warps in the grid
    (1, 4099, 32, 8, 128, 128, False),   # several tokens per warp, ragged tail
    (1, 700, 16, 4, 64, 32, True),
    (1, 300, 80, 8, 256, 128, False),    # many steps per token
])
def test_fast_prologue_contiguous_and_strided_heads_agree(sk, B, S, Hq, Hkv, D, rot, inter):
    """The fp32 instance on contiguous heads and on heads spaced two rows
    apart (a different address stream through the same copy ring): bit-
    identical outputs, the rows in between untouched, both within the bound."""
    gen = torch.Generator().manual_seed(B + S + Hq + D)
    q = (torch.randn(B, S, Hq, D, generator=gen) * 1.5).to(torch.bfloat16)
    k = torch.randn(B, S, Hkv, D, generator=gen).to(torch.bfloat16)
    wq = (1 + 0.1 * torch.randn(D, generator=gen)).to(torch.bfloat16)
    wk = (1 + 0.1 * torch.randn(D, generator=gen)).to(torch.bfloat16)
    tab = _table(S, rot)
    qa, ka = q.cuda(), k.cuda()
    qb_big = torch.zeros(B, S, 2 * Hq, D, dtype=torch.bfloat16, device="cuda")
    kb_big = torch.zeros(B, S, 2 * Hkv, D, dtype=torch.bfloat16, device="cuda")
    qb, kb = qb_big[:, :, ::2], kb_big[:, :, ::2]
    qb.copy_(qa)
    kb.copy_(ka)
    args = (wq.cuda(), wk.cuda(), tab.cuda())
    sk.qk_rmsnorm_rope(qa, ka, *args, rot_dim=rot, interleaved=inter, eps=1e-6)
    sk.qk_rmsnorm_rope(qb, kb, *args, rot_dim=rot, interleaved=inter, eps=1e-6)
    torch.cuda.synchronize()
    assert torch.equal(qa.view(torch.int16), qb.view(torch.int16))
    assert torch.equal(ka.view(torch.int16), kb.view(torch.int16))
    # the rows between the strided heads are untouched
    assert not qb_big[:, :, 1::2].any() and not kb_big[:, :, 1::2].any()
    eps32 = float(np.float32(1e-6))
    _fast_check(_bits(qa.cpu()), q, wq, tab, rot, inter, eps32)
    _fast_check(_bits(ka.cpu()), k, wk, tab, rot, inter, eps32)
