"""Parity of the packed variable-length entry point (attn_fwd_varlen, through
the C ABI) with the fp64 oracle: unequal segment lengths around the 128/256-row
tile edges, GQA, both head dims, hundreds of segments in one launch (and more
than one launch holds), pad exclusion through seqused_q/k (bitwise invariance
to pad contents, including NaN/Inf in the rows that share a segment's last
key tile; exact zero pad rows), rows outside every segment left untouched.
Same bar as the other parity tests: max-abs <= 2e-2, relative L2 <= 1e-2."""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-2
REL_L2 = 1e-2


@pytest.fixture(scope="module")
def sk():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    from varlen_flash_attention_b200 import build

    build.build()
    import varlen_flash_attention_b200 as m

    return m


def _packed(seed, q_lens, k_lens, Hq, Hkv, D):
    g = torch.Generator().manual_seed(seed)
    cq, ck = [0], [0]
    for lq, lk in zip(q_lens, k_lens):
        cq.append(cq[-1] + lq)
        ck.append(ck[-1] + lk)
    q = torch.randn(cq[-1], Hq, D, generator=g).to(torch.bfloat16)
    k = torch.randn(ck[-1], Hkv, D, generator=g).to(torch.bfloat16)
    v = torch.randn(ck[-1], Hkv, D, generator=g).to(torch.bfloat16)
    return q, k, v, cq, ck


def _compare(got, ref, what=""):
    diff = np.abs(got.astype(np.float64) - ref)
    max_abs = float(diff.max()) if diff.size else 0.0
    denom = float(np.sqrt((ref ** 2).sum()))
    rel = float(np.sqrt((diff ** 2).sum()) / denom) if denom > 0 else max_abs
    assert np.all(np.isfinite(got)), what
    assert max_abs <= MAX_ABS, f"{what} max_abs={max_abs}"
    assert rel <= REL_L2, f"{what} rel_l2={rel}"


@pytest.mark.parametrize("seed, D, Hq, Hkv, q_lens, k_lens", [
    (0, 128, 4, 4, [1, 127, 128, 129, 300], [5, 128, 129, 257, 40]),
    (1, 64, 8, 2, [256, 257, 33, 600], [513, 1, 200, 96]),
    (2, 128, 6, 2, [64] * 11, [100, 1, 37, 128, 255, 256, 64, 3, 90, 500, 17]),  # 11 segments: two launches
])
def test_varlen_matches_oracle(sk, seed, D, Hq, Hkv, q_lens, k_lens):
    q, k, v, cq, ck = _packed(seed, q_lens, k_lens, Hq, Hkv, D)
    out = sk.attn_fwd_varlen(q.cuda(), k.cuda(), v.cuda(), cq, ck)
    torch.cuda.synchronize()
    got = out.float().cpu().numpy()
    ref = oracle.attn_varlen(q, k, v, cq, ck)
    _compare(got, ref, f"seed {seed}")
    assert sk.sk_device_status() == 0


def test_varlen_pad_exclusion_and_untouched_rows(sk):
    """Three segments with pad (seqused < segment length), separated by 5-row
    gaps described as key-less segments (written as zeros), with 3 rows before
    the first and 4 after the last segment that no segment covers (untouched)."""
    D, Hq, Hkv = 128, 4, 2
    g = torch.Generator().manual_seed(7)
    seg_q, seg_k = [200, 77, 300], [260, 90, 129]
    used_q, used_k = [190, 77, 131], [250, 1, 129]
    lead, gap, tail = 3, 5, 4
    cu_q, cu_k, uq, uk = [lead], [0], [], []
    for i in range(3):
        cu_q.append(cu_q[-1] + seg_q[i]); cu_k.append(cu_k[-1] + seg_k[i]); uq.append(used_q[i]); uk.append(used_k[i])
        if i < 2:
            cu_q.append(cu_q[-1] + gap); cu_k.append(cu_k[-1]); uq.append(0); uk.append(0)
    Tq, Tk = cu_q[-1] + tail, cu_k[-1]
    q = torch.randn(Tq, Hq, D, generator=g).to(torch.bfloat16)
    k = torch.randn(Tk, Hkv, D, generator=g).to(torch.bfloat16)
    v = torch.randn(Tk, Hkv, D, generator=g).to(torch.bfloat16)
    canary = torch.full((Tq, Hq, D), 3.0, dtype=torch.bfloat16, device="cuda")
    dq, dk, dv = q.cuda(), k.cuda(), v.cuda()
    out = sk.attn_fwd_varlen(dq, dk, dv, cu_q, cu_k, seqused_q=uq, seqused_k=uk, out=canary.clone())
    torch.cuda.synchronize()
    got = out.float().cpu().numpy()
    ref = oracle.attn_varlen(q, k, v, cu_q, cu_k, seqused_q=uq, seqused_k=uk)
    assert np.all(got[:lead] == 3.0) and np.all(got[Tq - tail:] == 3.0)  # outside every segment
    for s_i in range(len(uq)):
        a, b = cu_q[s_i], cu_q[s_i + 1]
        if uq[s_i]:
            _compare(got[a:a + uq[s_i]], ref[a:a + uq[s_i]], f"segment {s_i}")
        assert np.all(got[a + uq[s_i]:b] == 0.0)  # pad rows and key-less gap segments
    # poison every pad key / pad query row: bitwise identical output
    k2, v2, q2 = dk.clone(), dv.clone(), dq.clone()
    for s_i in range(len(uq)):
        k2[cu_k[s_i] + uk[s_i]:cu_k[s_i + 1]] = float("nan")
        v2[cu_k[s_i] + uk[s_i]:cu_k[s_i + 1]] = float("inf")
        q2[cu_q[s_i] + uq[s_i]:cu_q[s_i + 1]] = float("nan")
    out2 = sk.attn_fwd_varlen(q2, k2, v2, cu_q, cu_k, seqused_q=uq, seqused_k=uk, out=canary.clone())
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16))
    assert sk.sk_device_status() == 0


def test_varlen_single_segment_equals_split_kv(sk):
    g = torch.Generator().manual_seed(9)
    q = torch.randn(1, 700, 4, 128, generator=g).to(torch.bfloat16).cuda()
    k = torch.randn(1, 900, 4, 128, generator=g).to(torch.bfloat16).cuda()
    v = torch.randn(1, 900, 4, 128, generator=g).to(torch.bfloat16).cuda()
    a = sk.attn_fwd_varlen(q, k, v, [0, 700], [0, 900])
    b = sk.attn_fwd_split_kv(q, k[:, :0], v[:, :0], k, v)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_varlen_rejections_raise(sk):
    q = torch.zeros(64, 2, 64, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(80, 2, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(sk.SplitKVError):
        sk.attn_fwd_varlen(q, k, k, [0, 70], [0, 80])
    with pytest.raises(sk.SplitKVError):
        sk.attn_fwd_varlen(q, k, k, [0, 64], [0, 80], seqused_k=[81])


def _kernel_launches(fn):
    """Attention kernel launches made by fn(), counted by the CUDA profiler."""
    from torch.profiler import ProfilerActivity, profile

    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        fn()
        torch.cuda.synchronize()
    return sum(e.count for e in prof.key_averages() if "attn_fwd" in e.key)


@pytest.mark.parametrize("seed, n, D, Hq, Hkv, lo, hi", [
    (20, 64, 128, 4, 2, 1, 700),
    (21, 300, 64, 2, 1, 1, 200),
])
def test_many_segments_one_launch(sk, seed, n, D, Hq, Hkv, lo, hi):
    g = torch.Generator().manual_seed(seed)
    q_lens = torch.randint(lo, hi + 1, (n,), generator=g).tolist()
    k_lens = torch.randint(lo, hi + 1, (n,), generator=g).tolist()
    q, k, v, cq, ck = _packed(seed, q_lens, k_lens, Hq, Hkv, D)
    dq, dk, dv = q.cuda(), k.cuda(), v.cuda()
    out = torch.empty_like(dq)
    launches = _kernel_launches(lambda: sk.attn_fwd_varlen(dq, dk, dv, cq, ck, out=out))
    assert launches == 1, launches
    rows = sorted(set(torch.randint(0, cq[-1], (400,), generator=g).tolist()) | set(cq[:-1]))
    ref = oracle.attn_varlen(q, k, v, cq, ck, rows=rows)
    _compare(out[rows].float().cpu().numpy(), ref, f"{n} segments")
    assert sk.sk_device_status() == 0


def test_more_segments_than_one_launch_holds(sk):
    """1100 short segments: two launches (1024 segments each at most)."""
    n = 1100
    g = torch.Generator().manual_seed(33)
    q_lens = torch.randint(1, 40, (n,), generator=g).tolist()
    k_lens = torch.randint(1, 40, (n,), generator=g).tolist()
    q, k, v, cq, ck = _packed(33, q_lens, k_lens, 2, 2, 64)
    dq, dk, dv = q.cuda(), k.cuda(), v.cuda()
    out = torch.empty_like(dq)
    launches = _kernel_launches(lambda: sk.attn_fwd_varlen(dq, dk, dv, cq, ck, out=out))
    assert launches == 2, launches
    _compare(out.float().cpu().numpy(), oracle.attn_varlen(q, k, v, cq, ck), "1100 segments")


def test_nan_rows_sharing_the_last_key_tile(sk):
    """Segments whose last key tile is partial, followed by pad rows (seqused_k)
    full of NaN and Inf: the pad rows share the tile with valid keys but must
    not reach any output (the PV product must not see 0 * NaN)."""
    D, Hq, Hkv = 128, 2, 2
    g = torch.Generator().manual_seed(44)
    seg = [(300, 150, 137), (200, 257, 250), (129, 129, 1)]  # (q rows, key rows, valid keys)
    cq, ck, uk = [0], [0], []
    for lq, lk, nk in seg:
        cq.append(cq[-1] + lq); ck.append(ck[-1] + lk); uk.append(nk)
    q = torch.randn(cq[-1], Hq, D, generator=g).to(torch.bfloat16)
    k = torch.randn(ck[-1], Hkv, D, generator=g).to(torch.bfloat16)
    v = torch.randn(ck[-1], Hkv, D, generator=g).to(torch.bfloat16)
    ref = oracle.attn_varlen(q, k, v, cq, ck, seqused_k=uk)
    for i, (lq, lk, nk) in enumerate(seg):
        k[ck[i] + nk:ck[i + 1]] = float("nan")
        v[ck[i] + nk:ck[i + 1]] = float("inf") if i % 2 else float("nan")
    out = sk.attn_fwd_varlen(q.cuda(), k.cuda(), v.cuda(), cq, ck, seqused_k=uk)
    torch.cuda.synchronize()
    got = out.float().cpu().numpy()
    assert np.all(np.isfinite(got))
    _compare(got, ref, "NaN/Inf pad keys in the last tile")
    assert sk.sk_device_status() == 0


def test_varlen_repeated_calls_bitwise_identical(sk):
    """64 unequal segments: repeated calls give identical bits (each row is
    written once, by the thread that owns it)."""
    g = torch.Generator().manual_seed(31)
    lens = torch.randint(1, 900, (64,), generator=g).tolist()
    q, k, v, cq, ck = _packed(31, lens, lens, 4, 2, 128)
    dq, dk, dv = q.cuda(), k.cuda(), v.cuda()
    first = sk.attn_fwd_varlen(dq, dk, dv, cq, ck)
    out = torch.full_like(first, float("nan"))
    for _ in range(3):
        sk.attn_fwd_varlen(dq, dk, dv, cq, ck, out=out)
        torch.cuda.synchronize()
        assert torch.equal(first.view(torch.int16), out.view(torch.int16))
        out.fill_(float("nan"))
    assert sk.sk_device_status() == 0
