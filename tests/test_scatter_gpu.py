"""Fused output all-to-all (attn_fwd_split_kv_scatter) on one GPU.

The Ulysses form ("sglang PR 26973", _forward_with_replicated_kv_prefix_split)
runs attention on a rank's head shard over the whole gathered sequence, then
an all-to-all returns each sequence chunk to the rank that owns it.  Here
every rank's receive buffer is a tensor on this GPU: each emulated rank calls
the scatter entry on its heads, writing straight into all ranks' buffers.
Each buffer must match the fp64 oracle's output for its sequence chunk
(max-abs <= 2e-2, relative L2 <= 1e-2, pad rows exactly 0), and equal the
chunk of the plain kernel's output bit for bit (each (query tile, head) is
computed the same way in both launches).  The
cross-GPU form (peer-mapped buffers, a barrier before the readers) needs
several GPUs and is not run here.
"""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu

SENTINEL = 7.0
MAX_ABS = 2e-2
REL_L2 = 1e-2


def _compare(got, ref, what):
    got = got.astype(np.float64)
    diff = np.abs(got - ref)
    max_abs = float(diff.max())
    rel = float(np.sqrt((diff ** 2).sum()) / max(np.sqrt((ref ** 2).sum()), 1e-300))
    assert np.all(np.isfinite(got)), what
    assert max_abs <= MAX_ABS, f"{what} max_abs={max_abs}"
    assert rel <= REL_L2, f"{what} rel_l2={rel}"


@pytest.fixture(scope="module")
def sk():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    from varlen_flash_attention_b200 import build

    build.build()
    import varlen_flash_attention_b200 as m

    return m


@pytest.mark.parametrize("sp,L,Hq,Hkv,D,B,pad", [
    (2, 256, 4, 4, 128, 1, 0),      # chunks aligned to 128-row tiles
    (2, 200, 4, 2, 128, 1, 0),      # tiles straddle the chunk boundary, GQA
    (4, 77, 8, 2, 64, 2, 5),        # 4 chunks, tail pad on the last rank's chunk, B = 2
    (8, 33, 8, 8, 128, 1, 9),       # one head per rank, short chunks, tail pad
])
def test_scatter_equals_plain_output_chunks(sk, sp, L, Hq, Hkv, D, B, pad):
    g = torch.Generator().manual_seed(sp * 100 + L)
    Sq = sp * L
    Sp = 48
    dev = "cuda"

    def r(*shape):
        return torch.randn(*shape, generator=g).to(torch.bfloat16)

    host = dict(q=r(B, Sq, Hq, D), k_prefix=r(B, Sp, Hkv, D), v_prefix=r(B, Sp, Hkv, D),
                k_suffix=r(B, Sq, Hkv, D), v_suffix=r(B, Sq, Hkv, D))
    q, kp, vp, ks, vs = (host[k].to(dev) for k in ("q", "k_prefix", "v_prefix", "k_suffix", "v_suffix"))
    real_len = [Sp + Sq - pad] * B
    q_valid = [Sq - pad] * B
    want_oracle = oracle.attn_split_kv(**host, real_len=real_len, q_valid=q_valid)
    ref = sk.attn_fwd_split_kv(q, kp, vp, ks, vs, real_len=real_len, q_valid=q_valid)
    # receive buffers: [B, L, Hq + 2 canary heads, D], canaries hold SENTINEL
    recv = [torch.full((B, L, Hq + 2, D), SENTINEL, dtype=torch.bfloat16, device=dev) for _ in range(sp)]
    hl = Hq // sp  # query heads per rank; its KV heads are the ones they read (q head h reads h // group)
    for rank in range(sp):
        h0 = rank * hl
        kv0 = h0 // (Hq // Hkv)
        sl = slice(kv0, kv0 + max(1, hl // (Hq // Hkv)))
        sk.attn_fwd_split_kv_scatter(q[:, :, h0:h0 + hl], kp[:, :, sl], vp[:, :, sl], ks[:, :, sl], vs[:, :, sl],
                                     recv, head_offset=h0, real_len=real_len, q_valid=q_valid)
    torch.cuda.synchronize()
    for rank in range(sp):
        got = recv[rank]
        _compare(got[:, :, :Hq].float().cpu().numpy(), want_oracle[:, rank * L:(rank + 1) * L],
                 f"rank {rank} vs oracle")
        want = ref[:, rank * L:(rank + 1) * L]
        assert torch.equal(got[:, :, :Hq].view(torch.int16), want.view(torch.int16)), rank
        assert bool((got[:, :, Hq:] == SENTINEL).all()), "canary heads written"
    if pad:
        assert bool((recv[-1][:, L - pad:, :Hq] == 0).all())
    assert sk.sk_device_status(0) == 0


def test_scatter_single_destination_is_the_plain_call(sk):
    g = torch.Generator().manual_seed(3)
    qh = torch.randn(1, 300, 2, 128, generator=g).to(torch.bfloat16)
    kh = torch.randn(1, 260, 2, 128, generator=g).to(torch.bfloat16)
    vh = torch.randn(1, 260, 2, 128, generator=g).to(torch.bfloat16)
    q, k, v = qh.cuda(), kh.cuda(), vh.cuda()
    ref = sk.attn_fwd_split_kv(q, k[:, :60], v[:, :60], k[:, 60:], v[:, 60:], real_len=[250])
    out = torch.empty_like(ref)
    sk.attn_fwd_split_kv_scatter(q, k[:, :60], v[:, :60], k[:, 60:], v[:, 60:], [out], real_len=[250])
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    want = oracle.attn_split_kv(qh, kh[:, :60], vh[:, :60], kh[:, 60:], vh[:, 60:], real_len=[250])
    _compare(out.float().cpu().numpy(), want, "single destination vs oracle")


def test_fused_ulysses_single_rank_uses_the_scatter_kernel(sk):
    """ulysses_attn_fwd_split_kv_fused at sp = 1 (no process group): the
    scatter kernel writes the output into the rank's own receive buffer."""
    from varlen_flash_attention_b200 import sp_shard as sps
    from varlen_flash_attention_b200 import ulysses

    g = torch.Generator().manual_seed(9)
    B, S, Hq, Hkv, D, Sp = 1, 333, 8, 2, 128, 64
    mk = lambda *sh: torch.randn(*sh, generator=g).to(torch.bfloat16)
    host = [mk(B, S, Hq, D), mk(B, S, Hkv, D), mk(B, S, Hkv, D), mk(B, Sp, Hkv, D), mk(B, Sp, Hkv, D)]
    q, ks, vs, kp, vp = (t.cuda() for t in host)
    plan = sps.build_shard_plan(S, 1, 0)
    recv = [torch.full((B, S, Hq, D), SENTINEL, dtype=torch.bfloat16, device="cuda")]
    out = ulysses.ulysses_attn_fwd_split_kv_fused(q, kp, vp, ks, vs, plan, recv)
    ref = ulysses.ulysses_attn_fwd_split_kv(q, kp, vp, ks, vs, plan)
    torch.cuda.synchronize()
    assert out.data_ptr() == recv[0].data_ptr()
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    want = oracle.attn_split_kv(host[0], host[3], host[4], host[1], host[2])
    _compare(out.float().cpu().numpy(), want, "fused Ulysses sp=1 vs oracle")
