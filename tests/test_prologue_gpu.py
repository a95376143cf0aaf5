"""Parity of the fused Q/K RMSNorm + RoPE prologue kernel with the fp64 oracle.

Bar: every output element within 1 bf16 ulp of the oracle and at least
99.99% bit-identical.  The kernel computes in fp64 with the oracle's rounding
points, so in practice every element is identical; the ulp allowance covers a
sum-of-squares reduction order that differs from the oracle's sequential one.
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
    sk.qk_rmsnorm_rope(qd, kd, wq.cuda(), wk.cuda(), tabd, rot_dim=rot, interleaved=inter, eps=1e-6)
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
    sk.qk_rmsnorm_rope(d[:, :, :Hq], d[:, :, Hq:Hq + Hkv], wq.cuda(), wk.cuda(), tab.cuda(), eps=1e-5)
    torch.cuda.synchronize()
    got = d.cpu()
    assert torch.equal(got[:, :, Hq + Hkv:], qkv[:, :, Hq + Hkv:])  # v untouched
    eps = float(np.float32(1e-5))
    ref_q = oracle.qk_rmsnorm_rope(qkv[:, :, :Hq].contiguous(), wq, tab.numpy(), eps=eps)
    ref_k = oracle.qk_rmsnorm_rope(qkv[:, :, Hq:Hq + Hkv].contiguous(), wk, tab.numpy(), eps=eps)
    _ulp_check(got[:, :, :Hq].contiguous().view(torch.int16).numpy().view(np.uint16), ref_q)
    _ulp_check(got[:, :, Hq:Hq + Hkv].contiguous().view(torch.int16).numpy().view(np.uint16), ref_k)
