"""Pins of the packed-varlen oracle against things other than itself: dense
fp64 attention (torch SDPA) over the whole packed sequence with an explicit
block-diagonal mask, packing-order invariance, and zeros where a segment has
no valid key ("vLLM-Omni performance patterns": check packed samples of
unequal lengths against dense attention, including padding exclusion)."""
import numpy as np
import pytest
import torch
import torch.nn.functional as F


def _packed(seed, q_lens, k_lens, Hq=4, Hkv=2, D=64):
    g = torch.Generator().manual_seed(seed)
    Tq, Tk = sum(q_lens), sum(k_lens)
    q = torch.randn(Tq, Hq, D, generator=g).to(torch.bfloat16)
    k = torch.randn(Tk, Hkv, D, generator=g).to(torch.bfloat16)
    v = torch.randn(Tk, Hkv, D, generator=g).to(torch.bfloat16)
    cq = np.concatenate([[0], np.cumsum(q_lens)]).astype(int).tolist()
    ck = np.concatenate([[0], np.cumsum(k_lens)]).astype(int).tolist()
    return q, k, v, cq, ck


def _dense_block_diag(q, k, v, cq, ck, used_q=None, used_k=None):
    Tq, Hq, D = q.shape
    Tk, Hkv, _ = k.shape
    mask = torch.zeros(Tq, Tk, dtype=torch.bool)
    for i in range(len(cq) - 1):
        nk = (ck[i + 1] - ck[i]) if used_k is None else used_k[i]
        mask[cq[i]:cq[i + 1], ck[i]:ck[i] + nk] = True
    g = Hq // Hkv
    qd = q.double().permute(1, 0, 2)
    kd = k.double().repeat_interleave(g, dim=1).permute(1, 0, 2)
    vd = v.double().repeat_interleave(g, dim=1).permute(1, 0, 2)
    o = F.scaled_dot_product_attention(qd, kd, vd, attn_mask=mask, scale=D ** -0.5)
    return o.permute(1, 0, 2).numpy(), mask


@pytest.mark.parametrize("seed, q_lens, k_lens", [
    (0, [5, 17, 1, 40], [9, 3, 25, 40]),
    (1, [64, 200, 33], [64, 130, 257]),
    (2, [1], [1]),
])
def test_varlen_oracle_equals_dense_block_diagonal(oracle_mod, seed, q_lens, k_lens):
    q, k, v, cq, ck = _packed(seed, q_lens, k_lens)
    got = oracle_mod.attn_varlen(q, k, v, cq, ck)
    ref, _ = _dense_block_diag(q, k, v, cq, ck)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_varlen_oracle_seqused_excludes_pad(oracle_mod):
    q, k, v, cq, ck = _packed(3, [20, 30], [25, 40])
    used_q, used_k = [15, 30], [21, 33]
    got = oracle_mod.attn_varlen(q, k, v, cq, ck, seqused_q=used_q, seqused_k=used_k)
    ref, _ = _dense_block_diag(q, k, v, cq, ck, used_k=used_k)
    for i in range(2):
        a, b = cq[i], cq[i] + used_q[i]
        np.testing.assert_allclose(got[a:b], ref[a:b], rtol=0, atol=1e-12)
        assert np.all(got[b:cq[i + 1]] == 0)
    # pad contents never matter
    k2, v2 = k.clone(), v.clone()
    k2[ck[0] + used_k[0]:ck[1]] = float("nan")
    v2[ck[1] + used_k[1]:ck[2]] = 1e4
    got2 = oracle_mod.attn_varlen(q, k2, v2, cq, ck, seqused_q=used_q, seqused_k=used_k)
    assert np.array_equal(got, got2)


def test_varlen_oracle_packing_order_and_empty_segments(oracle_mod):
    q, k, v, cq, ck = _packed(4, [7, 0, 12, 9], [5, 6, 0, 11])
    got = oracle_mod.attn_varlen(q, k, v, cq, ck)
    # the segment with no keys (third) gives zeros; the one with no queries nothing
    assert np.all(got[cq[2]:cq[3]] == 0)
    # reversing the packing order permutes the outputs
    order = [3, 2, 1, 0]
    qs = [q[cq[i]:cq[i + 1]] for i in order]
    ks = [k[ck[i]:ck[i + 1]] for i in order]
    vs = [v[ck[i]:ck[i + 1]] for i in order]
    cq2 = np.concatenate([[0], np.cumsum([len(t) for t in qs])]).tolist()
    ck2 = np.concatenate([[0], np.cumsum([len(t) for t in ks])]).tolist()
    got2 = oracle_mod.attn_varlen(torch.cat(qs), torch.cat(ks), torch.cat(vs), cq2, ck2)
    for j, i in enumerate(order):
        assert np.array_equal(got2[cq2[j]:cq2[j + 1]], got[cq[i]:cq[i + 1]])


def test_varlen_oracle_single_segment_is_plain_attention(oracle_mod):
    q, k, v, cq, ck = _packed(5, [33], [70])
    got = oracle_mod.attn_varlen(q, k, v, cq, ck)
    empty = k[:0].unsqueeze(0)
    ref = oracle_mod.attn_split_kv(q.unsqueeze(0), empty, empty, k.unsqueeze(0), v.unsqueeze(0))
    assert np.array_equal(got, ref[0])


def test_row_sample_equals_the_full_result(oracle_mod):
    """oracle.attn_varlen(rows=...) returns exactly the selected rows of the
    full result (sorted, duplicates dropped), including rows of empty
    segments and rows outside every segment (zeros)."""
    import numpy as np
    import torch

    g = torch.Generator().manual_seed(5)
    q = torch.randn(70, 3, 64, generator=g).to(torch.bfloat16)
    k = torch.randn(90, 3, 64, generator=g).to(torch.bfloat16)
    v = torch.randn(90, 3, 64, generator=g).to(torch.bfloat16)
    cq, ck = [2, 20, 20, 60], [0, 25, 40, 90]
    full = oracle_mod.attn_varlen(q, k, v, cq, ck, seqused_k=[25, 0, 31])
    rows = [65, 3, 19, 20, 59, 0, 3]
    sub = oracle_mod.attn_varlen(q, k, v, cq, ck, seqused_k=[25, 0, 31], rows=rows)
    assert np.array_equal(sub, full[sorted(set(rows))])
