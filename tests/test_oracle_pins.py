"""Pins for the CPU oracle: each checks it against something other than itself.

- torch scaled_dot_product_attention (fp64, CPU) on an explicit torch.cat of
  prefix and suffix with a boolean key mask: the pages' non-SP branch
  ("sglang PR 26973", forward_with_replicated_kv_prefix) through a library
  routine the oracle does not use;
- closed forms and hand-derived worked examples (tests/golden/);
- invariants the pages fix: any split point (prefix/suffix) gives the same
  result as the concatenation; tail pad of any content changes no real row
  ("sglang PR 30107", layout invariant + tail_attn_meta); non-causal
  attention is invariant to a joint permutation of keys; GQA head grouping;
- planted mistakes in the oracle that must each fail at least one pin.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")


def _bf16(x):
    return torch.as_tensor(x, dtype=torch.float32).to(torch.bfloat16)


def _sdpa_reference(t, real_len, q_valid, scale):
    """fp64 torch SDPA over an explicit concatenation with a key mask."""
    q = t["q"].double()
    k = torch.cat([t["k_prefix"], t["k_suffix"]], dim=1).double()
    v = torch.cat([t["v_prefix"], t["v_suffix"]], dim=1).double()
    B, Sq, Hq, D = q.shape
    Skv, Hkv = k.shape[1], k.shape[2]
    g = Hq // Hkv
    k = k.repeat_interleave(g, dim=2)
    v = v.repeat_interleave(g, dim=2)
    mask = torch.zeros(B, 1, 1, Skv, dtype=torch.bool)
    for b in range(B):
        mask[b, ..., : real_len[b]] = True
    out = F.scaled_dot_product_attention(
        q.transpose(1, 2), k.transpose(1, 2), v.transpose(1, 2), attn_mask=mask, scale=scale
    ).transpose(1, 2)
    out = out.clone()
    for b in range(B):
        if real_len[b] == 0:
            out[b] = 0.0
        out[b, q_valid[b]:] = 0.0
    return out.numpy()


def _random_case(seed, D=None):
    gen = torch.Generator().manual_seed(seed)
    if D is None:
        D = [32, 64, 128][seed % 3]
    w = workloads.random_workload(gen, D=D, max_sq=40, max_skv=90)
    t = workloads.make_inputs(w)
    return w, t


# --------------------------------------------------------------------------
# library cross-check


@pytest.mark.parametrize("seed", range(12))
def test_matches_torch_sdpa_on_explicit_concat(oracle_mod, seed):
    w, t = _random_case(seed)
    rl = w.real_lens()
    qv = oracle_mod.q_valid_rule(w.Sq, w.Skv, rl)
    scale = w.D ** -0.5
    got = oracle_mod.attn_split_kv(**t, real_len=rl, softmax_scale=scale)
    ref = _sdpa_reference(t, rl, qv, scale)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_tiny_workload_matches_sdpa(oracle_mod):
    w = workloads.get("tiny")
    t = workloads.make_inputs(w)
    got = oracle_mod.attn_split_kv(**t)
    ref = _sdpa_reference(t, w.real_lens(), [w.Sq], w.D ** -0.5)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_row_subset_equals_full(oracle_mod):
    w, t = _random_case(3)
    full = oracle_mod.attn_split_kv(**t, real_len=w.real_lens())
    rows = [w.Sq - 1, 0, w.Sq // 2]
    sub = oracle_mod.attn_split_kv(**t, real_len=w.real_lens(), rows=rows)
    assert np.array_equal(sub, full[:, rows])


# --------------------------------------------------------------------------
# worked examples (hand-derived, tests/golden)


def _vec(spec, D, dtype=np.float32):
    v = np.zeros(D, dtype=dtype)
    for k, x in spec.items():
        v[int(k)] = x
    return v


def _golden_attention_cases():
    with open(GOLDEN) as f:
        return json.load(f)["attention"]


@pytest.mark.parametrize("case", _golden_attention_cases(), ids=lambda c: c["name"])
def test_golden_attention(oracle_mod, case):
    D, Hq, Hkv = case["D"], case["Hq"], case["Hkv"]
    q = np.stack([np.stack([_vec(h, D) for h in row]) for row in case["q"]])[None]
    q = q.reshape(1, len(case["q"]), Hq, D)

    def kv(name):
        rows = case[name]
        a = np.zeros((1, len(rows), Hkv, D), dtype=np.float32)
        for i, spec in enumerate(rows):
            a[0, i, :] = _vec(spec, D)
        return _bf16(a)

    got = oracle_mod.attn_split_kv(
        _bf16(q), kv("k_prefix"), kv("v_prefix"), kv("k_suffix"), kv("v_suffix"),
        real_len=[case["real_len"]], softmax_scale=case["scale"])
    exp = np.stack([np.stack([_vec(h, D, np.float64) for h in row]) for row in case["expected"]])[None]
    # expected values are given to 16 significant digits
    np.testing.assert_allclose(got, exp.reshape(got.shape), rtol=0, atol=1e-15 * 8)


# --------------------------------------------------------------------------
# invariants


@pytest.mark.parametrize("p", [0, 1, 15, 16, 17, 80])
def test_split_invariance_tiny_bitwise(oracle_mod, p):
    w = workloads.get("tiny")
    t = workloads.make_inputs(w)
    base = oracle_mod.attn_split_kv(**t)
    k = torch.cat([t["k_prefix"], t["k_suffix"]], 1)
    v = torch.cat([t["v_prefix"], t["v_suffix"]], 1)
    s = dict(q=t["q"], k_prefix=k[:, :p], v_prefix=v[:, :p], k_suffix=k[:, p:], v_suffix=v[:, p:])
    got = oracle_mod.attn_split_kv(**s)
    assert np.array_equal(got, base)


@pytest.mark.parametrize("p", [0, 127, 128, 129, 512, 700])
def test_split_invariance_mid_bitwise(oracle_mod, p):
    gen = torch.Generator().manual_seed(11)
    q = _bf16(torch.randn(1, 24, 2, 64, generator=gen))
    k = _bf16(torch.randn(1, 700, 1, 64, generator=gen))
    v = _bf16(torch.randn(1, 700, 1, 64, generator=gen))
    base = oracle_mod.attn_split_kv(q, k[:, :300], v[:, :300], k[:, 300:], v[:, 300:], real_len=[650])
    got = oracle_mod.attn_split_kv(q, k[:, :p], v[:, :p], k[:, p:], v[:, p:], real_len=[650])
    assert np.array_equal(got, base)


@pytest.mark.parametrize("fill", [0.0, 1e4, float("nan"), float("inf"), "randn"])
@pytest.mark.parametrize("npad", [1, 3, 40, 130])
def test_pad_invariance_bitwise(oracle_mod, fill, npad):
    gen = torch.Generator().manual_seed(5)
    B, Sp, Ss, H, D = 2, 20, 50, 2, 64
    Sq = Sp + Ss  # joint self-attention: the pad covers queries too
    q = _bf16(torch.randn(B, Sq, H, D, generator=gen))
    kp = _bf16(torch.randn(B, Sp, H, D, generator=gen))
    vp = _bf16(torch.randn(B, Sp, H, D, generator=gen))
    ks = _bf16(torch.randn(B, Ss, H, D, generator=gen))
    vs = _bf16(torch.randn(B, Ss, H, D, generator=gen))
    base = oracle_mod.attn_split_kv(q, kp, vp, ks, vs)

    def padded(x, n):
        if fill == "randn":
            p = _bf16(torch.randn(x.shape[0], n, *x.shape[2:], generator=gen))
        else:
            p = torch.full((x.shape[0], n, *x.shape[2:]), fill, dtype=torch.bfloat16)
        return torch.cat([x, p], dim=1)

    got = oracle_mod.attn_split_kv(padded(q, npad), kp, vp, padded(ks, npad), padded(vs, npad),
                                   real_len=[Sp + Ss] * B)
    assert np.array_equal(got[:, :Sq], base)
    assert np.all(got[:, Sq:] == 0.0)


def test_pad_inside_prefix(oracle_mod):
    """real_len < Sp: the prefix is clipped and the whole suffix is pad."""
    gen = torch.Generator().manual_seed(6)
    q = _bf16(torch.randn(1, 9, 1, 64, generator=gen))
    kp = _bf16(torch.randn(1, 12, 1, 64, generator=gen))
    vp = _bf16(torch.randn(1, 12, 1, 64, generator=gen))
    ks = torch.full((1, 30, 1, 64), float("nan"), dtype=torch.bfloat16)
    vs = ks.clone()
    got = oracle_mod.attn_split_kv(q, kp, vp, ks, vs, real_len=[5])
    ref = oracle_mod.attn_split_kv(q, kp[:, :5], vp[:, :5], ks[:, :0], vs[:, :0])
    assert np.array_equal(got, ref)


def test_joint_key_permutation(oracle_mod):
    gen = torch.Generator().manual_seed(7)
    q = _bf16(torch.randn(2, 17, 4, 64, generator=gen))
    k = _bf16(torch.randn(2, 90, 2, 64, generator=gen))
    v = _bf16(torch.randn(2, 90, 2, 64, generator=gen))
    base = oracle_mod.attn_split_kv(q, k[:, :33], v[:, :33], k[:, 33:], v[:, 33:])
    perm = torch.randperm(90, generator=gen)
    kk, vv = k[:, perm], v[:, perm]
    got = oracle_mod.attn_split_kv(q, kk[:, :50], vv[:, :50], kk[:, 50:], vv[:, 50:])
    np.testing.assert_allclose(got, base, rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# closed forms


def test_scale_zero_gives_mean_of_valid_values(oracle_mod):
    gen = torch.Generator().manual_seed(8)
    q = _bf16(torch.randn(2, 10, 3, 64, generator=gen))
    kp = _bf16(torch.randn(2, 7, 3, 64, generator=gen))
    vp = _bf16(torch.randn(2, 7, 3, 64, generator=gen))
    ks = _bf16(torch.randn(2, 25, 3, 64, generator=gen))
    vs = _bf16(torch.randn(2, 25, 3, 64, generator=gen))
    rl = [19, 4]
    got = oracle_mod.attn_split_kv(q, kp, vp, ks, vs, real_len=rl, softmax_scale=0.0)
    vcat = torch.cat([vp, vs], 1).double().numpy()
    for b in range(2):
        mean = vcat[b, : rl[b]].mean(axis=0)  # [H, D]
        np.testing.assert_allclose(got[b], np.broadcast_to(mean, got[b].shape), rtol=0, atol=1e-14)


def test_uniform_v_is_exactly_one(oracle_mod):
    gen = torch.Generator().manual_seed(9)
    q = _bf16(torch.randn(1, 33, 2, 128, generator=gen) * 3)
    kp = _bf16(torch.randn(1, 16, 2, 128, generator=gen) * 3)
    ks = _bf16(torch.randn(1, 64, 2, 128, generator=gen) * 3)
    ones_p = torch.ones(1, 16, 2, 128, dtype=torch.bfloat16)
    ones_s = torch.ones(1, 64, 2, 128, dtype=torch.bfloat16)
    got = oracle_mod.attn_split_kv(q, kp, ones_p, ks, ones_s, real_len=[71])
    assert np.all(got == 1.0)


def test_equal_value_rows_give_that_row(oracle_mod):
    gen = torch.Generator().manual_seed(10)
    vrow = _bf16(torch.randn(64, generator=gen))
    q = _bf16(torch.randn(1, 5, 1, 64, generator=gen))
    kp = _bf16(torch.randn(1, 3, 1, 64, generator=gen))
    ks = _bf16(torch.randn(1, 9, 1, 64, generator=gen))
    vp = vrow.expand(1, 3, 1, 64).contiguous()
    vs = vrow.expand(1, 9, 1, 64).contiguous()
    got = oracle_mod.attn_split_kv(q, kp, vp, ks, vs)
    np.testing.assert_allclose(got[0, :, 0], np.broadcast_to(vrow.double().numpy(), (5, 64)),
                               rtol=1e-14, atol=1e-14)


def test_gqa_head_mapping(oracle_mod):
    gen = torch.Generator().manual_seed(12)
    Hq, Hkv = 12, 3
    g = Hq // Hkv
    q = _bf16(torch.randn(1, 6, Hq, 64, generator=gen))
    kp = _bf16(torch.randn(1, 4, Hkv, 64, generator=gen))
    ks = _bf16(torch.randn(1, 8, Hkv, 64, generator=gen))
    vp = torch.empty(1, 4, Hkv, 64, dtype=torch.bfloat16)
    vs = torch.empty(1, 8, Hkv, 64, dtype=torch.bfloat16)
    for h in range(Hkv):
        vp[:, :, h] = h + 1
        vs[:, :, h] = h + 1
    got = oracle_mod.attn_split_kv(q, kp, vp, ks, vs)
    for hq in range(Hq):
        np.testing.assert_allclose(got[0, :, hq], hq // g + 1, rtol=1e-14, atol=0, err_msg=str(hq))


def test_one_valid_key_gives_its_value_exactly(oracle_mod):
    gen = torch.Generator().manual_seed(13)
    q = _bf16(torch.randn(1, 4, 2, 64, generator=gen))
    kp = _bf16(torch.randn(1, 0, 2, 64, generator=gen))
    vp = _bf16(torch.randn(1, 0, 2, 64, generator=gen))
    ks = _bf16(torch.randn(1, 6, 2, 64, generator=gen))
    vs = _bf16(torch.randn(1, 6, 2, 64, generator=gen))
    got = oracle_mod.attn_split_kv(q, kp, vp, ks, vs, real_len=[1])
    for h in range(2):
        assert np.array_equal(got[0, :, h], np.broadcast_to(vs[0, 0, h].double().numpy(), (4, 64)))


def test_huge_logit_selects_its_value(oracle_mod):
    gen = torch.Generator().manual_seed(14)
    D = 64
    q = torch.zeros(1, 1, 1, D, dtype=torch.bfloat16)
    q[..., 0] = 64.0
    kp = _bf16(torch.randn(1, 10, 1, D, generator=gen) * 0.01)
    ks = _bf16(torch.randn(1, 10, 1, D, generator=gen) * 0.01)
    vp = _bf16(torch.randn(1, 10, 1, D, generator=gen))
    vs = _bf16(torch.randn(1, 10, 1, D, generator=gen))
    j0 = 13  # a suffix key
    ks[0, j0 - 10, 0, 0] = 64.0
    got = oracle_mod.attn_split_kv(q, kp, vp, ks, vs, softmax_scale=1.0)
    np.testing.assert_allclose(got[0, 0, 0], vs[0, j0 - 10, 0].double().numpy(), rtol=0, atol=1e-12)


def test_no_valid_key_and_pad_rows_are_zero(oracle_mod):
    gen = torch.Generator().manual_seed(15)
    q = _bf16(torch.randn(2, 8, 1, 64, generator=gen))
    kv = [_bf16(torch.randn(2, n, 1, 64, generator=gen)) for n in (3, 3, 5, 5)]
    got = oracle_mod.attn_split_kv(q, *kv, real_len=[0, 8])
    assert np.all(got[0] == 0.0)
    assert np.all(np.isfinite(got[1]))
    got = oracle_mod.attn_split_kv(q, *kv, real_len=[8, 8], q_valid=[3, 0])
    assert np.all(got[0, 3:] == 0.0) and np.all(got[1] == 0.0)
    assert np.all(got[0, :3] != 0.0)


def test_q_valid_rule():
    import oracle

    assert oracle.q_valid_rule(4432, 4432, [4429, 4429]) == [4429, 4429]
    assert oracle.q_valid_rule(4096, 4608, [4608]) == [4096]
    assert oracle.q_valid_rule(25088, 25088, [25048]) == [25048]


# --------------------------------------------------------------------------
# negative control: treating zero pad as keys (the bug the tail layout fixes)


def test_negative_control_unmasked_zero_pad(oracle_mod):
    """1 pad per 16 tokens, zero-filled, counted as keys, visibly changes real rows."""
    gen = torch.Generator().manual_seed(16)
    B, S, H, D = 1, 240, 2, 64
    npad = S // 15  # 16 pad per 240 real -> 1 pad per 16 tokens overall
    q = _bf16(torch.randn(B, S, H, D, generator=gen))
    k = _bf16(torch.randn(B, S, H, D, generator=gen))
    v = _bf16(torch.randn(B, S, H, D, generator=gen))
    zp = torch.zeros(B, npad, H, D, dtype=torch.bfloat16)
    kz, vz = torch.cat([k, zp], 1), torch.cat([v, zp], 1)
    empty = k[:, :0]
    right = oracle_mod.attn_split_kv(q, empty, empty, kz, vz, real_len=[S], q_valid=[S])
    wrong = oracle_mod.attn_split_kv(q, empty, empty, kz, vz, real_len=[S + npad], q_valid=[S])
    mae = np.abs(right[:, :S] - wrong[:, :S]).mean()
    # magnitude depends on the value distribution (parity unpinned); it must be visible
    assert mae > 1e-3, mae


# --------------------------------------------------------------------------
# planted mistakes must each fail at least one pin


def _pins_pass(oracle_mod, mutate):
    """Run a compact set of pins with a mutated oracle; True if all pass."""
    ok = True
    # 1. SDPA comparison on GQA random cases (with pad, prefix and suffix)
    for seed in (1, 4, 7):
        gen = torch.Generator().manual_seed(100 + seed)
        B, Sq, Sp, Ss, Hkv, g, D = 2, 9, 7, 13, 2, 2, 64
        t = dict(
            q=_bf16(torch.randn(B, Sq, Hkv * g, D, generator=gen)),
            k_prefix=_bf16(torch.randn(B, Sp, Hkv, D, generator=gen)),
            v_prefix=_bf16(torch.randn(B, Sp, Hkv, D, generator=gen)),
            k_suffix=_bf16(torch.randn(B, Ss, Hkv, D, generator=gen)),
            v_suffix=_bf16(torch.randn(B, Ss, Hkv, D, generator=gen)),
        )
        rl = [17, 20]
        got = oracle_mod.attn_split_kv(**t, real_len=rl, softmax_scale=0.3, mutate=mutate)
        ref = _sdpa_reference(t, rl, [Sq, Sq], 0.3)
        if not np.allclose(got, ref, rtol=0, atol=1e-12):
            ok = False
    # 2. pad invariance with NaN pad
    gen = torch.Generator().manual_seed(200)
    q = _bf16(torch.randn(1, 6, 2, 64, generator=gen))
    k = _bf16(torch.randn(1, 10, 2, 64, generator=gen))
    v = _bf16(torch.randn(1, 10, 2, 64, generator=gen))
    nan = torch.full((1, 3, 2, 64), float("nan"), dtype=torch.bfloat16)
    a = oracle_mod.attn_split_kv(q, k[:, :4], v[:, :4], k[:, 4:], v[:, 4:], mutate=mutate)
    b = oracle_mod.attn_split_kv(q, k[:, :4], v[:, :4], torch.cat([k[:, 4:], nan], 1),
                                 torch.cat([v[:, 4:], nan], 1), real_len=[10], mutate=mutate)
    if not np.array_equal(a, b):
        ok = False
    return ok


@pytest.mark.parametrize("name", sorted(__import__("oracle").MUTATIONS))
def test_planted_mistake_fails_a_pin(oracle_mod, name):
    assert _pins_pass(oracle_mod, 0)
    assert not _pins_pass(oracle_mod, oracle_mod.MUTATIONS[name]), name


# --------------------------------------------------------------------------
# fp64 -> bf16 rounding used by the prologue oracle


def test_round_bf16_ties_and_values(oracle_mod):
    r = oracle_mod.round_bf16
    assert r(1.0) == 0x3F80
    assert r(1.0 + 2.0 ** -8) == 0x3F80          # exact tie -> even
    assert r(1.0 + 3 * 2.0 ** -8) == 0x3F82      # exact tie -> even (up)
    assert r(1.0 + 2.0 ** -8 + 2.0 ** -40) == 0x3F81  # just above the tie
    assert r(-0.2) == 0xBE4D
    assert r(1.4) == 0x3FB3
    assert r(float("inf")) == 0x7F80
    assert r(3.5e38) == 0x7F80                   # overflow rounds to inf
    for x in np.random.default_rng(0).standard_normal(2000):
        want = torch.tensor(float(x), dtype=torch.float32).to(torch.bfloat16)
        # fp32 -> bf16 in torch is RNE; x is an fp32 value here, so both agree
        x32 = float(np.float32(x))
        assert r(x32) == int(want.view(torch.int16).item()) & 0xFFFF
