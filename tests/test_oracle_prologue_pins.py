"""Pins for the oracle's fused Q/K RMSNorm + RoPE prologue.

The pages ("vLLM-Omni performance patterns", Q/K RMSNorm + RoPE section;
"sglang PR 26973", cosmos3video.py) fix: RMSNorm over head_dim with a weight
and epsilon, then rotary embedding from a [cos | sin] table, NeoX half-split
or interleaved pairing, partial rotary passes the remaining dims through,
and bf16 rounding wherever the unfused path stores bf16.  Pins:
- torch F.rms_norm in fp64 (a library routine the oracle does not use), with
  the oracle's bf16 output required to be the nearest bf16 to it;
- rotation written as complex multiplication (numpy complex128);
- interleaved and half-split pairings agree under the matching permutation;
- worked examples from tests/golden/.
"""
import json
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")


def _bits_to_f64(bits):
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def _is_nearest_bf16(bits, ref):
    """Each bf16 in ``bits`` is a nearest bf16 to the fp64 value ``ref``."""
    bits = np.asarray(bits, dtype=np.uint16).ravel()
    ref = np.asarray(ref, dtype=np.float64).ravel()
    val = _bits_to_f64(bits)
    up = _bits_to_f64((bits.astype(np.int32) + 1).astype(np.uint16))
    dn = _bits_to_f64((bits.astype(np.int32) - 1).astype(np.uint16))
    err = np.abs(val - ref)
    return np.all(err <= np.abs(up - ref)) and np.all(err <= np.abs(dn - ref))


def _rand(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(*shape, generator=g) * scale).to(torch.bfloat16)


def _table(S, rot_dim, seed, theta=10000.0):
    pos = np.arange(S, dtype=np.float64)[:, None]
    inv = theta ** (-np.arange(0, rot_dim, 2, dtype=np.float64) / rot_dim)
    ang = pos * inv[None, :]
    return np.concatenate([np.cos(ang), np.sin(ang)], axis=1).astype(np.float32)


def test_identity_rotation_is_rmsnorm(oracle_mod):
    B, S, H, D = 2, 7, 3, 128
    x = _rand((B, S, H, D), 1, 2.0)
    w = _rand((D,), 2, 0.5)
    tab = np.concatenate([np.ones((S, 48), np.float32), np.zeros((S, 48), np.float32)], 1)
    got = oracle_mod.qk_rmsnorm_rope(x, w, tab, rot_dim=96, eps=1e-6)
    ref = F.rms_norm(x.double(), (D,), weight=w.double(), eps=1e-6).numpy()
    assert _is_nearest_bf16(got, ref)


def test_unit_rms_with_unit_weight(oracle_mod):
    x = _rand((1, 5, 2, 64), 3, 7.0)
    w = torch.ones(64, dtype=torch.bfloat16)
    tab = np.concatenate([np.ones((5, 32), np.float32), np.zeros((5, 32), np.float32)], 1)
    got = _bits_to_f64(oracle_mod.qk_rmsnorm_rope(x, w, tab, eps=0.0)).reshape(5, 2, 64)
    rms = np.sqrt((got ** 2).mean(-1))
    np.testing.assert_allclose(rms, 1.0, rtol=2.0 ** -8)


@pytest.mark.parametrize("rot_dim", [128, 96, 64])
def test_interleaved_rotation_is_complex_multiplication(oracle_mod, rot_dim):
    B, S, H, D = 1, 9, 2, 128
    x = _rand((B, S, H, D), 4)
    w = _rand((D,), 5)
    tab = _table(S, rot_dim, 0)
    got = oracle_mod.qk_rmsnorm_rope(x, w, tab, rot_dim=rot_dim, interleaved=True, eps=1e-6)
    # independent: library RMSNorm rounded to bf16, then complex rotation
    y = F.rms_norm(x.double(), (D,), weight=w.double(), eps=1e-6).to(torch.float32)
    y = y.to(torch.bfloat16).double().numpy()  # values are fp32-exact; one rounding to bf16
    c = tab[:, : rot_dim // 2].astype(np.float64)[None, :, None, :]
    s = tab[:, rot_dim // 2:].astype(np.float64)[None, :, None, :]
    zc = (y[..., 0:rot_dim:2] + 1j * y[..., 1:rot_dim:2]) * (c + 1j * s)
    ref = y.copy()
    ref[..., 0:rot_dim:2] = zc.real
    ref[..., 1:rot_dim:2] = zc.imag
    assert _is_nearest_bf16(got, ref)


@pytest.mark.parametrize("rot_dim", [128, 96])
def test_half_split_equals_interleaved_under_permutation(oracle_mod, rot_dim):
    D = 128
    h = rot_dim // 2
    x = _rand((1, 6, 2, D), 6)
    w = _rand((D,), 7)
    tab = _table(6, rot_dim, 0)
    # interleaved position 2i <- half-split position i ; 2i+1 <- i + h
    perm = np.arange(D)
    perm[0:rot_dim:2] = np.arange(h)
    perm[1:rot_dim:2] = np.arange(h, rot_dim)
    xi = x[..., perm].contiguous()
    wi = w[perm].contiguous()
    half = oracle_mod.qk_rmsnorm_rope(x, w, tab, rot_dim=rot_dim, interleaved=False)
    inter = oracle_mod.qk_rmsnorm_rope(xi, wi, tab, rot_dim=rot_dim, interleaved=True)
    assert np.array_equal(inter, half[..., perm])


def test_rotation_preserves_pair_norm(oracle_mod):
    D = 128
    x = _rand((1, 11, 1, D), 8)
    w = torch.ones(D, dtype=torch.bfloat16)
    tab = _table(11, 128, 0)
    ident = np.concatenate([np.ones((11, 64), np.float32), np.zeros((11, 64), np.float32)], 1)
    z = _bits_to_f64(oracle_mod.qk_rmsnorm_rope(x, w, tab)).reshape(11, D)
    y = _bits_to_f64(oracle_mod.qk_rmsnorm_rope(x, w, ident)).reshape(11, D)
    nz = z[:, :64] ** 2 + z[:, 64:] ** 2
    ny = y[:, :64] ** 2 + y[:, 64:] ** 2
    np.testing.assert_allclose(nz, ny, rtol=2.0 ** -6, atol=1e-6)


def _golden_rope_cases():
    with open(GOLDEN) as f:
        return json.load(f)["rmsnorm_rope"]


def _expand_bits(spec, D):
    out = np.zeros(D, dtype=np.uint16)
    for key, val in spec.items():
        v = int(val, 16)
        if key == "even":
            out[0::2] = v
        elif key == "odd":
            out[1::2] = v
        elif "-" in key:
            a, b = (int(t) for t in key.split("-"))
            out[a: b + 1] = v
        else:
            out[int(key)] = v
    return out


@pytest.mark.parametrize("case", _golden_rope_cases(), ids=lambda c: c["name"])
def test_golden_rmsnorm_rope(oracle_mod, case):
    D, rot = case["D"], case["rot_dim"]
    if "x" in case:
        x = torch.tensor(case["x"], dtype=torch.bfloat16).reshape(1, 1, 1, D)
    else:
        x = torch.full((1, 1, 1, D), case["x_all"], dtype=torch.bfloat16)
    w = torch.full((D,), case["w_all"], dtype=torch.bfloat16)
    tab = np.array([[case["cos"]] * (rot // 2) + [case["sin"]] * (rot // 2)], dtype=np.float32)
    got = oracle_mod.qk_rmsnorm_rope(x, w, tab, rot_dim=rot, interleaved=case["interleaved"],
                                     eps=case["eps"]).reshape(D)
    assert np.array_equal(got, _expand_bits(case["expected_bits"], D))
