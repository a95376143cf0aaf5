"""Pins of the oracle's tail-padded shard chunk (oracle.shard_chunk) to what
the "sglang PR 30107" page fixes: hand-derived chunks (tests/golden/
shard_chunks.json), torch's own padding routines (F.pad with zeros, and with
mode="replicate" for repeat_last) followed by a slice, the layout invariant
(all pad rows at the tail of the stream, so gathering every rank's chunk and
trimming to orig_len gives the input back), and planted mistakes that must
each fail one of these pins."""
import json
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "shard_chunks.json")


def _rows(n, width=3):
    """Row t holds the value t + 1 in every column (0 is left for zero pad)."""
    return np.repeat(np.arange(1, n + 1, dtype=np.float64)[None, :, None], width, axis=2)


def _ids(chunk):
    """Source index of each row of a chunk built from _rows (-1 = zero row)."""
    return [int(v) - 1 for v in chunk[0, :, 0]]


def test_golden_chunks():
    g = json.load(open(GOLDEN))
    for c in g["cases"]:
        n, sp = c["orig_len"], c["sp_size"]
        x = _rows(n)
        for mode in ("zeros", "repeat_last"):
            chunks = [oracle.shard_chunk(x, n, sp, r, mode) for r in range(sp)]
            assert all(ch.shape[1] == c["local_len"] for ch in chunks)
            assert c["local_len"] * sp - n == c["num_pad"]
            if "chunks" in c:
                assert [_ids(ch) for ch in chunks] == c["chunks"][mode], (n, sp, mode)
            else:
                assert _ids(chunks[-1])[-6:] == c["last_chunk_tail"][mode], (n, sp, mode)


def _library_chunk(x, n, sp, rank, mode):
    """torch's padding routine on the sequence axis, then the rank's slice."""
    local = -(-n // sp)
    pad = local * sp - n
    t = torch.from_numpy(x)                                   # [B, S, C]
    if mode == "zeros":
        full = F.pad(t, (0, 0, 0, pad))                       # pad axis 1 at its end
    else:
        full = F.pad(t.transpose(1, 2), (0, pad), mode="replicate").transpose(1, 2)
    return full[:, rank * local:(rank + 1) * local].numpy()


@pytest.mark.parametrize("n", [1, 2, 3, 7, 16, 33, 100, 333, 4429])
@pytest.mark.parametrize("sp", [1, 2, 3, 4, 8, 16])
@pytest.mark.parametrize("mode", ["zeros", "repeat_last"])
def test_matches_torch_padding(n, sp, mode):
    rng = np.random.default_rng(n * 31 + sp)
    x = rng.standard_normal((2, n, 5))
    for r in range(sp):
        got = oracle.shard_chunk(x, n, sp, r, mode)
        assert np.array_equal(got, _library_chunk(x, n, sp, r, mode)), (n, sp, r)


@pytest.mark.parametrize("n,sp", [(5, 2), (7, 3), (1, 4), (4429, 8), (333, 16), (10, 4)])
def test_gather_then_trim_is_identity(n, sp):
    x = _rows(n)
    for mode in ("zeros", "repeat_last"):
        gathered = np.concatenate([oracle.shard_chunk(x, n, sp, r, mode) for r in range(sp)], axis=1)
        assert np.array_equal(gathered[:, :n], x)
        tail = gathered[:, n:]
        want = 0.0 if mode == "zeros" else float(n)
        assert np.all(tail == want)


def test_bf16_bits_pass_through_exactly():
    g = torch.Generator().manual_seed(0)
    x = torch.randn(2, 13, 3, 8, generator=g).to(torch.bfloat16)
    x[0, 12, 0, 0] = float("nan")
    x[1, 3, 2, 1] = float("-inf")
    bits = x.view(torch.int16).numpy().view(np.uint16)
    for r in range(4):
        got = oracle.shard_chunk(x, 13, 4, r, "repeat_last")
        want = oracle.shard_chunk(bits, 13, 4, r, "repeat_last")
        assert got.dtype == np.uint16 and np.array_equal(got, want)


@pytest.mark.parametrize("mutate", ["floor_len", "pad_first", "repeat_first"])
def test_planted_mistakes_fail_a_pin(mutate):
    failed = False
    for n, sp in ((5, 2), (7, 3), (1, 4), (10, 4)):
        x = _rows(n)
        for mode in ("zeros", "repeat_last"):
            for r in range(sp):
                try:
                    got = oracle.shard_chunk(x, n, sp, r, mode, mutate=mutate)
                except (ValueError, IndexError):
                    failed = True
                    continue
                if got.shape != _library_chunk(x, n, sp, r, mode).shape or \
                        not np.array_equal(got, _library_chunk(x, n, sp, r, mode)):
                    failed = True
    assert failed, mutate
