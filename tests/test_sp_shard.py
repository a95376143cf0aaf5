"""Sequence-parallel shard helpers ("sglang PR 30107", unified SP shard utils),
checked against the shard math the page states: equal chunks of
ceil(S / sp) tokens, all pad at the global tail, tail metadata with
max_seqlen_tail >= num_pad, zero / repeat_last tail fill, and gather as the
inverse of shard.  Multi-rank cases run as gloo ranks on CPU."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from varlen_flash_attention_b200 import sp_shard as sps


def test_plan_divisible():
    for r in range(8):
        p = sps.build_shard_plan(4096, sp_size=8, sp_rank=r)
        assert (p.local_len, p.num_pad, p.local_pad, p.local_real_len) == (512, 0, 0, 512)
        assert sps.tail_attn_meta(p) is None


@pytest.mark.parametrize("sp, local_len", [(8, 554), (16, 277)])
def test_plan_padded_last_rank_tail_padded_workload(sp, local_len):
    # 333 text + 4096 image tokens = 4429, padded to 4432 (3 pad tokens).
    plans = [sps.build_shard_plan(4429, sp_size=sp, sp_rank=r) for r in range(sp)]
    for p in plans:
        assert p.local_len == local_len and p.num_pad == 3 and p.padded_len == 4432
    assert [p.local_pad for p in plans] == [0] * (sp - 1) + [3]
    assert sum(p.local_real_len for p in plans) == 4429
    meta_last = sps.tail_attn_meta(plans[-1])
    assert meta_last == {"tail": True, "valid_len": local_len - 3, "max_seqlen_tail": local_len - 3}
    meta_first = sps.tail_attn_meta(plans[0])
    assert meta_first["valid_len"] == local_len
    assert sps.tail_attn_meta(plans[-1], seqlen_multiplier=2)["valid_len"] == 2 * (local_len - 3)
    assert sps.attn_real_len(plans[0], batch=2) == [4429, 4429]


def test_plan_degenerate_pad_outnumbers_tokens():
    # one token over four ranks: local_len 1, three pad tokens
    plans = [sps.build_shard_plan(1, sp_size=4, sp_rank=r) for r in range(4)]
    assert all(p.local_len == 1 and p.num_pad == 3 for p in plans)
    assert [p.local_real_len for p in plans] == [1, 0, 0, 0]
    assert all(p.local_real_len >= 0 for p in plans)
    for p in plans:
        m = sps.tail_attn_meta(p)
        assert m["max_seqlen_tail"] >= p.num_pad and m["max_seqlen_tail"] >= m["valid_len"]


def test_plan_identity_and_validation():
    p = sps.build_shard_plan(100, sp_size=1, sp_rank=0)
    assert (p.orig_len, p.local_len, p.num_pad, p.sp_size) == (100, 100, 0, 1)
    x = torch.randn(2, 100, 3)
    assert sps.shard_like(x, p) is x
    with pytest.raises(ValueError):
        sps.build_shard_plan(10, sp_size=4, sp_rank=4)
    with pytest.raises(ValueError):
        sps.build_shard_plan(-1, sp_size=2, sp_rank=0)
    # not initialised: defaults to a one-rank plan
    assert sps.build_shard_plan(7).sp_size == 1


@pytest.mark.parametrize("S, sp", [(10, 4), (9, 3), (4429, 8), (3, 5), (1, 4)])
def test_padded_chunks_cover_sequence_exactly(S, sp):
    """Brute force: concatenating every rank's chunk gives the sequence followed
    by exactly num_pad zero rows, and each chunk's real/pad split matches."""
    x = torch.arange(1, S + 1, dtype=torch.float32).view(1, S, 1)
    plans = [sps.build_shard_plan(S, sp_size=sp, sp_rank=r) for r in range(sp)]
    chunks = [sps.shard_like(x, p) for p in plans]
    full = torch.cat(chunks, dim=1)
    assert full.shape[1] == plans[0].padded_len
    assert torch.equal(full[:, :S], x)
    assert torch.all(full[:, S:] == 0) and full.shape[1] - S == plans[0].num_pad
    for p, c in zip(plans, chunks):
        assert int((c != 0).sum()) == p.local_real_len
        assert int((c == 0).sum()) == p.local_pad


def test_shard_like_zero_and_repeat_last_tail():
    x = torch.arange(10, dtype=torch.float32).view(1, 10, 1) + 1
    p3 = sps.build_shard_plan(10, sp_size=4, sp_rank=3)  # local 3, pad 2
    assert sps.shard_like(x, p3).flatten().tolist() == [10.0, 0.0, 0.0]
    assert sps.shard_like(x, p3, pad_mode="repeat_last").flatten().tolist() == [10.0, 10.0, 10.0]
    p0 = sps.build_shard_plan(10, sp_size=4, sp_rank=0)
    assert sps.shard_like(x, p0).flatten().tolist() == [1.0, 2.0, 3.0]
    # sharding along another dim (a RoPE table [S, rot]) keeps chunks aligned
    t = torch.arange(20, dtype=torch.float32).view(10, 2)
    assert torch.equal(sps.shard_like(t, p0, dim=0), t[:3])
    with pytest.raises(ValueError):
        sps.shard_like(x, sps.build_shard_plan(11, sp_size=4, sp_rank=0))
    with pytest.raises(ValueError):
        sps.shard_like(x, p3, pad_mode="reflect")


def test_join_split_moves_pad_to_tail_and_back():
    txt = torch.cat([torch.ones(1, 5, 2), torch.zeros(1, 2, 2)], dim=1)  # 5 real + 2 pad
    img = torch.full((1, 4, 2), 7.0)
    (joint,) = sps.join_seqs([txt], [img], local_pad=2)
    assert joint[0, :, 0].tolist() == [1, 1, 1, 1, 1, 7, 7, 7, 7, 0, 0]
    ((t2, i2),) = sps.split_seqs([joint], first_len=7, local_pad=2)
    assert torch.equal(t2, txt) and torch.equal(i2, img)
    (j0,) = sps.join_seqs([txt], [img], local_pad=0)
    assert torch.equal(j0, torch.cat([txt, img], dim=1))
    with pytest.raises(ValueError):
        sps.join_seqs([txt], [img], local_pad=8)


def test_should_shard_text_policy():
    assert sps.should_shard_text(333, 8)
    assert not sps.should_shard_text(333, 1)
    assert not sps.should_shard_text(100, 8, min_len=256)
    assert sps.should_shard_text(256, 8, min_len=256)


def test_gathered_tail_pad_attention_equals_unpadded(oracle_mod):
    """The shard layout feeds attn_fwd_split_kv directly: attention over the
    gathered (tail-padded) joint sequence with real_len = orig_len equals
    attention over the unpadded sequence, for any pad contents."""
    gen = torch.Generator().manual_seed(11)
    S, H, D, sp = 45, 2, 64, 4
    plan = sps.build_shard_plan(S, sp_size=sp, sp_rank=0)
    q, k, v = (torch.randn(1, S, H, D, generator=gen).to(torch.bfloat16) for _ in range(3))
    pad = plan.num_pad
    assert pad == 3
    garbage = torch.full((1, pad, H, D), 1e4, dtype=torch.bfloat16)
    qp, kp_, vp_ = (torch.cat([t, garbage], dim=1) for t in (q, k, v))
    empty = k[:, :0]
    ref = oracle_mod.attn_split_kv(q, empty, empty, k, v, real_len=[S])
    got = oracle_mod.attn_split_kv(qp, empty, empty, kp_, vp_, real_len=sps.attn_real_len(plan))
    assert np.array_equal(got[:, :S], ref)
    assert np.all(got[:, S:] == 0)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _gather_worker(rank, world, port, S, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        plan = sps.build_shard_plan(S)  # size and rank from the process group
        x = torch.arange(S * 3, dtype=torch.float32).view(1, S, 3)
        local = sps.shard_seq(x, plan)
        back = sps.gather_seq(local, plan)
        q.put((rank, plan.sp_size, plan.sp_rank, plan.local_pad, bool(torch.equal(back, x))))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world, S", [(2, 7), (3, 10), (2, 8)])
def test_gather_inverts_shard_on_gloo_ranks(world, S):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_gather_worker, args=(r, world, port, S, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    local_len = -(-S // world)
    num_pad = local_len * world - S
    for rank, size, r, lp, ok in res:
        assert size == world and r == rank and ok
        assert lp == (num_pad if rank == world - 1 else 0)


@pytest.mark.gpu
@pytest.mark.parametrize("S, sp, mode", [(4429, 8, "zeros"), (10, 4, "repeat_last"), (1, 4, "zeros"),
                                          (1, 4, "repeat_last"), (333, 16, "zeros"), (4429, 8, "repeat_last")])
def test_shard_copy_kernel_matches_oracle(S, sp, mode):
    """The CUDA one-pass copy (sk_shard_pad_copy, used for chunks that hold
    pad; other chunks are views) equals the oracle's padded chunk bit for bit,
    and the CPU torch branch of shard_like agrees too."""
    import oracle

    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    from varlen_flash_attention_b200 import build

    build.build()
    g = torch.Generator().manual_seed(S)
    x = torch.randn(2, S, 3, 64, generator=g).to(torch.bfloat16)
    x[:, -1] = float("nan")  # the repeated row's bits must survive the copy
    xd = x.cuda()
    for r in range(sp):
        p = sps.build_shard_plan(S, sp_size=sp, sp_rank=r)
        want = oracle.shard_chunk(x, S, sp, r, mode)
        got = sps.shard_like(xd, p, pad_mode=mode)         # CUDA: view or the copy kernel
        torch.cuda.synchronize()
        got_bits = got.cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
        assert got_bits.shape == want.shape and np.array_equal(got_bits, want), f"rank {r}"
        cpu = sps.shard_like(x, p, pad_mode=mode).contiguous().view(torch.int16).numpy().view(np.uint16)
        assert np.array_equal(cpu, want), f"rank {r} (torch branch)"
