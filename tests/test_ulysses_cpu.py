"""Ulysses split path ("sglang PR 26973", _forward_with_replicated_kv_prefix_split)
on gloo ranks: sequence->head all-to-all of Q and the K/V suffix, local head
slice of the replicated prefix, attention, head->sequence all-to-all of O.
The local attention is the oracle here (this file is test infrastructure), so
every rank's chunk must equal the single-process oracle over the whole
sequence exactly: the exchange only moves rows, and each output row depends
only on its query and the valid keys in prefix-then-suffix order.  Covers a
tail-padded shard, GQA, and KV-head padding when Hkv does not divide sp."""
import datetime
import os
import socket
import warnings

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _problem(B, Hq, Hkv, D, Sp, S, seed=0):
    g = torch.Generator().manual_seed(seed)
    mk = lambda *sh: torch.randn(*sh, generator=g).to(torch.bfloat16)
    return mk(B, S, Hq, D), mk(B, Sp, Hkv, D), mk(B, Sp, Hkv, D), mk(B, S, Hkv, D), mk(B, S, Hkv, D)


def _oracle_local_attn(q, kp, vp, ks, vs, real_len, q_valid, softmax_scale):
    import oracle

    bf = lambda t: t.to(torch.bfloat16)  # values are bf16-exact: the exchange ran in fp32
    out = oracle.attn_split_kv(bf(q), bf(kp), bf(vp), bf(ks), bf(vs), real_len=real_len, q_valid=q_valid,
                               softmax_scale=softmax_scale)
    return torch.from_numpy(out)


def _worker(rank, world, port, cfg, q_out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import sys

        sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
        from varlen_flash_attention_b200 import sp_shard as sps
        from varlen_flash_attention_b200 import ulysses

        B, Hq, Hkv, D, Sp, S = cfg
        q, kp, vp, ks, vs = _problem(B, Hq, Hkv, D, Sp, S)
        plan = sps.build_shard_plan(S)
        f32 = lambda t: t.float()
        ql, ksl, vsl = (sps.shard_like(f32(t), plan) for t in (q, ks, vs))
        with warnings.catch_warnings(record=True) as wl:
            warnings.simplefilter("always")
            out = ulysses.ulysses_attn_fwd_split_kv(ql, f32(kp), f32(vp), ksl, vsl, plan,
                                                    local_attn=_oracle_local_attn)
        q_out.put((rank, plan.local_len, plan.local_real_len, out.numpy(), len(wl)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world, cfg, expect_warn", [
    (2, (1, 4, 2, 64, 5, 23), False),     # GQA 2, shard pad 1
    (4, (2, 6, 3, 64, 7, 30), False),     # Hkv 3 over 4 ranks: KV heads padded to 4, Q heads to 8
    (4, (1, 2, 1, 64, 0, 9), True),       # MQA over 4 ranks: Q heads 2 -> 8 (warned), no prefix
])
def test_ulysses_matches_single_process_oracle(oracle_mod, world, cfg, expect_warn):
    B, Hq, Hkv, D, Sp, S = cfg
    q, kp, vp, ks, vs = _problem(B, Hq, Hkv, D, Sp, S)
    ref = oracle_mod.attn_split_kv(q, kp, vp, ks, vs)  # Sq = S != Sp + S: every query row is real
    ctx = mp.get_context("spawn")
    qq = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, cfg, qq)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((qq.get(timeout=180) for _ in range(world)), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, local_len, real, out, nwarn in res:
        assert out.shape == (B, local_len, Hq, D)
        a = rank * local_len
        assert np.array_equal(out[:, :real], ref[:, a:a + real]), f"rank {rank}"
        assert np.all(out[:, real:] == 0)  # this rank's shard pad rows
        assert (nwarn > 0) == expect_warn


def _oracle_scatter(q, kp, vp, ks, vs, dst, head_offset, real_len, q_valid, softmax_scale):
    """Stand-in for the scatter kernel: the oracle's head-shard output, row s
    stored into dst[s // L] at this rank's head slot."""
    out = _oracle_local_attn(q, kp, vp, ks, vs, real_len, q_valid, softmax_scale)
    L, hl = dst[0].shape[1], out.shape[2]
    for r, buf in enumerate(dst):
        buf[:, :, head_offset:head_offset + hl] = out[:, r * L:(r + 1) * L].to(buf.dtype)


def _worker_fused(rank, world, port, cfg, recv, q_out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import sys

        sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
        from varlen_flash_attention_b200 import sp_shard as sps
        from varlen_flash_attention_b200 import ulysses

        B, Hq, Hkv, D, Sp, S = cfg
        q, kp, vp, ks, vs = _problem(B, Hq, Hkv, D, Sp, S)
        plan = sps.build_shard_plan(S)
        f32 = lambda t: t.float()
        ql, ksl, vsl = (sps.shard_like(f32(t), plan) for t in (q, ks, vs))
        with warnings.catch_warnings():
            warnings.simplefilter("ignore")
            out = ulysses.ulysses_attn_fwd_split_kv_fused(ql, f32(kp), f32(vp), ksl, vsl, plan, recv,
                                                          local_attn_scatter=_oracle_scatter)
        q_out.put((rank, plan.local_len, plan.local_real_len, out.numpy().copy()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world, cfg", [
    (2, (1, 4, 2, 64, 5, 23)),     # GQA 2, shard pad 1
    (4, (2, 6, 3, 64, 7, 30)),     # KV heads padded 3 -> 4, Q heads 6 -> 8
])
def test_fused_output_exchange_matches_single_process_oracle(oracle_mod, world, cfg):
    """The fused form: every rank stores its head shard's rows straight into
    the other ranks' receive buffers (shared memory standing in for buffers
    mapped from the other GPUs), then a barrier; each rank's chunk equals the
    single-process oracle exactly, pad rows included."""
    from varlen_flash_attention_b200 import sp_shard as sps
    from varlen_flash_attention_b200 import ulysses

    B, Hq, Hkv, D, Sp, S = cfg
    q, kp, vp, ks, vs = _problem(B, Hq, Hkv, D, Sp, S)
    ref = oracle_mod.attn_split_kv(q, kp, vp, ks, vs)
    L = sps.build_shard_plan(S, world, 0).local_len
    Hq_p, _ = ulysses.gqa_head_padding(Hq, Hkv, world)
    recv = [torch.full((B, L, Hq_p, D), float("nan"), dtype=torch.float64).share_memory_() for _ in range(world)]
    ctx = mp.get_context("spawn")
    qq = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker_fused, args=(r, world, port, cfg, recv, qq)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((qq.get(timeout=180) for _ in range(world)), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, local_len, real, out in res:
        assert out.shape == (B, local_len, Hq, D)
        a = rank * local_len
        assert np.array_equal(out[:, :real], ref[:, a:a + real]), f"rank {rank}"
        assert np.all(out[:, real:] == 0)  # this rank's shard pad rows


def test_head_padding_rule():
    from varlen_flash_attention_b200 import ulysses

    assert ulysses.gqa_head_padding(32, 8, 8) == (32, 8)
    assert ulysses.gqa_head_padding(24, 24, 16) == (32, 32)
    assert ulysses.gqa_head_padding(6, 3, 4) == (8, 4)
    with pytest.raises(ValueError):
        ulysses.gqa_head_padding(6, 4, 2)


def test_fused_form_needs_one_receive_buffer_per_rank():
    from varlen_flash_attention_b200 import sp_shard as sps
    from varlen_flash_attention_b200 import ulysses

    plan = sps.build_shard_plan(10, 2, 0)
    x = torch.zeros(1, plan.local_len, 2, 64)
    kv = torch.zeros(1, 3, 2, 64)
    with pytest.raises(ValueError):
        ulysses.ulysses_attn_fwd_split_kv_fused(x, kv, kv, x, x, plan, [torch.zeros(1, 5, 2, 64)])
