"""The N > 1 bench path on CPU: two gloo ranks combine their timings the way
bench.py does on GPUs (weak scaling: every rank runs its own copy of the
workload; value = all ranks' FLOPs / slowest rank's time)."""
import os
import socket

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


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import sys

    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    import workloads

    w = workloads.get("cosmos_self")
    fl = bench.flops_of(w)
    dt = 10.0 + 5.0 * rank  # rank 1 is slower
    dt_max, value = bench.combine_ranks(fl, 20, dt, dist, device="cpu")
    q.put((rank, dt_max, value, fl))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_weak_scaling_combination():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    (_, dt0, v0, fl), (_, dt1, v1, _) = res
    assert dt0 == dt1 == 15.0  # both ranks see the slowest rank's time
    expect = 2 * fl * 20 / (15.0 / 1e3) / 1e12
    assert v0 == pytest.approx(expect) and v1 == pytest.approx(expect)


def test_flops_count_only_valid_rows_and_keys():
    import bench
    import workloads

    w = workloads.get("long_gqa")
    assert bench.flops_of(w) == 4.0 * 128 * 32 * 25048 * 25048
    w = workloads.get("cross_short_kv")
    assert bench.flops_of(w) == 4.0 * 128 * 16 * 32760 * 1024


def test_peak_choice_burst_vs_sustained():
    import json
    import sys

    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench

    peaks = os.path.join(bench.ROOT, "MEASURED_PEAKS.json")
    if not os.path.exists(peaks):
        pytest.skip("no measured peaks on this machine")
    d = json.load(open(peaks))
    p_short, k_short = bench.measured_peaks(0.05)
    p_long, k_long = bench.measured_peaks(5.0)
    assert p_short == d["bf16_tflops"] and "burst" in k_short
    if "bf16_tflops_sustained" in d:
        assert p_long == d["bf16_tflops_sustained"] and "sustained" in k_long
