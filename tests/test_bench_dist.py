"""The multi-rank plumbing of bench.py on CPU: two gloo ranks.

bench.py runs one independent batch per rank (weak scaling, no data-path
collective); the only collective is the max over ranks of the device time.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    import datetime
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        ms = bench.reduce_max_ms(10.0 + 5.0 * rank, world, "cpu")
        out[rank] = (ms, bench.rank_seed(100, rank),
                     bench.weak_scaling_value(1000, 10, world, ms))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_weak_scaling():
    world = 2
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    ms = [out[r][0] for r in range(world)]
    assert ms == [15.0, 15.0], "every rank sees the slowest rank's time"
    assert out[0][1] != out[1][1], "ranks draw different batches"
    # 1000 tokens x 10 steps x 2 ranks in 15 ms
    assert out[0][2] == pytest.approx(1000 * 10 * 2 / 0.015)


def test_reference_arm_prints_the_contract_line():
    """bench.py --impl reference (the fp64 oracle on the host) prints one JSON
    line with the contract's keys, on the tiny Mamba-1 workload."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--workload",
                          "mamba1_tiny_f32", "--steps", "1", "--warmup", "0"], capture_output=True, text=True,
                         timeout=300, cwd=root)
    assert out.returncode == 0, out.stderr[-2000:]
    line = [l for l in out.stdout.splitlines() if l.startswith("{")][-1]
    d = json.loads(line)
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
