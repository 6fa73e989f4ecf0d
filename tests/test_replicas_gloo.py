"""Multi-process plumbing of `bench.py --gpus N` (replicas only: the hot path has
no exchange step), run as world_size-2 gloo ranks on the CPU.

Every rank takes the same collective steps; the reported time is the slowest
rank's and the value counts every rank's units (weak scaling)."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        local_s = [0.25, 0.75][rank]                  # rank 1 is the slow one
        t_max = bench.reduce_max(local_s, world)
        value, t = bench.aggregate(1000.0, [t_max] * world)
        bench.barrier(world)
        out.put((rank, t_max, value, t))
    finally:
        dist.destroy_process_group()


def test_replicas_report_slowest_rank_and_all_units():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=5) for _ in range(world))
    for rank, t_max, value, t in res:
        assert t_max == 0.75 and t == 0.75                 # max over ranks, on every rank
        assert value == pytest.approx(2 * 1000.0 / 0.75)   # all ranks' units over the slowest time


def test_aggregate_is_weak_scaling_over_the_slowest_rank():
    sys.path.insert(0, ROOT)
    import bench
    v, t = bench.aggregate(10.0, [1.0, 2.0, 4.0])
    assert t == 4.0 and v == pytest.approx(30.0 / 4.0)
    v1, _ = bench.aggregate(10.0, [2.0])
    assert v1 == pytest.approx(5.0)


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "1"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""                            # only rank 0 prints the line


def test_clock_sampler_reads_nvidia_smi_csv_without_nvml(tmp_path):
    sys.path.insert(0, ROOT)
    import bench
    cs = bench.ClockSampler.__new__(bench.ClockSampler)
    cs.thread, cs.nvml, cs.reasons = None, None, set()
    cs.path = str(tmp_path / "clk.csv")
    with open(cs.path, "w") as f:
        f.write("0, 1965, 1965, 250.5, 0x0, Not Active, Not Active, Not Active, Not Active\n")
        f.write("0, 1905, 1965, 999.0, 0x4, Not Active, Not Active, Not Active, Active\n")
        f.write("garbage line\n")

    class _Done:
        def terminate(self):
            pass

        def wait(self, timeout=None):
            return 0
    cs.proc = _Done()
    r = cs.stop()
    assert r["samples"] == 2 and r["sm_mhz"] == pytest.approx(1935.0) and r["sm_max_mhz"] == 1965.0
    assert r["reasons"] == ["sw_power_cap"] and r["power_w_max"] == 999.0
    json.dumps(r)
