"""The multi-process (N > 1) plumbing of bench.py, on CPU with gloo ranks.

Attention here shards with no exchange, so N GPUs run N independent replicas;
what N > 1 adds is the launch contract: ranks from torch.distributed.run, a
barrier around the timed region, the maximum over ranks of the timed value,
and a single JSON line from rank 0. These tests run that plumbing with two
gloo ranks on the host (no GPU): the helpers directly, and the reference arm
end to end under torch.distributed.run.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    r, w, local = bench.dist_setup(world)
    assert (r, w, local) == (rank, world, rank)
    assert dist.get_backend() == "gloo"
    bench.dist_barrier(w)
    # each rank's "timed value" differs; every rank must see the maximum
    got = bench.dist_max(100.0 + 7.5 * rank, w)
    bench.dist_barrier(w)
    with open(os.path.join(out_dir, "rank%d.txt" % rank), "w") as f:
        f.write(repr(got))
    dist.destroy_process_group()


def test_dist_helpers_take_the_max_over_two_gloo_ranks(tmp_path):
    world = 2
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    vals = [float(open(tmp_path / ("rank%d.txt" % r)).read()) for r in range(world)]
    assert vals == [107.5, 107.5]


def test_single_process_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    env = {k: os.environ.pop(k) for k in ("RANK", "WORLD_SIZE") if k in os.environ}
    try:
        assert bench.dist_setup(1) == (0, 1, 0)
        assert bench.dist_max(3.25, 1) == 3.25
        bench.dist_barrier(1)  # a no-op without a process group
    finally:
        os.environ.update(env)


@pytest.mark.timeout(600)
def test_reference_arm_under_torchrun_prints_one_line_from_rank0():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
           "--steps", "2", "--warmup", "3", "--workload", "tiny", "--ref-budget-seconds", "30"]
    env = dict(os.environ, OMP_NUM_THREADS="2")
    p = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=540)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [ln for ln in p.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, p.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2
    assert d["value"] > 0 and d["unit"] == "us/call" and d["higher_is_better"] is False
    assert d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    # full oracle calls, the steps that ran reported as such
    assert d["steps"] == 2 and d["warmup"] == 0 and "unsampled" in d["cpu_baseline"]["sample"]


def test_clock_summary_reads_medians_power_and_throttle_reasons():
    # nvidia-smi csv,noheader,nounits lines in ClockSampler.FIELDS order:
    # clocks.sm, clocks.max.sm, power.draw, reasons.active, hw_slowdown,
    # hw_thermal_slowdown, sw_thermal_slowdown, sw_power_cap
    sys.path.insert(0, ROOT)
    import bench
    c = bench.ClockSampler(0)
    c.lines = [
        "1965, 1965, 250.0, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "1530, 1965, 990.5, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "1540, 1965, 991.5, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "1550, 1965, 992.5, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "garbage line",
    ]
    s = bench.ClockSampler.summary(c)
    assert s["sm_mhz"] == 1545.0 and s["sm_max_mhz"] == 1965.0 and s["samples"] == 4
    assert s["reasons"] == ["sw_power_cap"]
    # a window of the samples (the sustained timing skips its settling second)
    w = c.summary(1, 4)
    assert w["sm_mhz"] == 1540.0 and w["power_w"] == 991.5 and w["samples"] == 3
    c.lines = []
    assert c.summary()["reasons"] == ["unavailable"]
