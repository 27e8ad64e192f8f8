"""Multi-rank host logic of bench.py on the CPU (gloo, world size 2).

The path partitions by request: every rank runs its own replica of the
workload and the only cross-rank step is the timing reduction (max over
ranks) and the whole-job rate.  Two spawned ranks check that both see the
same maximum, that the rate counts every rank's units over the slowest
rank's time, and that the reference arm (of the step metric and of the
calibration fit) runs and prints on rank 0 only.
"""
import multiprocessing
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    from datetime import timedelta

    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    import bench
    from speculative_decoding_05_b200 import workloads as WL
    ms_local = [2.0, 3.5][rank]
    mx = bench.reduce_max(ms_local)
    rate = bench.whole_job_rate(16, world, mx)

    class Args:
        steps, warmup = 1, 0

    ref = bench.run_reference(Args, WL.get("tiny"), rank, world)

    class CalArgs:
        impl, steps, warmup = "reference", 1, 0

    os.environ["DSPARK_REF_SEQUENCES"] = "2000"
    import contextlib
    import io
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.run_calibration(CalArgs, WL.CALIBRATIONS["calibration_small"], rank, world)
    cal_lines = [l for l in buf.getvalue().splitlines() if l.startswith("{")]
    q.put((rank, mx, rate, ref is None, len(cal_lines)))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_timing_reduction_and_reference_arm():
    ctx = multiprocessing.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=240)
    alive = [p for p in procs if p.is_alive()]
    for p in alive:
        p.kill()
    assert not alive, "a rank hung"
    assert all(p.exitcode == 0 for p in procs)
    res = sorted(q.get(timeout=5) for _ in range(2))
    for rank, mx, rate, ref_none, n_cal in res:
        assert mx == 3.5
        assert rate == pytest.approx(16 * 2 / 3.5e-3)
        assert ref_none == (rank != 0)  # rank 0 alone runs the reference arm
        assert n_cal == (1 if rank == 0 else 0)  # also for the calibration line


def test_single_process_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max(1.25) == 1.25
    assert bench.whole_job_rate(16, 1, 2.0) == pytest.approx(8000.0)


def test_launcher_for_gpus_n():
    """--gpus N without a launcher re-runs the script as N ranks through
    torch.distributed.run on 127.0.0.1; under a launcher --gpus must match
    its world size."""
    sys.path.insert(0, ROOT)
    import bench
    argv = bench.launcher_argv(4, ["--gpus", "4", "--steps", "3"], 29512)
    assert argv[1:3] == ["-m", "torch.distributed.run"]
    assert "--nproc-per-node=4" in argv and "--master-addr=127.0.0.1" in argv
    assert "--master-port=29512" in argv and argv[-4:] == ["--gpus", "4", "--steps", "3"]
    assert bench.check_world(2, {"WORLD_SIZE": "2"}) == 2
    assert bench.check_world(1, {}) == 1
    with pytest.raises(SystemExit):
        bench.check_world(4, {"WORLD_SIZE": "2"})
    with pytest.raises(SystemExit):
        bench.check_world(2, {"WORLD_SIZE": "1"})
