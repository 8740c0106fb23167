"""The N-GPU bench path is N independent replicas: its only collectives are the timing
barrier and the max of the device times over ranks.  Checked here on CPU with two gloo
ranks (no GPU), plus the reference arm's rank gating."""
import io
import os
import socket
import sys
from contextlib import redirect_stdout

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch
    reps = bench.Replicas("gloo", torch.device("cpu"), timeout_s=60)
    reps.barrier()
    local_ms = 10.0 + 5.0 * rank          # rank 1 is the slow replica
    ms = reps.max(local_ms)
    value = reps.throughput(51200, 4, ms)
    reps.barrier()
    reps.close()
    out.put((rank, reps.world, ms, value))


def test_two_gloo_replicas_agree_on_the_slowest_time_and_the_job_rate():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, world, ms, value in res:
        assert world == 2
        assert ms == 15.0                      # the max over ranks, on every rank
        assert abs(value - 51200 * 4 * 2 / 15e-3) < 1e-6 * value


def test_single_process_needs_no_process_group(monkeypatch):
    for k in ("WORLD_SIZE", "RANK"):
        monkeypatch.delenv(k, raising=False)
    reps = bench.Replicas("gloo")
    assert reps.world == 1 and reps.max(3.5) == 3.5
    assert reps.throughput(100, 10, 1000.0) == 1000.0
    reps.barrier()
    reps.close()


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    buf = io.StringIO()
    with redirect_stdout(buf):
        sys_argv = sys.argv
        sys.argv = ["bench.py", "--impl", "reference", "--gpus", "2", "--steps", "1",
                    "--warmup", "0"]
        try:
            bench.run_reference(bench.parse_args(sys.argv[1:]))
        finally:
            sys.argv = sys_argv
    assert buf.getvalue() == ""              # the other ranks exit without work or output


def test_gpus_flag_starts_that_many_ranks_through_the_launcher():
    # `bench.py --gpus 2` without torchrun re-launches itself as 2 ranks; the replica check
    # runs the same plumbing the GPU arm uses (gloo on CPU here) and every rank reports
    import json
    import subprocess
    env = {k: v for k, v in os.environ.items()
           if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_PORT")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2",
                        "--replica-check"], env=env, capture_output=True, text=True,
                       timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stdout + r.stderr
    lines = [json.loads(l) for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout                  # rank 0 alone prints
    views = lines[0]["ranks"]
    assert sorted(v["rank"] for v in views) == [0, 1], r.stdout
    for l in views:
        assert l["world"] == 2 and l["max_ms"] == 15.0
        assert abs(l["value"] - 1000 * 4 * 2 / 15e-3) < 1e-6 * l["value"]


def test_launch_command_is_one_local_node_on_loopback():
    cmd = bench.launch_command(4, ["--gpus", "4", "--steps", "3"], 29555)
    assert cmd[1:3] == ["-m", "torch.distributed.run"]
    assert "--nproc-per-node=4" in cmd and "--nnodes=1" in cmd
    assert cmd[cmd.index("--master-addr") + 1] == "127.0.0.1"
    assert cmd[-4:] == ["--gpus", "4", "--steps", "3"]
    assert cmd[-5].endswith("bench.py")
