"""Multi-rank host logic of bench.py on CPU (gloo, world size 2): rank set-up, the max-over-ranks
reduction of the timed duration, barriers, the whole-job throughput, and the reference arm under
torchrun (rank 0 alone prints; the other rank exits 0 without work)."""
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


def _rank_main(rank: int, world: int, port: int, out_dir: str) -> None:
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist
    import bench
    ws, r = bench.dist_init("gloo", timeout_s=60)
    assert (ws, r) == (world, rank)
    # each rank "timed" a different duration; the job time is the slowest rank's
    mine = 10.0 + 5.0 * rank
    mx = bench.reduce_max(mine, torch.device("cpu"))
    bench.barrier(torch.device("cpu"))
    thr = bench.job_throughput(1000, ws, 4, mx)
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump({"max_ms": mx, "throughput": thr, "env": bench.dist_env()}, f)
    dist.destroy_process_group()


def test_reduce_max_barrier_and_job_throughput_two_ranks(tmp_path):
    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, str(tmp_path))) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(2)]
    for r, d in enumerate(res):
        assert d["max_ms"] == 15.0                      # the slower rank's time on every rank
        assert d["throughput"] == pytest.approx(1000 * 2 * 4 / 0.015)
        assert d["env"] == [2, r, r]


def test_single_process_helpers_are_identities():
    sys.path.insert(0, ROOT)
    import torch
    import bench
    assert bench.reduce_max(3.5, torch.device("cpu")) == 3.5
    bench.barrier(torch.device("cpu"))                  # no process group: no-op
    assert bench.job_throughput(4096 * 4096, 1, 10, 59.6) == pytest.approx(4096 * 4096 * 10 / 0.0596)


@pytest.mark.slow
def test_reference_arm_under_torchrun_rank0_prints_only():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl",
           "reference", "--gpus", "2", "--steps", "1", "--warmup", "0", "--ref-rows", "4",
           "--workload", "tiny_256x512"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
