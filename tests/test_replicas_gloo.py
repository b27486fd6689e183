"""The multi-GPU benchmark path (independent replicas, one process per GPU) on
the CPU: world-size-2 gloo process groups for the rank bookkeeping, a rank that
never joins, and the reference arm launched by torch.distributed.run."""
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


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import torch

    from expert_router_gemm_b200 import replicas
    r = replicas.from_env()
    assert replicas.init(r, "gloo", timeout_s=30)
    replicas.barrier()
    slowest = replicas.max_over_ranks(1.5 + r.rank, torch.device("cpu"))
    thr = replicas.job_throughput(1000, r.world, slowest)
    out.put((r.rank, r.leader, slowest, thr))
    replicas.finish()


def test_two_gloo_ranks_agree_on_the_slowest_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(world))
    assert [g[0] for g in got] == [0, 1]
    assert [g[1] for g in got] == [True, False]          # only rank 0 prints the line
    for _, _, slowest, thr in got:
        assert slowest == 2.5                            # the max of 1.5 and 2.5
        assert thr == pytest.approx(2 * 1000 / 2.5)      # all ranks' units over the slowest time


def _lonely_rank(port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK="0", WORLD_SIZE="2", LOCAL_RANK="0")
    from expert_router_gemm_b200 import replicas
    try:
        replicas.init(replicas.from_env(), "gloo", timeout_s=3)
        out.put("joined")
    except Exception as e:  # the peer never arrives: an error, not a hang
        out.put(type(e).__name__)


def test_a_rank_that_never_joins_ends_the_wait_with_an_error():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    p = ctx.Process(target=_lonely_rank, args=(_free_port(), q))
    p.start()
    p.join(timeout=120)
    assert p.exitcode == 0
    assert q.get(timeout=5) != "joined"


def test_single_rank_needs_no_process_group():
    from expert_router_gemm_b200 import replicas
    r = replicas.Ranks(0, 1, 0)
    assert not replicas.init(r, "gloo")
    import torch
    assert replicas.max_over_ranks(3.0, torch.device("cpu")) == 3.0
    replicas.barrier()
    replicas.finish()


def test_reference_arm_under_torchrun_two_ranks():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--config", "tiny", "--gpus", "2", "--steps", "2", "--warmup", "3"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]
    lines = [json.loads(x) for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1                               # rank 0 alone prints
    line = lines[0]
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
