"""The N>1 path of bench.py on CPU: two `gloo` ranks.

The matvec does not shard, so `bench.py --gpus N` runs N independent replicas.
The host logic is checked here: each rank builds different matrices, the step
time is the slowest rank's, and the whole-job value counts all ranks' matvecs.
The reference arm does its work on rank 0 only.
"""
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

WORKER = r"""
import os, sys, datetime
sys.path.insert(0, {root!r})
import torch, torch.distributed as dist
import bench
rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
dev = torch.device("cpu")
mine = 10.0 + 5.0 * rank                     # this rank's step time
slowest = bench.max_over_ranks(mine, world, dev)
seeds = [bench.replica_seed(rank, m) for m in range(3)]
allseeds = [None] * world
dist.all_gather_object(allseeds, seeds)
value = bench.whole_job_us_per_matvec(slowest, world)
print("RESULT", rank, slowest, value, sorted(set(sum(allseeds, []))) == sorted(sum(allseeds, [])), flush=True)
dist.barrier()
dist.destroy_process_group()
"""


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks_time_the_slowest_and_use_distinct_replicas(tmp_path):
    script = tmp_path / "worker.py"
    script.write_text(WORKER.format(root=ROOT))
    port = str(free_port())
    procs = []
    for r in range(2):
        env = dict(os.environ, RANK=str(r), WORLD_SIZE="2", MASTER_ADDR="127.0.0.1", MASTER_PORT=port,
                   LOCAL_RANK=str(r))
        procs.append(subprocess.Popen([sys.executable, str(script)], env=env, stdout=subprocess.PIPE,
                                      stderr=subprocess.STDOUT, text=True))
    outs = []
    for p in procs:
        out, _ = p.communicate(timeout=120)
        assert p.returncode == 0, out
        outs.append(out)
    results = {}
    for out in outs:
        line = [l for l in out.splitlines() if l.startswith("RESULT")][0].split()
        results[int(line[1])] = (float(line[2]), float(line[3]), line[4] == "True")
    for r in (0, 1):
        slowest, value, distinct = results[r]
        assert slowest == 15.0            # rank 1's 15 us is the job's step time
        assert value == 7.5               # two matvecs per 15 us step
        assert distinct                   # no two ranks share a matrix seed


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")

    class A:
        steps, warmup, gpus = 1, 0, 2

    bench.run_reference(A())  # returns at once: no oracle work on other ranks
    assert capsys.readouterr().out == ""
