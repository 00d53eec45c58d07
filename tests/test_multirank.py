"""The N > 1 path of bench.py on CPU: world size 2 over gloo (127.0.0.1).

Ranks are replicas (each decodes its own batch, no collective on the data path); the
only cross-rank steps are the barrier and the max of the timings.  These tests run the
helpers under two spawned gloo ranks and the whole reference arm under
torch.distributed.run with two ranks.
"""

import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out_dir):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = 3.0 + 2.0 * rank                  # this rank's duration
        got = bench.max_over_ranks(mine, dist)   # every rank sees the slowest
        seed = bench.rank_seed("llama32k", rank)
        with open(os.path.join(out_dir, "r%d.json" % rank), "w") as f:
            json.dump({"max": got, "seed": seed}, f)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_share_the_max_and_own_their_seeds(tmp_path):
    import torch.multiprocessing as mp
    port = _free_port()
    mp.spawn(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True)
    r0 = json.load(open(tmp_path / "r0.json"))
    r1 = json.load(open(tmp_path / "r1.json"))
    assert r0["max"] == r1["max"] == 5.0
    assert r0["seed"] != r1["seed"]


def test_whole_job_rate_counts_every_rank():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.whole_job_rate(1000, 1, 1.0) == pytest.approx(1e6)
    assert bench.whole_job_rate(1000, 4, 2.0) == pytest.approx(2e6)
    assert bench.max_over_ranks(7.5, None) == 7.5


def test_reference_arm_under_torchrun_two_ranks():
    # rank 0 alone prints the line; rank 1 exits 0 without work
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl",
           "reference", "--gpus", "2", "--steps", "2", "--warmup", "3", "--workload", "tiny",
           "--cpu-seconds", "0.3"]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    p = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=240, env=env)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [ln for ln in p.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, p.stdout
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2
    assert rec["cpu_baseline"]["kind"] == "oracle" and rec["value"] > 0
