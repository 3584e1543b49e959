"""The bench's multi-rank host logic on CPU ranks (gloo, world size 2): how a
rank reads its place in the job, the max-over-ranks reduction of a timing,
the job-level config, and the reference arm under torchrun (rank 0 alone
runs the oracle and prints the line; the other rank exits 0 without work).
No GPU is used."""
import json
import os
import socket
import subprocess
import sys
from pathlib import Path

import pytest
import torch.multiprocessing as mp

ROOT = Path(__file__).resolve().parent.parent


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import datetime
    import types
    import torch.distributed as dist
    sys.path.insert(0, str(ROOT))
    import bench
    from neighborhood_attention_na2d_b200.inputs import WORKLOADS
    os.environ.update(WORLD_SIZE=str(world), RANK=str(rank), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        got_world, got_rank, got_local = bench.dist_setup(types.SimpleNamespace(gpus=world))
        # a different timing on every rank: the job takes the slowest
        slowest = bench.max_over_ranks(1.0 + 0.25 * rank, dist, "cpu")
        again = bench.max_over_ranks(5.0 - rank, dist, "cpu")
        wl = WORKLOADS["nat_tiny_s1_fp16"]
        cfg = bench.config_dict(wl, got_world)
        res = dict(world=got_world, rank=got_rank, local=got_local, slowest=slowest, again=again,
                   global_batch=cfg["global_batch"], parallelism=cfg["parallelism"], B=wl.shapes[0].B)
        Path(out_dir, f"rank{rank}.json").write_text(json.dumps(res))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_gloo_two_ranks_reduce_and_config(tmp_path):
    world, port = 2, _free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path)), nprocs=world, start_method="spawn", join=True)
    res = [json.loads((tmp_path / f"rank{r}.json").read_text()) for r in range(world)]
    for r, x in enumerate(res):
        assert (x["world"], x["rank"], x["local"]) == (world, r, r)
        assert x["slowest"] == 1.25 and x["again"] == 5.0   # the same maximum on every rank
        assert x["global_batch"] == world * x["B"] and x["parallelism"] == f"replicas{world}"


def test_reference_arm_under_torchrun_two_ranks():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes", "1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "3"]
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="", OMP_NUM_THREADS="1")
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["config"]["parallelism"] == "replicas2"
