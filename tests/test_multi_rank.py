"""Host-side logic of bench.py's multi-GPU path, on CPU ranks (gloo).

With N GPUs every rank runs the same layer on its own tokens (independent
batches, no data exchange) and the step time is the slowest rank's.  These
tests run two gloo ranks on the CPU: the max-over-ranks reduction, the
per-rank inputs, and the reference arm printing from rank 0 only.
"""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    import datetime
    import bench
    from int4_weight_quantized_block_b200 import inputs
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        slowest = bench.max_over_ranks(1.5 + rank, torch.device("cpu"))
        x, _ = inputs.layer_inputs(bench.MAIN, seed=bench.rank_seed(rank), M=4)
        xs = [None] * world
        dist.all_gather_object(xs, x[:, :64].copy())
        q.put((rank, slowest, not np.array_equal(xs[0], xs[1])))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_and_distinct_inputs():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, slowest, distinct in out:
        assert slowest == 2.5          # both ranks see the slowest rank's time
        assert distinct                # each rank draws its own tokens


def test_single_process_max_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.25, torch.device("cpu")) == 3.25


@pytest.mark.parametrize("rank", [0, 1])
def test_reference_arm_prints_on_rank0_only(rank):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank))
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3", "--cpu-seconds", "0.2"],
                       capture_output=True, text=True, env=env, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    if rank == 0:
        assert len(lines) == 1
        d = json.loads(lines[0])
        assert d["impl"] == "reference" and d["unit"] == "TOPS" and d["value"] > 0
        assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
    else:
        assert lines == []


def test_gpus_flag_launches_the_ranks_itself():
    """bench.py --gpus 2 outside a launcher starts two ranks itself (torch's
    launcher on this node); the reference arm then prints one line, from rank
    0, and both ranks exit 0."""
    env = {k: v for k, v in os.environ.items()
           if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--impl",
                        "reference", "--steps", "1", "--warmup", "3", "--cpu-seconds", "0.2"],
                       capture_output=True, text=True, env=env, timeout=900)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [l for l in r.stdout.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0
