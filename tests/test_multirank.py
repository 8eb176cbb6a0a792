"""Multi-rank host logic of the benchmark on CPU with two gloo ranks: every
rank gets its own batch (same shapes, own seed), the timing reduction is the
max over ranks on every rank, and the reference arm runs on rank 0 only."""
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = bench.rank_workload("decoder", rank)
        local = [1.0 + rank, 5.0 - rank, 0.25 * (rank + 1)]
        red = bench.max_over_ranks(local, world, torch.device("cpu"))
        buf = io.StringIO()
        with redirect_stdout(buf):
            bench.main(["--impl", "reference", "--workload", "decoder", "--steps", "1",
                        "--warmup", "0", "--gpus", str(world)])
        dist.barrier()
        q.put((rank, w.seed, red, buf.getvalue()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(2):
        r, seed, red, out = q.get(timeout=300)
        res[r] = (seed, red, out)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[0][0] != res[1][0]  # own seed per rank
    assert res[0][1] == res[1][1] == [2.0, 5.0, 0.5]  # max over ranks, on every rank
    line = json.loads(res[0][2].strip())
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert res[1][2].strip() == ""  # rank 1 prints nothing
