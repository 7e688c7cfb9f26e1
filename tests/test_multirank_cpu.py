"""The bench's multi-process path on CPU (gloo, world size 2).  With N > 1
processes every rank runs its own independent call (replicas, no data-path
collective); the only cross-rank step is the max-over-ranks reduction of the
timings, which this test checks."""
import json
import multiprocessing as mp
import os
import socket
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, outdir):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import torch
    import torch.distributed as dist

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench

        vals = torch.tensor([1.0 + rank, 10.0 - rank, 3.0], dtype=torch.float64)
        red = bench.max_over_ranks(vals, world).tolist()
        with open(os.path.join(outdir, f"rank{rank}.json"), "w") as f:
            json.dump({"red": red}, f)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_gloo_max_over_ranks(tmp_path):
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_worker, args=(r, world, port, str(tmp_path))) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    for r in range(world):
        with open(tmp_path / f"rank{r}.json") as f:
            assert json.load(f)["red"] == [2.0, 10.0, 3.0]
