"""The multi-rank path on CPU (gloo, world size 2): the max-over-ranks timing
reduction of the bench, and the head decomposition of one call -- oracle
results of each rank's head shard equal the slices of the full run (heads are
independent problems, so the split needs no data exchange)."""
import json
import multiprocessing as mp
import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SHAPE = (2, 3, 64, 3, 9, 13)  # B, H, d, F, Hv, Wv: 6 (batch, head) units


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
        from oracle import oracle as O
        from video_dit_sparse_da2_b200.inputs import make_qkv
        from video_dit_sparse_da2_b200.sharding import head_shard

        vals = torch.tensor([1.0 + rank, 10.0 - rank, 3.0], dtype=torch.float64)
        red = bench.max_over_ranks(vals, world).tolist()

        B, H, d, F, Hv, Wv = SHAPE
        q, k, v = make_qkv(B, H, F * Hv * Wv, d, 0)
        lo, hi = head_shard(B * H, world, rank)
        # flatten (batch, head) units, take this rank's shard as a batch of units
        sl = lambda t: t.reshape(B * H, 1, *t.shape[2:])[lo:hi].reshape(1, hi - lo, *t.shape[2:])
        prep, A, plan, out = O.run(sl(q), sl(k), sl(v), F, Hv, Wv, 2500, 2500, 0.2)
        np.savez(os.path.join(outdir, f"rank{rank}.npz"), out=out, prec=plan.prec, cnt=plan.cnt, lo=lo, hi=hi)
        with open(os.path.join(outdir, f"rank{rank}.json"), "w") as f:
            json.dump({"red": red}, f)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_gloo(tmp_path):
    from oracle import oracle as O
    from video_dit_sparse_da2_b200.inputs import make_qkv

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

    B, H, d, F, Hv, Wv = SHAPE
    q, k, v = make_qkv(B, H, F * Hv * Wv, d, 0)
    _, _, plan, out = O.run(q, k, v, F, Hv, Wv, 2500, 2500, 0.2)
    out_u = out.reshape(B * H, *out.shape[2:])
    prec_u = plan.prec.reshape(B * H, *plan.prec.shape[2:])
    cnt_u = plan.cnt.reshape(2, B * H, -1)
    covered = []
    for r in range(world):
        z = np.load(tmp_path / f"rank{r}.npz")
        lo, hi = int(z["lo"]), int(z["hi"])
        covered += list(range(lo, hi))
        assert np.array_equal(z["out"].reshape(hi - lo, *out.shape[2:]), out_u[lo:hi])
        assert np.array_equal(z["prec"].reshape(hi - lo, *plan.prec.shape[2:]), prec_u[lo:hi])
        assert np.array_equal(z["cnt"].reshape(2, hi - lo, -1), cnt_u[:, lo:hi])
    assert covered == list(range(B * H))


@pytest.mark.parametrize("n,world", [(6, 2), (7, 3), (2, 4), (0, 2)])
def test_head_shard_partition(n, world):
    from video_dit_sparse_da2_b200.sharding import head_shard
    ranges = [head_shard(n, world, r) for r in range(world)]
    assert ranges[0][0] == 0 and ranges[-1][1] == n
    assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
    sizes = [hi - lo for lo, hi in ranges]
    assert max(sizes) - min(sizes) <= 1
