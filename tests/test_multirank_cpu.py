"""The multi-process plumbing of bench.py on CPU (gloo, world size 2): one process per
rank, max over ranks of the per-rank time, barriers, disjoint per-rank token streams, and
the reference arm doing its work on rank 0 only.  The decode layer of one token stream has
no exchange step, so N ranks are N independent replicas (weak scaling) and nothing else
crosses ranks."""
import os
import socket
import sys

import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update({"RANK": str(rank), "LOCAL_RANK": str(rank), "WORLD_SIZE": str(world),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    import bench
    import synth
    import torch.distributed as dist
    r, ws = bench.init_dist("gloo")
    assert (r, ws) == (rank, world) and dist.is_initialized()
    dev = torch.device("cpu")
    # each rank's "step time" differs; every rank must see the max
    t = bench.reduce_max(1.5 + rank, dev)
    bench.barrier(dev)
    # ranks draw disjoint token streams of the same workload
    w = synth.WORKLOADS["tiny"]
    x = synth.activations(w, bench.rank_step_seed(rank, 0), tokens=2)
    gathered = [torch.empty_like(x) for _ in range(world)]
    dist.all_gather(gathered, x)
    distinct = not torch.equal(gathered[0], gathered[1])
    # the reference arm returns nothing on ranks other than 0 (they exit without work)
    ref_none = rank == 0 or bench.run_reference(bench.parse(["--impl", "reference"]), w, 2) is None
    dist.destroy_process_group()
    q.put((rank, t, distinct, ref_none))


def test_two_rank_plumbing_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[0] for r in res] == [0, 1]
    assert all(r[1] == 2.5 for r in res)  # max over ranks
    assert all(r[2] for r in res)         # disjoint token streams
    assert all(r[3] for r in res)         # reference arm: rank 1 returns None
