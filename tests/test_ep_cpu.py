"""Expert parallelism on CPU (gloo, world size 2): the partition of a layer's experts over
ranks and the all-reduce of the ranks' partial sums, with the fp64 oracle standing in for
each rank's kernels.  Each rank holds the experts e with e % world == rank (its pool shard,
slot e // world); rank 0 adds the shared expert; the summed partials plus the residual must
equal the one-rank layer.  (The GPU kernels of a rank's share are checked against the same
oracle in tests/test_gpu_ep.py.)"""
import os
import socket
import sys

import numpy as np
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _layer(w):
    import synth
    L = synth.make_layer(w, 0, "cpu")
    x = synth.activations(w, 3, tokens=w.tokens)
    bits = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)  # noqa: E731
    return L, x, bits


def _rank_partial(w, rank, world):
    """This rank's share, from its own pool shard and slot table (the oracle's primitives)."""
    import oracle
    from int4_expert_gemv_router_b200 import ep
    L, x, bits = _layer(w)
    pool = ep.shard_pool(L.pool, rank, world).numpy()
    table = ep.local_slot_table(w.n_experts, rank, world).numpy()
    b = None if L.router_bias is None else L.router_bias.numpy()
    logits = oracle.router_logits(bits(x), bits(L.w_router), b)
    idx, p = oracle.route(logits, w.top_k)  # every rank routes the same tokens
    xf = oracle.bf16_to_f64(bits(x))
    part = np.zeros((x.shape[0], w.hidden))
    for t in range(x.shape[0]):
        for j in range(w.top_k):
            slot = int(table[idx[t, j]])
            if slot == ep.SLOT_REMOTE:
                continue
            wts = oracle.read_expert(pool[slot], w.hidden, w.inter, w.bits)
            part[t] += p[t, j] * oracle.expert_forward(wts, xf[t])
    if rank == 0:
        gate = oracle.sigmoid(xf @ oracle.bf16_to_f64(bits(L.w_sg)))
        part += gate[:, None] * oracle.expert_forward(oracle.read_expert(L.shared.numpy(), w.hidden, w.shared_inter,
                                                                         w.bits), xf)
    return part, idx


def _worker(rank, world, port, q):
    os.environ.update({"RANK": str(rank), "LOCAL_RANK": str(rank), "WORLD_SIZE": str(world),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    import datetime
    import torch.distributed as dist
    import synth
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
    w = synth.WORKLOADS["tiny"].with_(router="zipf", seed=91)
    part, idx = _rank_partial(w, rank, world)
    t = torch.from_numpy(part)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    ids = torch.from_numpy(idx.astype(np.int64))
    gathered = [torch.empty_like(ids) for _ in range(world)]
    dist.all_gather(gathered, ids)
    dist.destroy_process_group()
    q.put((rank, t.numpy(), all(torch.equal(g, ids) for g in gathered)))


def test_partition_covers_every_expert_once():
    from int4_expert_gemv_router_b200 import ep
    for E, world in ((16, 2), (512, 8), (13, 4), (3, 4)):
        owners = [[r for r in range(world) if ep.local_slot_table(E, r, world)[e] >= 0] for e in range(E)]
        assert all(len(o) == 1 for o in owners)
        for r in range(world):
            table = ep.local_slot_table(E, r, world)
            mine = ep.local_experts(E, r, world)
            assert [int(table[e]) for e in mine] == list(range(len(mine)))
            assert all(ep.owner(e, world) == r for e in mine)
        pool = torch.arange(E).reshape(E, 1)
        for r in range(world):
            assert ep.shard_pool(pool, r, world).reshape(-1).tolist() == ep.local_experts(E, r, world)


def test_two_rank_partials_sum_to_the_layer():
    import oracle
    import synth
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=240) for _ in procs), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert all(r[2] for r in res)  # the ranks routed identically
    summed = res[0][1]
    assert np.array_equal(summed, res[1][1])  # the all-reduce leaves the same sum on both
    w = synth.WORKLOADS["tiny"].with_(router="zipf", seed=91)
    L, x, bits = _layer(w)
    ref = oracle.layer_forward(bits(x), bits(L.w_router), L.router_bias.numpy(), w.top_k,
                               lambda e: L.pool[e].numpy(), L.shared.numpy(), bits(L.w_sg), w.hidden, w.inter,
                               w.shared_inter, w.bits, residual_bits=bits(x))
    got = summed + oracle.bf16_to_f64(bits(x))
    assert np.allclose(got, ref["out"], rtol=1e-12, atol=1e-12)
