"""GPU checks of the bounded slot pool (moe_expert_pool_load): slot decisions equal the
oracle's LFU + recency simulation step by step (and its LRU / pure LFU variants for the
eviction ablation), missed blobs land byte-for-byte, the
pool-mode forward is bit-identical to the all-resident forward, and failures leave the
pool consistent."""
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import assert_close, forward, oracle_forward, ws_for
from int4_expert_gemv_router_b200 import abi, build

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build()


class Pool:
    def __init__(self, w, n_slots, layer=0):
        self.w = w
        self.L = synth.make_layer(w, layer, DEV)  # all-resident copy (reference path)
        self.host = self.L.pool.cpu().pin_memory()
        self.stride = self.L.pool.shape[1]
        self.dev = torch.zeros(n_slots, self.stride, dtype=torch.uint8, device=DEV)
        self.table = torch.empty(w.n_experts, dtype=torch.int32, device=DEV)
        self.n_slots = n_slots
        self.shape = abi.shape_of(w)
        self.h = abi.moe_pool_create(self.shape, n_slots, self.host, self.dev, self.table)

    def close(self):
        abi.moe_pool_destroy(self.h)


def _route(P, x):
    w = P.w
    T = x.shape[0]
    ws = ws_for(P.shape, T)
    idx = torch.empty(T, w.top_k, dtype=torch.int32, device=DEV)
    p = torch.empty(T, w.top_k, dtype=torch.float32, device=DEV)
    abi.moe_router_topk(P.shape, x, T, P.L.w_router, P.L.router_bias, idx, p, ws)
    return idx, p


@pytest.mark.parametrize("wname,steps,T", [("pool_int4", 48, 1), ("pool_int8", 32, 1), ("pool_int4", 12, 8)])
def test_pool_matches_oracle_cache_and_resident_forward(wname, steps, T):
    w = synth.WORKLOADS[wname]
    P = Pool(w, w.n_slots)
    sim = oracle.SlotCache(w.n_experts, w.n_slots)
    try:
        assert torch.all(P.table == -1)
        for s in range(steps):
            x = synth.activations(w, s, tokens=T, device=DEV)
            idx, p = _route(P, x)
            abi.moe_expert_pool_load(P.h, idx, T)
            sim.step(idx.cpu().numpy().reshape(-1).tolist())
            slot_of, expert_in = abi.moe_pool_slot_table(P.h, w.n_experts, w.n_slots)
            assert slot_of == sim.slot_of.tolist()
            assert expert_in == sim.expert_in.tolist()
            torch.cuda.synchronize()
            assert P.table.cpu().tolist() == slot_of
            # the selected experts' slots hold their blobs byte for byte
            for e in set(idx.cpu().numpy().reshape(-1).tolist()):
                assert torch.equal(P.dev[slot_of[e]].cpu(), P.host[e])
            out_pool, *_ = forward(w, P.L, x, residual=x, pool=P.dev, slot_table=P.table, n_slots=P.n_slots,
                                   topk=(idx, p))
            out_res, *_ = forward(w, P.L, x, residual=x, topk=(idx, p))
            assert torch.equal(out_pool, out_res)
        st = abi.moe_pool_stats(P.h)
        assert (st["lookups"], st["hits"], st["misses"], st["evictions"]) == (sim.lookups, sim.hits, sim.misses,
                                                                              sim.evictions)
        assert st["h2d_bytes"] == sim.misses * P.stride
        assert st["steps"] == steps
    finally:
        P.close()


@pytest.mark.parametrize("policy", ["lru", "lfu", "lfu_recency"])
def test_pool_policies_match_oracle(policy):
    """Eviction ablation: each policy's slot decisions equal the oracle's simulation of the
    same policy, step by step, on Zipf routing with a small pool (many evictions)."""
    w = synth.WORKLOADS["pool_int4"]
    n_slots = 24
    P = Pool(w, n_slots)
    sim = oracle.SlotCache(w.n_experts, n_slots, policy)
    try:
        abi.moe_pool_set_policy(P.h, policy)
        with pytest.raises(abi.MoeError):
            abi.lib()  # the binding maps names; an out-of-range code is rejected by the library
            abi._check(abi.lib().moe_pool_set_policy(P.h, 7))
        for s in range(40):
            x = synth.activations(w, 1000 + s, tokens=1, device=DEV)
            idx, _ = _route(P, x)
            abi.moe_expert_pool_load(P.h, idx, 1)
            sim.step(idx.cpu().numpy().reshape(-1).tolist())
            slot_of, expert_in = abi.moe_pool_slot_table(P.h, w.n_experts, n_slots)
            assert slot_of == sim.slot_of.tolist()
            assert expert_in == sim.expert_in.tolist()
        torch.cuda.synchronize()
        assert P.table.cpu().tolist() == slot_of
        st = abi.moe_pool_stats(P.h)
        assert (st["lookups"], st["hits"], st["misses"], st["evictions"]) == (sim.lookups, sim.hits, sim.misses,
                                                                              sim.evictions)
        assert sim.evictions > 0
    finally:
        P.close()


def test_pool_capacity_error_changes_nothing():
    w = synth.WORKLOADS["tiny"].with_(n_experts=16, top_k=4, seed=31)
    P = Pool(w, 3)
    try:
        x = synth.activations(w, 0, tokens=1, device=DEV)
        idx, _ = _route(P, x)
        with pytest.raises(abi.MoeError) as ei:
            abi.moe_expert_pool_load(P.h, idx, 1)
        assert ei.value.status == -3
        slot_of, expert_in = abi.moe_pool_slot_table(P.h, 16, 3)
        assert all(s == -1 for s in slot_of) and all(e == -1 for e in expert_in)
        assert abi.moe_pool_stats(P.h)["lookups"] == 0
    finally:
        P.close()


def test_pool_bad_id_rejected():
    w = synth.WORKLOADS["tiny"].with_(seed=32)
    P = Pool(w, 8)
    try:
        bad = torch.tensor([[3, 16]], dtype=torch.int32, device=DEV)
        with pytest.raises(abi.MoeError) as ei:
            abi.moe_expert_pool_load(P.h, bad, 1)
        assert ei.value.status == -1
    finally:
        P.close()


def test_pool_injected_copy_failure_leaves_consistent_state():
    w = synth.WORKLOADS["tiny"].with_(n_experts=16, top_k=2, seed=33)
    P = Pool(w, 4)
    try:
        ids = torch.tensor([[5, 9]], dtype=torch.int32, device=DEV)
        abi.moe_pool_inject_copy_failure(P.h, 1)  # the second copy fails
        with pytest.raises(abi.MoeError) as ei:
            abi.moe_expert_pool_load(P.h, ids, 1)
        assert ei.value.status == -2
        slot_of, expert_in = abi.moe_pool_slot_table(P.h, 16, 4)
        assert slot_of[5] == 0 and slot_of[9] == -1 and expert_in == [5, -1, -1, -1]
        torch.cuda.synchronize()
        assert P.table.cpu().tolist() == slot_of
        # retry succeeds and lands the blob
        abi.moe_expert_pool_load(P.h, ids, 1)
        slot_of, _ = abi.moe_pool_slot_table(P.h, 16, 4)
        assert slot_of[9] == 1
        torch.cuda.synchronize()
        assert torch.equal(P.dev[1].cpu(), P.host[9])
    finally:
        P.close()


@pytest.mark.parametrize("wname,steps,T", [("pool_int4", 24, 1), ("pool_int8", 12, 1), ("pool_int4", 8, 8)])
def test_pool_overlap_mode_bit_identical(wname, steps, T):
    """Overlap mode: the forward is enqueued right after the load, while the misses are still
    being copied; the fused kernel waits per expert for its pending slot-table entry.  Same
    slot decisions as the oracle, the table settles to the host mirror, no device error, and
    the output equals the all-resident forward bit for bit."""
    w = synth.WORKLOADS[wname]
    P = Pool(w, w.n_slots)
    sim = oracle.SlotCache(w.n_experts, w.n_slots)
    try:
        abi.moe_pool_set_overlap(P.h, True)
        for s in range(steps):
            x = synth.activations(w, 100 + s, tokens=T, device=DEV)
            idx, p = _route(P, x)
            abi.moe_expert_pool_load(P.h, idx, T)
            sim.step(idx.cpu().numpy().reshape(-1).tolist())
            out_pool, _, _, ws = forward(w, P.L, x, residual=x, pool=P.dev, slot_table=P.table,
                                         n_slots=P.n_slots, topk=(idx, p))
            assert abi.moe_ws_check(ws) == 0
            slot_of, expert_in = abi.moe_pool_slot_table(P.h, w.n_experts, w.n_slots)
            assert slot_of == sim.slot_of.tolist()
            assert expert_in == sim.expert_in.tolist()
            assert P.table.cpu().tolist() == slot_of  # every pending entry settled
            out_res, *_ = forward(w, P.L, x, residual=x, topk=(idx, p))
            assert torch.equal(out_pool, out_res)
        st = abi.moe_pool_stats(P.h)
        assert (st["lookups"], st["hits"], st["misses"]) == (sim.lookups, sim.hits, sim.misses)
        assert st["h2d_bytes"] == sim.misses * P.stride
    finally:
        P.close()


def test_pool_overlap_mode_needs_fused_shape():
    w = synth.WORKLOADS["tiny"].with_(hidden=384, inter=64, shared_inter=64)  # no fused kernel
    P = Pool(w, 8)
    try:
        with pytest.raises(abi.MoeError) as ei:
            abi.moe_pool_set_overlap(P.h, True)
        assert ei.value.status == -5  # MOE_ERR_UNSUPPORTED
        abi.moe_pool_set_overlap(P.h, False)
    finally:
        P.close()


def test_pool_many_token_step():
    """A many-token step through the pool: moe_router_topk and moe_expert_pool_load on 40
    tokens (more than the decode path's 8), then the many-token layer forward reading the
    experts through the slot table.  Slot decisions equal the oracle's, and the output matches
    both the all-resident forward and the oracle within tolerance (the many-token path sums
    its down products with atomics, so bits may differ in the last place)."""
    w = synth.WORKLOADS["tiny"].with_(n_experts=16, top_k=2, seed=34)
    n_slots = 12
    P = Pool(w, n_slots)
    sim = oracle.SlotCache(w.n_experts, n_slots)
    try:
        T = 40
        for s in range(3):
            x = synth.activations(w, 200 + s, tokens=T, device=DEV)
            # a router bias that keeps the step within the pool's 12 slots
            P.L.router_bias = torch.zeros(w.n_experts, dtype=torch.float32, device=DEV)
            P.L.router_bias[(s * 5 + torch.arange(6)) % w.n_experts] = 40.0
            idx, p = _route(P, x)
            abi.moe_expert_pool_load(P.h, idx, T)
            sim.step(idx.cpu().numpy().reshape(-1).tolist())
            slot_of, expert_in = abi.moe_pool_slot_table(P.h, w.n_experts, n_slots)
            assert slot_of == sim.slot_of.tolist() and expert_in == sim.expert_in.tolist()
            out_pool, _, _, ws = forward(w, P.L, x, residual=x, pool=P.dev, slot_table=P.table, n_slots=n_slots,
                                         topk=(idx, p))
            assert abi.moe_ws_check(ws) == 0
            out_res, *_ = forward(w, P.L, x, residual=x, topk=(idx, p))
            a, b = out_pool.float(), out_res.float()
            assert (a - b).abs().max().item() <= 1e-2 * b.abs().max().item() + 1e-3
            ref = oracle_forward(w, P.L, x, residual=x, idx=idx.cpu().numpy(), p=p.cpu().numpy().astype(np.float64))
            assert_close(out_pool, ref["out"])
    finally:
        P.close()


@pytest.mark.parametrize("wname,direct,overlap,T", [("pool_int4", True, False, 1), ("pool_int4", False, True, 1),
                                                    ("pool_int8", True, True, 8)])
def test_file_backed_pool(tmp_path, wname, direct, overlap, T):
    """The storage tier: misses read from a file of fixed-stride blobs (one pread per blob,
    O_DIRECT where the file system allows it) instead of pinned host memory.  Slot decisions
    equal the oracle's, slot bytes equal the file's, and the forward through the slots is
    bit-identical to the all-resident forward."""
    w = synth.WORKLOADS[wname]
    L = synth.make_layer(w, 0, DEV)
    path = str(tmp_path / "experts.blobs")
    L.pool.cpu().numpy().tofile(path)
    host = torch.from_numpy(np.fromfile(path, dtype=np.uint8).reshape(w.n_experts, -1))
    shape = abi.shape_of(w)
    dev = torch.zeros(w.n_slots, L.pool.shape[1], dtype=torch.uint8, device=DEV)
    table = torch.empty(w.n_experts, dtype=torch.int32, device=DEV)
    h = abi.moe_pool_create_file(shape, w.n_slots, path, dev, table, direct=direct)
    sim = oracle.SlotCache(w.n_experts, w.n_slots)
    try:
        if overlap:
            abi.moe_pool_set_overlap(h, True)
        for s in range(12):
            x = synth.activations(w, 300 + s, tokens=T, device=DEV)
            ws = ws_for(shape, T)
            idx = torch.empty(T, w.top_k, dtype=torch.int32, device=DEV)
            p = torch.empty(T, w.top_k, dtype=torch.float32, device=DEV)
            abi.moe_router_topk(shape, x, T, L.w_router, L.router_bias, idx, p, ws)
            abi.moe_expert_pool_load(h, idx, T)
            sim.step(idx.cpu().numpy().reshape(-1).tolist())
            out_pool, _, _, ws2 = forward(w, L, x, residual=x, pool=dev, slot_table=table, n_slots=w.n_slots,
                                          topk=(idx, p))
            assert abi.moe_ws_check(ws2) == 0
            slot_of, expert_in = abi.moe_pool_slot_table(h, w.n_experts, w.n_slots)
            assert slot_of == sim.slot_of.tolist() and expert_in == sim.expert_in.tolist()
            assert table.cpu().tolist() == slot_of
            for e in set(idx.cpu().numpy().reshape(-1).tolist()):
                assert torch.equal(dev[slot_of[e]].cpu(), host[e])
            out_res, *_ = forward(w, L, x, residual=x, topk=(idx, p))
            assert torch.equal(out_pool, out_res)
        st = abi.moe_pool_stats(h)
        assert (st["lookups"], st["hits"], st["misses"]) == (sim.lookups, sim.hits, sim.misses)
        assert st["h2d_bytes"] == sim.misses * L.pool.shape[1]
    finally:
        abi.moe_pool_destroy(h)


def test_file_backed_pool_read_errors(tmp_path):
    """A file too short for E blobs is refused at creation; a blob that cannot be read later
    (the file shrank) fails its load with MOE_ERR_IO and leaves its slot empty."""
    w = synth.WORKLOADS["tiny"].with_(n_experts=16, top_k=2, seed=35)
    L = synth.make_layer(w, 0, DEV)
    shape = abi.shape_of(w)
    stride = L.pool.shape[1]
    dev = torch.zeros(4, stride, dtype=torch.uint8, device=DEV)
    table = torch.empty(w.n_experts, dtype=torch.int32, device=DEV)
    short = str(tmp_path / "short.blobs")
    L.pool[:8].cpu().numpy().tofile(short)
    with pytest.raises(abi.MoeError) as ei:
        abi.moe_pool_create_file(shape, 4, short, dev, table)
    assert ei.value.status == -8
    path = str(tmp_path / "full.blobs")
    L.pool.cpu().numpy().tofile(path)
    h = abi.moe_pool_create_file(shape, 4, path, dev, table)
    try:
        abi.moe_expert_pool_load(h, torch.tensor([[1, 2]], dtype=torch.int32, device=DEV), 1)
        os.truncate(path, 10 * stride)  # experts 10.. can no longer be read
        with pytest.raises(abi.MoeError) as ei:
            abi.moe_expert_pool_load(h, torch.tensor([[3, 12]], dtype=torch.int32, device=DEV), 1)
        assert ei.value.status == -8
        slot_of, expert_in = abi.moe_pool_slot_table(h, 16, 4)
        assert slot_of[12] == -1 and slot_of[3] >= 0 and slot_of[1] >= 0 and slot_of[2] >= 0
        assert 12 not in expert_in
        torch.cuda.synchronize()
        assert table.cpu().tolist() == slot_of
        assert torch.equal(dev[slot_of[3]].cpu(), L.pool[3].cpu())
    finally:
        abi.moe_pool_destroy(h)
