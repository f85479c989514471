"""GPU checks of one expert-parallel rank's share of a layer (moe_layer_forward_partial) and
of the combine (moe_combine_partials), through the C ABI.  The ranks are run one after the
other on one GPU, each with its own pool shard and slot table (no kernel waits for another
rank), and their fp32 partials are summed by moe_combine_partials in rank order, which is
what an all-reduce followed by the combine computes.  Bar: routing identical on every rank
and equal to the single-GPU routing, the layer within the oracle tolerance, and with one rank
the partial path bit-identical to moe_layer_forward."""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import assert_close, assert_routing, forward, host_bits, oracle_forward, ws_for
from int4_expert_gemv_router_b200 import abi, build, ep

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build()


def _rank_partial(w, L, x, rank, world):
    shape = abi.shape_of(w)
    T = x.shape[0]
    pool = ep.shard_pool(L.pool, rank, world)
    table = ep.local_slot_table(w.n_experts, rank, world, DEV)
    part = torch.full((T, w.hidden), float("nan"), dtype=torch.float32, device=DEV)
    idx = torch.empty(T, w.top_k, dtype=torch.int32, device=DEV)
    p = torch.empty(T, w.top_k, dtype=torch.float32, device=DEV)
    ws = ws_for(shape, T)
    abi.moe_layer_forward_partial(shape, x, T, L.w_router, L.router_bias, None, None, pool, table, pool.shape[0],
                                  L.shared, L.w_sg, 1 if rank == 0 else 0, part, idx, p, ws)
    torch.cuda.synchronize()
    assert abi.moe_ws_check(ws) == 0  # remote experts raise no error bit
    return part, idx, p


@pytest.mark.parametrize("wname,world,T", [("tiny", 2, 4), ("tiny", 4, 1), ("decode80b", 2, 1),
                                           ("decode80b", 8, 1), ("decode35b", 4, 8)])
def test_ranks_sum_to_the_layer(wname, world, T):
    w = synth.WORKLOADS[wname].with_(layers=1)
    L = synth.make_layer(w, 0, DEV)
    x = synth.activations(w, 61, tokens=T, device=DEV)
    parts, ids = [], []
    for r in range(world):
        part, idx, p = _rank_partial(w, L, x, r, world)
        assert torch.isfinite(part).all()
        parts.append(part)
        ids.append((idx, p))
    for idx, p in ids[1:]:
        assert torch.equal(idx, ids[0][0]) and torch.equal(p, ids[0][1])
    out = torch.empty(T, w.hidden, dtype=torch.bfloat16, device=DEV)
    abi.moe_combine_partials(parts, T, w.hidden, x, out)
    torch.cuda.synchronize()
    ref = oracle_forward(w, L, x, residual=x)
    assert_routing(ids[0][0], ref["idx"], ref["logits"])
    assert_close(out, ref["out"])
    out1, idx1, _, _ = forward(w, L, x, residual=x)
    assert torch.equal(idx1, ids[0][0])


@pytest.mark.parametrize("wname,T", [("tiny", 3), ("decode80b", 1), ("decode35b", 8)])
def test_one_rank_partial_is_bit_identical(wname, T):
    w = synth.WORKLOADS[wname].with_(layers=1)
    L = synth.make_layer(w, 0, DEV)
    x = synth.activations(w, 62, tokens=T, device=DEV)
    part, idx, p = _rank_partial(w, L, x, 0, 1)
    out = torch.empty(T, w.hidden, dtype=torch.bfloat16, device=DEV)
    abi.moe_combine_partials([part], T, w.hidden, x, out)
    out_ref, idx_ref, p_ref, _ = forward(w, L, x, residual=x)
    assert torch.equal(idx, idx_ref) and torch.equal(p, p_ref)
    assert torch.equal(out, out_ref)


def test_combine_partials_order_and_tail():
    """The combine alone: a ragged element count (not a multiple of 4) and four partials."""
    T, H = 3, 70
    g = torch.Generator(device=DEV).manual_seed(5)
    parts = [torch.randn(T, H, device=DEV, generator=g) for _ in range(4)]
    res = torch.randn(T, H, device=DEV, generator=g).to(torch.bfloat16)
    out = torch.empty(T, H, dtype=torch.bfloat16, device=DEV)
    abi.moe_combine_partials(parts, T, H, res, out)
    torch.cuda.synchronize()
    ref = ((parts[0].double() + parts[1].double() + parts[2].double() + parts[3].double()) + res.double())
    assert (out.double() - ref).abs().max().item() <= 2 ** -8 * ref.abs().max().item()


def test_partial_rejects_unsupported():
    """A shape neither path takes (hidden 192: no fused decode instantiation, and the
    prefill GEMMs need hidden % 128 == 0), with one token and with many."""
    w = synth.WORKLOADS["tiny"].with_(hidden=192)
    shape = abi.shape_of(w)
    t = torch.zeros(1 << 16, dtype=torch.uint8, device=DEV)
    for T in (1, 9):
        with pytest.raises(abi.MoeError) as ei:
            abi.moe_layer_forward_partial(shape, t, T, t, None, None, None, t, t, 1, t, t, 1, t, None, None, t)
        assert ei.value.status == -5


@pytest.mark.parametrize("wname,world,T", [("tiny", 2, 40), ("decode80b", 2, 64), ("decode80b", 4, 300)])
def test_prefill_ranks_sum_to_the_layer(wname, world, T):
    """More than 8 tokens take the prefill path: each rank groups only the pairs of its own
    experts (the others' slot entries are -3) and runs the grouped GEMMs over them, the
    shared expert on rank 0; the fp32 partials summed by the combine give the layer."""
    w = synth.WORKLOADS[wname].with_(layers=1)
    L = synth.make_layer(w, 0, DEV)
    x = synth.activations(w, 63, tokens=T, device=DEV)
    parts, ids = [], []
    for r in range(world):
        part, idx, p = _rank_partial(w, L, x, r, world)
        assert torch.isfinite(part).all()
        parts.append(part)
        ids.append((idx, p))
    for idx, p in ids[1:]:
        assert torch.equal(idx, ids[0][0]) and torch.equal(p, ids[0][1])
    out = torch.empty(T, w.hidden, dtype=torch.bfloat16, device=DEV)
    abi.moe_combine_partials(parts, T, w.hidden, x, out)
    torch.cuda.synchronize()
    # the oracle with each selected expert decoded once for all its tokens
    xb, wrb = host_bits(x), host_bits(L.w_router)
    bias = None if L.router_bias is None else L.router_bias.cpu().numpy()
    logits = oracle.router_logits(xb, wrb, bias)
    ref_idx, ref_p = oracle.route(logits, w.top_k)
    assert_routing(ids[0][0], ref_idx, logits)
    pool = L.pool.cpu().numpy()
    ref = oracle.layer_forward_by_expert(xb, wrb, bias, w.top_k, lambda e: pool[e], L.shared.cpu().numpy(),
                                         host_bits(L.w_sg), w.hidden, w.inter, w.shared_inter, w.bits,
                                         residual_bits=xb, idx=ref_idx, p=ref_p)
    assert_close(out, ref["out"])
