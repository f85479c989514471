"""GPU parity on the method's edge cases, against the fp64 oracle through the C ABI:

* every logit equal (an all-zero router): the selection is experts 0..k-1 with weights 1/k
  (the tie rule of the router: larger logit first, ties to the lower expert id), which drives
  the decode top-k past its 64-candidate fast path and the many-token router past its
  96-candidate certified path into their exact fallbacks;
* an exact two-way tie at the k-th place: the lower id is selected;
* logits that differ by less than the fp32 router's rounding (half an ulp): the exact order
  decides, through both routers;
* the int8 layer at the full 80B-like width (hidden 2048, 512 experts, top-10), whose fused
  decode kernel no smaller case instantiates;
* the router alone on many tokens (4096 on the prefill shape, and a shape the tensor-core
  router does not cover, routed eight tokens at a time);
* a bounded device wait that runs out: a slot-table entry left pending with nothing to settle
  it ends in MOE_DEVERR_TIMEOUT | MOE_DEVERR_BAD_SLOT, the expert is skipped and the rest of
  the layer still matches the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import assert_close, assert_routing, forward, host_bits, oracle_forward, ws_for
from int4_expert_gemv_router_b200 import abi, build

pytestmark = pytest.mark.gpu
DEV = "cuda"
TINY = synth.WORKLOADS["tiny"]


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build()


def _layer_80b_shape(bits=4, seed=71):
    w = synth.WORKLOADS["decode80b"].with_(bits=bits, seed=seed, layers=1)
    return w, synth.make_layer(w, 0, DEV)


@pytest.mark.parametrize("T", [1, 8, 64])
def test_all_equal_logits_pick_lowest_ids(T):
    """Zero router weights, no bias: every logit is 0, so ids 0..k-1 in order and p = 1/k.
    T = 1 and 8 run the fused decode kernel (more than 64 keys at the threshold: k rounds of
    warp arg-max); T = 64 runs the many-token router (more than 96 candidates within the fp32
    bound: every logit recomputed exactly)."""
    w, L = _layer_80b_shape()
    L.w_router.zero_()
    L.router_bias = None
    x = synth.activations(w, 5, tokens=T, device=DEV)
    out, idx, p, ws = forward(w, L, x, residual=x)
    assert abi.moe_ws_check(ws) == 0
    want = np.tile(np.arange(w.top_k, dtype=np.int32), (T, 1))
    assert np.array_equal(idx.cpu().numpy(), want)
    assert np.allclose(p.cpu().numpy(), 1.0 / w.top_k, rtol=1e-7, atol=0)
    ref = oracle_forward(w, L, x, residual=x)
    assert np.array_equal(ref["idx"], want)  # the oracle's own closed form
    assert_close(out, ref["out"])


@pytest.mark.parametrize("T", [1, 16])
def test_exact_tie_at_kth_place_goes_to_lower_id(T):
    """Token 0's k-th and (k+1)-th experts get identical router rows, so their logits are
    equal whatever x is; the lower of the two ids must be selected (fused decode kernel at
    T = 1, many-token router at T = 16)."""
    w, L = _layer_80b_shape(seed=72)
    L.router_bias = None
    x = synth.activations(w, 6, tokens=T, device=DEV)
    logits = oracle.router_logits(host_bits(x), host_bits(L.w_router), None)
    order = np.lexsort((np.arange(w.n_experts), -logits[0]))
    c, d = int(order[w.top_k - 1]), int(order[w.top_k])
    L.w_router[d] = L.w_router[c]
    ref = oracle_forward(w, L, x, residual=x)
    assert ref["logits"][0, c] == ref["logits"][0, d]
    assert min(c, d) in ref["idx"][0].tolist() and max(c, d) not in ref["idx"][0].tolist()
    out, idx, p, ws = forward(w, L, x, residual=x)
    assert abi.moe_ws_check(ws) == 0
    assert np.array_equal(idx.cpu().numpy(), ref["idx"])
    assert np.allclose(p.cpu().numpy(), ref["p"], rtol=2e-6, atol=1e-7)
    assert_close(out, ref["out"])


def test_many_near_equal_candidates_take_the_exact_fallback():
    """Token 0's best router row copied to 200 rows, each copy nudged by one bf16 ulp in a
    column of its own: their logits differ by far less than the fp32 error bound, so token 0
    has more than 96 candidates and the many-token router takes its fallback (every expert's
    exact value, skipped by the certified bound once k are kept).  Ids must be the oracle's
    fp64 selection."""
    w, L = _layer_80b_shape(seed=73)
    L.router_bias = None
    T = 16
    x = synth.activations(w, 7, tokens=T, device=DEV)
    logits = oracle.router_logits(host_bits(x), host_bits(L.w_router), None)
    best = int(np.argmax(logits[0]))
    base = L.w_router[best].clone().view(torch.int16)
    others = [e for e in range(w.n_experts) if e != best][:199]
    for j, e in enumerate(others):
        r = base.clone()
        r[(37 * j) % w.hidden] += 1  # the next bf16 away from zero
        L.w_router[e] = r.view(torch.bfloat16)
    ref = oracle_forward(w, L, x, residual=x)
    near = np.abs(ref["logits"][0, others + [best]] - ref["logits"][0, best])
    assert near.max() < 1e-2 and np.unique(ref["logits"][0, others]).size > 150  # near-equal, mostly distinct
    out, idx, p, ws = forward(w, L, x, residual=x)
    assert abi.moe_ws_check(ws) == 0
    assert_routing(idx, ref["idx"], ref["logits"])
    assert np.allclose(p.cpu().numpy(), ref["p"], rtol=2e-6, atol=1e-7)
    assert_close(out, ref["out"])


@pytest.mark.parametrize("T", [1, 8])
def test_int8_full_width_layer(T):
    """The int8 layer of the bounded-pool workload's shape (hidden 2048, inter 512, 512
    experts, top-10), all experts resident, against the oracle."""
    w = synth.WORKLOADS["pool_int8"]
    L = synth.make_layer(w, 0, DEV)
    x = synth.activations(w, 40 + T, tokens=T, device=DEV)
    out, idx, p, ws = forward(w, L, x, residual=x)
    assert abi.moe_ws_check(ws) == 0
    ref = oracle_forward(w, L, x, residual=x)
    assert_routing(idx, ref["idx"], ref["logits"])
    assert np.allclose(p.cpu().numpy(), ref["p"], rtol=2e-6, atol=1e-7)
    assert_close(out, ref["out"])


def test_router_topk_many_tokens_prefill_shape():
    """moe_router_topk on the prefill workload's 4096 tokens: certified tensor-core routing,
    ids bit-exact against the oracle's selection, weights within 2e-6."""
    w = synth.WORKLOADS["prefill"]
    wr, bias, _ = synth.router_weights(w, 0, DEV)
    T = w.tokens
    x = synth.activations(w, 77, tokens=T, device=DEV)
    shape = abi.shape_of(w)
    ws = ws_for(shape, T)
    idx = torch.full((T, w.top_k), -7, dtype=torch.int32, device=DEV)
    p = torch.full((T, w.top_k), -7.0, dtype=torch.float32, device=DEV)
    abi.moe_router_topk(shape, x, T, wr, bias, idx, p, ws)
    torch.cuda.synchronize()
    assert abi.moe_ws_check(ws) == 0
    logits = oracle.router_logits(host_bits(x), host_bits(wr), None if bias is None else bias.cpu().numpy())
    ref_idx, ref_p = oracle.route(logits, w.top_k)
    assert_routing(idx, ref_idx, logits)
    assert np.allclose(p.cpu().numpy(), ref_p, rtol=2e-6, atol=1e-7)


@pytest.mark.parametrize("T", [4, 16])
def test_router_orders_logits_fp32_cannot_tell_apart(T):
    """Every expert has the same router row except coordinate 0, where expert e has
    (e + 1) * 2^-10, and every token has x_0 = 2^-18: the logits (0.05 to 0.55 here) differ
    only by (e + 1) * 2^-28, below the resolution of an fp32 sum (a sequential fp32 sum gives
    3 to 17 distinct values for the 64 experts), while the exact sums order them.  The router
    must select the k highest ids in decreasing order (T = 4: the fused decode router;
    T = 16: the many-token certified router, whose candidates are then every expert)."""
    w = TINY.with_(n_experts=64, top_k=4, seed=79)
    wr, _, _ = synth.router_weights(w, 0, DEV)
    base = wr[0].clone()
    wr = base.repeat(w.n_experts, 1)
    wr[:, 0] = ((torch.arange(w.n_experts, dtype=torch.float32) + 1) * 2.0 ** -10).to(torch.bfloat16).to(DEV)
    x = synth.activations(w, 79, tokens=T, device=DEV)
    x[:, 0] = 2.0 ** -18
    shape = abi.shape_of(w)
    ws = ws_for(shape, T)
    idx = torch.full((T, w.top_k), -7, dtype=torch.int32, device=DEV)
    p = torch.full((T, w.top_k), -7.0, dtype=torch.float32, device=DEV)
    abi.moe_router_topk(shape, x, T, wr, None, idx, p, ws)
    torch.cuda.synchronize()
    assert abi.moe_ws_check(ws) == 0
    logits = oracle.router_logits(host_bits(x), host_bits(wr), None)
    ref_idx, ref_p = oracle.route(logits, w.top_k)
    want = np.tile(np.arange(w.n_experts - 1, w.n_experts - 1 - w.top_k, -1, dtype=np.int32), (T, 1))
    assert np.array_equal(ref_idx, want)  # the construction does what it says
    assert np.array_equal(idx.cpu().numpy(), want)
    assert np.allclose(p.cpu().numpy(), ref_p, rtol=2e-6, atol=1e-7)


def test_router_topk_many_tokens_in_groups_of_eight():
    """A shape outside the tensor-core router (E > 512) routes any T in groups of 8."""
    w = TINY.with_(n_experts=600, top_k=6, seed=73, router="zipf")
    wr, bias, _ = synth.router_weights(w, 0, DEV)
    T = 21
    x = synth.activations(w, 78, tokens=T, device=DEV)
    shape = abi.shape_of(w)
    ws = ws_for(shape, T)
    idx = torch.full((T, w.top_k), -7, dtype=torch.int32, device=DEV)
    p = torch.full((T, w.top_k), -7.0, dtype=torch.float32, device=DEV)
    abi.moe_router_topk(shape, x, T, wr, bias, idx, p, ws)
    torch.cuda.synchronize()
    logits = oracle.router_logits(host_bits(x), host_bits(wr), bias.cpu().numpy())
    ref_idx, ref_p = oracle.route(logits, w.top_k)
    assert_routing(idx, ref_idx, logits)
    assert np.allclose(p.cpu().numpy(), ref_p, rtol=2e-6, atol=1e-7)


@pytest.mark.parametrize("T", [1, 3])
def test_pending_slot_wait_runs_out(T):
    """Failure detection by a bounded device wait: one selected expert's slot-table entry is
    left pending (-2, what a pool in overlap mode writes until the blob has landed) and nothing
    ever settles it.  With the wait bound set to 1 ms the kernel gives up on that expert, flags
    TIMEOUT and BAD_SLOT, and finishes the layer without it; the output equals the oracle's
    with that expert's weight set to zero.  The workspace then serves a normal call again."""
    w = synth.WORKLOADS["decode80b"].with_(layers=1, seed=74)
    L = synth.make_layer(w, 0, DEV)
    x = synth.activations(w, 9, tokens=T, device=DEV)
    _, idx, p, _ = forward(w, L, x, residual=x)
    lost = int(idx[0, 0].item())
    table = torch.arange(w.n_experts, dtype=torch.int32, device=DEV)
    table[lost] = -2
    shape = abi.shape_of(w)
    ws = ws_for(shape, T)
    abi.moe_ws_set_slot_wait(ws, 1000)
    out, _, _, _ = forward(w, L, x, residual=x, slot_table=table, ws=ws, topk=(idx, p))
    flags = abi.moe_ws_check(ws)
    assert flags == abi.DEVERR_TIMEOUT | abi.DEVERR_BAD_SLOT, hex(flags)
    ih, ph = idx.cpu().numpy(), p.cpu().numpy()
    ref = oracle_forward(w, L, x, residual=x, idx=ih, p=np.where(ih == lost, 0.0, ph))
    assert_close(out, ref["out"])
    # the setting stays with the workspace; restored to the default, a normal call is clean
    abi.moe_ws_set_slot_wait(ws, 0)
    out2, idx2, _, _ = forward(w, L, x, residual=x, ws=ws)
    assert abi.moe_ws_check(ws) == 0
    assert torch.equal(idx2, idx)
    ref2 = oracle_forward(w, L, x, residual=x)
    assert_close(out2, ref2["out"])
