"""GPU parity of the decode path (moe_layer_forward / moe_router_topk through the C ABI)
against the fp64 oracle on the same seeded inputs.

Bar: top-k ids bit-exact (ties at fp64 precision excepted and checked), routing weights
within fp32 rounding, outputs within max|diff| <= 1e-2 * max|ref| + 1e-3.
"""
import numpy as np
import pytest
import torch

import synth
from helpers import (assert_close, assert_routing, forward, host_bits, oracle_forward, ws_for)
from int4_expert_gemv_router_b200 import abi, build

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build()


TINY = synth.WORKLOADS["tiny"]

# (name, workload overrides, T): span several tiles and ragged tails of every kernel.
CASES = [
    ("tiny", {}, 4),
    ("tiny_int8", dict(bits=8), 4),
    ("tiny_T1", {}, 1),
    ("tiny_T8_bias", dict(router="zipf"), 8),
    ("E33_k5", dict(hidden=512, inter=128, shared_inter=128, n_experts=33, top_k=5, seed=11), 3),
    ("k_eq_E", dict(n_experts=8, top_k=8, seed=12), 5),
    ("k1", dict(top_k=1, seed=13), 6),
    ("E1_k1", dict(n_experts=1, top_k=1, seed=14), 2),
    ("H1024_int8_T8", dict(hidden=1024, inter=256, shared_inter=256, n_experts=64, top_k=8, bits=8, seed=15), 8),
    ("H4096_I1024", dict(hidden=4096, inter=1024, shared_inter=1024, n_experts=20, top_k=4, seed=16), 2),
    ("k32", dict(n_experts=64, top_k=32, seed=17), 2),
    ("E1024", dict(n_experts=1024, top_k=16, seed=18), 2),
]


@pytest.mark.parametrize("name,over,T", CASES, ids=[c[0] for c in CASES])
def test_layer_parity(name, over, T):
    w = TINY.with_(**over)
    L = synth.make_layer(w, 0, DEV)
    x = synth.activations(w, 0, tokens=T, device=DEV)
    res = synth.activations(w, 1, tokens=T, device=DEV)
    out, idx, p, ws = forward(w, L, x, residual=res)
    ref = oracle_forward(w, L, x, residual=res)
    assert_routing(idx, ref["idx"], ref["logits"])
    assert np.allclose(p.cpu().numpy(), ref["p"], rtol=2e-6, atol=1e-7)
    assert np.allclose(p.sum(1).cpu().numpy(), 1.0, atol=1e-5)
    assert_close(out, ref["out"])
    assert abi.moe_ws_check(ws) == 0


@pytest.mark.parametrize("wname,T,layers", [("decode80b", 1, (0, 47)), ("decode35b", 1, (0,)),
                                            ("decode35b", 4, (39,)), ("decode35b", 8, (5,))])
def test_full_size_layer_parity(wname, T, layers):
    w = synth.WORKLOADS[wname]
    for l in layers:
        L = synth.make_layer(w, l, DEV)
        x = synth.activations(w, 1000 + l, tokens=T, device=DEV)
        out, idx, p, ws = forward(w, L, x, residual=x)
        ref = oracle_forward(w, L, x, residual=x)
        assert_routing(idx, ref["idx"], ref["logits"])
        assert np.allclose(p.cpu().numpy(), ref["p"], rtol=2e-6, atol=1e-7)
        assert_close(out, ref["out"])
        assert abi.moe_ws_check(ws) == 0
        del L
        torch.cuda.empty_cache()


def test_stacked_layers_chain_80b():
    """Three chained 80B-like layers as the benchmark chains them (input of layer l+1 =
    bf16(x_0 + moe_l(x_l))); each layer is checked against the oracle on the GPU's own x_l,
    so rounding does not compound into routing flips."""
    w = synth.WORKLOADS["decode80b"]
    x0 = synth.activations(w, 7, device=DEV)
    x = x0
    for l in range(3):
        L = synth.make_layer(w, l, DEV)
        out, idx, p, ws = forward(w, L, x, residual=x0)
        ref = oracle_forward(w, L, x, residual=x0)
        assert_routing(idx, ref["idx"], ref["logits"])
        assert_close(out, ref["out"])
        x = out
        del L
        torch.cuda.empty_cache()


def test_precomputed_topk_is_bit_identical():
    w = TINY.with_(router="zipf", seed=21)
    L = synth.make_layer(w, 0, DEV)
    x = synth.activations(w, 0, tokens=5, device=DEV)
    out1, idx, p, _ = forward(w, L, x, residual=x)
    out2, _, _, _ = forward(w, L, x, residual=x, topk=(idx.clone(), p.clone()))
    assert torch.equal(out1, out2)


def test_router_only_matches_layer_routing():
    w = synth.WORKLOADS["decode80b"]
    L = synth.make_layer(w, 3, DEV)
    x = synth.activations(w, 3, device=DEV)
    shape = abi.shape_of(w)
    ws = ws_for(shape, 1)
    idx = torch.empty(1, w.top_k, dtype=torch.int32, device=DEV)
    p = torch.empty(1, w.top_k, dtype=torch.float32, device=DEV)
    abi.moe_router_topk(shape, x, 1, L.w_router, L.router_bias, idx, p, ws)
    _, idx2, p2, _ = forward(w, L, x)
    assert torch.equal(idx, idx2) and torch.equal(p, p2)


def test_slot_permutation_is_bit_identical_and_deterministic():
    """Experts read through a permuted slot table give the same bits (pool-mode invariant)."""
    w = TINY.with_(n_experts=16, top_k=3, seed=22)
    L = synth.make_layer(w, 0, DEV)
    x = synth.activations(w, 0, tokens=4, device=DEV)
    out1, *_ = forward(w, L, x, residual=x)
    out1b, *_ = forward(w, L, x, residual=x)
    assert torch.equal(out1, out1b)
    perm = torch.randperm(16, generator=torch.Generator().manual_seed(0))
    n_slots = 20
    pool2 = torch.zeros(n_slots, L.pool.shape[1], dtype=torch.uint8, device=DEV)
    slot_of = perm + 3  # expert e lives in slot perm[e] + 3
    pool2[slot_of.to(DEV).long()] = L.pool
    out2, *_ = forward(w, L, x, residual=x, pool=pool2, slot_table=slot_of.to(torch.int32).to(DEV), n_slots=n_slots)
    assert torch.equal(out1, out2)


def test_device_error_flags():
    w = TINY.with_(seed=23)
    L = synth.make_layer(w, 0, DEV)
    x = synth.activations(w, 0, tokens=2, device=DEV)
    # a selected expert's slot out of range -> BAD_SLOT, no fault
    _, idx, p, _ = forward(w, L, x)
    st = torch.arange(w.n_experts, dtype=torch.int32, device=DEV)
    st[idx[0, 0].item()] = 10_000
    _, _, _, ws = forward(w, L, x, slot_table=st)
    assert abi.moe_ws_check(ws) & abi.DEVERR_BAD_SLOT
    assert abi.moe_ws_check(ws) == 0  # cleared by the read
    # a caller-given id out of range -> BAD_EXPERT, the pair is skipped
    bad = idx.clone()
    bad[1, 1] = w.n_experts + 5
    out, _, _, ws = forward(w, L, x, topk=(bad, p))
    assert abi.moe_ws_check(ws) & abi.DEVERR_BAD_EXPERT
    ref = oracle_forward(w, L, x, idx=np.where(bad.cpu().numpy() < w.n_experts, bad.cpu().numpy(), 0),
                         p=np.where(bad.cpu().numpy() < w.n_experts, p.cpu().numpy(), 0.0))
    assert_close(out, ref["out"])


def test_stack_forward_equals_layer_by_layer():
    """moe_stack_forward (one launch for the stack) gives the same bits as one
    moe_layer_forward per layer, and each layer matches the oracle on its own input."""
    w = synth.WORKLOADS["decode80b"].with_(layers=3)
    T = 1
    layers = [synth.make_layer(w, l, DEV) for l in range(3)]
    shape = abi.shape_of(w)
    x0 = synth.activations(w, 11, tokens=T, device=DEV)
    bufs = [x0] + [torch.empty(T, w.hidden, dtype=torch.bfloat16, device=DEV) for _ in range(3)]
    idx = [torch.empty(T, w.top_k, dtype=torch.int32, device=DEV) for _ in range(3)]
    p = [torch.empty(T, w.top_k, dtype=torch.float32, device=DEV) for _ in range(3)]
    slots = torch.arange(w.n_experts, dtype=torch.int32, device=DEV)
    descs = [abi.layer_desc(x=bufs[l] if l == 0 else None, w_router=L.w_router, router_bias=L.router_bias,
                            pool=L.pool, slot_table=slots, n_slots=w.n_experts, shared_blob=L.shared,
                            w_shared_gate=L.w_sg, residual=x0, out=bufs[l + 1], topk_idx_out=idx[l],
                            topk_w_out=p[l]) for l, L in enumerate(layers)]
    ws = ws_for(shape, T)
    abi.moe_stack_forward(shape, T, descs, ws)
    torch.cuda.synchronize()
    assert abi.moe_ws_check(ws) == 0
    x = x0
    for l, L in enumerate(layers):
        out, i2, p2, _ = forward(w, L, x, residual=x0)
        assert torch.equal(out, bufs[l + 1]) and torch.equal(i2, idx[l]) and torch.equal(p2, p[l])
        ref = oracle_forward(w, L, x, residual=x0)
        assert_routing(idx[l], ref["idx"], ref["logits"])
        assert_close(bufs[l + 1], ref["out"])
        x = bufs[l + 1]


@pytest.mark.parametrize("T", [1, 3, 8])
def test_stack_forward_unfused_shape_falls_back(T):
    """A shape without a fused kernel (E > 512) runs layer by layer with the same results."""
    w = TINY.with_(n_experts=600, top_k=6, seed=41, layers=2)
    layers = [synth.make_layer(w, l, DEV) for l in range(2)]
    shape = abi.shape_of(w)
    x0 = synth.activations(w, 12, tokens=T, device=DEV)
    outs = [torch.empty(T, w.hidden, dtype=torch.bfloat16, device=DEV) for _ in range(2)]
    slots = torch.arange(w.n_experts, dtype=torch.int32, device=DEV)
    descs = [abi.layer_desc(x=x0 if l == 0 else None, w_router=L.w_router, router_bias=L.router_bias, pool=L.pool,
                            slot_table=slots, n_slots=w.n_experts, shared_blob=L.shared, w_shared_gate=L.w_sg,
                            residual=None, out=outs[l]) for l, L in enumerate(layers)]
    ws = ws_for(shape, T)
    abi.moe_stack_forward(shape, T, descs, ws)
    torch.cuda.synchronize()
    x = x0
    for l, L in enumerate(layers):
        ref = oracle_forward(w, L, x)
        assert_close(outs[l], ref["out"])
        x = outs[l]
