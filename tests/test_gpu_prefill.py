"""GPU parity of the many-token (prefill) path against the fp64 oracle: certified routing
(ids bit-exact), stable grouping by expert (bit-exact), tcgen05 grouped GEMMs on bf16-
dequantised weights (outputs within max|diff| <= 1e-2 * max|ref| + 1e-3), and agreement
of each token's prefill output with its one-token decode output."""
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


def _group(w, idx):
    shape = abi.shape_of(w)
    T = idx.shape[0]
    order = torch.full((T * w.top_k,), -1, dtype=torch.int32, device=DEV)
    offsets = torch.full((w.n_experts + 1,), -1, dtype=torch.int32, device=DEV)
    ws = ws_for(shape, T)
    abi.moe_group_pairs(shape, T, idx, order, offsets, ws)
    torch.cuda.synchronize()
    return order.cpu().numpy(), offsets.cpu().numpy(), ws


@pytest.mark.parametrize("E,k,T", [(16, 2, 5), (512, 10, 4096), (64, 8, 333), (7, 7, 40), (512, 1, 1)])
def test_group_pairs_bit_exact(E, k, T):
    g = torch.Generator().manual_seed(E * 31 + T)
    # skewed: low ids much more likely, so some experts get far more than 256 pairs
    idx = torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(T)])
    idx = torch.where(torch.rand(T, k, generator=g) < 0.3, idx % 3, idx)
    # keep ids distinct per token
    for t in range(T):
        seen = set()
        for j in range(k):
            e = int(idx[t, j])
            while e in seen:
                e = (e + 1) % E
            idx[t, j] = e
            seen.add(e)
    w = TINY.with_(n_experts=E, top_k=k)
    order, offsets, ws = _group(w, idx.to(torch.int32).to(DEV))
    _, ref_off, ref_order = oracle.group_pairs(idx.numpy(), E)
    assert np.array_equal(offsets, ref_off)
    assert np.array_equal(order, ref_order)
    assert abi.moe_ws_check(ws) == 0


def test_group_pairs_flags_bad_ids():
    w = TINY.with_(n_experts=16, top_k=2)
    idx = torch.tensor([[3, 16], [-1, 3], [5, 3]], dtype=torch.int32, device=DEV)
    order, offsets, ws = _group(w, idx)
    assert abi.moe_ws_check(ws) & abi.DEVERR_BAD_EXPERT
    assert offsets[-1] == 4  # the two bad pairs are left out
    assert order[:4].tolist() == [0, 3, 5, 4]  # expert 3: pairs 0, 3, 5; expert 5: pair 4


PREFILL_CASES = [
    ("tiny_T40", dict(seed=51), 40),
    ("tiny_T9_int8", dict(bits=8, seed=52), 9),
    ("H2048_E64_T300", dict(hidden=2048, inter=512, shared_inter=512, n_experts=64, top_k=4, seed=53), 300),
    ("H2048_E32_T520_int8", dict(hidden=2048, inter=512, shared_inter=512, n_experts=32, top_k=6, bits=8,
                                 seed=54, router="zipf"), 520),
    ("H512_E20_T64", dict(hidden=512, inter=128, shared_inter=128, n_experts=20, top_k=3, seed=55), 64),
]


@pytest.mark.parametrize("name,over,T", PREFILL_CASES, ids=[c[0] for c in PREFILL_CASES])
def test_prefill_layer_parity(name, over, T):
    w = TINY.with_(**over)
    L = synth.make_layer(w, 0, DEV)
    x = synth.activations(w, 3, tokens=T, device=DEV)
    res = synth.activations(w, 4, tokens=T, device=DEV)
    out, idx, p, ws = forward(w, L, x, residual=res)
    assert abi.moe_ws_check(ws) == 0
    ref = oracle_forward(w, L, x, residual=res)
    assert_routing(idx, ref["idx"], ref["logits"])
    assert np.allclose(p.cpu().numpy(), ref["p"], rtol=2e-6, atol=1e-7)
    assert_close(out, ref["out"])


def test_prefill_expert_with_more_than_256_tokens():
    """A router bias that puts every token on experts 0 and 1: each gets T > 256 pairs, so
    its work is split over several token tiles."""
    w = TINY.with_(n_experts=16, top_k=2, seed=56)
    L = synth.make_layer(w, 0, DEV)
    L.router_bias = torch.zeros(16, dtype=torch.float32, device=DEV)
    L.router_bias[:2] = 50.0
    T = 600
    x = synth.activations(w, 5, tokens=T, device=DEV)
    out, idx, p, ws = forward(w, L, x, residual=x)
    assert set(np.unique(idx.cpu().numpy()).tolist()) == {0, 1}
    ref = oracle_forward(w, L, x, residual=x)
    assert_routing(idx, ref["idx"], ref["logits"])
    assert_close(out, ref["out"])


def test_prefill_given_topk_matches_routed():
    w = TINY.with_(hidden=2048, inter=512, shared_inter=512, n_experts=48, top_k=5, seed=57)
    L = synth.make_layer(w, 0, DEV)
    x = synth.activations(w, 6, tokens=100, device=DEV)
    out1, idx, p, _ = forward(w, L, x, residual=x)
    out2, _, _, _ = forward(w, L, x, residual=x, topk=(idx.clone(), p.clone()))
    # same routing, same GEMMs; the fp32 scatter order may differ in the last bits
    ref = oracle_forward(w, L, x, residual=x)
    assert_close(out2, ref["out"])
    assert (out1.float() - out2.float()).abs().max().item() <= 1e-2 * out1.float().abs().max().item()


def test_prefill_full_size_every_output_and_routing_margin():
    """The prefill workload itself (hidden 2048, 512 experts, top-10, 4096 tokens): routing of
    every token bit-exact, every output row against the oracle (experts evaluated one at a time
    over their tokens), and the measured margin of the certified routing: the largest
    |fp32 tensor-core logit - exact logit| over all 4096 x 512 logits, as a fraction of the
    bound H * 2^-22 * ||x_t|| * ||w_e|| that the certification assumes, must stay <= 0.25."""
    w = synth.WORKLOADS["prefill"]
    L = synth.make_layer(w, 0, DEV)
    T = w.tokens
    x = synth.activations(w, 0, tokens=T, device=DEV)
    out, idx, p, ws = forward(w, L, x, residual=x)
    assert abi.moe_ws_check(ws) == 0
    l32 = abi.moe_ws_router_logits(abi.shape_of(w), T, ws)[:, :w.n_experts].cpu().numpy().astype(np.float64)
    xb, wrb = host_bits(x), host_bits(L.w_router)
    logits = oracle.router_logits(xb, wrb, None)
    ref_idx, ref_p = oracle.route(logits, w.top_k)
    assert_routing(idx, ref_idx, logits)
    assert np.allclose(p.cpu().numpy(), ref_p, rtol=2e-6, atol=1e-7)
    xn = np.sqrt((oracle.bf16_to_f64(xb) ** 2).sum(1))
    wn = np.sqrt((oracle.bf16_to_f64(wrb) ** 2).sum(1))
    bound = w.hidden * 2.0 ** -22 * xn[:, None] * wn[None, :]
    margin = float((np.abs(l32 - logits) / bound).max())
    print(f"certified routing: max |fp32 - exact| / bound = {margin:.3e}")
    assert margin <= 0.25, margin
    # every expert has a real matrix of tokens
    counts = np.bincount(ref_idx.reshape(-1), minlength=w.n_experts)
    assert counts.sum() == T * w.top_k
    pool = L.pool.cpu().numpy()
    ref = oracle.layer_forward_by_expert(xb, wrb, None, w.top_k, lambda e: pool[e], L.shared.cpu().numpy(),
                                         host_bits(L.w_sg), w.hidden, w.inter, w.shared_inter, w.bits,
                                         residual_bits=xb, idx=ref_idx, p=ref_p)
    assert_close(out, ref["out"])
    # and per token, not only over the whole matrix
    got = out.float().cpu().numpy().astype(np.float64)
    err = np.abs(got - ref["out"]).max(1)
    tol = 1e-2 * np.abs(ref["out"]).max(1) + 1e-3
    assert np.all(err <= tol), int(np.argmax(err - tol))


def test_prefill_matches_token_by_token_decode():
    """Full-sequence vs incremental: each token's prefill output equals (within tolerance)
    its output through the one-token decode path, with the same routing."""
    w = synth.WORKLOADS["prefill"].with_(n_experts=128, seed=58)
    L = synth.make_layer(w, 0, DEV)
    T = 48
    x = synth.activations(w, 9, tokens=T, device=DEV)
    out, idx, p, _ = forward(w, L, x, residual=x)
    for t0 in range(0, T, 8):
        xd = x[t0:t0 + 8].contiguous()
        od, idd, pd, _ = forward(w, L, xd, residual=xd)
        assert torch.equal(idd, idx[t0:t0 + 8])
        a, b = od.float(), out[t0:t0 + 8].float()
        assert (a - b).abs().max().item() <= 1e-2 * b.abs().max().item() + 1e-3


def test_prefill_device_error_flags():
    """Many-token path: a selected expert with an out-of-range slot is flagged and contributes
    nothing (its weights read as zeros); a caller-given id out of range is flagged and its pair
    is skipped.  The rest of the output still matches the oracle."""
    w = TINY.with_(hidden=512, inter=128, shared_inter=128, n_experts=20, top_k=3, seed=61)
    L = synth.make_layer(w, 0, DEV)
    T = 40
    x = synth.activations(w, 7, tokens=T, device=DEV)
    _, idx, p, _ = forward(w, L, x, residual=x)
    bad_e = int(idx[0, 0].item())
    st = torch.arange(w.n_experts, dtype=torch.int32, device=DEV)
    st[bad_e] = 10_000
    out, idx2, p2, ws = forward(w, L, x, residual=x, slot_table=st)
    assert abi.moe_ws_check(ws) & abi.DEVERR_BAD_SLOT
    assert torch.equal(idx2, idx)
    ih, ph = idx.cpu().numpy(), p.cpu().numpy()
    ref = oracle_forward(w, L, x, residual=x, idx=ih, p=np.where(ih == bad_e, 0.0, ph))
    assert_close(out, ref["out"])
    # caller-given routing with one id out of range
    bad = idx.clone()
    bad[3, 1] = w.n_experts + 5
    out, _, _, ws = forward(w, L, x, residual=x, topk=(bad, p))
    assert abi.moe_ws_check(ws) & abi.DEVERR_BAD_EXPERT
    bh = bad.cpu().numpy()
    ref = oracle_forward(w, L, x, residual=x, idx=np.where(bh < w.n_experts, bh, 0),
                         p=np.where(bh < w.n_experts, ph, 0.0))
    assert_close(out, ref["out"])


@pytest.mark.parametrize("bits", [4, 8])
def test_prefill_large_hidden(bits):
    """hidden 4096 / inter 1024: longer K loops, the fewest tile stages shared memory allows."""
    w = TINY.with_(hidden=4096, inter=1024, shared_inter=1024, n_experts=12, top_k=3, bits=bits, seed=62 + bits)
    L = synth.make_layer(w, 0, DEV)
    T = 64
    x = synth.activations(w, 8, tokens=T, device=DEV)
    out, idx, p, ws = forward(w, L, x, residual=x)
    assert abi.moe_ws_check(ws) == 0
    ref = oracle_forward(w, L, x, residual=x)
    assert_close(out, ref["out"])
    assert np.array_equal(idx.cpu().numpy(), ref["idx"])
