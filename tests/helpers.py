"""Shared test helpers: build seeded layers on the device, run the C-ABI path and the oracle."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import synth
from int4_expert_gemv_router_b200 import abi

# Output tolerance of the layer: max|out - ref| <= REL * max|ref| + ABS (bf16 output of an
# fp32 computation against the fp64 oracle).
REL, ABS = 1e-2, 1e-3


def assert_close(out_bf16: torch.Tensor, ref: np.ndarray, rel=REL, atol=ABS, what="out"):
    got = out_bf16.float().cpu().numpy().astype(np.float64)
    err = np.abs(got - ref).max()
    bound = rel * np.abs(ref).max() + atol
    assert err <= bound, f"{what}: max|diff| {err:.3e} > {bound:.3e} (max|ref| {np.abs(ref).max():.3e})"
    return err, bound


def assert_routing(idx_gpu: torch.Tensor, idx_ref: np.ndarray, logits_ref=None, k=None):
    """Top-k ids bit-exact; where they differ only by a tie at fp64 precision both sets are valid."""
    g = idx_gpu.cpu().numpy()
    if np.array_equal(g, idx_ref):
        return 0
    assert logits_ref is not None, f"routing differs:\n{g}\nvs\n{idx_ref}"
    n_ties = 0
    for t in range(g.shape[0]):
        if np.array_equal(g[t], idx_ref[t]):
            continue
        lt = logits_ref[t]
        gap = np.abs(lt[g[t]] - lt[idx_ref[t]]).max()
        scale = np.abs(lt).max()
        assert gap <= 1e-12 * max(scale, 1.0), f"token {t}: ids {g[t]} vs {idx_ref[t]} (gap {gap:.3e})"
        n_ties += 1
    return n_ties


def host_bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> uint16 numpy patterns."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def ws_for(shape, T, device="cuda"):
    n = abi.moe_workspace_size(shape, T)
    return torch.zeros(n, dtype=torch.uint8, device=device)


def forward(w: synth.Workload, L: synth.Layer, x: torch.Tensor, residual=None, slot_table=None, pool=None,
            n_slots=None, topk=None, ws=None, want_topk=True):
    """Run moe_layer_forward; returns (out, idx, p, ws)."""
    shape = abi.shape_of(w)
    T = x.shape[0]
    dev = x.device
    if slot_table is None:
        slot_table = torch.arange(w.n_experts, dtype=torch.int32, device=dev)
    if pool is None:
        pool = L.pool
    if n_slots is None:
        n_slots = pool.shape[0]
    if ws is None:
        ws = ws_for(shape, T, dev)
    out = torch.empty(T, w.hidden, dtype=torch.bfloat16, device=dev)
    idx = torch.full((T, w.top_k), -7, dtype=torch.int32, device=dev)
    p = torch.full((T, w.top_k), -7.0, dtype=torch.float32, device=dev)
    if topk is not None:
        abi.moe_layer_forward(shape, x, T, L.w_router, L.router_bias, topk[0], topk[1], pool, slot_table, n_slots,
                              L.shared, L.w_sg, residual, out, None, None, ws)
        idx, p = topk
    else:
        abi.moe_layer_forward(shape, x, T, L.w_router, L.router_bias, None, None, pool, slot_table, n_slots,
                              L.shared, L.w_sg, residual, out, idx if want_topk else None,
                              p if want_topk else None, ws)
    torch.cuda.synchronize()
    return out, idx, p, ws


def oracle_forward(w: synth.Workload, L: synth.Layer, x: torch.Tensor, residual=None, idx=None, p=None):
    """fp64 oracle on host copies of the generator's bytes (never the kernels' outputs)."""
    pool_host = {}

    def blob(e):
        if e not in pool_host:
            pool_host[e] = L.pool[e].cpu().numpy()
        return pool_host[e]

    bias = None if L.router_bias is None else L.router_bias.cpu().numpy()
    return oracle.layer_forward(host_bits(x), host_bits(L.w_router), bias, w.top_k, blob, L.shared.cpu().numpy(),
                                host_bits(L.w_sg), w.hidden, w.inter, w.shared_inter, w.bits,
                                residual_bits=None if residual is None else host_bits(residual), idx=idx, p=p)
