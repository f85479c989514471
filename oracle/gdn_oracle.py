"""fp64 CPU oracle of one Gated DeltaNet decode step (the linear-attention layers).

TEST INFRASTRUCTURE ONLY, like moe_oracle: only the test suite, the smoke check and the
benchmark's CPU-baseline leg may import it; it imports nothing from the product package.

The Swiftlet pages say that three quarters of the hybrid model's layers are Gated DeltaNet
linear attention with a fixed-size recurrent state instead of a growing key/value cache
(«Paquets Swiftlet 80B Qwen dans Mac…», xix.ai, paragraph 6; «Swiftlet: 在 Mac 和 iPhone 上
執行…», agentlenshq.com, section 技術譜系與正確性).  They print no formula.  The plainest
reading is the gated delta rule that names the layer: per value head, a state matrix
S (d_v x d_k) that maps keys to values, updated per token by

    S_t = alpha_t * S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,    o_t = S_t q_t

with alpha_t = exp(g_t) in (0, 1] (decay), beta_t in [0, 1] (write strength), k_t and q_t
L2-normalised and q_t scaled by d_k^-1/2.  Expanded,
S_t = alpha_t S_{t-1} + beta_t (v_t - alpha_t S_{t-1} k_t) k_t^T: the state is decayed, then
moved so that it maps k_t closer to v_t (exactly onto it when beta_t = 1).  Value head h
reads key head h // (H_v / H_k) (key heads shared by groups of value heads).  The gates and
the q/k/v projections are inputs; only the recurrence and its read-out are the step.
"""
from __future__ import annotations

import numpy as np


def l2_normalize(v: np.ndarray, eps: float = 1e-6) -> np.ndarray:
    """v / max(||v||, eps) along the last axis (float64)."""
    v = np.asarray(v, dtype=np.float64)
    n = np.sqrt((v * v).sum(-1, keepdims=True))
    return v / np.maximum(n, eps)


def gdn_step(S: np.ndarray, q: np.ndarray, k: np.ndarray, v: np.ndarray, g: np.ndarray, beta: np.ndarray):
    """One decode step of one sequence.

    S    [H_v, d_v, d_k] state (float64; a new array is returned)
    q, k [H_k, d_k]      queries and keys (normalised here)
    v    [H_v, d_v]      values
    g    [H_v]           log decay (alpha = exp(g))
    beta [H_v]           write strength
    Returns (S_new [H_v, d_v, d_k], o [H_v, d_v]).
    """
    S = np.asarray(S, dtype=np.float64)
    Hv, dv, dk = S.shape
    Hk = q.shape[0]
    assert Hv % Hk == 0
    qn = l2_normalize(q) / np.sqrt(dk)
    kn = l2_normalize(k)
    S_new = np.empty_like(S)
    o = np.empty((Hv, dv))
    for h in range(Hv):
        kh, qh = kn[h // (Hv // Hk)], qn[h // (Hv // Hk)]
        alpha = np.exp(float(g[h]))
        b = float(beta[h])
        # S (alpha (I - b k k^T)) + b v k^T, with the matrices written out
        A = alpha * (np.eye(dk) - b * np.outer(kh, kh))
        S_new[h] = S[h] @ A + b * np.outer(v[h], kh)
        o[h] = S_new[h] @ qh
    return S_new, o


def gdn_steps(S: np.ndarray, q, k, v, g, beta):
    """Several consecutive decode steps of one sequence: inputs with a leading token axis.
    Returns (S after the last step, o [T, H_v, d_v])."""
    outs = []
    for t in range(len(q)):
        S, o = gdn_step(S, q[t], k[t], v[t], g[t], beta[t])
        outs.append(o)
    return S, np.stack(outs)
