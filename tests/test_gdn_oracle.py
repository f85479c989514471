"""Pins of the Gated DeltaNet decode-step oracle (oracle/gdn_oracle.py) to things other than
itself: closed forms of the gated delta rule, its defining property, an independent expanded
formulation, and invariances.  CPU only."""
import numpy as np
import pytest

import oracle


def _inputs(rng, Hk=2, Hv=4, dk=8, dv=6):
    S = rng.standard_normal((Hv, dv, dk))
    q = rng.standard_normal((Hk, dk))
    k = rng.standard_normal((Hk, dk))
    v = rng.standard_normal((Hv, dv))
    g = -rng.uniform(0.0, 1.0, Hv)
    beta = rng.uniform(0.0, 1.0, Hv)
    return S, q, k, v, g, beta


def test_no_write_only_decays():
    # beta = 0: S' = alpha S and o = alpha S q^ / sqrt(d_k)
    rng = np.random.default_rng(0)
    S, q, k, v, g, _ = _inputs(rng)
    S1, o = oracle.gdn_step(S, q, k, v, g, np.zeros(4))
    qn = q / np.linalg.norm(q, axis=1, keepdims=True) / np.sqrt(8)
    for h in range(4):
        a = np.exp(g[h])
        assert np.allclose(S1[h], a * S[h], rtol=1e-14, atol=0)
        assert np.allclose(o[h], a * S[h] @ qn[h // 2], rtol=1e-13, atol=1e-15)


def test_full_write_maps_key_onto_value():
    # the delta rule's defining property: with alpha = 1 and beta = 1 the new state maps the
    # (normalised) key exactly onto the value, whatever the old state
    rng = np.random.default_rng(1)
    S, q, k, v, _, _ = _inputs(rng)
    S1, _ = oracle.gdn_step(S, q, k, v, np.zeros(4), np.ones(4))
    kn = k / np.linalg.norm(k, axis=1, keepdims=True)
    for h in range(4):
        assert np.allclose(S1[h] @ kn[h // 2], v[h], rtol=1e-13, atol=1e-13)
        # and leaves directions orthogonal to the key unchanged
        w = rng.standard_normal(8)
        w -= (w @ kn[h // 2]) * kn[h // 2]
        assert np.allclose(S1[h] @ w, S[h] @ w, rtol=1e-12, atol=1e-12)


def test_zero_state_closed_form():
    rng = np.random.default_rng(2)
    _, q, k, v, g, beta = _inputs(rng)
    S1, o = oracle.gdn_step(np.zeros((4, 6, 8)), q, k, v, g, beta)
    kn = k / np.linalg.norm(k, axis=1, keepdims=True)
    qn = q / np.linalg.norm(q, axis=1, keepdims=True)
    for h in range(4):
        assert np.allclose(S1[h], beta[h] * np.outer(v[h], kn[h // 2]), rtol=1e-14, atol=1e-16)
        assert np.allclose(o[h], beta[h] * v[h] * (kn[h // 2] @ qn[h // 2]) / np.sqrt(8), rtol=1e-13, atol=1e-16)


def test_expanded_form_and_head_groups():
    # S' = alpha S + beta (v - alpha S k) k^T, written with einsum over all heads at once;
    # value head h reads key head h // (H_v / H_k)
    rng = np.random.default_rng(3)
    for Hk, Hv in ((1, 1), (2, 4), (4, 4), (2, 8)):
        S, q, k, v, g, beta = _inputs(rng, Hk=Hk, Hv=Hv)
        S1, o = oracle.gdn_step(S, q, k, v, g, beta)
        grp = np.arange(Hv) // (Hv // Hk)
        kn = (k / np.linalg.norm(k, axis=1, keepdims=True))[grp]
        qn = (q / np.linalg.norm(q, axis=1, keepdims=True))[grp] / np.sqrt(8)
        a = np.exp(g)[:, None, None]
        Sd = a * S
        u = np.einsum("hij,hj->hi", Sd, kn)
        ref = Sd + beta[:, None, None] * np.einsum("hi,hj->hij", v - u, kn)
        assert np.allclose(S1, ref, rtol=1e-12, atol=1e-13)
        assert np.allclose(o, np.einsum("hij,hj->hi", ref, qn), rtol=1e-12, atol=1e-13)


def test_steps_decay_product_and_scale_invariance():
    rng = np.random.default_rng(4)
    S, q, k, v, _, _ = _inputs(rng)
    T = 5
    g = -rng.uniform(0, 0.5, (T, 4))
    qs, ks, vs = (np.stack([x] * T) for x in (q, k, v))
    ST, _ = oracle.gdn_steps(S, qs, ks, vs, g, np.zeros((T, 4)))
    assert np.allclose(ST, np.exp(g.sum(0))[:, None, None] * S, rtol=1e-13)
    # q and k enter normalised: positive rescaling changes nothing
    gg = -rng.uniform(0, 1, 4)
    bb = rng.uniform(0, 1, 4)
    a1 = oracle.gdn_step(S, q, k, v, gg, bb)
    a2 = oracle.gdn_step(S, 3.5 * q, 0.25 * k, v, gg, bb)
    assert np.allclose(a1[0], a2[0], rtol=1e-13) and np.allclose(a1[1], a2[1], rtol=1e-13)
