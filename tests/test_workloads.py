"""Checks of the seeded workload generator against the workloads it stands in for."""
import numpy as np

import oracle
import synth
from helpers import host_bits


def _fitted_exponent(counts):
    c = np.sort(counts)[::-1]
    c = c[c > 0]
    r = np.arange(1, len(c) + 1)
    return -np.polyfit(np.log(r), np.log(c), 1)[0]


def test_zipf_router_bias_gives_zipf_one_popularity():
    """The 80B-like router (512 experts, top-10, per-expert bias) routes tokens so that the
    expert of popularity rank r is selected with frequency ~ r^-1 (fitted exponent 1 +- 0.15)."""
    w = synth.WORKLOADS["decode80b"]
    wr, bias, _ = synth.router_weights(w, 0, "cpu")
    x = synth.activations(w, 0, tokens=2500, device="cpu")
    logits = oracle.router_logits(host_bits(x), host_bits(wr), bias.numpy())
    idx, _ = oracle.route(logits, w.top_k)
    s = _fitted_exponent(np.bincount(idx.reshape(-1), minlength=w.n_experts))
    assert abs(s - 1.0) < 0.15, s


def test_uniform_router_has_flat_popularity():
    """The 35B-like router (uniform init, no bias): no expert is favoured; the most popular
    expert is chosen at most ~2x the mean rate."""
    w = synth.WORKLOADS["decode35b"]
    wr, bias, _ = synth.router_weights(w, 0, "cpu")
    assert bias is None
    x = synth.activations(w, 0, tokens=2500, device="cpu")
    idx, _ = oracle.route(oracle.router_logits(host_bits(x), host_bits(wr), None), w.top_k)
    c = np.bincount(idx.reshape(-1), minlength=w.n_experts)
    assert c.max() < 2.0 * c.mean() and c.min() > 0.3 * c.mean()
