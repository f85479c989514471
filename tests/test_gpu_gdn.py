"""GPU parity of the Gated DeltaNet decode step (moe_gdn_decode_step through the C ABI)
against the fp64 oracle (oracle/gdn_oracle.py), over several consecutive steps so that the
state the kernel wrote is what the next step reads.

Bar: every step's output within max|diff| <= 1e-2 * max|ref| + 1e-3 (the layer tolerance);
the fp32 state within 1e-4 * max|S| + 1e-6 of the fp64 state after the last step (fp32
rounding of d_k-term sums, compounded over the steps)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from int4_expert_gemv_router_b200 import abi, build

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build()


def _run(Hk, Hv, dk, dv, B, T, seed, start_random):
    shape = abi.moe_gdn_shape(Hk, Hv, dk, dv)
    q, k, v, g, beta = synth.gdn_inputs(Hk, Hv, dk, dv, B, T, seed, DEV)
    S = synth.gdn_state(Hv, dk, dv, B, seed, DEV) if start_random else torch.zeros(B, Hv, dv, dk, device=DEV)
    S_host = S.double().cpu().numpy()
    outs = []
    for t in range(T):
        o = torch.empty(B, Hv, dv, dtype=torch.bfloat16, device=DEV)
        abi.moe_gdn_decode_step(shape, B, S, q[t].contiguous(), k[t].contiguous(), v[t].contiguous(),
                                g[t].contiguous(), beta[t].contiguous(), o)
        outs.append(o)
    torch.cuda.synchronize()
    f = lambda t: t.float().double().cpu().numpy()  # noqa: E731
    for b in range(B):
        Sb = S_host[b]
        for t in range(T):
            Sb, o_ref = oracle.gdn_step(Sb, f(q[t, b]), f(k[t, b]), f(v[t, b]), f(g[t, b]), f(beta[t, b]))
            got = f(outs[t][b])
            err = np.abs(got - o_ref).max()
            assert err <= 1e-2 * np.abs(o_ref).max() + 1e-3, (b, t, err)
        Sg = S[b].double().cpu().numpy()
        assert np.abs(Sg - Sb).max() <= 1e-4 * np.abs(Sb).max() + 1e-6, (b, np.abs(Sg - Sb).max())


@pytest.mark.parametrize("Hk,Hv,dk,dv,B,T,start_random", [
    (16, 32, 128, 128, 1, 6, False),   # the 80B-like linear-attention shape, from a zero state
    (16, 32, 128, 128, 3, 4, True),    # three sequences, from a random state: 4 rows per warp
    (16, 32, 128, 128, 8, 2, True),    # eight sequences: 8 rows per warp
    (4, 8, 256, 200, 12, 2, True),     # 4 rows per warp with d_k 256 and a ragged d_v
    (2, 2, 64, 40, 2, 5, True),        # d_k 64 (two elements per lane), ragged d_v
    (1, 4, 256, 24, 1, 3, True),       # d_k 256, four value heads on one key head
])
def test_gdn_steps_match_oracle(Hk, Hv, dk, dv, B, T, start_random):
    _run(Hk, Hv, dk, dv, B, T, seed=Hk * 7 + dk + B, start_random=start_random)


def test_gdn_full_write_recalls_value():
    """alpha = 1, beta = 1 from a random state: the step's state maps the normalised key onto
    v, so reading with q = k returns v / sqrt(d_k) (the delta rule's defining property)."""
    Hk = Hv = 4
    dk = dv = 128
    shape = abi.moe_gdn_shape(Hk, Hv, dk, dv)
    q, k, v, _, _ = synth.gdn_inputs(Hk, Hv, dk, dv, 1, 1, 3, DEV)
    S = synth.gdn_state(Hv, dk, dv, 1, 3, DEV)
    o = torch.empty(1, Hv, dv, dtype=torch.bfloat16, device=DEV)
    g = torch.zeros(1, Hv, device=DEV)
    beta = torch.ones(1, Hv, device=DEV)
    abi.moe_gdn_decode_step(shape, 1, S, k[0].contiguous(), k[0].contiguous(), v[0].contiguous(), g, beta, o)
    torch.cuda.synchronize()
    want = v[0].float() / np.sqrt(dk)
    assert (o.float() - want).abs().max().item() <= 1e-2 * want.abs().max().item() + 1e-3


def test_gdn_rejects_bad_shapes():
    t = torch.zeros(64, device=DEV)
    with pytest.raises(abi.MoeError) as ei:
        abi.moe_gdn_decode_step(abi.moe_gdn_shape(2, 3, 128, 128), 1, t, t, t, t, t, t, t)
    assert ei.value.status == -1
    with pytest.raises(abi.MoeError) as ei:
        abi.moe_gdn_decode_step(abi.moe_gdn_shape(2, 2, 96, 128), 1, t, t, t, t, t, t, t)
    assert ei.value.status == -5


@pytest.mark.parametrize("B,graph", [(1, False), (1, True), (8, True)])
def test_gdn_early_state_chain_matches_plain(B, graph):
    """A chain of layers (each its own state) run for two steps with MOE_GDN_EARLY_STATE —
    each step launched as a programmatic dependent of the one before, reading its state rows
    early — gives bit for bit the outputs and states of the same chain launched plainly, and
    the first layer matches the oracle."""
    Hk, Hv, dk, dv, nL, steps = 16, 32, 128, 128, 4, 2
    shape = abi.moe_gdn_shape(Hk, Hv, dk, dv)
    ins = [synth.gdn_inputs(Hk, Hv, dk, dv, B, steps, 300 + l, DEV) for l in range(nL)]
    S0 = [synth.gdn_state(Hv, dk, dv, B, 400 + l, DEV) for l in range(nL)]

    def chain(flags):
        S = [s.clone() for s in S0]
        outs = torch.empty(steps, nL, B, Hv, dv, dtype=torch.bfloat16, device=DEV)
        stream = torch.cuda.Stream()

        def one_step(t):
            for l in range(nL):
                q, k, v, g, beta = (x[t].contiguous() for x in ins[l])
                abi.moe_gdn_decode_step(shape, B, S[l], q, k, v, g, beta, outs[t, l], stream=stream, flags=flags)

        with torch.cuda.stream(stream):
            if graph:
                # the inputs are made contiguous once, outside the captured calls
                flat = [[tuple(x[t].contiguous() for x in ins[l]) for l in range(nL)] for t in range(steps)]
                graphs = []
                for t in range(steps):
                    gr = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(gr, stream=stream):
                        for l in range(nL):
                            abi.moe_gdn_decode_step(shape, B, S[l], *flat[t][l], outs[t, l], stream=stream,
                                                    flags=flags)
                    graphs.append(gr)
                # capture ran nothing: reset the states the captures did not touch, then replay
                for l in range(nL):
                    S[l].copy_(S0[l])
                for gr in graphs:
                    gr.replay()
            else:
                for t in range(steps):
                    one_step(t)
        stream.synchronize()
        return outs, S

    o0, s0 = chain(0)
    o1, s1 = chain(abi.MOE_GDN_EARLY_STATE)
    assert torch.equal(o0, o1)
    for a_, b_ in zip(s0, s1):
        assert torch.equal(a_, b_)
    f = lambda t: t.float().double().cpu().numpy()  # noqa: E731
    Sb = S0[0][0].double().cpu().numpy()
    q, k, v, g, beta = ins[0]
    for t in range(steps):
        Sb, o_ref = oracle.gdn_step(Sb, f(q[t, 0]), f(k[t, 0]), f(v[t, 0]), f(g[t, 0]), f(beta[t, 0]))
        err = np.abs(f(o1[t, 0, 0]) - o_ref).max()
        assert err <= 1e-2 * np.abs(o_ref).max() + 1e-3, (t, err)


def test_gdn_rejects_unknown_flags():
    shape = abi.moe_gdn_shape(2, 2, 64, 16)
    S = torch.zeros(1, 2, 16, 64, device=DEV)
    q = torch.zeros(1, 2, 64, dtype=torch.bfloat16, device=DEV)
    v = torch.zeros(1, 2, 16, dtype=torch.bfloat16, device=DEV)
    g = torch.zeros(1, 2, device=DEV)
    out = torch.empty(1, 2, 16, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(abi.MoeError):
        abi.moe_gdn_decode_step(shape, 1, S, q, q, v, g, g, out, flags=6)
