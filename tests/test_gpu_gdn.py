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
