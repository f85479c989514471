"""Seeded synthetic inputs for the routed-MoE layer.

This module is the one piece shared by the GPU path's tests/benchmarks and by the
fp64 oracle's tests.  It only draws random numbers and formats them into the
input byte layout that a repacking tool would write; it computes nothing of the
layer's forward pass (no routing, no dequantisation, no GEMV).

Workloads (the pages' decode / prefill / bounded-pool shapes):

* ``tiny``      hidden 256, 16 experts, intermediate 64, top-2, 4 tokens, 1 layer.
* ``decode80b`` hidden 2048, 512 experts, intermediate 512, top-10, 1 token/step,
  48 layers, router bias giving Zipf(1.0) popularity (Swiftlet pages: "each layer
  routes each token to 10 of 512 experts (80B)").
* ``decode35b`` hidden 2048, 256 experts, intermediate 512, top-8, 1/4/8
  tokens/step, 40 layers, uniform router init ("8 of 256 (35B)").
* ``prefill``   hidden 2048, 512 experts, top-10, 4096 tokens, 1 layer.
* ``pool``      hidden 2048, 512 experts, top-10, int4 or int8, 128 slots,
  1024 decode steps, Zipf(1.0) routing.

Every expert of every layer has its own seed, so any single expert can be
regenerated without generating the rest (the oracle checks a sample of experts
of a 43 GB pool this way).

Quantisation recipe (MLX-style affine, group 64 along the input dimension; the
pages say only "MLX-style int4/int8 group quantisation"): per group
``scale = bf16((max - min) / (2**bits - 1))``, ``bias = bf16(min)``,
``q = clamp(round_half_even((w - bias) / scale), 0, 2**bits - 1)`` (q = 0 when
scale = 0).  This is data preparation only: the forward pass consumes the codes
as given.

Blob byte layout (one fixed-stride blob per expert, "one read = one fetch"):
sections, each starting on a 256-byte boundary, in the order
Wg.q [I, H*b/8], Wu.q [I, H*b/8], Wd.q [H, I*b/8], Wg.s [I, H/64], Wg.bias,
Wu.s, Wu.bias, Wd.s [H, I/64], Wd.bias; scales/biases bf16; codes packed
little-endian (for int4, byte n holds element 2n in its low nibble, element
2n+1 in its high nibble).  stride = total rounded up to 256 bytes.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import Optional

import torch

GROUP = 64
ALIGN = 256


# ----------------------------------------------------------------------------
# workload registry
# ----------------------------------------------------------------------------
@dataclass(frozen=True)
class Workload:
    name: str
    hidden: int
    n_experts: int
    inter: int
    shared_inter: int
    top_k: int
    bits: int
    tokens: int
    layers: int
    router: str  # "normal" | "zipf" | "uniform"
    seed: int = 0
    weight_std: float = 0.02
    router_std: float = 0.02
    zipf_s: float = 1.0       # target exponent of the measured expert popularity
    zipf_alpha: float = 0.39  # router bias scale that yields it (see router_weights)
    n_slots: Optional[int] = None
    steps: int = 1
    extra: dict = field(default_factory=dict)

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", hidden=256, n_experts=16, inter=64, shared_inter=64, top_k=2,
                     bits=4, tokens=4, layers=1, router="normal", seed=0),
    "decode80b": Workload("decode80b", hidden=2048, n_experts=512, inter=512, shared_inter=512,
                          top_k=10, bits=4, tokens=1, layers=48, router="zipf", seed=1),
    "decode35b": Workload("decode35b", hidden=2048, n_experts=256, inter=512, shared_inter=512,
                          top_k=8, bits=4, tokens=1, layers=40, router="uniform", seed=2),
    "prefill": Workload("prefill", hidden=2048, n_experts=512, inter=512, shared_inter=512,
                        top_k=10, bits=4, tokens=4096, layers=1, router="normal", seed=3),
    "pool_int4": Workload("pool_int4", hidden=2048, n_experts=512, inter=512, shared_inter=512,
                          top_k=10, bits=4, tokens=1, layers=1, router="zipf", seed=4,
                          n_slots=128, steps=1024),
    "pool_int8": Workload("pool_int8", hidden=2048, n_experts=512, inter=512, shared_inter=512,
                          top_k=10, bits=8, tokens=1, layers=1, router="zipf", seed=5,
                          n_slots=128, steps=1024),
}


# ----------------------------------------------------------------------------
# seeds
# ----------------------------------------------------------------------------
_M64 = (1 << 64) - 1


def _splitmix64(z: int) -> int:
    z = (z + 0x9E3779B97F4A7C15) & _M64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _M64
    return z ^ (z >> 31)


def mix_seed(*vals: int) -> int:
    """Combine integers into one 63-bit generator seed."""
    h = 0x243F6A8885A308D3
    for v in vals:
        h = _splitmix64(h ^ (int(v) & _M64))
    return h & ((1 << 63) - 1)


def _gen(device, *vals) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(mix_seed(*vals))
    return g


# ----------------------------------------------------------------------------
# byte layout (formatting of the input, as a repacking tool writes it)
# ----------------------------------------------------------------------------
def _up(n: int, a: int = ALIGN) -> int:
    return (n + a - 1) // a * a


def blob_sections(hidden: int, inter: int, bits: int):
    """[(offset, nbytes)] for the 9 sections, and the stride."""
    H, I, b = hidden, inter, bits
    sizes = [I * H * b // 8, I * H * b // 8, H * I * b // 8,
             I * (H // GROUP) * 2, I * (H // GROUP) * 2,
             I * (H // GROUP) * 2, I * (H // GROUP) * 2,
             H * (I // GROUP) * 2, H * (I // GROUP) * 2]
    secs, off = [], 0
    for s in sizes:
        off = _up(off)
        secs.append((off, s))
        off += s
    return secs, _up(off)


def blob_stride(hidden: int, inter: int, bits: int) -> int:
    return blob_sections(hidden, inter, bits)[1]


# ----------------------------------------------------------------------------
# weights
# ----------------------------------------------------------------------------
def quantize(w: torch.Tensor, bits: int):
    """Affine group-64 quantisation of w [..., rows, K] (fp32) -> (q u8, scale bf16, bias bf16)."""
    *lead, rows, K = w.shape
    g = w.reshape(*lead, rows, K // GROUP, GROUP)
    wmin = g.amin(-1)
    wmax = g.amax(-1)
    qmax = (1 << bits) - 1
    scale = ((wmax - wmin) / qmax).to(torch.bfloat16)
    bias = wmin.to(torch.bfloat16)
    s32 = scale.float().unsqueeze(-1)
    b32 = bias.float().unsqueeze(-1)
    safe = torch.where(s32 == 0, torch.ones_like(s32), s32)
    q = torch.round((g - b32) / safe).clamp_(0, qmax)
    q = torch.where(s32 == 0, torch.zeros_like(q), q)
    return q.to(torch.uint8).reshape(*lead, rows, K), scale, bias


def pack_codes(q: torch.Tensor, bits: int) -> torch.Tensor:
    """u8 codes [..., K] -> packed bytes [..., K*bits/8] (int4: low nibble = even element)."""
    if bits == 8:
        return q.contiguous()
    lo = q[..., 0::2]
    hi = q[..., 1::2]
    return (lo | (hi << 4)).contiguous()


def _bf16_bytes(t: torch.Tensor) -> torch.Tensor:
    return t.contiguous().view(torch.uint8)


def pack_blobs(parts: dict, hidden: int, inter: int, bits: int, out: torch.Tensor) -> None:
    """Write experts into blobs.

    parts: dict with qg, qu [n, I, H] u8; qd [n, H, I] u8; sg, bg, su, bu [n, I, H/64] bf16;
    sd, bd [n, H, I/64] bf16.  out: u8 [n, stride] (a view into a pool is fine).
    """
    secs, stride = blob_sections(hidden, inter, bits)
    n = parts["qg"].shape[0]
    assert out.shape == (n, stride) and out.dtype == torch.uint8
    payload = [pack_codes(parts["qg"], bits), pack_codes(parts["qu"], bits),
               pack_codes(parts["qd"], bits),
               _bf16_bytes(parts["sg"]), _bf16_bytes(parts["bg"]),
               _bf16_bytes(parts["su"]), _bf16_bytes(parts["bu"]),
               _bf16_bytes(parts["sd"]), _bf16_bytes(parts["bd"])]
    out.zero_()
    for (off, size), p in zip(secs, payload):
        out[:, off:off + size] = p.reshape(n, -1)


def expert_parts(hidden: int, inter: int, bits: int, seeds, device, std: float = 0.02) -> dict:
    """Draw W ~ N(0, std) for gate/up/down of each seed's expert and quantise them."""
    n = len(seeds)
    wg = torch.empty(n, inter, hidden, device=device)
    wu = torch.empty(n, inter, hidden, device=device)
    wd = torch.empty(n, hidden, inter, device=device)
    for i, s in enumerate(seeds):
        g = _gen(device, s)
        wg[i].normal_(0.0, std, generator=g)
        wu[i].normal_(0.0, std, generator=g)
        wd[i].normal_(0.0, std, generator=g)
    qg, sg, bg = quantize(wg, bits)
    del wg
    qu, su, bu = quantize(wu, bits)
    del wu
    qd, sd, bd = quantize(wd, bits)
    del wd
    return dict(qg=qg, qu=qu, qd=qd, sg=sg, bg=bg, su=su, bu=bu, sd=sd, bd=bd)


def expert_seed(w: Workload, layer: int, expert: int) -> int:
    """expert == -1 is the shared expert."""
    return mix_seed(w.seed, 101, layer, expert)


def make_blobs(w: Workload, layer: int, experts, device, out: Optional[torch.Tensor] = None,
               shared: bool = False, chunk: int = 32) -> torch.Tensor:
    """Blobs [len(experts), stride] u8 of the given experts of one layer."""
    inter = w.shared_inter if shared else w.inter
    stride = blob_stride(w.hidden, inter, w.bits)
    experts = list(experts)
    if out is None:
        out = torch.empty(len(experts), stride, dtype=torch.uint8, device=device)
    for c0 in range(0, len(experts), chunk):
        ids = experts[c0:c0 + chunk]
        parts = expert_parts(w.hidden, inter, w.bits,
                             [expert_seed(w, layer, -1 if shared else e) for e in ids],
                             device, w.weight_std)
        pack_blobs(parts, w.hidden, inter, w.bits, out[c0:c0 + len(ids)])
        del parts
    return out


def expert_parts_of(w: Workload, layer: int, experts, device, shared: bool = False) -> dict:
    inter = w.shared_inter if shared else w.inter
    return expert_parts(w.hidden, inter, w.bits,
                        [expert_seed(w, layer, -1 if shared else e) for e in experts],
                        device, w.weight_std)


def router_weights(w: Workload, layer: int, device):
    """(W_r bf16 [E, H], bias fp32 [E] or None, w_sg bf16 [H])."""
    g = _gen(device, w.seed, 202, layer)
    E, H = w.n_experts, w.hidden
    if w.router == "uniform":
        a = w.router_std * math.sqrt(3.0)
        wr = torch.empty(E, H, device=device).uniform_(-a, a, generator=g)
    else:
        wr = torch.empty(E, H, device=device).normal_(0.0, w.router_std, generator=g)
    bias = None
    if w.router == "zipf":
        # bias_e = -alpha * ln(rank_e), rank a seeded permutation of 1..E.  alpha is chosen so
        # that the measured top-k selection frequency of the expert of popularity rank r falls
        # as r^-zipf_s: with logits ~ N(0, 0.905^2) (x ~ N(0,1), W_r ~ N(0, 0.02), H = 2048)
        # and top-10 of 512, alpha = 0.39 fits an exponent of 1.00 (alpha = 1 would fit ~2.7,
        # because selection sharpens the bias).
        gp = torch.Generator(device="cpu")
        gp.manual_seed(mix_seed(w.seed, 303, layer))
        rank = torch.randperm(E, generator=gp).to(torch.float64) + 1.0
        bias = (-w.zipf_alpha * torch.log(rank)).to(torch.float32).to(device)
    wsg = torch.empty(H, device=device).normal_(0.0, w.weight_std, generator=g)
    return wr.to(torch.bfloat16), bias, wsg.to(torch.bfloat16)


def activations(w: Workload, step: int, tokens: Optional[int] = None, device="cpu") -> torch.Tensor:
    """x bf16 [T, H] ~ N(0, 1)."""
    T = w.tokens if tokens is None else tokens
    g = _gen(device, w.seed, 404, step)
    return torch.empty(T, w.hidden, device=device).normal_(0.0, 1.0, generator=g).to(torch.bfloat16)


@dataclass
class Layer:
    pool: torch.Tensor          # u8 [E, stride] (all experts resident, slot e holds expert e)
    shared: torch.Tensor        # u8 [stride_s]
    w_router: torch.Tensor      # bf16 [E, H]
    router_bias: Optional[torch.Tensor]  # fp32 [E]
    w_sg: torch.Tensor          # bf16 [H]


def make_layer(w: Workload, layer: int, device, pool_out: Optional[torch.Tensor] = None) -> Layer:
    pool = make_blobs(w, layer, range(w.n_experts), device, out=pool_out)
    shared = make_blobs(w, layer, [0], device, shared=True)[0]
    wr, b, wsg = router_weights(w, layer, device)
    return Layer(pool=pool, shared=shared, w_router=wr, router_bias=b, w_sg=wsg)


def bf16_bits(t: torch.Tensor) -> torch.Tensor:
    """bf16 tensor -> int16 view -> the same bits as uint16 numpy-friendly int32."""
    return t.contiguous().view(torch.int16).to(torch.int32) & 0xFFFF


# ----------------------------------------------------------------------------
# Gated DeltaNet decode-step inputs
# ----------------------------------------------------------------------------
# Linear-attention shape of the 80B-like model: 16 query/key heads, 32 value heads, head
# width 128 (the pages give no dimensions; this is the published layout of the model family
# they run), hidden 2048, 36 of its 48 layers (three quarters).
GDN_WORKLOADS = {
    "gdn80b": dict(n_k_heads=16, n_v_heads=32, d_k=128, d_v=128, layers=36, batch=1, seed=7),
    "gdn80b_b8": dict(n_k_heads=16, n_v_heads=32, d_k=128, d_v=128, layers=36, batch=8, seed=8),
}


def gdn_inputs(Hk: int, Hv: int, dk: int, dv: int, B: int, T: int, seed: int, device="cpu"):
    """T tokens of decode-step inputs for B sequences: q, k bf16 [T, B, Hk, dk] and v bf16
    [T, B, Hv, dv] ~ N(0, 1); log decay g fp32 [T, B, Hv] uniform in [-0.3, 0) (alpha = e^g
    in (0.74, 1]); write strength beta fp32 [T, B, Hv] = sigmoid(N(0, 1))."""
    g_ = _gen(device, seed, 505)
    q = torch.empty(T, B, Hk, dk, device=device).normal_(generator=g_).to(torch.bfloat16)
    k = torch.empty(T, B, Hk, dk, device=device).normal_(generator=g_).to(torch.bfloat16)
    v = torch.empty(T, B, Hv, dv, device=device).normal_(generator=g_).to(torch.bfloat16)
    g = -0.3 * torch.rand(T, B, Hv, device=device, generator=g_)
    beta = torch.sigmoid(torch.empty(T, B, Hv, device=device).normal_(generator=g_))
    return q, k, v, g.float(), beta.float()


def gdn_state(Hv: int, dk: int, dv: int, B: int, seed: int, device="cpu", std: float = 0.1):
    """A seeded fp32 starting state [B, Hv, dv, dk] ~ N(0, std)."""
    g_ = _gen(device, seed, 606)
    return torch.empty(B, Hv, dv, dk, device=device).normal_(0.0, std, generator=g_)
