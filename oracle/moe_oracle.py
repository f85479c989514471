"""fp64 CPU oracle of the routed-MoE layer forward.

TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
benchmark's CPU-baseline leg may import this module; the product path never
does, and this module imports nothing from the product package.

It is a plain, slow, obviously-correct restatement of what the layer computes,
in float64, written from the Swiftlet pages:

* «Paquets Swiftlet 80B Qwen dans Mac avec 4,3 Go de mémoire…» (xix.ai), ¶5:
  each layer routes each token to 10 of 512 experts (80B) or 8 of 256 (35B);
  routed experts live in fixed-stride blobs so that fetching one is one read;
  a bounded pool caches the hot experts with LFU combined with recency.
* same page, ¶9: MLX-style int4/int8 group quantisation, byte-addressable with
  64-bit offsets; the MoE is high-sparsity with shared experts.
* «Swiftlet: 在 Mac 和 iPhone 上執行 80B 與 35B Qwen 模型» (agentlenshq.com),
  section 記憶體管理與權重串流: fixed-stride blobs in a .qpack container, a
  bounded LFU + recency pool.
* «Swiftlet — это Swift + Metal рантайм…» (news.bugfactory.tech), ¶3: the same
  routing counts, shared experts kept resident, LFU plus recency eviction.

The pages name the blocks but print no formulas.  Where they are silent this
oracle takes the plain reading of a Qwen-style MoE block (each reading is
listed in the design notes):

* router:     l[t,e] = sum_i x[t,i] * Wr[e,i] (+ b[e]);  top-k by l descending,
              ties to the lower expert index;  p = softmax over the k selected
              logits (so the k weights sum to 1).
* expert:     SwiGLU, y = Wd @ (silu(Wg @ x) * (Wu @ x)),  silu(a) = a / (1 + e^-a).
* shared:     always-on expert, scaled by sigmoid(w_sg . x) (bias-free gate).
* combine:    out = sum_k p_k y_k + sigmoid(w_sg . x) y_shared (+ residual).
* weights:    w = scale * q + bias per group of 64 along the input dimension,
              q unsigned, scale and bias bf16.  In float64 this dequantisation
              is exact (a bf16 times an 8-bit integer plus a bf16 fits in 53 bits).

Parity pins (what ties this file to something other than itself) live in
tests/test_oracle_pins.py; every function below has at least one.
"""
from __future__ import annotations

import math
from typing import Callable, Optional, Sequence

import numpy as np

GROUP = 64
ALIGN = 256


# ----------------------------------------------------------------------------
# number formats
# ----------------------------------------------------------------------------
def bf16_to_f64(bits) -> np.ndarray:
    """bf16 bit patterns (any integer dtype holding 16 bits) -> float64 values.

    A bf16 value is the upper half of an IEEE float32, so the conversion is a
    16-bit left shift of the pattern reinterpreted as float32 (exact).
    """
    u = np.asarray(bits).astype(np.uint32) & 0xFFFF
    return (u << 16).view(np.float32).astype(np.float64)


def f64_to_bf16_bits(v) -> np.ndarray:
    """Round float64 values to the nearest bf16 (ties to even), once -> uint16 patterns.

    A bf16 number has 8 significant bits and float32's exponent range: normal numbers
    m * 2^(e-8) with 128 <= m < 256, subnormal ones n * 2^-133 with n < 128.  The float64
    value is rounded directly onto that grid (not through float32, which would round twice
    and can move a value that lies just off a bf16 midpoint onto it).  Values at or beyond
    the midpoint between the largest bf16 (2^128 - 2^120) and 2^128 become infinity; NaN
    becomes the quiet NaN 0x7FC0.  Used to form the next stacked layer's input in tests and
    the CPU baseline.
    """
    a = np.abs(np.asarray(v, dtype=np.float64))
    neg = np.signbit(np.asarray(v, dtype=np.float64))
    out = np.empty(a.shape, dtype=np.float64)
    with np.errstate(over="ignore", invalid="ignore"):
        m, e = np.frexp(a)                          # a = m * 2^e, 0.5 <= m < 1
        normal = a >= 2.0 ** -126
        # normal range: 8 significant bits, m * 2^8 in [128, 256), rounded half to even
        out[normal] = np.ldexp(np.round(np.ldexp(m[normal], 8)), e[normal] - 8)
        # subnormal range: multiples of 2^-133
        out[~normal] = np.ldexp(np.round(np.ldexp(a[~normal], 133)), -133)
        f32 = out.astype(np.float32)                # exact: a bf16 value, or inf past the top
    u = (f32.view(np.uint32) >> 16).astype(np.uint32)
    u = np.where(neg, u | 0x8000, u)
    u = np.where(np.isnan(a), 0x7FC0, u)
    return u.astype(np.uint16)


# ----------------------------------------------------------------------------
# fixed-stride blob (one expert = one contiguous read)
# ----------------------------------------------------------------------------
SECTION_NAMES = ("wg_q", "wu_q", "wd_q", "wg_s", "wg_b", "wu_s", "wu_b", "wd_s", "wd_b")


def blob_layout(hidden: int, inter: int, bits: int):
    """Offsets and sizes (bytes) of the nine sections of an expert blob, and the stride.

    Order: gate codes [I, H], up codes [I, H], down codes [H, I], then gate
    scale, gate bias, up scale, up bias [I, H/64] and down scale, down bias
    [H, I/64] (bf16).  Every section starts on a 256-byte boundary and the
    stride is the total rounded up to 256, so expert e of a pool sits at byte
    e * stride (a 64-bit offset for multi-GB pools).
    """
    H, I, b = hidden, inter, bits
    codes_gu = I * H * b // 8
    codes_d = H * I * b // 8
    sb_gu = I * (H // GROUP) * 2
    sb_d = H * (I // GROUP) * 2
    sizes = [codes_gu, codes_gu, codes_d, sb_gu, sb_gu, sb_gu, sb_gu, sb_d, sb_d]
    offs = []
    pos = 0
    for s in sizes:
        pos = -(-pos // ALIGN) * ALIGN
        offs.append(pos)
        pos += s
    stride = -(-pos // ALIGN) * ALIGN
    return offs, sizes, stride


def unpack_codes(packed: np.ndarray, bits: int, K: int) -> np.ndarray:
    """Packed code bytes [rows, K*bits/8] -> unsigned codes [rows, K] (int64).

    MLX packs codes little-endian into 32-bit words: element j of a word sits
    at bits [bits*j, bits*j + bits).  Read byte by byte this means: for int8,
    byte n is element n; for int4, byte n holds element 2n in its low nibble
    and element 2n+1 in its high nibble.
    """
    p = np.asarray(packed, dtype=np.uint8)
    rows = p.shape[0]
    if bits == 8:
        return p.reshape(rows, K).astype(np.int64)
    if bits == 4:
        out = np.empty((rows, K), dtype=np.int64)
        out[:, 0::2] = p & 0x0F
        out[:, 1::2] = p >> 4
        return out
    raise ValueError("bits must be 4 or 8")


def dequantize(q: np.ndarray, scale: np.ndarray, bias: np.ndarray) -> np.ndarray:
    """w[r, i] = scale[r, i // 64] * q[r, i] + bias[r, i // 64]   (float64, exact)."""
    rows, K = q.shape
    s = np.repeat(np.asarray(scale, dtype=np.float64), GROUP, axis=1)
    b = np.repeat(np.asarray(bias, dtype=np.float64), GROUP, axis=1)
    assert s.shape == (rows, K)
    return s * q + b


def read_expert(blob: np.ndarray, hidden: int, inter: int, bits: int):
    """Decode one blob into dequantised (Wg [I,H], Wu [I,H], Wd [H,I]) float64 matrices."""
    blob = np.asarray(blob, dtype=np.uint8).reshape(-1)
    offs, sizes, stride = blob_layout(hidden, inter, bits)
    assert blob.size >= offs[-1] + sizes[-1]
    H, I = hidden, inter

    def sec(i):
        return blob[offs[i]:offs[i] + sizes[i]]

    def sb(i, rows, cols):
        return bf16_to_f64(sec(i).view(np.uint16).reshape(rows, cols))

    qg = unpack_codes(sec(0).reshape(I, -1), bits, H)
    qu = unpack_codes(sec(1).reshape(I, -1), bits, H)
    qd = unpack_codes(sec(2).reshape(H, -1), bits, I)
    wg = dequantize(qg, sb(3, I, H // GROUP), sb(4, I, H // GROUP))
    wu = dequantize(qu, sb(5, I, H // GROUP), sb(6, I, H // GROUP))
    wd = dequantize(qd, sb(7, H, I // GROUP), sb(8, H, I // GROUP))
    return wg, wu, wd


# ----------------------------------------------------------------------------
# router
# ----------------------------------------------------------------------------
def router_logits(x_bits, wr_bits, bias: Optional[np.ndarray] = None) -> np.ndarray:
    """l[t, e] = sum_i x[t, i] Wr[e, i] (+ b[e]) in float64; x, Wr given as bf16 patterns."""
    x = bf16_to_f64(x_bits)
    wr = bf16_to_f64(wr_bits)
    l = x @ wr.T
    if bias is not None:
        l = l + np.asarray(bias, dtype=np.float32).astype(np.float64)[None, :]
    return l


def route(logits: np.ndarray, k: int):
    """Top-k experts per token and their softmax weights.

    Order: logit descending, ties to the lower expert index.  The weights are a
    softmax over the k selected logits (equal to the full softmax renormalised
    over the selected set), so each row sums to 1.
    """
    T, E = logits.shape
    idx = np.empty((T, k), dtype=np.int32)
    p = np.empty((T, k), dtype=np.float64)
    cols = np.arange(E)
    for t in range(T):
        order = np.lexsort((cols, -logits[t]))  # primary: -logit, secondary: index
        sel = order[:k]
        idx[t] = sel
        z = logits[t, sel] - logits[t, sel].max()
        e = np.exp(z)
        p[t] = e / e.sum()
    return idx, p


def sigmoid(v):
    return 1.0 / (1.0 + np.exp(-v))


def silu(a):
    return a / (1.0 + np.exp(-a))


# ----------------------------------------------------------------------------
# experts and the layer
# ----------------------------------------------------------------------------
def expert_forward(weights, x: np.ndarray) -> np.ndarray:
    """SwiGLU expert: y = Wd @ (silu(Wg @ x) * (Wu @ x)); x [H] or [n, H] float64."""
    wg, wu, wd = weights
    xx = np.atleast_2d(x)
    a = xx @ wg.T
    u = xx @ wu.T
    h = silu(a) * u
    y = h @ wd.T
    return y if np.ndim(x) == 2 else y[0]


def expert_hidden(weights, x: np.ndarray) -> np.ndarray:
    """The SwiGLU intermediate h = silu(Wg x) * (Wu x) (for checking the gate/up stage alone)."""
    wg, wu, _ = weights
    xx = np.atleast_2d(x)
    h = silu(xx @ wg.T) * (xx @ wu.T)
    return h if np.ndim(x) == 2 else h[0]


def layer_forward(x_bits, wr_bits, bias, top_k: int, expert_blob: Callable[[int], np.ndarray],
                  shared_blob, wsg_bits, hidden: int, inter: int, shared_inter: int, bits: int,
                  residual_bits=None, idx: Optional[np.ndarray] = None,
                  p: Optional[np.ndarray] = None, cache: Optional[dict] = None):
    """Routed-MoE layer forward for T tokens, float64.

    expert_blob(e) returns the blob bytes of routed expert e.  If idx/p are
    given the routing step is skipped and they are used as the top-k.
    Returns dict(out [T,H], idx [T,k], p [T,k], logits, gate [T]).
    """
    x = bf16_to_f64(x_bits)
    T = x.shape[0]
    logits = None
    if idx is None:
        logits = router_logits(x_bits, wr_bits, bias)
        idx, p = route(logits, top_k)
    cache = {} if cache is None else cache

    def weights_of(e):
        if e not in cache:
            cache[e] = read_expert(expert_blob(e), hidden, inter, bits)
        return cache[e]

    out = np.zeros((T, hidden), dtype=np.float64)
    for t in range(T):
        for j in range(idx.shape[1]):
            out[t] += p[t, j] * expert_forward(weights_of(int(idx[t, j])), x[t])
    ws = read_expert(shared_blob, hidden, shared_inter, bits)
    gate = sigmoid(x @ bf16_to_f64(wsg_bits))
    out += gate[:, None] * expert_forward(ws, x)
    if residual_bits is not None:
        out += bf16_to_f64(residual_bits)
    return dict(out=out, idx=idx, p=p, logits=logits, gate=gate)


def layer_forward_by_expert(x_bits, wr_bits, bias, top_k: int, expert_blob: Callable[[int], np.ndarray],
                            shared_blob, wsg_bits, hidden: int, inter: int, shared_inter: int, bits: int,
                            residual_bits=None, idx: Optional[np.ndarray] = None,
                            p: Optional[np.ndarray] = None):
    """The same layer as layer_forward, with the loops turned round for many tokens.

    Each selected expert is decoded once and applied to all the tokens routed to it
    (y = expert_forward(W_e, x[tokens of e])), then dropped, so a call over thousands of
    tokens holds one expert's weights at a time.  Per token the arithmetic is that of
    layer_forward: out[t] = sum_j p[t, j] y_{idx[t, j]}(x_t) + sigmoid(w_sg . x_t) y_s(x_t)
    (+ residual), each term an fp64 matrix product; only the order in which the terms of
    different tokens are formed changes.  Returns the same dict as layer_forward.
    """
    x = bf16_to_f64(x_bits)
    T = x.shape[0]
    logits = None
    if idx is None:
        logits = router_logits(x_bits, wr_bits, bias)
        idx, p = route(logits, top_k)
    out = np.zeros((T, hidden), dtype=np.float64)
    for e in np.unique(idx):
        tok, slot = np.nonzero(idx == e)
        y = expert_forward(read_expert(expert_blob(int(e)), hidden, inter, bits), x[tok])
        for n in range(tok.size):
            out[tok[n]] += p[tok[n], slot[n]] * y[n]
    ws = read_expert(shared_blob, hidden, shared_inter, bits)
    gate = sigmoid(x @ bf16_to_f64(wsg_bits))
    out += gate[:, None] * expert_forward(ws, x)
    if residual_bits is not None:
        out += bf16_to_f64(residual_bits)
    return dict(out=out, idx=idx, p=p, logits=logits, gate=gate)


def layer_forward_dense_masked(x_bits, wr_bits, bias, top_k: int, blobs: Sequence[np.ndarray],
                               shared_blob, wsg_bits, hidden: int, inter: int,
                               shared_inter: int, bits: int, residual_bits=None) -> np.ndarray:
    """Brute force: evaluate ALL E experts on every token, then mask to the top-k.

    Independent formulation of the same layer: a full softmax over all E
    logits, a 0/1 mask of the k largest (full stable sort), renormalisation of
    the masked softmax, and a dense weighted sum over every expert.
    """
    x = bf16_to_f64(x_bits)
    T = x.shape[0]
    E = len(blobs)
    logits = router_logits(x_bits, wr_bits, bias)
    full = np.exp(logits - logits.max(axis=1, keepdims=True))
    full = full / full.sum(axis=1, keepdims=True)
    mask = np.zeros((T, E))
    for t in range(T):
        ranked = sorted(range(E), key=lambda e: (-logits[t, e], e))
        mask[t, ranked[:top_k]] = 1.0
    w = full * mask
    w = w / w.sum(axis=1, keepdims=True)
    ys = np.stack([expert_forward(read_expert(b, hidden, inter, bits), x) for b in blobs], 1)
    out = np.einsum("te,teh->th", w, ys)
    ws = read_expert(shared_blob, hidden, shared_inter, bits)
    gate = sigmoid(x @ bf16_to_f64(wsg_bits))
    out = out + gate[:, None] * expert_forward(ws, x)
    if residual_bits is not None:
        out = out + bf16_to_f64(residual_bits)
    return out


# ----------------------------------------------------------------------------
# prefill grouping
# ----------------------------------------------------------------------------
def group_pairs(idx: np.ndarray, n_experts: int):
    """Stable counting sort of the (token, slot) pairs by expert.

    Pair number n = t * k + j refers to idx[t, j].  Returns (counts [E],
    offsets [E+1] exclusive prefix sums, order [T*k] pair numbers sorted by
    expert, ties kept in pair order).
    """
    flat = np.asarray(idx, dtype=np.int64).reshape(-1)
    counts = np.bincount(flat, minlength=n_experts).astype(np.int32)
    offsets = np.zeros(n_experts + 1, dtype=np.int32)
    offsets[1:] = np.cumsum(counts)
    order = np.empty(flat.size, dtype=np.int32)
    fill = offsets[:-1].copy()
    for n, e in enumerate(flat):
        order[fill[e]] = n
        fill[e] += 1
    return counts, offsets, order


# ----------------------------------------------------------------------------
# bounded slot pool: LFU + recency
# ----------------------------------------------------------------------------
SLOT_POLICIES = ("lfu_recency", "lru", "lfu")


class SlotCache:
    """Bounded pool of expert slots with LFU + recency eviction.

    Per slot: the resident expert, a use count (set to 1 when the expert is
    loaded, +1 on every later step that uses it) and the step of last use.
    Each step looks up its unique experts in first-appearance order: a
    resident expert is a hit; the misses are then loaded in the same order,
    into the lowest-numbered empty slot if any, otherwise into the slot with
    the smallest (count, last use, slot index) among slots whose expert this
    step does not need (those are pinned for the step).  A step that needs more
    unique experts than there are slots is a capacity error.

    For the eviction ablation, `policy` may instead be "lru" (smallest (last use, slot))
    or "lfu" (smallest (count, slot)); "lfu_recency" is the pages' policy and the default.
    """

    def __init__(self, n_experts: int, n_slots: int, policy: str = "lfu_recency"):
        if policy not in SLOT_POLICIES:
            raise ValueError(f"unknown policy {policy!r}")
        self.policy = policy
        self.E, self.S = n_experts, n_slots
        self.slot_of = np.full(n_experts, -1, dtype=np.int32)
        self.expert_in = np.full(n_slots, -1, dtype=np.int32)
        self.count = np.zeros(n_slots, dtype=np.int64)
        self.last = np.full(n_slots, -1, dtype=np.int64)
        self.lookups = self.hits = self.misses = self.evictions = 0
        self.step_no = 0

    def step(self, experts: Sequence[int]):
        """Process one step's expert ids (any order, duplicates allowed).

        Returns the list of (expert, slot) loads of this step, in load order.
        """
        uniq = []
        seen = set()
        for e in experts:
            e = int(e)
            if e not in seen:
                seen.add(e)
                uniq.append(e)
        if len(uniq) > self.S:
            raise OverflowError("step needs more unique experts than slots")
        s_no = self.step_no
        loads = []
        for e in uniq:
            self.lookups += 1
            s = self.slot_of[e]
            if s >= 0:
                self.hits += 1
                self.count[s] += 1
                self.last[s] = s_no
        for e in uniq:
            if self.slot_of[e] >= 0:
                continue
            self.misses += 1
            empty = np.nonzero(self.expert_in < 0)[0]
            if empty.size:
                s = int(empty[0])
            else:
                best = None
                for c in range(self.S):
                    if int(self.expert_in[c]) in seen:
                        continue
                    if self.policy == "lru":
                        key = (int(self.last[c]), c)
                    elif self.policy == "lfu":
                        key = (int(self.count[c]), c)
                    else:
                        key = (int(self.count[c]), int(self.last[c]), c)
                    if best is None or key < best:
                        best = key
                s = best[-1]
                self.slot_of[self.expert_in[s]] = -1
                self.evictions += 1
            self.expert_in[s] = e
            self.slot_of[e] = s
            self.count[s] = 1
            self.last[s] = s_no
            loads.append((e, s))
        self.step_no += 1
        return loads
