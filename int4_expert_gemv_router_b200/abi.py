"""Thin ctypes binding of libmoe.so (include/moe.h): same names, argument marshalling only.

Every function takes torch tensors (or None for optional pointers) and passes
their data pointers; `stream` defaults to torch's current CUDA stream.  A
non-OK status raises MoeError with the library's message.  Nothing here
computes any part of the layer: there is no fallback if the library is
missing; loading fails loudly instead.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe.so")

MOE_OK = 0
STATUS = {0: "MOE_OK", -1: "MOE_ERR_INVALID", -2: "MOE_ERR_CUDA", -3: "MOE_ERR_CAPACITY",
          -4: "MOE_ERR_NOT_RESIDENT", -5: "MOE_ERR_UNSUPPORTED", -6: "MOE_ERR_TIMEOUT",
          -7: "MOE_ERR_DEVICE", -8: "MOE_ERR_IO"}
DEVERR_BAD_EXPERT, DEVERR_BAD_SLOT, DEVERR_NONFINITE, DEVERR_TIMEOUT = 1, 2, 4, 8


class MoeError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


class moe_shape(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int32), ("inter", ctypes.c_int32), ("shared_inter", ctypes.c_int32),
                ("n_experts", ctypes.c_int32), ("top_k", ctypes.c_int32), ("bits", ctypes.c_int32),
                ("group", ctypes.c_int32)]


class moe_pool_stats_t(ctypes.Structure):
    _fields_ = [("steps", ctypes.c_int64), ("lookups", ctypes.c_int64), ("hits", ctypes.c_int64),
                ("misses", ctypes.c_int64), ("evictions", ctypes.c_int64), ("h2d_bytes", ctypes.c_int64)]

    def as_dict(self):
        return {k: int(getattr(self, k)) for k, _ in self._fields_}


class moe_layer_desc(ctypes.Structure):
    _fields_ = [("x", ctypes.c_void_p), ("w_router", ctypes.c_void_p), ("router_bias", ctypes.c_void_p),
                ("topk_idx_in", ctypes.c_void_p), ("topk_w_in", ctypes.c_void_p), ("pool", ctypes.c_void_p),
                ("slot_table", ctypes.c_void_p), ("n_slots", ctypes.c_int64), ("shared_blob", ctypes.c_void_p),
                ("w_shared_gate", ctypes.c_void_p), ("residual", ctypes.c_void_p), ("out", ctypes.c_void_p),
                ("topk_idx_out", ctypes.c_void_p), ("topk_w_out", ctypes.c_void_p)]


class moe_gdn_shape(ctypes.Structure):
    _fields_ = [("n_k_heads", ctypes.c_int32), ("n_v_heads", ctypes.c_int32), ("d_k", ctypes.c_int32),
                ("d_v", ctypes.c_int32)]


_P = ctypes.c_void_p
_I32, _I64, _SZ = ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
_SIGS = {
    "moe_blob_layout": (ctypes.c_int, [_I32, _I32, _I32, _I32, ctypes.POINTER(_I64), ctypes.POINTER(_I64)]),
    "moe_workspace_size": (ctypes.c_int, [ctypes.POINTER(moe_shape), _I32, ctypes.POINTER(_SZ)]),
    "moe_router_topk": (ctypes.c_int, [ctypes.POINTER(moe_shape), _P, _I32, _P, _P, _P, _P, _P, _SZ, _P]),
    "moe_layer_forward": (ctypes.c_int, [ctypes.POINTER(moe_shape), _P, _I32, _P, _P, _P, _P, _P, _P, _I64,
                                         _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "moe_layer_forward_static": (ctypes.c_int, [ctypes.POINTER(moe_shape), _P, _I32, _P, _P, _P, _P, _P, _P,
                                                _I64, _P, _P, _P, _P, _P, _P, _P]),
    "moe_layer_forward_partial": (ctypes.c_int, [ctypes.POINTER(moe_shape), _P, _I32, _P, _P, _P, _P, _P, _P, _I64,
                                                 _P, _P, _I32, _P, _P, _P, _P, _SZ, _P]),
    "moe_combine_partials": (ctypes.c_int, [_P, _I32, _I32, _I32, _P, _P, _P]),
    "moe_stack_forward": (ctypes.c_int, [ctypes.POINTER(moe_shape), _I32, ctypes.POINTER(moe_layer_desc), _I32, _P,
                                         _SZ, _P]),
    "moe_group_pairs": (ctypes.c_int, [ctypes.POINTER(moe_shape), _I32, _P, _P, _P, _P, _SZ, _P]),
    "moe_ws_check": (ctypes.c_int, [_P, _P, ctypes.POINTER(ctypes.c_uint32)]),
    "moe_ws_set_slot_wait": (ctypes.c_int, [_P, ctypes.c_uint32, _P]),
    "moe_ws_router_logits": (ctypes.c_int, [ctypes.POINTER(moe_shape), _I32, _P, _SZ, ctypes.POINTER(_P)]),
    "moe_gdn_decode_step": (ctypes.c_int, [ctypes.POINTER(moe_gdn_shape), _I32, _P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_gdn_decode_step_ex": (ctypes.c_int, [ctypes.POINTER(moe_gdn_shape), _I32, _P, _P, _P, _P, _P, _P, _P, _I32,
                                              _P]),
    "moe_pool_create": (ctypes.c_int, [ctypes.POINTER(moe_shape), _I32, _P, _P, _P, ctypes.POINTER(_P)]),
    "moe_pool_create_file": (ctypes.c_int, [ctypes.POINTER(moe_shape), _I32, ctypes.c_char_p, _I32, _P, _P,
                                            ctypes.POINTER(_P)]),
    "moe_expert_pool_load": (ctypes.c_int, [_P, _P, _I32, _P]),
    "moe_pool_stats": (ctypes.c_int, [_P, ctypes.POINTER(moe_pool_stats_t)]),
    "moe_pool_slot_table": (ctypes.c_int, [_P, _P, _P]),
    "moe_pool_inject_copy_failure": (ctypes.c_int, [_P, _I64]),
    "moe_pool_set_policy": (ctypes.c_int, [_P, ctypes.c_int32]),
    "moe_pool_set_overlap": (ctypes.c_int, [_P, ctypes.c_int32]),
    "moe_pool_destroy": (None, [_P]),
    "moe_profile_events": (ctypes.c_int, [_P, _I32]),
    "moe_last_error": (ctypes.c_char_p, []),
    "moe_version": (ctypes.c_char_p, []),
}

_lib = None


def lib() -> ctypes.CDLL:
    """Load libmoe.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m int4_expert_gemv_router_b200.build`")
        l = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(l, name)
            f.restype = res
            f.argtypes = args
        _lib = l
    return _lib


def exported_symbols():
    return list(_SIGS)


def _check(st: int):
    if st != MOE_OK:
        raise MoeError(st, lib().moe_last_error().decode())


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if isinstance(t, torch.Tensor):
        if not t.is_contiguous():
            raise ValueError("tensor must be contiguous")
        return t.data_ptr()
    raise TypeError(f"expected a tensor, an int address or None, got {type(t)}")


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def make_shape(hidden, inter, shared_inter, n_experts, top_k, bits, group=64) -> moe_shape:
    return moe_shape(hidden, inter, shared_inter, n_experts, top_k, bits, group)


def shape_of(w) -> moe_shape:
    """moe_shape from any object with hidden/inter/shared_inter/n_experts/top_k/bits attributes."""
    return make_shape(w.hidden, w.inter, w.shared_inter, w.n_experts, w.top_k, w.bits)


def moe_version() -> str:
    return lib().moe_version().decode()


def moe_blob_layout(hidden: int, inter: int, bits: int, group: int = 64):
    offs = (_I64 * 9)()
    stride = _I64()
    _check(lib().moe_blob_layout(hidden, inter, bits, group, offs, ctypes.byref(stride)))
    return list(offs), int(stride.value)


def moe_workspace_size(shape: moe_shape, T: int) -> int:
    n = _SZ()
    _check(lib().moe_workspace_size(ctypes.byref(shape), T, ctypes.byref(n)))
    return int(n.value)


def moe_router_topk(shape, x, T, w_router, router_bias, topk_idx, topk_w, ws, stream=None):
    _check(lib().moe_router_topk(ctypes.byref(shape), _ptr(x), T, _ptr(w_router), _ptr(router_bias),
                                 _ptr(topk_idx), _ptr(topk_w), _ptr(ws), ws.numel() * ws.element_size(),
                                 _stream(stream)))


def moe_layer_forward(shape, x, T, w_router, router_bias, topk_idx_in, topk_w_in, pool, slot_table, n_slots,
                      shared_blob, w_shared_gate, residual, out, topk_idx_out, topk_w_out, ws, stream=None):
    _check(lib().moe_layer_forward(ctypes.byref(shape), _ptr(x), T, _ptr(w_router), _ptr(router_bias),
                                   _ptr(topk_idx_in), _ptr(topk_w_in), _ptr(pool), _ptr(slot_table), n_slots,
                                   _ptr(shared_blob), _ptr(w_shared_gate), _ptr(residual), _ptr(out),
                                   _ptr(topk_idx_out), _ptr(topk_w_out), _ptr(ws),
                                   ws.numel() * ws.element_size(), _stream(stream)))


def moe_layer_forward_partial(shape, x, T, w_router, router_bias, topk_idx_in, topk_w_in, pool, slot_table, n_slots,
                              shared_blob, w_shared_gate, include_shared, partial_out, topk_idx_out, topk_w_out, ws,
                              stream=None):
    """One expert-parallel rank's fp32 share of the layer (slot_table -3: held by another rank)."""
    _check(lib().moe_layer_forward_partial(ctypes.byref(shape), _ptr(x), T, _ptr(w_router), _ptr(router_bias),
                                           _ptr(topk_idx_in), _ptr(topk_w_in), _ptr(pool), _ptr(slot_table), n_slots,
                                           _ptr(shared_blob), _ptr(w_shared_gate), int(include_shared),
                                           _ptr(partial_out), _ptr(topk_idx_out), _ptr(topk_w_out), _ptr(ws),
                                           ws.numel() * ws.element_size(), _stream(stream)))


def moe_combine_partials(partials, T, hidden, residual, out, stream=None):
    """out = bf16(sum of the fp32 partials in order + residual)."""
    arr = (ctypes.c_void_p * len(partials))(*[_ptr(t) for t in partials])
    _check(lib().moe_combine_partials(arr, len(partials), T, hidden, _ptr(residual), _ptr(out), _stream(stream)))


def layer_desc(x=None, w_router=None, router_bias=None, topk_idx_in=None, topk_w_in=None, pool=None,
               slot_table=None, n_slots=0, shared_blob=None, w_shared_gate=None, residual=None, out=None,
               topk_idx_out=None, topk_w_out=None) -> moe_layer_desc:
    """A moe_layer_desc from tensors (None -> NULL)."""
    return moe_layer_desc(_ptr(x), _ptr(w_router), _ptr(router_bias), _ptr(topk_idx_in), _ptr(topk_w_in), _ptr(pool),
                          _ptr(slot_table), int(n_slots), _ptr(shared_blob), _ptr(w_shared_gate), _ptr(residual),
                          _ptr(out), _ptr(topk_idx_out), _ptr(topk_w_out))


def moe_stack_forward(shape, T, layers, ws, stream=None):
    """layers: a list of moe_layer_desc (see layer_desc)."""
    arr = (moe_layer_desc * len(layers))(*layers)
    _check(lib().moe_stack_forward(ctypes.byref(shape), T, arr, len(layers), _ptr(ws),
                                   ws.numel() * ws.element_size(), _stream(stream)))


def moe_layer_forward_static(shape, x, T, w_router, router_bias, topk_idx_in, topk_w_in, pool, slot_table, n_slots,
                             shared_blob, w_shared_gate, residual, out, topk_idx_out, topk_w_out, stream=None):
    """moe_layer_forward without a workspace argument (the library's fixed device scratch)."""
    _check(lib().moe_layer_forward_static(ctypes.byref(shape), _ptr(x), T, _ptr(w_router), _ptr(router_bias),
                                          _ptr(topk_idx_in), _ptr(topk_w_in), _ptr(pool), _ptr(slot_table),
                                          n_slots, _ptr(shared_blob), _ptr(w_shared_gate), _ptr(residual),
                                          _ptr(out), _ptr(topk_idx_out), _ptr(topk_w_out), _stream(stream)))


def moe_group_pairs(shape, T, topk_idx, order, offsets, ws, stream=None):
    _check(lib().moe_group_pairs(ctypes.byref(shape), T, _ptr(topk_idx), _ptr(order), _ptr(offsets), _ptr(ws),
                                 ws.numel() * ws.element_size(), _stream(stream)))


def moe_ws_check(ws, stream=None, raise_on_error: bool = False) -> int:
    flags = ctypes.c_uint32()
    st = lib().moe_ws_check(_ptr(ws), _stream(stream), ctypes.byref(flags))
    if st not in (MOE_OK, -7) or (raise_on_error and st != MOE_OK):
        _check(st)
    return int(flags.value)


def moe_ws_set_slot_wait(ws, microseconds: int, stream=None):
    """Bound (us; 0 = the 2 s default) of the decode kernel's waits for pending slot entries."""
    _check(lib().moe_ws_set_slot_wait(_ptr(ws), int(microseconds), _stream(stream)))


def moe_ws_router_logits(shape, T: int, ws) -> torch.Tensor:
    """The many-token router's fp32 logits [T, E+1] inside ws, as a view (column E unused)."""
    addr = _P()
    _check(lib().moe_ws_router_logits(ctypes.byref(shape), T, _ptr(ws), ws.numel() * ws.element_size(),
                                      ctypes.byref(addr)))
    off = addr.value - ws.data_ptr()
    n = T * (shape.n_experts + 1)
    return ws[off:off + 4 * n].view(torch.float32).view(T, shape.n_experts + 1)


MOE_GDN_EARLY_STATE = 1


def moe_gdn_decode_step(shape, B, state, q, k, v, g, beta, out, stream=None, flags=0):
    """One gated-delta-rule decode step of B sequences; state (fp32) is updated in place.
    flags=MOE_GDN_EARLY_STATE: the state rows may be read before the preceding kernel on the
    stream has finished (that kernel must not write this state)."""
    if flags:
        _check(lib().moe_gdn_decode_step_ex(ctypes.byref(shape), B, _ptr(state), _ptr(q), _ptr(k), _ptr(v),
                                            _ptr(g), _ptr(beta), _ptr(out), flags, _stream(stream)))
    else:
        _check(lib().moe_gdn_decode_step(ctypes.byref(shape), B, _ptr(state), _ptr(q), _ptr(k), _ptr(v), _ptr(g),
                                         _ptr(beta), _ptr(out), _stream(stream)))


def moe_pool_create(shape, n_slots, host_blobs, dev_pool, dev_slot_table) -> int:
    h = _P()
    _check(lib().moe_pool_create(ctypes.byref(shape), n_slots, _ptr(host_blobs), _ptr(dev_pool),
                                 _ptr(dev_slot_table), ctypes.byref(h)))
    return h.value


POOL_FILE_DIRECT = 1


def moe_pool_create_file(shape, n_slots, path: str, dev_pool, dev_slot_table, direct: bool = False) -> int:
    """A pool whose misses are read from a file of fixed-stride blobs (see moe.h)."""
    h = _P()
    _check(lib().moe_pool_create_file(ctypes.byref(shape), n_slots, os.fsencode(path), POOL_FILE_DIRECT if direct else 0,
                                      _ptr(dev_pool), _ptr(dev_slot_table), ctypes.byref(h)))
    return h.value


def moe_expert_pool_load(pool: int, topk_idx, T: int, stream=None):
    _check(lib().moe_expert_pool_load(pool, _ptr(topk_idx), T, _stream(stream)))


def moe_pool_stats(pool: int) -> dict:
    s = moe_pool_stats_t()
    _check(lib().moe_pool_stats(pool, ctypes.byref(s)))
    return s.as_dict()


def moe_pool_slot_table(pool: int, n_experts: int, n_slots: int):
    a = (ctypes.c_int32 * n_experts)()
    b = (ctypes.c_int32 * n_slots)()
    _check(lib().moe_pool_slot_table(pool, a, b))
    return list(a), list(b)


POOL_POLICIES = {"lfu_recency": 0, "lru": 1, "lfu": 2}


def moe_pool_set_policy(pool: int, policy: str):
    """Eviction policy of the pool's next loads: "lfu_recency" (default), "lru" or "lfu"."""
    _check(lib().moe_pool_set_policy(pool, POOL_POLICIES[policy]))


def moe_pool_set_overlap(pool: int, on: bool):
    """Overlap mode: the forward starts before the step's misses have landed (see moe.h)."""
    _check(lib().moe_pool_set_overlap(pool, 1 if on else 0))


def moe_pool_inject_copy_failure(pool: int, nth: int):
    _check(lib().moe_pool_inject_copy_failure(pool, nth))


def moe_pool_destroy(pool: int):
    lib().moe_pool_destroy(pool)


_prof_keep = None


def moe_profile_events(events, n: int = 0):
    """events: a list of torch.cuda.Event (2 per kernel) or None to disable."""
    global _prof_keep
    if events is None:
        _prof_keep = None
        _check(lib().moe_profile_events(None, 0))
        return
    arr = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
    _prof_keep = arr
    _check(lib().moe_profile_events(arr, n or len(events) // 2))
