"""C-ABI library checks that need no GPU: it builds, loads, exports every declared symbol,
and validates arguments on the host before touching the device."""
import ctypes
import os
import re
import subprocess

import pytest

import oracle
from int4_expert_gemv_router_b200 import abi, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build()


def _declared():
    names = set()
    inc = os.path.join(ROOT, "include")
    for f in os.listdir(inc):
        if f.endswith(".h"):
            src = open(os.path.join(inc, f)).read()
            names |= set(re.findall(r"^MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", src, flags=re.M))
    return names


def test_exports_every_declared_symbol():
    decl = _declared()
    assert len(decl) >= 13
    out = subprocess.run(["nm", "-D", "--defined-only", abi.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (moe_\w+)", out))
    assert decl <= exported, f"missing: {decl - exported}"
    lib = ctypes.CDLL(abi.LIB_PATH)
    for n in decl:
        getattr(lib, n)
    assert decl == set(abi.exported_symbols())


def test_version():
    assert "sm_100a" in abi.moe_version()


@pytest.mark.parametrize("H,I,b", [(2048, 512, 4), (2048, 512, 8), (256, 64, 4), (192, 64, 4), (4096, 1024, 8)])
def test_blob_layout_matches_oracle(H, I, b):
    offs, stride = abi.moe_blob_layout(H, I, b)
    o_offs, _, o_stride = oracle.blob_layout(H, I, b)
    assert offs == o_offs and stride == o_stride


@pytest.mark.parametrize("args", [(2048, 512, 5, 64), (2048, 512, 4, 32), (100, 512, 4, 64), (2048, 0, 4, 64)])
def test_blob_layout_rejects(args):
    with pytest.raises(abi.MoeError) as ei:
        abi.moe_blob_layout(*args)
    assert ei.value.status == -1


def test_workspace_size_grows_with_tokens():
    s = abi.make_shape(2048, 512, 512, 512, 10, 4)
    a, b = abi.moe_workspace_size(s, 1), abi.moe_workspace_size(s, 8)
    assert 0 < a < b and a % 256 == 0


@pytest.mark.parametrize("field,val", [("group", 32), ("bits", 3), ("hidden", 100), ("n_experts", 0),
                                       ("top_k", 0), ("top_k", 600), ("n_experts", 4096)])
def test_shape_validation(field, val):
    s = abi.make_shape(2048, 512, 512, 512, 10, 4)
    setattr(s, field, val)
    with pytest.raises(abi.MoeError) as ei:
        abi.moe_workspace_size(s, 1)
    assert ei.value.status == -1


def test_layer_forward_rejects_before_any_device_work():
    s = abi.make_shape(2048, 512, 512, 512, 10, 4)
    # NULL pointers: rejected on the host
    with pytest.raises(abi.MoeError) as ei:
        abi.lib()
        st = abi.lib().moe_layer_forward(ctypes.byref(s), None, 1, None, None, None, None, None, None, 1, None, None,
                                         None, None, None, None, None, 0, None)
        abi._check(st)
    assert ei.value.status == -1
    # unsupported shape (shared_inter != inter)
    s2 = abi.make_shape(2048, 512, 256, 512, 10, 4)
    st = abi.lib().moe_layer_forward(ctypes.byref(s2), 16, 1, 16, None, None, None, 256, 16, 1, 256, 16, None, 16,
                                     None, None, 256, 1 << 20, None)
    assert st == -5
    # many tokens on a shape without a prefill kernel (E > 512)
    s3 = abi.make_shape(2048, 512, 512, 600, 10, 4)
    st = abi.lib().moe_layer_forward(ctypes.byref(s3), 16, 9, 16, None, None, None, 256, 16, 1, 256, 16, None, 16,
                                     None, None, 256, 1 << 30, None)
    assert st == -5
    # misaligned x
    st = abi.lib().moe_layer_forward(ctypes.byref(s), 18, 1, 16, None, None, None, 256, 16, 1, 256, 16, None, 16,
                                     None, None, 256, 1 << 30, None)
    assert st == -1
    assert "aligned" in abi.lib().moe_last_error().decode()


def test_pool_create_rejects_bad_args():
    s = abi.make_shape(2048, 512, 512, 512, 10, 4)
    h = ctypes.c_void_p()
    assert abi.lib().moe_pool_create(ctypes.byref(s), 0, 16, 256, 16, ctypes.byref(h)) == -1
    assert abi.lib().moe_pool_create(ctypes.byref(s), 4, None, 256, 16, ctypes.byref(h)) == -1
    abi.moe_pool_destroy(None)


def test_pool_calls_reject_a_null_pool():
    """Every pool call checks its handle before touching anything (no device needed)."""
    L = abi.lib()
    assert L.moe_pool_set_policy(None, 0) == -1
    assert L.moe_pool_set_overlap(None, 1) == -1
    assert L.moe_pool_inject_copy_failure(None, 0) == -1
    assert L.moe_expert_pool_load(None, None, 1, None) == -1
    assert "NULL" in L.moe_last_error().decode()
