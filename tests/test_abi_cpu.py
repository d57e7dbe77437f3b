"""C-ABI library checks that need no GPU: the shared library loads, exports
every function the header declares, and rejects invalid arguments on the host
before touching the device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_layer.h")


@pytest.fixture(scope="module")
def bq():
    from bit_quantized_moe_top_b200 import build
    build.build()
    import bit_quantized_moe_top_b200 as m
    return m


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_\w+)\s*\(", text)))


def test_header_and_binding_agree(bq):
    assert header_functions() == sorted(bq.EXPORTS)


def test_library_exports_every_symbol(bq):
    lib = ctypes.CDLL(bq.LIB_PATH)
    for name in header_functions():
        assert hasattr(lib, name), name


def test_status_strings(bq):
    lib = bq._lib()
    for s in range(9):
        assert lib.moe_status_string(s)
    assert bq.moe_status_string(99) == "unknown status"


def _desc(bq, bits=(4, 4), fmt=0, group=64, rank=0):
    return bq.ExpertDesc((ctypes.c_int * 2)(*bits), fmt, group, rank)


@pytest.mark.parametrize("args", [
    dict(E=0), dict(E=300), dict(K=100), dict(N=192), dict(max_tokens=0), dict(top_k=9), dict(top_k=5, E=4),
    dict(bits=(5, 4)), dict(bits=(1, 4)), dict(group=48), dict(group=32), dict(rank=65), dict(rank=-1),
    dict(fmt=2, bits=(4, 4)), dict(fmt=7), dict(flags=4),
])
def test_create_rejects_invalid_args(bq, args):
    E = args.get("E", 4)
    descs = [_desc(bq, args.get("bits", (4, 4)), args.get("fmt", 0), args.get("group", 64), args.get("rank", 0))
             for _ in range(max(E, 1))]
    arr = (bq.ExpertDesc * max(E, 1))(*descs)
    out = ctypes.c_void_p(1234)
    st = bq._lib().moe_layer_create(E, args.get("K", 256), args.get("N", 256), args.get("max_tokens", 8),
                                    args.get("top_k", 2), arr, args.get("flags", 0), ctypes.byref(out))
    assert st == 1  # MOE_ERR_INVALID_ARG
    assert out.value is None


def test_null_handles_are_rejected(bq):
    lib = bq._lib()
    assert lib.moe_layer_set_bits(None, 0, 0, 3) == 1
    assert lib.moe_layer_set_path(None, 0) == 1
    assert lib.moe_layer_forward(None, None, None, 1, 1, None, None) == 1
    assert lib.moe_layer_forward_host(None, None, None, 1, 1, None, None) == 1
    assert lib.moe_layer_get_routing(None, None, None, None, None, None, None) == 1
    assert lib.moe_layer_debug_unpack(None, 0, 0, None) == 1
    assert lib.moe_layer_sync_status(None) == 1
    assert lib.moe_layer_last_launch_count(None) == 0
    assert lib.moe_layer_create(4, 256, 256, 8, 2, None, 0, None) == 1
    lib.moe_layer_destroy(None)
