"""The C ABI library loads without a GPU, exports every symbol the public
header declares, and its host-side checks reject bad shapes before anything
is launched."""
import ctypes
import os
import re

import pytest

from combine_moe_route_07_b200 import _binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if not fn.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", fn)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^\s*[A-Za-z_][\w\s\*]*?\b(moe_\w+)\s*\(", text, flags=re.M):
            names.add(m.group(1))
    return names


@pytest.fixture(scope="module")
def lib():
    import __graft_entry__  # noqa: F401  (build() keeps the library current)
    from combine_moe_route_07_b200 import build
    build.build()
    return _binding.lib()


def test_header_declares_the_four_steps():
    d = _declared()
    for name in ("moe_route", "moe_layout", "moe_dispatch", "moe_combine"):
        assert name in d


def test_every_declared_symbol_is_exported(lib):
    d = _declared()
    assert d, "no declarations found"
    missing = [n for n in d if not hasattr(lib, n)]
    assert not missing, missing
    assert set(_binding.EXPORTS) <= d


def test_abi_version_and_status_strings(lib):
    assert lib.moe_abi_version() == 1
    for code in range(8):
        assert lib.moe_status_string(code)
    assert lib.moe_status_string(0) == b"ok"


def _shape(**kw):
    base = dict(tokens=4096, hidden=4096, experts=128, k=8, ranks=16, capacity=0, align=1,
                flags=1)
    base.update(kw)
    return _binding.MoeShapeC(**base)


def test_rows_and_workspace_sizes(lib):
    s = _shape()
    assert lib.moe_layout_rows(ctypes.byref(s)) == 4096 * 8
    assert lib.moe_layout_rows(ctypes.byref(_shape(capacity=1229, experts=256, ranks=32))) \
        == 256 * 1229
    assert lib.moe_layout_rows(ctypes.byref(_shape(align=128))) == 4096 * 8 + 128 * 127
    ws = lib.moe_workspace_bytes(ctypes.byref(s))
    assert ws >= 256 + 32 * 128 * 4 and ws % 256 == 0


@pytest.mark.parametrize("bad", [
    dict(k=0), dict(k=33, experts=64, ranks=1), dict(k=9, experts=8, ranks=1),
    dict(experts=0), dict(experts=1025, ranks=1), dict(ranks=3), dict(hidden=12),
    dict(hidden=0), dict(flags=3, hidden=136), dict(flags=8), dict(tokens=-1),
    dict(capacity=-1), dict(align=0), dict(capacity=4, align=2),
    dict(tokens=1 << 27, k=8), dict(capacity=1 << 24, experts=256, ranks=1),
])
def test_invalid_shapes_are_rejected_on_the_host(lib, bad):
    s = _shape(**bad)
    assert lib.moe_layout_rows(ctypes.byref(s)) == -1
    assert lib.moe_workspace_bytes(ctypes.byref(s)) == 0
    fake = ctypes.c_void_p(0x1000)
    # rejected before any CUDA call: no GPU needed
    assert lib.moe_route(ctypes.byref(s), fake, None, fake, fake, fake, 1 << 20, None) == 1
    assert lib.moe_layout(ctypes.byref(s), fake, fake, fake, fake, fake, fake, fake, fake,
                          1 << 20, None) == 1
    assert lib.moe_dispatch(ctypes.byref(s), fake, fake, fake, fake, fake, 1 << 20, None) == 1
    assert lib.moe_combine(ctypes.byref(s), fake, fake, fake, None, None, fake, fake, 1 << 20,
                           None) == 1


def test_bad_pointers_and_workspace_are_rejected_on_the_host(lib):
    s = _shape()
    fake = ctypes.c_void_p(0x1000)
    odd = ctypes.c_void_p(0x1008)  # 8-byte aligned, not 16
    null = None
    assert lib.moe_route(ctypes.byref(s), null, None, fake, fake, fake, 1 << 20, None) == 1
    assert lib.moe_dispatch(ctypes.byref(s), odd, fake, fake, None, fake, 1 << 20, None) == 1
    assert lib.moe_combine(ctypes.byref(s), fake, fake, fake, odd, None, fake, fake, 1 << 20,
                           None) == 1
    # workspace: NULL, misaligned, too small
    assert lib.moe_route(ctypes.byref(s), fake, None, fake, fake, null, 1 << 20, None) == 3
    assert lib.moe_route(ctypes.byref(s), fake, None, fake, fake, odd, 1 << 20, None) == 3
    assert lib.moe_layout(ctypes.byref(s), fake, fake, fake, fake, fake, fake, fake, fake, 64,
                          None) == 3
    fp8 = _shape(flags=3)
    assert lib.moe_dispatch(ctypes.byref(fp8), fake, fake, fake, null, fake, 1 << 20, None) == 1
