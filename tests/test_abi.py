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


def _extra_calls(lib, s, fake):
    """Every entry point beyond the four steps, with plausible pointers."""
    p = ctypes.byref(s)
    big = 1 << 20
    return {
        "moe_route_limited": lambda: lib.moe_route_limited(p, fake, None, 4, fake, fake, fake, big,
                                                           None),
        "moe_layout_remote_first": lambda: lib.moe_layout_remote_first(
            p, fake, 0, fake, fake, fake, fake, fake, fake, None, fake, big, None),
        "moe_route_round_robin": lambda: lib.moe_route_round_robin(p, fake, fake, None),
        "moe_bias_update": lambda: lib.moe_bias_update(p, fake, 0.001, fake, None),
        "moe_layout_src": lambda: lib.moe_layout_src(p, fake, fake, fake, fake, fake, fake, fake,
                                                     fake, fake, big, None),
        "moe_route_layout": lambda: lib.moe_route_layout(p, fake, None, fake, fake, fake, fake,
                                                         fake, fake, fake, fake, fake, big, None),
        "moe_route_layout_dispatch": lambda: lib.moe_route_layout_dispatch(
            p, fake, None, fake, fake, fake, fake, fake, fake, fake, fake, fake, fake, None, fake,
            big, None),
        "moe_layout_noalloc": lambda: lib.moe_layout_noalloc(p, fake, fake, fake, fake, fake, fake,
                                                             fake, None),
    }


@pytest.mark.parametrize("bad", [dict(k=0), dict(ranks=3), dict(hidden=12), dict(tokens=-1)])
def test_every_other_entry_point_rejects_a_bad_shape_on_the_host(lib, bad):
    fake = ctypes.c_void_p(0x1000)
    for name, call in _extra_calls(lib, _shape(**bad), fake).items():
        assert call() == _binding.MOE_ERR_INVALID_ARG, name


def test_rank_limit_arguments(lib):
    fake = ctypes.c_void_p(0x1000)
    s = _shape()  # E = 128 on R = 16: 8 experts a rank
    call = lambda m, shape=s: lib.moe_route_limited(ctypes.byref(shape), fake, None, m, fake,
                                                     fake, fake, 1 << 20, None)
    assert call(0) == _binding.MOE_ERR_INVALID_ARG     # max_ranks < 1
    assert call(-3) == _binding.MOE_ERR_INVALID_ARG
    k9 = _shape(k=9)
    assert call(1, k9) == _binding.MOE_ERR_INVALID_ARG  # k > max_ranks * E/R = 8


def test_home_rank_must_be_one_of_the_ranks(lib):
    fake = ctypes.c_void_p(0x1000)
    s = _shape()
    for home in (-1, 16, 1 << 30):
        assert lib.moe_layout_remote_first(ctypes.byref(s), fake, home, fake, fake, fake, fake,
                                           fake, fake, None, fake, 1 << 20,
                                           None) == _binding.MOE_ERR_INVALID_ARG, home


def test_bias_update_arguments(lib):
    fake = ctypes.c_void_p(0x1000)
    odd = ctypes.c_void_p(0x1002)
    s = ctypes.byref(_shape())
    for gamma in (-0.5, float("inf"), float("nan")):
        assert lib.moe_bias_update(s, fake, gamma, fake, None) == _binding.MOE_ERR_INVALID_ARG
    assert lib.moe_bias_update(s, None, 0.1, fake, None) == _binding.MOE_ERR_INVALID_ARG
    assert lib.moe_bias_update(s, fake, 0.1, None, None) == _binding.MOE_ERR_INVALID_ARG
    assert lib.moe_bias_update(s, odd, 0.1, fake, None) == _binding.MOE_ERR_INVALID_ARG


def test_the_source_layout_flag_picks_its_own_calls(lib):
    """A shape with MOE_F_SRC_LAYOUT is refused by the plain, fused and
    allocation-free layout calls, and one without it by moe_layout_src."""
    fake = ctypes.c_void_p(0x1000)
    src = _shape(flags=_binding.MOE_F_RENORM | _binding.MOE_F_SRC_LAYOUT)
    calls = _extra_calls(lib, src, fake)
    for name in ("moe_layout_remote_first", "moe_route_layout", "moe_route_layout_dispatch",
                 "moe_layout_noalloc"):
        assert calls[name]() == _binding.MOE_ERR_INVALID_ARG, name
    assert lib.moe_layout(ctypes.byref(src), fake, fake, fake, fake, fake, fake, fake, fake,
                          1 << 20, None) == _binding.MOE_ERR_INVALID_ARG
    plain = _extra_calls(lib, _shape(), fake)
    assert plain["moe_layout_src"]() == _binding.MOE_ERR_INVALID_ARG


def test_allocation_free_layout_refuses_shapes_past_its_array(lib):
    """min(ceil(T/16), 128) * E above 65536 words a table: unsupported, with
    nothing launched (checked before any CUDA call)."""
    fake = ctypes.c_void_p(0x1000)
    ok_shape = _shape(tokens=1024, experts=1024, ranks=16)   # 64 * 1024 = 65536: fits
    big = _shape(tokens=1040, experts=1024, ranks=16)        # 65 * 1024: does not
    wide = _shape(tokens=4096, experts=1024, ranks=16)       # 128 * 1024
    for s in (big, wide):
        assert lib.moe_layout_noalloc(ctypes.byref(s), fake, fake, fake, fake, fake, fake, fake,
                                      None) == _binding.MOE_ERR_UNSUPPORTED
    assert lib.moe_layout_noalloc(ctypes.byref(ok_shape), fake, fake, fake, fake, fake, fake,
                                  ctypes.c_void_p(0x1002), None) == _binding.MOE_ERR_INVALID_ARG


def test_self_test_and_error_read_check_their_arguments(lib):
    fake = ctypes.c_void_p(0x1000)
    odd = ctypes.c_void_p(0x1008)
    assert lib.moe_selftest_wait_timeout(fake, 0, None) == _binding.MOE_ERR_INVALID_ARG
    assert lib.moe_selftest_wait_timeout(fake, 2000001, None) == _binding.MOE_ERR_INVALID_ARG
    assert lib.moe_selftest_wait_timeout(None, 1000, None) == _binding.MOE_ERR_WORKSPACE
    assert lib.moe_selftest_wait_timeout(odd, 1000, None) == _binding.MOE_ERR_WORKSPACE
    detail = ctypes.c_int32(0)
    assert lib.moe_get_device_error(None, ctypes.byref(detail), None) == _binding.MOE_ERR_WORKSPACE
    assert lib.moe_get_device_error(odd, ctypes.byref(detail), None) == _binding.MOE_ERR_WORKSPACE
    assert lib.moe_workspace_init(None, 1 << 20, None) == _binding.MOE_ERR_WORKSPACE
    assert lib.moe_workspace_init(fake, 16, None) == _binding.MOE_ERR_WORKSPACE


def test_fused_calls_check_alignment_and_pointers(lib):
    fake = ctypes.c_void_p(0x1000)
    odd = ctypes.c_void_p(0x1008)  # 8-byte aligned, not 16
    s = ctypes.byref(_shape())
    # x and out must be 16-byte aligned
    assert lib.moe_route_layout_dispatch(s, fake, None, odd, fake, fake, fake, fake, fake, fake,
                                         fake, fake, fake, None, fake, 1 << 20,
                                         None) == _binding.MOE_ERR_INVALID_ARG
    assert lib.moe_route_layout_dispatch(s, fake, None, fake, fake, fake, fake, fake, fake, fake,
                                         fake, fake, odd, None, fake, 1 << 20,
                                         None) == _binding.MOE_ERR_INVALID_ARG
    # no logits, or a workspace that is too small
    assert lib.moe_route_layout(s, None, None, fake, fake, fake, fake, fake, fake, fake, fake,
                                fake, 1 << 20, None) == _binding.MOE_ERR_INVALID_ARG
    assert lib.moe_route_layout(s, fake, None, fake, fake, fake, fake, fake, fake, fake, fake,
                                fake, 64, None) == _binding.MOE_ERR_WORKSPACE
    # the round-robin router's outputs must be 4-byte aligned
    assert lib.moe_route_round_robin(s, ctypes.c_void_p(0x1002), fake,
                                     None) == _binding.MOE_ERR_INVALID_ARG
