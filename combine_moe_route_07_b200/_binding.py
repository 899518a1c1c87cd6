"""ctypes binding to libmoe_route07.so (include/moe_route07.h).

Argument marshalling only: every function here forwards device pointers,
sizes and the current CUDA stream to the C ABI and maps the status code to an
exception.  There is no fallback: if the library is missing the import of
the entry points fails loudly.
"""
import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.environ.get("MOE_ROUTE07_LIB", os.path.join(PKG, "libmoe_route07.so"))

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_UNSUPPORTED = 2
MOE_ERR_WORKSPACE = 3
MOE_ERR_CUDA = 4
MOE_ERR_DEVICE_RANGE = 5
MOE_ERR_DEVICE_TIMEOUT = 6
MOE_ERR_DEVICE_NAN = 7

MOE_F_RENORM = 0x1
MOE_F_FP8 = 0x2
MOE_F_SRC_LAYOUT = 0x4

# Every extern "C" symbol of include/moe_route07.h.
EXPORTS = (
    "moe_abi_version", "moe_status_string", "moe_layout_rows", "moe_workspace_bytes",
    "moe_workspace_init", "moe_route", "moe_layout", "moe_dispatch", "moe_combine",
    "moe_get_device_error", "moe_layout_noalloc", "moe_route_layout",
    "moe_route_layout_dispatch", "moe_layout_src", "moe_route_limited",
    "moe_bias_update", "moe_layout_remote_first", "moe_route_round_robin",
    "moe_selftest_wait_timeout",
)


class MoeShapeC(ctypes.Structure):
    _fields_ = [("tokens", ctypes.c_int32), ("hidden", ctypes.c_int32),
                ("experts", ctypes.c_int32), ("k", ctypes.c_int32), ("ranks", ctypes.c_int32),
                ("capacity", ctypes.c_int32), ("align", ctypes.c_int32),
                ("flags", ctypes.c_uint32)]


class MoeError(RuntimeError):
    def __init__(self, status, what, detail=None):
        self.status = status
        self.detail = detail
        msg = f"{what}: {status_string(status)} (status {status})"
        if detail is not None:
            msg += f", detail {detail}"
        super().__init__(msg)


_lib = None


def lib(path: str = None):
    """Load the library (once) and declare every entry point's signature."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise ImportError(f"{p} is missing: build it with `python -m combine_moe_route_07_b200.build`"
                          " (or __graft_entry__.build()); there is no fallback")
    L = ctypes.CDLL(p)
    vp, sz, i32, i64 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32, ctypes.c_int64
    sp = ctypes.POINTER(MoeShapeC)
    L.moe_abi_version.argtypes, L.moe_abi_version.restype = [], i32
    L.moe_status_string.argtypes, L.moe_status_string.restype = [i32], ctypes.c_char_p
    L.moe_layout_rows.argtypes, L.moe_layout_rows.restype = [sp], i64
    L.moe_workspace_bytes.argtypes, L.moe_workspace_bytes.restype = [sp], sz
    L.moe_workspace_init.argtypes, L.moe_workspace_init.restype = [vp, sz, vp], i32
    L.moe_route.argtypes = [sp, vp, vp, vp, vp, vp, sz, vp]
    L.moe_route.restype = i32
    L.moe_layout.argtypes = [sp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.moe_layout.restype = i32
    L.moe_route_layout.argtypes = [sp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.moe_route_layout.restype = i32
    L.moe_route_layout_dispatch.argtypes = [sp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                            vp, sz, vp]
    L.moe_route_layout_dispatch.restype = i32
    L.moe_dispatch.argtypes = [sp, vp, vp, vp, vp, vp, sz, vp]
    L.moe_dispatch.restype = i32
    L.moe_combine.argtypes = [sp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.moe_combine.restype = i32
    L.moe_layout_remote_first.argtypes = [sp, vp, i32, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.moe_layout_remote_first.restype = i32
    L.moe_route_round_robin.argtypes = [sp, vp, vp, vp]
    L.moe_route_round_robin.restype = i32
    L.moe_selftest_wait_timeout.argtypes = [vp, ctypes.c_uint32, vp]
    L.moe_selftest_wait_timeout.restype = i32
    L.moe_bias_update.argtypes = [sp, vp, ctypes.c_float, vp, vp]
    L.moe_bias_update.restype = i32
    L.moe_route_limited.argtypes = [sp, vp, vp, i32, vp, vp, vp, sz, vp]
    L.moe_route_limited.restype = i32
    L.moe_layout_src.argtypes = [sp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.moe_layout_src.restype = i32
    L.moe_layout_noalloc.argtypes = [sp, vp, vp, vp, vp, vp, vp, vp, vp]
    L.moe_layout_noalloc.restype = i32
    L.moe_get_device_error.argtypes = [vp, ctypes.POINTER(i32), vp]
    L.moe_get_device_error.restype = i32
    if path is None:
        _lib = L
    return L


def status_string(status: int) -> str:
    try:
        return lib().moe_status_string(int(status)).decode()
    except ImportError:
        return "unknown"
