"""ctypes declarations of the libgla C ABI (include/gla.h).

Loading fails loudly: there is no Python or CPU fallback for any entry point.
"""
from __future__ import annotations

import ctypes
import os
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
# GLA_CHECKS=1 in the environment selects the checking build (every call runs the library's checks).
LIB_PATH = os.path.join(HERE, "libgla_checks.so" if os.environ.get("GLA_CHECKS") == "1" else "libgla.so")

GLA_OK = 0
GLA_ERR_INVALID_ARG = 1
GLA_ERR_UNSUPPORTED = 2
GLA_ERR_WORKSPACE = 3
GLA_ERR_TIMEOUT = 5
STATUS_NAMES = {0: "GLA_OK", 1: "GLA_ERR_INVALID_ARG", 2: "GLA_ERR_UNSUPPORTED", 3: "GLA_ERR_WORKSPACE",
                4: "GLA_ERR_CUDA", 5: "GLA_ERR_TIMEOUT"}
DTYPE = {"f32": 0, "bf16": 1}
STATE_MODE = {"auto": 0, "materialized": 1, "nonmaterialized": 2}
IMPL = {"auto": 0, "simt": 1, "tc": 2}
GATE = {"channel": 0, "scalar": 1, "head": 2, "preact": 3}
FLAG_WS_FROM_FWD = 0x1
FLAG_CHECKS = 0x2

# Every function the header declares, for the ABI-completeness test.
EXPORTS = (
    "gla_fwd_workspace_size", "gla_bwd_workspace_size", "gla_fwd", "gla_bwd", "gla_step", "gla_chunk_cumsum",
    "gla_check_device_error", "gla_status_string", "gla_abi_version", "gla_resolve", "gla_launch_count",
    "gla_launch_count_reset", "gla_profile_enable", "gla_profile_read", "gla_profile_reset", "gla_fwd_noalloc",
    "gla_selftest_wait_timeout", "gla_last_device_error", "gla_fwd_workspace_bytes", "gla_bwd_workspace_bytes",
    "gla_segment_decay", "gla_state_combine", "gla_fwd_final_state", "gla_bwd_initial_grad",
    "gla_gsa_resolve", "gla_gsa_fwd_workspace_size", "gla_gsa_bwd_workspace_size", "gla_gsa_fwd", "gla_gsa_bwd",
    "gla_gsa_step",
)


class GlaDesc(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int64), ("H", ctypes.c_int64), ("L", ctypes.c_int64), ("Dk", ctypes.c_int64),
                ("Dv", ctypes.c_int64), ("dtype", ctypes.c_int32), ("chunk", ctypes.c_int32),
                ("subchunk", ctypes.c_int32), ("state_mode", ctypes.c_int32), ("impl", ctypes.c_int32),
                ("flags", ctypes.c_int32), ("gate", ctypes.c_int32), ("gate_tau", ctypes.c_float)]


_lock = threading.Lock()
_lib = None


class GlaError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__("%s failed: %s (%s)" % (what, STATUS_NAMES.get(status, status), status_string(status)))


def _declare(lib):
    vp, sz, i32, u64 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32, ctypes.c_uint64
    dp = ctypes.POINTER(GlaDesc)
    lib.gla_fwd_workspace_size.argtypes = [dp]
    lib.gla_fwd_workspace_size.restype = sz
    lib.gla_bwd_workspace_size.argtypes = [dp]
    lib.gla_bwd_workspace_size.restype = sz
    lib.gla_fwd.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.gla_fwd.restype = ctypes.c_int
    lib.gla_bwd.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.gla_bwd.restype = ctypes.c_int
    lib.gla_step.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp]
    lib.gla_step.restype = ctypes.c_int
    lib.gla_chunk_cumsum.argtypes = [dp, vp, vp, vp]
    lib.gla_chunk_cumsum.restype = ctypes.c_int
    lib.gla_check_device_error.argtypes = [vp]
    lib.gla_check_device_error.restype = ctypes.c_int
    lib.gla_last_device_error.argtypes = [vp]
    lib.gla_last_device_error.restype = ctypes.c_int
    lib.gla_fwd_workspace_bytes.argtypes = [dp]
    lib.gla_fwd_workspace_bytes.restype = sz
    lib.gla_bwd_workspace_bytes.argtypes = [dp]
    lib.gla_bwd_workspace_bytes.restype = sz
    lib.gla_selftest_wait_timeout.argtypes = [ctypes.c_longlong, vp]
    lib.gla_selftest_wait_timeout.restype = ctypes.c_int
    lib.gla_status_string.argtypes = [ctypes.c_int]
    lib.gla_status_string.restype = ctypes.c_char_p
    lib.gla_abi_version.restype = ctypes.c_int
    lib.gla_resolve.argtypes = [dp, ctypes.POINTER(i32), ctypes.POINTER(i32), ctypes.POINTER(i32),
                                ctypes.POINTER(i32)]
    lib.gla_resolve.restype = ctypes.c_int
    lib.gla_launch_count.restype = u64
    lib.gla_launch_count_reset.restype = None
    lib.gla_profile_enable.argtypes = [ctypes.c_int]
    lib.gla_profile_enable.restype = None
    lib.gla_profile_read.argtypes = [ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(u64),
                                     ctypes.POINTER(ctypes.c_double), ctypes.c_int]
    lib.gla_profile_read.restype = ctypes.c_int
    lib.gla_profile_reset.restype = None
    lib.gla_fwd_noalloc.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.gla_fwd_noalloc.restype = ctypes.c_int
    lib.gla_fwd_final_state.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.gla_fwd_final_state.restype = ctypes.c_int
    lib.gla_bwd_initial_grad.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.gla_bwd_initial_grad.restype = ctypes.c_int
    lib.gla_gsa_resolve.argtypes = [dp, i32, ctypes.POINTER(i32)]
    lib.gla_gsa_resolve.restype = ctypes.c_int
    lib.gla_gsa_fwd_workspace_size.argtypes = [dp, i32]
    lib.gla_gsa_fwd_workspace_size.restype = sz
    lib.gla_gsa_bwd_workspace_size.argtypes = [dp, i32]
    lib.gla_gsa_bwd_workspace_size.restype = sz
    lib.gla_gsa_fwd.argtypes = [dp, i32] + [vp] * 9 + [vp, sz, vp]
    lib.gla_gsa_fwd.restype = ctypes.c_int
    lib.gla_gsa_bwd.argtypes = [dp, i32] + [vp] * 15 + [vp, sz, vp]
    lib.gla_gsa_bwd.restype = ctypes.c_int
    lib.gla_gsa_step.argtypes = [dp, i32] + [vp] * 7 + [vp]
    lib.gla_gsa_step.restype = ctypes.c_int
    lib.gla_segment_decay.argtypes = [dp, vp, vp, vp]
    lib.gla_segment_decay.restype = ctypes.c_int
    i64 = ctypes.c_int64
    lib.gla_state_combine.argtypes = [i64, i64, i64, i64, vp, vp, vp, i32, i32, vp, vp]
    lib.gla_state_combine.restype = ctypes.c_int


def load(path: str = LIB_PATH):
    """Load libgla.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(path):
                raise ImportError("libgla.so not found at %s: build it with "
                                  "`python -m chunkwise_linear_rnn_gla_b200.build`" % path)
            lib = ctypes.CDLL(path)
            _declare(lib)
            _lib = lib
    return _lib


def status_string(status: int) -> str:
    try:
        return load().gla_status_string(int(status)).decode()
    except Exception:  # library not loadable: still produce a message
        return STATUS_NAMES.get(status, "unknown")
