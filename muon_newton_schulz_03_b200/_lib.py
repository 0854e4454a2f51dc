"""ctypes loader for libmuon_ns.so (the C ABI declared in include/muon_ns.h).

The library is built in-tree by ``muon_newton_schulz_03_b200.build``; a
missing or stale library is rebuilt on first load. If it cannot be built or
loaded, every entry point raises: there is no fallback implementation.
"""

from __future__ import annotations

import ctypes
import os
import threading

from . import build as _build

_LOCK = threading.Lock()
_LIB = None

c_int = ctypes.c_int
c_float = ctypes.c_float
c_double = ctypes.c_double
c_size_t = ctypes.c_size_t
c_void_p = ctypes.c_void_p
c_char_p = ctypes.c_char_p
P = ctypes.POINTER


class MuonConfig(ctypes.Structure):
    _fields_ = [
        ("scale_mode", c_int),
        ("extra_scale", c_float),
        ("ns_precision", c_int),
        ("check_nonfinite", c_int),
        ("num_sms", c_int),
        ("workspace_cap_bytes", c_size_t),
        ("wait_timeout_s", c_double),
        ("small_path", c_int),
        ("ns_algorithm", c_int),
        ("deterministic", c_int),
        ("cta_pair", c_int),
        ("fused_apply", c_int),
    ]


# name -> (restype, argtypes)
_SIGNATURES = {
    "muon_config_init": (c_int, [P(MuonConfig)]),
    "muon_init": (c_int, [c_int, P(MuonConfig), P(c_void_p)]),
    "muon_destroy": (c_int, [c_void_p]),
    "muon_step": (c_int, [c_void_p, P(c_void_p), P(c_void_p), P(c_void_p), P(ctypes.c_int32), c_int,
                          c_float, c_float, c_int, c_float, c_int, P(c_float), c_void_p]),
    "muon_step_schedule": (c_int, [c_void_p, P(c_void_p), P(c_void_p), P(c_void_p), P(ctypes.c_int32), c_int,
                                   c_float, c_float, c_int, c_float, c_int, P(c_float), c_int, c_void_p]),
    "muon_qk_clip": (c_int, [c_void_p, P(c_void_p), P(ctypes.c_int32), P(c_void_p), c_int, c_float, c_void_p]),
    "muon_step_host": (c_int, [c_void_p, P(c_void_p), P(c_void_p), P(c_void_p), P(ctypes.c_int32), c_int,
                               c_float, c_float, c_int, c_float, c_int, P(c_float), c_void_p]),
    "muon_momentum_norm": (c_int, [c_void_p, P(c_void_p), P(c_void_p), P(c_void_p), c_void_p,
                                   P(ctypes.c_int32), c_int, c_float, c_int, c_void_p]),
    "muon_newton_schulz": (c_int, [c_void_p, P(c_void_p), P(c_void_p), c_void_p, P(ctypes.c_int32), c_int,
                                   c_int, P(c_float), c_void_p]),
    "muon_apply": (c_int, [c_void_p, P(c_void_p), P(c_void_p), c_void_p, P(ctypes.c_int32), c_int,
                           c_float, c_float, c_void_p]),
    "muon_plan_query": (c_int, [P(ctypes.c_int32), c_int, c_int, c_int, P(ctypes.c_int64), P(ctypes.c_int64),
                                P(ctypes.c_int32), P(ctypes.c_int32), P(ctypes.c_int64)]),
    "muon_plan_groups": (c_int, [P(ctypes.c_int32), c_int, c_int, c_int, c_size_t, P(ctypes.c_int32),
                                 P(ctypes.c_int32), P(ctypes.c_int64), P(ctypes.c_int64)]),
    "muon_workspace_size": (c_int, [c_void_p, P(ctypes.c_int32), c_int, P(c_size_t)]),
    "muon_workspace_ptr": (c_int, [c_void_p, P(c_void_p), P(c_size_t)]),
    "muon_get_status": (c_int, [c_void_p, c_void_p, P(ctypes.c_int32), P(ctypes.c_uint64)]),
    "muon_last_launch_count": (c_int, [c_void_p, P(ctypes.c_int32)]),
    "muon_profile_enable": (c_int, [c_void_p, c_int]),
    "muon_profile_read": (c_int, [c_void_p, P(ctypes.c_int32), P(c_float), c_int, P(ctypes.c_int32)]),
    "muon_newton_schulz_noalloc": (c_int, [P(c_void_p), P(c_void_p), c_void_p, P(ctypes.c_int32), c_int, c_int,
                                           P(c_float), c_void_p, c_void_p]),
    "muon_last_error": (c_char_p, []),
    "muon_version": (c_char_p, []),
}

EXPORTED = tuple(_SIGNATURES)


def lib_path() -> str:
    return _build.LIB_PATH


def load():
    """Load (building first if needed) and return the ctypes library."""
    global _LIB
    with _LOCK:
        if _LIB is not None:
            return _LIB
        if _build.needs_build():
            _build.build()
        if not os.path.exists(_build.LIB_PATH):
            raise RuntimeError(f"{_build.LIB_PATH} is missing and could not be built")
        lib = ctypes.CDLL(_build.LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = lib
        return lib


class MuonError(RuntimeError):
    """A non-zero status from the C ABI."""

    NAMES = {
        1: "MUON_ERR_INVALID_ARG", 2: "MUON_ERR_CUDA", 3: "MUON_ERR_OOM", 4: "MUON_ERR_TIMEOUT",
        5: "MUON_ERR_NONFINITE", 6: "MUON_ERR_NO_DEVICE", 7: "MUON_ERR_UNSUPPORTED",
    }

    def __init__(self, code: int, message: str):
        self.code = code
        super().__init__(f"{self.NAMES.get(code, code)}: {message}")


def check(code: int):
    if code != 0:
        raise MuonError(code, load().muon_last_error().decode(errors="replace"))
