"""ctypes view of the C ABI in include/replay.h (libreplay.so, built in-tree).

Loading fails loudly when the library is missing: there is no other implementation.
"""

from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libreplay.so")

REPLAY_OK = 0
REPLAY_EINVAL = -1
REPLAY_EALIGN = -2
REPLAY_ECUDA = -3
REPLAY_EPENDING = -4
REPLAY_ENOPENDING = -5
REPLAY_EDEVICE = -6
REPLAY_ENOMEM = -7
REPLAY_ESCRATCH = -8

# size of the library's fixed query scratch (replay_verify_static_scratch)
STATIC_SCRATCH_BYTES = 32 << 20

REPLAY_F32 = 0
REPLAY_BF16 = 1
REPLAY_CKPT_F32 = 0
REPLAY_CKPT_F32_FP8READ = 1
REPLAY_CKPT_F32_FP4READ = 2

DEV_WAIT_TIMEOUT = 1
DEV_POINTER = 2
DEV_ROLLBACK = 4
DEV_SNAPSHOT = 8


class ReplayError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {strerror(code)} ({code})")


class CConfig(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("heads", ctypes.c_int32), ("groups", ctypes.c_int32),
                ("P", ctypes.c_int32), ("N", ctypes.c_int32), ("L", ctypes.c_int32),
                ("max_pos", ctypes.c_int32), ("io", ctypes.c_int32), ("ckpt", ctypes.c_int32)]


class CBuffers(ctypes.Structure):
    _fields_ = [("S0", ctypes.c_void_p), ("S0_codes", ctypes.c_void_p), ("S0_scale", ctypes.c_void_p),
                ("ring_k", ctypes.c_void_p), ("ring", ctypes.c_void_p), ("qpack", ctypes.c_void_p),
                ("counts", ctypes.c_void_p), ("status", ctypes.c_void_p)]


_lib = None


def load() -> ctypes.CDLL:
    """The loaded libreplay.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m linear_attention_decode_replay_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    cfgp = ctypes.POINTER(CConfig)
    sig = {
        "replay_ring_capacity": (i32, [cfgp]),
        "replay_ring_record_bytes": (i32, [cfgp]),
        "replay_ring_k_record_bytes": (i32, [cfgp]),
        "replay_init": (ctypes.c_int, [cfgp, ctypes.POINTER(CBuffers), vp, ctypes.POINTER(vp)]),
        "replay_step": (ctypes.c_int, [vp, vp, vp, vp, vp, vp, vp, vp, vp]),
        "replay_verify": (ctypes.c_int, [vp, i32, vp, vp, vp, vp, vp, vp, vp, vp]),
        "replay_verify_static_scratch": (ctypes.c_int, [vp, i32, vp, vp, vp, vp, vp, vp, vp, vp]),
        "replay_rollback": (ctypes.c_int, [vp, vp, vp]),
        "replay_append_slots": (ctypes.c_int, [vp, vp, vp]),
        "replay_snapshot_bytes": (i64, [cfgp]),
        "replay_export": (ctypes.c_int, [vp, vp, i32, vp, vp]),
        "replay_import": (ctypes.c_int, [vp, vp, i32, vp, vp]),
        "replay_step_resident": (ctypes.c_int, [vp, vp, vp, vp, vp]),
        "replay_verify_resident": (ctypes.c_int, [vp, i32, vp, vp, vp, vp]),
        "replay_flush": (ctypes.c_int, [vp, vp, vp]),
        "replay_read_counts": (ctypes.c_int, [vp, vp, vp]),
        "replay_check_status": (ctypes.c_int, [vp, ctypes.POINTER(i32), vp]),
        "replay_destroy": (None, [vp]),
        "eager_step": (ctypes.c_int, [cfgp, vp, vp, vp, vp, vp, vp, vp, vp]),
        "eager_step_fp8": (ctypes.c_int, [cfgp, vp, vp, vp, vp, vp, vp, vp, vp, vp]),
        "replay_quantize_rows_e4m3": (ctypes.c_int, [vp, i64, i32, vp, vp, vp]),
        "replay_quantize_rows_e2m1": (ctypes.c_int, [vp, i64, i32, vp, vp, vp]),
        "replay_strerror": (ctypes.c_char_p, [ctypes.c_int]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def strerror(code: int) -> str:
    return load().replay_strerror(code).decode()


def check(code: int, what: str) -> None:
    if code != REPLAY_OK:
        raise ReplayError(code, what)
