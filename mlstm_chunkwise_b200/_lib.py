"""ctypes view of ``include/mlstm_fw.h``: loads the in-tree ``libmlstm_fw.so``.

There is no fallback: if the library is missing or fails to load, every call
raises.  Build it with ``python -m mlstm_chunkwise_b200.build``.
"""
from __future__ import annotations

import ctypes
import os
import threading

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmlstm_fw.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_DEVICE = range(6)
ERR_SCRATCH_TOO_SMALL = 6
DT_F32, DT_BF16 = 0, 1
GATE_EXP, GATE_SIGMOID, GATE_SIGMOID_PLAIN = 0, 1, 2
ALGO_AUTO, ALGO_SIMT, ALGO_TC, ALGO_TC_FUSED = 0, 1, 2, 3
KERNEL_COUNT = 9

_vp = ctypes.c_void_p
_i = ctypes.c_int
_sz = ctypes.c_size_t

# name -> (restype, argtypes), in the order of include/mlstm_fw.h
SIGNATURES = {
    "mlstm_fw_workspace_size": (_i, [_i, _i, _i, _i, _i, _i, _i, _i, ctypes.POINTER(_sz)]),
    "mlstm_fw": (_i, [_vp] * 12 + [_i] * 9 + [_vp, _sz, _vp]),
    "mlstm_fw_substep_workspace_size": (_i, [_i, _i, _i, _i, _i, _i, _i, _i,
                                             ctypes.POINTER(_sz)]),
    "mlstm_fw_chunk_states": (_i, [_vp] * 13 + [_i] * 9 + [_vp, _sz, _vp]),
    "mlstm_fw_parallel": (_i, [_vp] * 11 + [_i] * 9 + [_vp, _sz, _vp]),
    "mlstm_fw_static_scratch": (_i, [_vp] * 12 + [_i] * 9 + [_vp]),
    "mlstm_fw_static_scratch_capacity": (_sz, []),
    "mlstm_bw_workspace_size": (_i, [_i] * 7 + [ctypes.POINTER(_sz)]),
    "mlstm_bw": (_i, [_vp] * 17 + [_i] * 8 + [_vp, _sz, _vp]),
    "mlstm_train_sizes": (_i, [_i] * 6 + [ctypes.POINTER(_sz)] * 3),
    "mlstm_fw_train": (_i, [_vp] * 13 + [_sz] + [_i] * 7 + [_vp, _sz, _vp]),
    "mlstm_bw_saved": (_i, [_vp] * 10 + [_sz] + [_vp] * 9 + [_i] * 7 + [_vp, _sz, _vp]),
    "mlstm_step": (_i, [_vp] * 9 + [_i] * 6 + [_vp]),
    "mlstm_last_device_error": (_i, [_vp]),
    "mlstm_last_device_error_word": (ctypes.c_uint32, []),
    "mlstm_set_watchdog": (None, [ctypes.c_uint64]),
    "mlstm_watchdog_selftest": (_i, [_vp]),
    "mlstm_kernel_launches": (ctypes.c_uint64, []),
    "mlstm_profile_enable": (None, [_i]),
    "mlstm_profile_read": (_i, [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_uint64),
                                _i]),
    "mlstm_kernel_name": (ctypes.c_char_p, [_i]),
    "mlstm_status_string": (ctypes.c_char_p, [_i]),
    "mlstm_abi_version": (_i, []),
}

_lock = threading.Lock()
_lib = None


class MlstmError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


def open_library(path: str):
    """Load a build of the library at ``path`` (for instance the bounds-checked
    ``libmlstm_fw_debug.so``) with the signatures of include/mlstm_fw.h."""
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing")
    h = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(h, name)
        fn.restype = res
        fn.argtypes = args
    return h


def lib():
    """The loaded library (loads it on first use; raises if it is missing)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"{LIB_PATH} is missing: build it with `python -m mlstm_chunkwise_b200.build`")
            h = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(h, name)
                fn.restype = res
                fn.argtypes = args
            _lib = h
    return _lib


def status_string(status: int) -> str:
    return lib().mlstm_status_string(int(status)).decode()


def check(status: int, where: str) -> None:
    if status != OK:
        raise MlstmError(status, where)
