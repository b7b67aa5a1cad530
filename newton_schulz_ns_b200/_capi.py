"""ctypes declarations of libmuon_ns (include/muon_ns.h, include/muon_ns_testing.h).

Argument marshalling only: every step of the optimizer runs in the CUDA
library.  Importing this module loads the library and fails loudly if it is
missing or lacks a symbol; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

_PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG_DIR, "libmuon_ns.so")

MUON_F32, MUON_BF16, MUON_F16 = 0, 1, 2

STATUS = {
    0: "MUON_OK", 1: "MUON_INVALID_ARG", 2: "MUON_BAD_SHAPE", 3: "MUON_UNSUPPORTED_DTYPE",
    4: "MUON_MISALIGNED", 5: "MUON_WORKSPACE_TOO_SMALL", 6: "MUON_CUDA_ERROR", 7: "MUON_UNSUPPORTED_DEVICE",
}


class MuonError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)} ({status_string(status)})")


class MuonView(ctypes.Structure):
    _fields_ = [("ptr", ctypes.c_void_p), ("ld", ctypes.c_int64), ("batch_stride", ctypes.c_int64),
                ("dtype", ctypes.c_int32), ("reserved", ctypes.c_int32)]


class MuonBatch(ctypes.Structure):
    _fields_ = [("n", ctypes.c_int64), ("rows", ctypes.c_int64), ("cols", ctypes.c_int64),
                ("grad", MuonView), ("momentum", MuonView), ("ns_in", MuonView), ("ns_out", MuonView),
                ("weight", MuonView), ("weight_copy", MuonView),
                ("sumsq", ctypes.c_void_p), ("variance", ctypes.c_void_p), ("row_sumsq", ctypes.c_void_p),
                ("fan_out", ctypes.c_int64), ("fan_in", ctypes.c_int64)]


class MuonHparams(ctypes.Structure):
    _fields_ = [("mu", ctypes.c_float), ("nesterov", ctypes.c_int32), ("ns_eps", ctypes.c_float),
                ("a", ctypes.c_float), ("b", ctypes.c_float), ("c", ctypes.c_float),
                ("ns_steps", ctypes.c_int32), ("beta2", ctypes.c_float), ("nor_eps", ctypes.c_float),
                ("lr", ctypes.c_float), ("weight_decay", ctypes.c_float),
                ("abc_schedule", ctypes.POINTER(ctypes.c_float)),
                ("scale_mode", ctypes.c_int32), ("extra_scale_factor", ctypes.c_float),
                ("gram_restart", ctypes.c_int32), ("reserved", ctypes.c_int32)]


class MuonTestingOptions(ctypes.Structure):
    _fields_ = [("fused_small", ctypes.c_int32), ("max_waves", ctypes.c_int32), ("max_problems", ctypes.c_int32),
                ("pdl", ctypes.c_int32), ("overlap", ctypes.c_int32)]


MUON_SCALE_SPECTRAL, MUON_SCALE_RMS_NORM = 0, 1
SCALE_MODES = {"spectral": MUON_SCALE_SPECTRAL, "rms_norm": MUON_SCALE_RMS_NORM}
MUON_GRAM_RESTART_DEFAULT = 3


EXPORTS = ("muon_workspace_size", "muon_momentum_norm", "muon_ns_batched", "muon_gram_ns_batched",
           "normuon_update", "muon_workspace_error", "muon_status_string", "muon_version",
           "muon_testing_gemm", "muon_kernel_launches", "muon_momentum_norm_noalloc",
           "muon_testing_bounded_wait", "muon_ns_auto_batched", "muon_polar_express_schedule", "muon_update_scale",
           "muon_testing_set_options")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python newton_schulz_ns_b200/build.py` "
            "(the Muon step has no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    for name in EXPORTS:
        if not hasattr(lib, name):
            raise ImportError(f"{LIB_PATH} does not export {name}")
    P = ctypes.c_void_p
    B = ctypes.POINTER(MuonBatch)
    H = ctypes.POINTER(MuonHparams)
    lib.muon_workspace_size.argtypes = [B, ctypes.c_int, ctypes.c_int]
    lib.muon_workspace_size.restype = ctypes.c_size_t
    for fn in (lib.muon_momentum_norm, lib.muon_ns_batched, lib.muon_gram_ns_batched):
        fn.argtypes = [B, ctypes.c_int, H, P, ctypes.c_size_t, P]
        fn.restype = ctypes.c_int
    lib.muon_momentum_norm_noalloc.argtypes = [B, ctypes.c_int, H, P]
    lib.muon_momentum_norm_noalloc.restype = ctypes.c_int
    lib.muon_ns_auto_batched.argtypes = [B, ctypes.c_int, H, ctypes.c_float, P, ctypes.c_size_t, P]
    lib.muon_ns_auto_batched.restype = ctypes.c_int
    lib.normuon_update.argtypes = [B, ctypes.c_int, H, ctypes.c_int, P, ctypes.c_size_t, P]
    lib.normuon_update.restype = ctypes.c_int
    lib.muon_workspace_error.argtypes = [P, P, ctypes.POINTER(ctypes.c_int32)]
    lib.muon_workspace_error.restype = ctypes.c_int
    lib.muon_status_string.argtypes = [ctypes.c_int]
    lib.muon_status_string.restype = ctypes.c_char_p
    lib.muon_kernel_launches.argtypes = []
    lib.muon_kernel_launches.restype = ctypes.c_uint64
    lib.muon_version.argtypes = []
    lib.muon_version.restype = ctypes.c_char_p
    lib.muon_polar_express_schedule.argtypes = [ctypes.c_double, ctypes.c_int, ctypes.c_double,
                                                ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_double)]
    lib.muon_polar_express_schedule.restype = ctypes.c_int
    i64, i32, f32 = ctypes.c_int64, ctypes.c_int, ctypes.c_float
    lib.muon_testing_gemm.argtypes = [i32, i32, i32, i32, i32, i32,
                                      P, i64, i64, i32, P, i64, i64, i32, P, i64, i64, i32,
                                      P, i64, i64, i32, f32, f32, f32, f32, i32, P, f32, P, i32, i32,
                                      P, ctypes.c_size_t, P]
    lib.muon_testing_gemm.restype = ctypes.c_int
    lib.muon_testing_bounded_wait.argtypes = [ctypes.c_uint64, P, ctypes.c_size_t, P]
    lib.muon_testing_bounded_wait.restype = ctypes.c_int
    lib.muon_update_scale.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_int32, ctypes.c_float,
                                      ctypes.POINTER(ctypes.c_float)]
    lib.muon_update_scale.restype = ctypes.c_int
    lib.muon_testing_set_options.argtypes = [ctypes.POINTER(MuonTestingOptions), ctypes.POINTER(MuonTestingOptions)]
    lib.muon_testing_set_options.restype = ctypes.c_int
    return lib


lib = _load()


def status_string(status: int) -> str:
    return lib.muon_status_string(int(status)).decode()


def check(status: int, what: str) -> None:
    if status != 0:
        raise MuonError(status, what)
