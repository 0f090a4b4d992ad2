"""ctypes mirror of include/ssm_scan.h. Declarations only: every computation happens in the CUDA
library. Loading fails loudly when the library has not been built; there is no fallback."""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libssm_scan.so")

SSM_F32, SSM_BF16 = 0, 1
SSM_ZOH, SSM_EULER = 0, 1
SSM_SCAN_LANES, SSM_SCAN_CHUNKED = 0, 1
SSM_SSD_AUTO, SSM_SSD_THREE_PASS, SSM_SSD_FUSED = 0, 1, 2
SSM_STATE_CHUNK = 16
SSM_NOALLOC_SCRATCH_BYTES = 72 << 20
SSM_ERR_TIMEOUT = 8

STATUS = {
    0: "SSM_OK", 1: "SSM_ERR_NULL", 2: "SSM_ERR_SHAPE", 3: "SSM_ERR_ALIGN", 4: "SSM_ERR_DTYPE",
    5: "SSM_ERR_UNSUPPORTED", 6: "SSM_ERR_CUDA", 7: "SSM_ERR_WORKSPACE", 8: "SSM_ERR_TIMEOUT",
}


class FwdArgs(ctypes.Structure):
    _fields_ = [
        ("x", ctypes.c_void_p), ("dt", ctypes.c_void_p), ("dt_bias", ctypes.c_void_p),
        ("A_log", ctypes.c_void_p), ("B", ctypes.c_void_p), ("C", ctypes.c_void_p),
        ("D", ctypes.c_void_p), ("z", ctypes.c_void_p), ("conv_w", ctypes.c_void_p),
        ("conv_b", ctypes.c_void_p), ("out", ctypes.c_void_p), ("chunk_states", ctypes.c_void_p),
        ("u_out", ctypes.c_void_p),
        ("Bt", ctypes.c_int64), ("Dn", ctypes.c_int64), ("N", ctypes.c_int64), ("L", ctypes.c_int64),
        ("K", ctypes.c_int32), ("in_dtype", ctypes.c_int32), ("out_dtype", ctypes.c_int32),
        ("delta_softplus", ctypes.c_int32),
        ("h0", ctypes.c_void_p), ("conv_hist", ctypes.c_void_p), ("h_last", ctypes.c_void_p),
        ("conv_hist_out", ctypes.c_void_p), ("discretization", ctypes.c_int32),
        ("n_segments", ctypes.c_int32), ("workspace", ctypes.c_void_p),
        ("workspace_bytes", ctypes.c_size_t), ("scan_form", ctypes.c_int32),
    ]


class BwdArgs(ctypes.Structure):
    _fields_ = [
        ("fwd", FwdArgs), ("dout", ctypes.c_void_p), ("chunk_states", ctypes.c_void_p),
        ("dx", ctypes.c_void_p), ("ddt", ctypes.c_void_p), ("dz", ctypes.c_void_p),
        ("dA_log", ctypes.c_void_p), ("dB", ctypes.c_void_p), ("dC", ctypes.c_void_p),
        ("dD", ctypes.c_void_p), ("ddt_bias", ctypes.c_void_p), ("dconv_w", ctypes.c_void_p),
        ("dconv_b", ctypes.c_void_p), ("workspace", ctypes.c_void_p),
        ("workspace_bytes", ctypes.c_size_t), ("timing_events", ctypes.c_void_p),
        ("dh_last", ctypes.c_void_p), ("dh0", ctypes.c_void_p), ("dconv_hist", ctypes.c_void_p),
    ]


class StepArgs(ctypes.Structure):
    _fields_ = [
        ("x", ctypes.c_void_p), ("dt", ctypes.c_void_p), ("dt_bias", ctypes.c_void_p),
        ("A_log", ctypes.c_void_p), ("B", ctypes.c_void_p), ("C", ctypes.c_void_p),
        ("D", ctypes.c_void_p), ("z", ctypes.c_void_p), ("conv_w", ctypes.c_void_p),
        ("conv_b", ctypes.c_void_p), ("h", ctypes.c_void_p), ("conv_hist", ctypes.c_void_p),
        ("out", ctypes.c_void_p), ("Bt", ctypes.c_int64), ("Dn", ctypes.c_int64),
        ("N", ctypes.c_int64), ("K", ctypes.c_int32), ("in_dtype", ctypes.c_int32),
        ("out_dtype", ctypes.c_int32), ("delta_softplus", ctypes.c_int32),
        ("discretization", ctypes.c_int32),
    ]


class SsdArgs(ctypes.Structure):
    _fields_ = [
        ("x", ctypes.c_void_p), ("dt", ctypes.c_void_p), ("dt_bias", ctypes.c_void_p),
        ("A_log", ctypes.c_void_p), ("B", ctypes.c_void_p), ("C", ctypes.c_void_p),
        ("D", ctypes.c_void_p), ("h0", ctypes.c_void_p), ("y", ctypes.c_void_p),
        ("h_last", ctypes.c_void_p),
        ("Bt", ctypes.c_int64), ("H", ctypes.c_int64), ("L", ctypes.c_int64), ("P", ctypes.c_int64),
        ("N", ctypes.c_int64),
        ("in_dtype", ctypes.c_int32), ("out_dtype", ctypes.c_int32),
        ("delta_softplus", ctypes.c_int32), ("discretization", ctypes.c_int32),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
        ("timing_events", ctypes.c_void_p), ("form", ctypes.c_int32),
    ]


# (name, restype, argtypes) of every exported function in include/ssm_scan.h
SIGNATURES = [
    ("ssm_num_state_chunks", ctypes.c_int64, [ctypes.c_int64]),
    ("ssm_scan_fwd", ctypes.c_int, [ctypes.POINTER(FwdArgs), ctypes.c_void_p]),
    ("ssm_fwd_workspace_size", ctypes.c_size_t, [ctypes.POINTER(FwdArgs)]),
    ("ssm_bwd_workspace_size", ctypes.c_size_t, [ctypes.POINTER(BwdArgs)]),
    ("ssm_workspace_size", ctypes.c_size_t, [ctypes.POINTER(FwdArgs), ctypes.c_int32]),
    ("ssm_scan_bwd", ctypes.c_int, [ctypes.POINTER(BwdArgs), ctypes.c_void_p]),
    ("ssm_scan_bwd_noalloc", ctypes.c_int, [ctypes.POINTER(BwdArgs), ctypes.c_void_p]),
    ("ssm_scan_step", ctypes.c_int, [ctypes.POINTER(StepArgs), ctypes.c_void_p]),
    ("ssm_ssd_workspace_size", ctypes.c_size_t, [ctypes.POINTER(SsdArgs)]),
    ("ssm_ssd_fwd", ctypes.c_int, [ctypes.POINTER(SsdArgs), ctypes.c_void_p]),
    ("ssm_ssd_check", ctypes.c_int, [ctypes.POINTER(SsdArgs), ctypes.c_void_p]),
    ("ssm_wait_selftest", ctypes.c_int, [ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p]),
    ("ssm_conv1d_silu", ctypes.c_int,
     [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
      ctypes.c_int64, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
      ctypes.c_void_p]),
    ("ssm_status_string", ctypes.c_char_p, [ctypes.c_int]),
    ("ssm_last_cuda_error", ctypes.c_int, []),
]

_lib = None


def load():
    """Load libssm_scan.so and declare its signatures. Raises if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                "libssm_scan.so is not built (expected at %s); run "
                "`python -m selective_state_space_34_b200.build`" % LIB_PATH)
        lib = ctypes.CDLL(LIB_PATH)
        for name, res, args in SIGNATURES:
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


class SSMError(RuntimeError):
    def __init__(self, fn: str, code: int):
        lib = load()
        msg = lib.ssm_status_string(code).decode()
        if code == 6:
            msg += " (cudaError %d)" % lib.ssm_last_cuda_error()
        super().__init__("%s: %s" % (fn, msg))
        self.code = code


def check(fn: str, code: int) -> None:
    if code != 0:
        raise SSMError(fn, code)
