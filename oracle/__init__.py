"""Float64 CPU oracle for the Mamba-1 selective scan (S6): Python marshalling around ssm_oracle.c.

TEST INFRASTRUCTURE ONLY. Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The product library (``selective_state_space_34_b200``)
never imports it, and this package never imports the product library: the two share no code.

The arithmetic lives in ``ssm_oracle.c`` (plain C, double precision, sequential loops in the
order the method is defined); this file only converts numpy arrays to contiguous float64 buffers
and calls it through ctypes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssm_oracle.c")
_LIB = os.path.join(_HERE, "libssm_oracle.so")
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_i64 = ctypes.c_int64


def build(force: bool = False) -> str:
    """Compile ssm_oracle.c into libssm_oracle.so (gcc, -O2, OpenMP, strict IEEE: no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-fno-fast-math",
               "-ffp-contract=off", "-Wall", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def bind(lib):
    """Declare the C signatures on a loaded copy of the oracle library and return it."""
    lib.ssm_oracle_softplus.restype = ctypes.c_double
    lib.ssm_oracle_softplus.argtypes = [ctypes.c_double]
    lib.ssm_oracle_sigmoid.restype = ctypes.c_double
    lib.ssm_oracle_sigmoid.argtypes = [ctypes.c_double]
    lib.ssm_oracle_silu.restype = ctypes.c_double
    lib.ssm_oracle_silu.argtypes = [ctypes.c_double]
    lib.ssm_oracle_zoh.restype = None
    lib.ssm_oracle_zoh.argtypes = [ctypes.c_double] * 3 + [_dp, _dp]
    lib.ssm_oracle_conv1d_silu.restype = None
    lib.ssm_oracle_conv1d_silu.argtypes = [_dp, _dp, _dp, _i64, _i64, _i64, _i64, _dp]
    common = [_dp] * 10 + [_i64] * 5 + [ctypes.c_int, ctypes.c_int, _dp, _dp]
    lib.ssm_oracle_fwd.restype = ctypes.c_int
    lib.ssm_oracle_fwd.argtypes = common + [_dp] * 5 + [ctypes.c_int]
    lib.ssm_oracle_bwd.restype = ctypes.c_int
    lib.ssm_oracle_bwd.argtypes = common + [_dp] * 2 + [_dp] * 12 + [ctypes.c_int]
    lib.ssm_oracle_ssd_fwd.restype = ctypes.c_int
    lib.ssm_oracle_ssd_fwd.argtypes = ([_dp] * 7 + [_i64] * 5 + [ctypes.c_int, ctypes.c_int] +
                                       [_dp] * 3 + [ctypes.c_int])
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = bind(ctypes.CDLL(build()))
    return _lib


def _in(a) -> Optional[np.ndarray]:
    if a is None:
        return None
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: Optional[np.ndarray]):
    if a is None:
        return None
    return a.ctypes.data_as(_dp)


def softplus(v: float) -> float:
    return _load().ssm_oracle_softplus(float(v))


def sigmoid(v: float) -> float:
    return _load().ssm_oracle_sigmoid(float(v))


def silu(v: float) -> float:
    return _load().ssm_oracle_silu(float(v))


def zoh(A: float, B: float, delta: float):
    """Exact zero-order hold of one diagonal entry: returns (A_bar, B_bar)."""
    ab, bb = ctypes.c_double(), ctypes.c_double()
    _load().ssm_oracle_zoh(float(A), float(B), float(delta), ctypes.byref(ab), ctypes.byref(bb))
    return ab.value, bb.value


def conv1d_silu(x, w, b=None):
    """x: (Bt, Dn, L); w: (Dn, K) newest-first taps; b: (Dn,) or None. Returns u (float64)."""
    x, w, b = _in(x), _in(w), _in(b)
    Bt, Dn, L = x.shape
    K = w.shape[1]
    u = np.empty_like(x)
    _load().ssm_oracle_conv1d_silu(_ptr(x), _ptr(w), _ptr(b), Bt, Dn, L, K, _ptr(u))
    return u


def _shapes(x, A_log, conv_w):
    Bt, Dn, L = x.shape
    N = A_log.shape[1]
    K = conv_w.shape[1] if conv_w is not None else 0
    return Bt, Dn, N, L, K


def fwd(x, dt, A_log, B, C, D=None, z=None, dt_bias=None, conv_w=None, conv_b=None,
        delta_softplus=True, want_u=False, want_y=False, n_threads=0, euler=False, h0=None,
        conv_hist=None, want_state=False):
    """Selective-scan forward. x, dt, z: (Bt, Dn, L); B, C: (Bt, N, L); A_log: (Dn, N);
    D, dt_bias, conv_b: (Dn,); conv_w: (Dn, K); h0: (Bt, Dn, N) carried state; conv_hist:
    (Bt, Dn, K-1) carried pre-conv inputs, newest-first. Returns out, or (out, extras) when extras
    are requested: 'u' (scan input), 'y' (pre-gate output incl. D*u), 'h_last' and
    'conv_hist' (the carried state after this chunk)."""
    x, dt, A_log, B, C = _in(x), _in(dt), _in(A_log), _in(B), _in(C)
    D, z, dt_bias, conv_w, conv_b = _in(D), _in(z), _in(dt_bias), _in(conv_w), _in(conv_b)
    h0, conv_hist = _in(h0), _in(conv_hist)
    Bt, Dn, N, L, K = _shapes(x, A_log, conv_w)
    out = np.empty_like(x)
    u = np.empty_like(x) if want_u else None
    y = np.empty_like(x) if want_y else None
    hl = np.empty((Bt, Dn, N)) if want_state else None
    ch = np.empty((Bt, Dn, max(K - 1, 0))) if (want_state and conv_w is not None) else None
    rc = _load().ssm_oracle_fwd(_ptr(x), _ptr(dt), _ptr(dt_bias), _ptr(A_log), _ptr(B), _ptr(C),
                                _ptr(D), _ptr(z), _ptr(conv_w), _ptr(conv_b), Bt, Dn, N, L, K,
                                int(bool(delta_softplus)), int(bool(euler)), _ptr(h0),
                                _ptr(conv_hist), _ptr(out), _ptr(u), _ptr(y), _ptr(hl), _ptr(ch),
                                int(n_threads))
    if rc != 0:
        raise MemoryError("ssm_oracle_fwd: allocation failed")
    if want_u or want_y or want_state:
        ex = {}
        if want_u:
            ex["u"] = u
        if want_y:
            ex["y"] = y
        if want_state:
            ex["h_last"] = hl
            ex["conv_hist"] = ch
        return out, ex
    return out


def bwd(x, dt, A_log, B, C, dout, D=None, z=None, dt_bias=None, conv_w=None, conv_b=None,
        delta_softplus=True, n_threads=0, euler=False, h0=None, conv_hist=None, dh_last=None):
    """Selective-scan backward (VJP of :func:`fwd` against ``dout`` and, optionally, ``dh_last``
    for the carried state). Returns a dict with dx, ddt, dA_log, dB, dC, dD, ddt_bias, dh0, and
    dz / dconv_w / dconv_b / dconv_hist where those inputs exist."""
    x, dt, A_log, B, C = _in(x), _in(dt), _in(A_log), _in(B), _in(C)
    D, z, dt_bias, conv_w, conv_b = _in(D), _in(z), _in(dt_bias), _in(conv_w), _in(conv_b)
    h0, conv_hist, dh_last = _in(h0), _in(conv_hist), _in(dh_last)
    dout = _in(dout)
    Bt, Dn, N, L, K = _shapes(x, A_log, conv_w)
    g = {
        "dx": np.empty_like(x), "ddt": np.empty_like(x), "dA_log": np.empty((Dn, N)),
        "dB": np.empty((Bt, N, L)), "dC": np.empty((Bt, N, L)), "dD": np.empty(Dn),
        "ddt_bias": np.empty(Dn),
    }
    if z is not None:
        g["dz"] = np.empty_like(x)
    g["dh0"] = np.empty((Bt, Dn, N))
    if conv_w is not None:
        g["dconv_w"] = np.empty((Dn, K))
        g["dconv_b"] = np.empty(Dn)
        g["dconv_hist"] = np.empty((Bt, Dn, max(K - 1, 0)))
    rc = _load().ssm_oracle_bwd(
        _ptr(x), _ptr(dt), _ptr(dt_bias), _ptr(A_log), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
        _ptr(conv_w), _ptr(conv_b), Bt, Dn, N, L, K, int(bool(delta_softplus)), int(bool(euler)),
        _ptr(h0), _ptr(conv_hist), _ptr(dout), _ptr(dh_last),
        _ptr(g["dx"]), _ptr(g["ddt"]), _ptr(g["dA_log"]), _ptr(g["dB"]), _ptr(g["dC"]),
        _ptr(g["dD"]), _ptr(g["ddt_bias"]), _ptr(g.get("dz")), _ptr(g.get("dconv_w")),
        _ptr(g.get("dconv_b")), _ptr(g["dh0"]), _ptr(g.get("dconv_hist")), int(n_threads))
    if rc != 0:
        raise MemoryError("ssm_oracle_bwd: allocation failed")
    return g


def ssd_fwd(x, dt, A_log, B, C, D=None, dt_bias=None, delta_softplus=True, euler=False, h0=None,
            want_state=False, n_threads=0):
    """Mamba-2 state-space-duality recurrence ("state-space models", "Mamba-2 and state-space
    duality"). x: (Bt, H, L, P); dt: (Bt, H, L); B, C: (Bt, L, N); A_log, D, dt_bias: (H,);
    h0: (Bt, H, N, P). Returns y (Bt, H, L, P), or (y, h_last) with want_state."""
    x, dt, A_log, B, C = _in(x), _in(dt), _in(A_log), _in(B), _in(C)
    D, dt_bias, h0 = _in(D), _in(dt_bias), _in(h0)
    Bt, H, L, P = x.shape
    N = B.shape[2]
    y = np.empty_like(x)
    hl = np.empty((Bt, H, N, P)) if want_state else None
    rc = _load().ssm_oracle_ssd_fwd(_ptr(x), _ptr(dt), _ptr(dt_bias), _ptr(A_log), _ptr(B), _ptr(C),
                                    _ptr(D), Bt, H, L, P, N, int(bool(delta_softplus)),
                                    int(bool(euler)), _ptr(h0), _ptr(y), _ptr(hl), int(n_threads))
    if rc != 0:
        raise MemoryError("ssm_oracle_ssd_fwd: allocation failed")
    return (y, hl) if want_state else y
