"""PyTorch-facing marshalling for the C ABI (include/ssm_scan.h).

Each function validates tensor devices/dtypes/contiguity, allocates outputs (and the backward's
scratch) with torch on the inputs' device, fills the C argument struct with raw device pointers
and calls the library on torch's current CUDA stream. Nothing is computed here.
"""
from __future__ import annotations

import ctypes
from typing import Dict, Optional

import torch

from . import _abi

_DT = {torch.float32: _abi.SSM_F32, torch.bfloat16: _abi.SSM_BF16}


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _need_cuda(name: str, t: torch.Tensor) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a torch.Tensor" % name)
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor (the library has no CPU path)" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)


def _opt(name, t, dtype=None):
    if t is None:
        return None
    _need_cuda(name, t)
    if dtype is not None and t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    return t


def _stream_handle(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def ssm_num_state_chunks(L: int) -> int:
    return int(_abi.load().ssm_num_state_chunks(int(L)))


_DISC = {"zoh": _abi.SSM_ZOH, "euler": _abi.SSM_EULER}


_SCAN = {"lanes": _abi.SSM_SCAN_LANES, "chunked": _abi.SSM_SCAN_CHUNKED}
_SSD_FORM = {"auto": _abi.SSM_SSD_AUTO, "three_pass": _abi.SSM_SSD_THREE_PASS, "fused": _abi.SSM_SSD_FUSED}


def _fwd_args(x, dt, A_log, B, C, D, z, dt_bias, conv_w, conv_b, delta_softplus, out_dtype,
              discretization="zoh", h0=None, conv_hist=None, scan_form="lanes"):
    for n, t in (("x", x), ("dt", dt), ("A_log", A_log), ("B", B), ("C", C)):
        _need_cuda(n, t)
    if x.dtype not in _DT:
        raise TypeError("x must be float32 or bfloat16")
    act = x.dtype
    for n, t in (("dt", dt), ("B", B), ("C", C)):
        if t.dtype != act:
            raise TypeError("%s must have the activation dtype %s" % (n, act))
    _opt("z", z, act)
    for n, t in (("A_log", A_log), ("D", D), ("dt_bias", dt_bias), ("conv_w", conv_w),
                 ("conv_b", conv_b)):
        _opt(n, t, torch.float32)
    if x.dim() != 3 or B.dim() != 3 or A_log.dim() != 2:
        raise ValueError("x must be (Bt, Dn, L), B/C (Bt, N, L), A_log (Dn, N)")
    Bt, Dn, L = x.shape
    N = A_log.shape[1]
    if tuple(dt.shape) != (Bt, Dn, L) or (z is not None and tuple(z.shape) != (Bt, Dn, L)):
        raise ValueError("dt and z must have the shape of x")
    if tuple(B.shape) != (Bt, N, L) or tuple(C.shape) != (Bt, N, L) or A_log.shape[0] != Dn:
        raise ValueError("B, C must be (Bt, N, L) and A_log (Dn, N)")
    for n, t in (("D", D), ("dt_bias", dt_bias), ("conv_b", conv_b)):
        if t is not None and tuple(t.shape) != (Dn,):
            raise ValueError("%s must be (Dn,)" % n)
    K = 0
    if conv_w is not None:
        if conv_w.dim() != 2 or conv_w.shape[0] != Dn:
            raise ValueError("conv_w must be (Dn, K)")
        K = conv_w.shape[1]
    od = act if out_dtype is None else out_dtype
    if od not in _DT:
        raise TypeError("out_dtype must be float32 or bfloat16")
    a = _abi.FwdArgs()
    a.x, a.dt, a.dt_bias, a.A_log = _ptr(x), _ptr(dt), _ptr(dt_bias), _ptr(A_log)
    a.B, a.C, a.D, a.z = _ptr(B), _ptr(C), _ptr(D), _ptr(z)
    a.conv_w, a.conv_b = _ptr(conv_w), _ptr(conv_b)
    a.Bt, a.Dn, a.N, a.L, a.K = Bt, Dn, N, L, K
    a.in_dtype, a.out_dtype = _DT[act], _DT[od]
    a.delta_softplus = 1 if delta_softplus else 0
    if discretization not in _DISC:
        raise ValueError("discretization must be 'zoh' or 'euler'")
    a.discretization = _DISC[discretization]
    if scan_form not in _SCAN:
        raise ValueError("scan_form must be 'lanes' or 'chunked'")
    a.scan_form = _SCAN[scan_form]
    if h0 is not None:
        _opt("h0", h0, torch.float32)
        if tuple(h0.shape) != (Bt, Dn, N):
            raise ValueError("h0 must be (Bt, Dn, N)")
        a.h0 = _ptr(h0)
    if conv_hist is not None:
        _opt("conv_hist", conv_hist, act)
        if conv_w is None or tuple(conv_hist.shape) != (Bt, Dn, K - 1):
            raise ValueError("conv_hist must be (Bt, Dn, K-1) and needs conv_w")
        a.conv_hist = _ptr(conv_hist)
    return a, od


def ssm_scan_fwd(x, dt, A_log, B, C, D=None, z=None, dt_bias=None, conv_w=None, conv_b=None,
                 delta_softplus: bool = True, out_dtype=None, save_states: bool = False,
                 return_u: bool = False, out: Optional[torch.Tensor] = None,
                 discretization: str = "zoh", h0=None, conv_hist=None, return_state: bool = False,
                 n_segments: int = 0, scan_form: str = "lanes"):
    """Fused forward. Returns ``out`` or a dict with ``out`` and, when asked, ``chunk_states``
    ((Bt, Dn, ceil(L/16), N) fp32, for ssm_scan_bwd), ``u`` (the scan input), and ``h_last`` /
    ``conv_hist`` (the state to carry into the next chunk). ``h0`` / ``conv_hist`` carry the state
    in from a previous chunk; ``discretization`` is "zoh" (exact) or "euler" (Delta * B).
    ``n_segments`` splits the sequence across CTAs (0/1: one pass; k >= 2: up to k segments;
    -1: the library decides from the device and the shape); the scratch it needs is allocated
    here. ``scan_form`` lays a one-pass scan out as "lanes" (a channel's states over lanes, each
    walking the sequence) or "chunked" (lanes over time steps, a warp-shuffle scan per chunk)."""
    a, od = _fwd_args(x, dt, A_log, B, C, D, z, dt_bias, conv_w, conv_b, delta_softplus, out_dtype,
                      discretization, h0, conv_hist, scan_form)
    Bt, Dn, L = x.shape
    N = A_log.shape[1]
    if out is None:
        out = torch.empty((Bt, Dn, L), dtype=od, device=x.device)
    else:
        _opt("out", out, od)
    a.out = _ptr(out)
    res: Dict[str, torch.Tensor] = {"out": out}
    if save_states:
        st = torch.empty((Bt, Dn, ssm_num_state_chunks(L), N), dtype=torch.float32, device=x.device)
        a.chunk_states = _ptr(st)
        res["chunk_states"] = st
    if return_u:
        u = torch.empty((Bt, Dn, L), dtype=od, device=x.device)
        a.u_out = _ptr(u)
        res["u"] = u
    if return_state:
        hl = torch.empty((Bt, Dn, N), dtype=torch.float32, device=x.device)
        a.h_last = _ptr(hl)
        res["h_last"] = hl
        if conv_w is not None and conv_w.shape[1] > 1:
            ch = torch.empty((Bt, Dn, conv_w.shape[1] - 1), dtype=x.dtype, device=x.device)
            a.conv_hist_out = _ptr(ch)
            res["conv_hist"] = ch
    lib = _abi.load()
    ws = None
    if n_segments:
        a.n_segments = int(n_segments)
        need = lib.ssm_fwd_workspace_size(ctypes.byref(a))
        if need:
            ws = torch.empty(need + 256, dtype=torch.uint8, device=x.device)
            a.workspace = (ws.data_ptr() + 255) & ~255
            a.workspace_bytes = need
    _abi.check("ssm_scan_fwd", lib.ssm_scan_fwd(ctypes.byref(a), _stream_handle(x.device)))
    return res if (save_states or return_u or return_state) else out


def _bwd_struct(dout, x, dt, A_log, B, C, D, z, dt_bias, conv_w, conv_b, delta_softplus,
                chunk_states, discretization="zoh", h0=None, conv_hist=None, dh_last=None):
    a, _ = _fwd_args(x, dt, A_log, B, C, D, z, dt_bias, conv_w, conv_b, delta_softplus, None,
                     discretization, h0, conv_hist)
    _need_cuda("dout", dout)
    if dout.dtype != x.dtype or dout.shape != x.shape:
        raise ValueError("dout must match x in shape and dtype")
    _opt("chunk_states", chunk_states, torch.float32)
    bw = _abi.BwdArgs()
    bw.fwd = a
    bw.dout = _ptr(dout)
    bw.chunk_states = _ptr(chunk_states)
    if dh_last is not None:
        _opt("dh_last", dh_last, torch.float32)
        bw.dh_last = _ptr(dh_last)
    return bw


def ssm_bwd_workspace_size(dout, x, dt, A_log, B, C, D=None, z=None, dt_bias=None, conv_w=None,
                           conv_b=None, delta_softplus=True, chunk_states=None,
                           n_segments: int = 0) -> int:
    bw = _bwd_struct(dout, x, dt, A_log, B, C, D, z, dt_bias, conv_w, conv_b, delta_softplus,
                     chunk_states)
    bw.fwd.n_segments = int(n_segments)
    return int(_abi.load().ssm_bwd_workspace_size(ctypes.byref(bw)))


def ssm_scan_bwd(dout, x, dt, A_log, B, C, D=None, z=None, dt_bias=None, conv_w=None,
                 conv_b=None, delta_softplus: bool = True, chunk_states=None,
                 workspace: Optional[torch.Tensor] = None, grads: Optional[Dict] = None,
                 timing_events=None, discretization: str = "zoh", h0=None, conv_hist=None,
                 dh_last=None, state_grads: bool = False, n_segments: int = 0,
                 scan_form: str = "lanes"):
    """Backward. Returns a dict of fp32 gradients: dx, ddt, dA_log, dB, dC, and dD / ddt_bias /
    dz / dconv_w / dconv_b where the corresponding input exists. ``workspace`` (uint8, at least
    ssm_bwd_workspace_size bytes) may be passed to avoid an allocation per call.
    ``timing_events``: optional pair of recorded-once torch.cuda.Event(enable_timing=True); the
    library records them just before and just after its main backward kernel. ``scan_form``
    selects the forward layout used to recompute the chunk states when none are passed."""
    bw = _bwd_struct(dout, x, dt, A_log, B, C, D, z, dt_bias, conv_w, conv_b, delta_softplus,
                     chunk_states, discretization, h0, conv_hist, dh_last)
    if scan_form not in _SCAN:
        raise ValueError("scan_form must be 'lanes' or 'chunked'")
    bw.fwd.scan_form = _SCAN[scan_form]
    Bt, Dn, L = x.shape
    N = A_log.shape[1]
    dev = x.device
    f32 = dict(dtype=torch.float32, device=dev)
    if grads is None:
        grads = {"dx": torch.empty((Bt, Dn, L), **f32), "ddt": torch.empty((Bt, Dn, L), **f32),
                 "dA_log": torch.empty((Dn, N), **f32), "dB": torch.empty((Bt, N, L), **f32),
                 "dC": torch.empty((Bt, N, L), **f32)}
        if D is not None:
            grads["dD"] = torch.empty((Dn,), **f32)
        if dt_bias is not None:
            grads["ddt_bias"] = torch.empty((Dn,), **f32)
        if z is not None:
            grads["dz"] = torch.empty((Bt, Dn, L), **f32)
        if conv_w is not None:
            grads["dconv_w"] = torch.empty(tuple(conv_w.shape), **f32)
            grads["dconv_b"] = torch.empty((Dn,), **f32)
        if state_grads or h0 is not None or dh_last is not None:
            grads["dh0"] = torch.empty((Bt, Dn, N), **f32)
        if conv_w is not None and conv_w.shape[1] > 1 and (state_grads or conv_hist is not None):
            grads["dconv_hist"] = torch.empty((Bt, Dn, conv_w.shape[1] - 1), **f32)
    for k, v in grads.items():
        _opt(k, v, torch.float32)
        setattr(bw, k, _ptr(v))
    lib = _abi.load()
    bw.fwd.n_segments = int(n_segments)  # split-L (see ssm_scan_fwd)
    need = int(lib.ssm_bwd_workspace_size(ctypes.byref(bw)))
    if need > 0:
        if workspace is None or workspace.numel() * workspace.element_size() < need:
            workspace = torch.empty(need + 256, dtype=torch.uint8, device=dev)
        base = workspace.data_ptr()
        aligned = (base + 255) & ~255
        if aligned + need > base + workspace.numel() * workspace.element_size():
            workspace = torch.empty(need + 256, dtype=torch.uint8, device=dev)
            base = workspace.data_ptr()
            aligned = (base + 255) & ~255
        bw.workspace = aligned
        bw.workspace_bytes = need
    ev_arr = None
    if timing_events is not None:
        ev_arr = (ctypes.c_void_p * 2)(*[ctypes.c_void_p(e.cuda_event) for e in timing_events])
        bw.timing_events = ctypes.cast(ev_arr, ctypes.c_void_p)
    _abi.check("ssm_scan_bwd", lib.ssm_scan_bwd(ctypes.byref(bw), _stream_handle(dev)))
    return grads


def ssm_scan_step(x, dt, A_log, B, C, h, conv_hist=None, D=None, z=None, dt_bias=None,
                  conv_w=None, conv_b=None, delta_softplus: bool = True, out_dtype=None,
                  discretization: str = "zoh", out: Optional[torch.Tensor] = None):
    """One decode step. x, dt, z: (Bt, Dn); B, C: (Bt, N); h: (Bt, Dn, N) fp32 and conv_hist:
    (Bt, Dn, K-1) are read and updated in place. Returns the output (Bt, Dn)."""
    for n, t in (("x", x), ("dt", dt), ("A_log", A_log), ("B", B), ("C", C), ("h", h)):
        _need_cuda(n, t)
    if x.dtype not in _DT:
        raise TypeError("x must be float32 or bfloat16")
    act = x.dtype
    for n, t in (("dt", dt), ("B", B), ("C", C)):
        if t.dtype != act:
            raise TypeError("%s must have the activation dtype %s" % (n, act))
    _opt("z", z, act)
    _opt("conv_hist", conv_hist, act)
    for n, t in (("A_log", A_log), ("D", D), ("dt_bias", dt_bias), ("conv_w", conv_w),
                 ("conv_b", conv_b), ("h", h)):
        _opt(n, t, torch.float32)
    Bt, Dn = x.shape
    N = A_log.shape[1]
    if tuple(h.shape) != (Bt, Dn, N) or tuple(B.shape) != (Bt, N) or tuple(C.shape) != (Bt, N):
        raise ValueError("h must be (Bt, Dn, N); B, C (Bt, N)")
    od = act if out_dtype is None else out_dtype
    if out is None:
        out = torch.empty((Bt, Dn), dtype=od, device=x.device)
    a = _abi.StepArgs()
    a.x, a.dt, a.dt_bias, a.A_log, a.B, a.C = _ptr(x), _ptr(dt), _ptr(dt_bias), _ptr(A_log), _ptr(B), _ptr(C)
    a.D, a.z, a.conv_w, a.conv_b = _ptr(D), _ptr(z), _ptr(conv_w), _ptr(conv_b)
    a.h, a.conv_hist, a.out = _ptr(h), _ptr(conv_hist), _ptr(out)
    a.Bt, a.Dn, a.N = Bt, Dn, N
    a.K = int(conv_w.shape[1]) if conv_w is not None else 0
    a.in_dtype, a.out_dtype = _DT[act], _DT[od]
    a.delta_softplus = 1 if delta_softplus else 0
    a.discretization = _DISC[discretization]
    lib = _abi.load()
    _abi.check("ssm_scan_step", lib.ssm_scan_step(ctypes.byref(a), _stream_handle(x.device)))
    return out


def ssm_conv1d_silu(x, w, b=None, out_dtype=None, out: Optional[torch.Tensor] = None):
    """Standalone causal depthwise conv1d + SiLU: x (Bt, Dn, L), w (Dn, K) newest-first."""
    _need_cuda("x", x)
    if x.dtype not in _DT:
        raise TypeError("x must be float32 or bfloat16")
    _opt("w", w, torch.float32)
    _opt("b", b, torch.float32)
    Bt, Dn, L = x.shape
    od = x.dtype if out_dtype is None else out_dtype
    if out is None:
        out = torch.empty((Bt, Dn, L), dtype=od, device=x.device)
    lib = _abi.load()
    _abi.check("ssm_conv1d_silu", lib.ssm_conv1d_silu(
        _ptr(x), _ptr(out), _ptr(w), _ptr(b), Bt, Dn, L, int(w.shape[1]), _DT[x.dtype], _DT[od],
        _stream_handle(x.device)))
    return out


def ssm_ssd_fwd(x, dt, A_log, B, C, D=None, dt_bias=None, h0=None, delta_softplus: bool = True,
                out_dtype=None, discretization: str = "zoh", return_state: bool = False,
                check: bool = False, timing_events=None, form: str = "auto"):
    """Mamba-2 state-space duality forward. x: (Bt, H, L, P) bf16; dt: (Bt, H, L) bf16; B, C:
    (Bt, L, N) bf16 shared by the heads; A_log, D, dt_bias: (H,) fp32; h0: (Bt, H, N, P) fp32.
    P and N must be 64 or 128. Returns y (Bt, H, L, P), or (y, h_last) with return_state.
    ``form``: "fused" (one launch, the state kept on chip; P = 64), "three_pass" (chunk states,
    their carry and the outputs as three launches) or "auto" (fused where it applies).
    check=True synchronises the stream afterwards and raises SSMError (code SSM_ERR_TIMEOUT) if a
    bounded wait for the tensor cores ran out. ``timing_events``: optional pair of
    torch.cuda.Event(enable_timing=True), recorded once already; the library records them just
    before and just after the fused kernel, or the output kernel of the three-pass form."""
    for n, t in (("x", x), ("dt", dt), ("A_log", A_log), ("B", B), ("C", C)):
        _need_cuda(n, t)
    for n, t in (("x", x), ("dt", dt), ("B", B), ("C", C)):
        if t.dtype != torch.bfloat16:
            raise TypeError("%s must be bfloat16" % n)
    for n, t in (("A_log", A_log), ("D", D), ("dt_bias", dt_bias), ("h0", h0)):
        _opt(n, t, torch.float32)
    Bt, H, L, P = x.shape
    N = B.shape[2]
    if tuple(dt.shape) != (Bt, H, L) or tuple(B.shape) != (Bt, L, N) or tuple(C.shape) != (Bt, L, N):
        raise ValueError("dt must be (Bt, H, L); B, C (Bt, L, N)")
    if h0 is not None and tuple(h0.shape) != (Bt, H, N, P):
        raise ValueError("h0 must be (Bt, H, N, P)")
    od = torch.bfloat16 if out_dtype is None else out_dtype
    y = torch.empty((Bt, H, L, P), dtype=od, device=x.device)
    hl = torch.empty((Bt, H, N, P), dtype=torch.float32, device=x.device) if return_state else None
    a = _abi.SsdArgs()
    a.x, a.dt, a.dt_bias, a.A_log, a.B, a.C = _ptr(x), _ptr(dt), _ptr(dt_bias), _ptr(A_log), _ptr(B), _ptr(C)
    a.D, a.h0, a.y, a.h_last = _ptr(D), _ptr(h0), _ptr(y), _ptr(hl)
    a.Bt, a.H, a.L, a.P, a.N = Bt, H, L, P, N
    a.in_dtype, a.out_dtype = _abi.SSM_BF16, _DT[od]
    a.delta_softplus = 1 if delta_softplus else 0
    if discretization not in _DISC:
        raise ValueError("discretization must be 'zoh' or 'euler'")
    a.discretization = _DISC[discretization]
    if form not in _SSD_FORM:
        raise ValueError("form must be 'auto', 'fused' or 'three_pass'")
    a.form = _SSD_FORM[form]
    lib = _abi.load()
    need = int(lib.ssm_ssd_workspace_size(ctypes.byref(a)))
    ws = None
    if need:
        ws = torch.empty(need + 256, dtype=torch.uint8, device=x.device)
        a.workspace = (ws.data_ptr() + 255) & ~255
        a.workspace_bytes = need
    ev_arr = None
    if timing_events is not None:
        ev_arr = (ctypes.c_void_p * 2)(*[ctypes.c_void_p(e.cuda_event) for e in timing_events])
        a.timing_events = ctypes.cast(ev_arr, ctypes.c_void_p)
    _abi.check("ssm_ssd_fwd", lib.ssm_ssd_fwd(ctypes.byref(a), _stream_handle(x.device)))
    if check:
        _abi.check("ssm_ssd_check", lib.ssm_ssd_check(ctypes.byref(a), _stream_handle(x.device)))
    return (y, hl) if return_state else y


def ssm_wait_selftest(arrive: bool, polls: int = 4096, device=None) -> bool:
    """Run the bounded-wait self-test on a CUDA device: one CTA waits, at most `polls` times, on an
    mbarrier that receives its arrival only when `arrive` is true. Returns True when the wait
    completed and False when it ran out (the library answered SSM_ERR_TIMEOUT); any other failure
    raises SSMError. Synchronises the device's current stream."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    if dev.type != "cuda":
        raise ValueError("ssm_wait_selftest needs a CUDA device")
    word = torch.empty(1, dtype=torch.int32, device=dev)
    code = _abi.load().ssm_wait_selftest(1 if arrive else 0, int(polls), _ptr(word), _stream_handle(dev))
    if code == _abi.SSM_ERR_TIMEOUT:
        return False
    _abi.check("ssm_wait_selftest", code)
    return True
