"""Host-side checks of the C ABI that need no GPU: the library loads, exports every function that
include/ssm_scan.h declares, and the synchronous argument validation returns the documented
status codes before anything is launched (only invalid or empty arguments are passed here, so
no CUDA call is ever reached)."""
import ctypes
import os
import re

import pytest

from selective_state_space_34_b200 import _abi, build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "ssm_scan.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _abi.load()


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*[A-Za-z_][\w\s\*]*?\b(ssm_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_every_declared_function_is_exported(lib):
    names = _declared_functions()
    assert {"ssm_scan_fwd", "ssm_scan_bwd", "ssm_conv1d_silu"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(n for n, _, _ in _abi.SIGNATURES) == names


def _header_fields(struct):
    src = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    body = src[src.index("typedef struct %s {" % struct) + len("typedef struct %s {" % struct):
               src.index("} %s;" % struct)]
    names = []
    for decl in body.split(";"):
        if decl.strip():
            names.extend(re.findall(r"(\w+)\s*$", part)[0] for part in decl.split(","))
    return names


@pytest.mark.parametrize("struct,cls,size", [
    # 18 pointers, 4 int64, 7 int32, one size (+4 bytes of tail padding)
    ("ssm_fwd_args", "FwdArgs", 18 * 8 + 4 * 8 + 7 * 4 + 8 + 4),
    # the forward block, 17 pointers and one size
    ("ssm_bwd_args", "BwdArgs", 216 + 17 * 8 + 8),
    # 13 pointers, 3 int64, 5 int32 (+4 bytes of tail padding)
    ("ssm_step_args", "StepArgs", 13 * 8 + 3 * 8 + 5 * 4 + 4),
    # 10 pointers, 5 int64, 4 int32, workspace pointer and size, timing events, the form (+4 bytes
    # of tail padding)
    ("ssm_ssd_args", "SsdArgs", 10 * 8 + 5 * 8 + 4 * 4 + 8 + 8 + 8 + 8),
])
def test_struct_layout_matches_header_field_order(struct, cls, size):
    ct = [f[0] for f in getattr(_abi, cls)._fields_]
    assert _header_fields(struct) == ct
    assert ctypes.sizeof(getattr(_abi, cls)) == size


def test_status_strings(lib):
    for code, name in _abi.STATUS.items():
        assert lib.ssm_status_string(code).decode().startswith(name)
    assert lib.ssm_status_string(99) == b"unknown ssm_status"


def test_state_chunk_count(lib):
    assert lib.ssm_num_state_chunks(0) == 0
    assert lib.ssm_num_state_chunks(1) == 1
    assert lib.ssm_num_state_chunks(16) == 1
    assert lib.ssm_num_state_chunks(17) == 2
    assert lib.ssm_num_state_chunks(65536) == 4096


def _args(**kw):
    a = _abi.FwdArgs()
    a.x, a.dt, a.A_log, a.B, a.C, a.out = 0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 0x6000
    a.Bt, a.Dn, a.N, a.L, a.K = 2, 8, 4, 32, 4
    a.in_dtype, a.out_dtype, a.delta_softplus = 0, 0, 1
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def _fwd(lib, a):
    return lib.ssm_scan_fwd(ctypes.byref(a), None)


def test_fwd_validation_codes(lib):
    assert lib.ssm_scan_fwd(None, None) == 1
    assert _fwd(lib, _args(x=None)) == 1
    assert _fwd(lib, _args(out=None)) == 1
    assert _fwd(lib, _args(in_dtype=7)) == 4
    assert _fwd(lib, _args(out_dtype=-1)) == 4
    assert _fwd(lib, _args(Dn=0)) == 2          # empty internal axes are rejected
    assert _fwd(lib, _args(N=0)) == 2
    assert _fwd(lib, _args(L=-1)) == 2
    assert _fwd(lib, _args(Bt=-3)) == 2
    assert _fwd(lib, _args(N=65)) == 5
    assert _fwd(lib, _args(conv_w=0x7000, K=5)) == 5
    assert _fwd(lib, _args(conv_w=0x7000, K=0)) == 2
    assert _fwd(lib, _args(Bt=1 << 40, Dn=1 << 30)) == 2   # size overflow
    assert _fwd(lib, _args(x=0x1001)) == 3      # fp32 tensor not 4-byte aligned
    assert _fwd(lib, _args(in_dtype=1, x=0x1001)) == 3
    assert _fwd(lib, _args(A_log=0x3002)) == 3
    assert _fwd(lib, _args(out_dtype=1, out=0x6001)) == 3
    assert _fwd(lib, _args(scan_form=2)) == 5   # unknown scan layout
    assert _fwd(lib, _args(discretization=2)) == 5


def test_empty_problems_are_noops(lib):
    # L = 0 or Bt = 0: nothing to do, no pointer is touched (even NULL ones)
    assert _fwd(lib, _args(L=0, x=None, out=None)) == 0
    assert _fwd(lib, _args(Bt=0, x=None)) == 0


def test_bwd_validation_codes(lib):
    bw = _abi.BwdArgs()
    bw.fwd = _args()
    assert lib.ssm_scan_bwd(None, None) == 1
    assert lib.ssm_scan_bwd(ctypes.byref(bw), None) == 1      # dout missing
    bw.dout = 0x8000
    need = lib.ssm_bwd_workspace_size(ctypes.byref(bw))
    assert need > 0
    assert lib.ssm_scan_bwd(ctypes.byref(bw), None) == 7      # no workspace
    bw.workspace, bw.workspace_bytes = 0x100000, need - 1
    assert lib.ssm_scan_bwd(ctypes.byref(bw), None) == 7      # too small
    bw.workspace, bw.workspace_bytes = 0x100010, need
    assert lib.ssm_scan_bwd(ctypes.byref(bw), None) == 7      # not 256-byte aligned
    bw.dx = 0x9002
    assert lib.ssm_scan_bwd(ctypes.byref(bw), None) == 3
    bw.dx = 0
    bw.dout = 0x8001
    assert lib.ssm_scan_bwd(ctypes.byref(bw), None) == 3
    bw.fwd = _args(L=0)
    assert lib.ssm_bwd_workspace_size(ctypes.byref(bw)) == 0
    assert lib.ssm_scan_bwd(ctypes.byref(bw), None) == 0
    # saved states shrink the workspace (no recompute buffer)
    bw.fwd = _args()
    bw.dout = 0x8000
    bw.chunk_states = 0
    full = lib.ssm_bwd_workspace_size(ctypes.byref(bw))
    bw.chunk_states = 0xA000
    assert lib.ssm_bwd_workspace_size(ctypes.byref(bw)) < full


def test_workspace_size_from_forward_arguments(lib):
    """ssm_workspace_size(fwd args, for_bwd): the forward's own size, or the backward's for a
    backward with that fwd block, handed saved states exactly when fwd.chunk_states is set."""
    for kw in (dict(), dict(n_segments=4, L=1000), dict(n_segments=-1, L=4096), dict(L=0)):
        a = _args(**kw)
        assert lib.ssm_workspace_size(ctypes.byref(a), 0) == lib.ssm_fwd_workspace_size(ctypes.byref(a))
        for states in (0, 0xA000):
            a.chunk_states = states
            bw = _abi.BwdArgs()
            bw.fwd = a
            bw.chunk_states = states
            assert lib.ssm_workspace_size(ctypes.byref(a), 1) == lib.ssm_bwd_workspace_size(ctypes.byref(bw))
    assert lib.ssm_workspace_size(None, 0) == 0 and lib.ssm_workspace_size(None, 1) == 0


def test_state_carry_validation_codes(lib):
    assert _fwd(lib, _args(discretization=2)) == 5
    assert _fwd(lib, _args(discretization=1, x=0x1001)) == 3   # Euler passes the flag check
    assert _fwd(lib, _args(h0=0x7002)) == 3
    assert _fwd(lib, _args(h_last=0x7001)) == 3
    assert _fwd(lib, _args(conv_w=0x7000, conv_hist=0x7001)) == 3
    assert _fwd(lib, _args(in_dtype=1, conv_w=0x7000, conv_hist_out=0x7001)) == 3
    # an empty chunk carries the state through without touching NULL pointers
    assert _fwd(lib, _args(L=0, x=None, out=None)) == 0


def test_split_l_workspace_and_codes(lib):
    size = lambda **kw: lib.ssm_fwd_workspace_size(ctypes.byref(_args(**kw)))
    assert size() == 0 and size(n_segments=1) == 0           # one pass needs no scratch
    assert size(n_segments=2, L=100) == 0                     # too short to split
    # L = 1000 in up to 4 segments: 256-step segments -> 4 of them; 2 (4 Bt Dn N) + 4 Bt Dn floats
    rnd = lambda x: (x + 255) // 256 * 256
    assert size(n_segments=4, L=1000) == 2 * rnd(4 * 2 * 8 * 4 * 4) + rnd(4 * 2 * 8 * 4)
    assert size(n_segments=7, L=1000) == 2 * rnd(6 * 2 * 8 * 4 * 4) + rnd(6 * 2 * 8 * 4)  # 192-step segs
    assert size(n_segments=-2) == 0
    assert _fwd(lib, _args(n_segments=-2)) == 2
    assert _fwd(lib, _args(n_segments=4, L=1000)) == 7                  # no workspace
    assert _fwd(lib, _args(n_segments=4, L=1000, workspace=0x100000, workspace_bytes=16)) == 7
    need = size(n_segments=4, L=1000)
    assert _fwd(lib, _args(n_segments=4, L=1000, workspace=0x100010, workspace_bytes=need)) == 7


def _step(**kw):
    a = _abi.StepArgs()
    a.x, a.dt, a.A_log, a.B, a.C, a.h, a.out = 0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 0x6000, 0x7000
    a.Bt, a.Dn, a.N, a.K = 2, 8, 4, 4
    a.in_dtype, a.out_dtype, a.delta_softplus = 0, 0, 1
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def test_step_validation_codes(lib):
    f = lambda a: lib.ssm_scan_step(ctypes.byref(a), None)
    assert lib.ssm_scan_step(None, None) == 1
    assert f(_step(h=None)) == 1
    assert f(_step(in_dtype=3)) == 4
    assert f(_step(discretization=5)) == 5
    assert f(_step(Dn=0)) == 2
    assert f(_step(N=0)) == 2
    assert f(_step(N=65)) == 5
    assert f(_step(conv_w=0x8000, K=5, conv_hist=0x9000)) == 5
    assert f(_step(conv_w=0x8000, K=4)) == 1          # a conv needs its history
    assert f(_step(conv_w=0x8000, K=4, conv_hist=0x9001)) == 3
    assert f(_step(h=0x6002)) == 3
    assert f(_step(Bt=0, x=None, h=None)) == 0        # no rows: nothing to do


def _ssd(**kw):
    a = _abi.SsdArgs()
    a.x, a.dt, a.A_log, a.B, a.C, a.y = 0x10000, 0x20000, 0x30000, 0x40000, 0x50000, 0x60000
    a.Bt, a.H, a.L, a.P, a.N = 2, 4, 300, 64, 128
    a.in_dtype, a.out_dtype, a.delta_softplus = 1, 1, 1
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def test_ssd_validation_codes(lib):
    f = lambda a: lib.ssm_ssd_fwd(ctypes.byref(a), None)
    size = lambda a: lib.ssm_ssd_workspace_size(ctypes.byref(a))
    assert lib.ssm_ssd_fwd(None, None) == 1
    assert f(_ssd(x=None)) == 1
    assert f(_ssd(in_dtype=0)) == 5            # fp32 inputs: tensor-core path is bf16 only
    assert f(_ssd(out_dtype=3)) == 4
    assert f(_ssd(P=32)) == 5 and f(_ssd(N=16)) == 5
    assert f(_ssd(H=0)) == 2 and f(_ssd(L=-1)) == 2
    assert f(_ssd(discretization=2)) == 5
    assert f(_ssd(form=3)) == 5 and f(_ssd(form=-1)) == 5
    assert f(_ssd(form=2, P=128)) == 5          # the fused form takes P = 64 only
    assert f(_ssd(x=0x10008)) == 3             # 16-byte alignment of the tile loads
    assert f(_ssd(dt=0x20001)) == 3
    assert f(_ssd(h0=0x70004)) == 3 and f(_ssd(h_last=0x70008)) == 3
    assert f(_ssd(Bt=0, x=None)) == 0          # empty: nothing launched
    assert f(_ssd()) == 7                      # no workspace
    need = size(_ssd())
    # 2 x 4 heads x 3 chunks: S (fp32) + H_in (bf16) of 128 x 64, one log-decay each, error word
    rnd = lambda v: (v + 255) // 256 * 256
    assert need == rnd(24 * 128 * 64 * 4) + rnd(24 * 128 * 64 * 2) + rnd(24 * 4) + 256
    assert f(_ssd(workspace=0x100010, workspace_bytes=need)) == 7


def test_failure_detection_validation_codes(lib):
    # Error paths only: each returns before any CUDA call.
    chk = lambda a: lib.ssm_ssd_check(ctypes.byref(a), None)
    assert lib.ssm_ssd_check(None, None) == 1
    assert chk(_ssd(P=32)) == 5                 # same argument checks as ssm_ssd_fwd
    assert chk(_ssd(Bt=0, x=None)) == 0         # empty: nothing ran, nothing to read
    assert chk(_ssd()) == 7                     # the error word lives in the workspace
    need = lib.ssm_ssd_workspace_size(ctypes.byref(_ssd()))
    assert chk(_ssd(workspace=0x100100, workspace_bytes=need - 1)) == 7
    assert chk(_ssd(workspace=0x100010, workspace_bytes=need)) == 7
    st = lib.ssm_wait_selftest
    assert st(0, 16, None, None) == 1
    assert st(0, 16, 0x1002, None) == 3
    assert st(0, 0, 0x1000, None) == 2 and st(0, (1 << 22) + 1, 0x1000, None) == 2
    assert lib.ssm_status_string(8).decode().startswith("SSM_ERR_TIMEOUT")


def test_conv_validation_codes(lib):
    f = lib.ssm_conv1d_silu
    assert f(0x1000, 0x2000, 0x3000, None, 2, 4, 8, 4, 9, 0, None) == 4
    assert f(0x1000, 0x2000, 0x3000, None, 2, 0, 8, 4, 0, 0, None) == 2
    assert f(0x1000, 0x2000, 0x3000, None, 2, 4, 8, 0, 0, 0, None) == 2
    assert f(0x1000, 0x2000, 0x3000, None, 2, 4, 8, 5, 0, 0, None) == 5
    assert f(None, 0x2000, 0x3000, None, 2, 4, 8, 4, 0, 0, None) == 1
    assert f(0x1001, 0x2000, 0x3000, None, 2, 4, 8, 4, 0, 0, None) == 3
    assert f(None, None, None, None, 2, 4, 0, 4, 0, 0, None) == 0


def test_binding_refuses_cpu_tensors():
    import torch
    import selective_state_space_34_b200 as ssm
    x = torch.zeros(1, 2, 8)
    with pytest.raises(ValueError, match="CUDA"):
        ssm.ssm_scan_fwd(x, x, torch.zeros(2, 4), torch.zeros(1, 4, 8), torch.zeros(1, 4, 8))
