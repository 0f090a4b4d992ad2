"""ssm_scan_bwd_noalloc: the backward for callers that cannot allocate device memory (a host
program or plugin that only receives device pointers, or code running where allocating is not
allowed), using the library's built-in scratch array instead of a caller workspace.

The GPU test calls the entry point through the C ABI twice in a row and checks both results
against the regular ssm_scan_bwd on the same inputs, with the gradient tolerance the other tests
use. The file is named to be collected last, so a run that stops at the first failure has run
every other test first; it also passes when run alone in a fresh process."""
import ctypes

import numpy as np
import pytest

from selective_state_space_34_b200 import _abi, build


def test_oversize_problem_is_rejected_before_any_device_work():
    # pure host path: the size check precedes every CUDA call
    build.build()
    lib = _abi.load()
    bw = _abi.BwdArgs()
    a = bw.fwd
    a.x, a.dt, a.A_log, a.B, a.C = 0x1000, 0x2000, 0x3000, 0x4000, 0x5000
    a.Bt, a.Dn, a.N, a.L, a.K = 4, 4096, 16, 4096, 4
    a.in_dtype, a.out_dtype, a.delta_softplus = 1, 1, 1
    bw.dout = 0x8000
    assert lib.ssm_bwd_workspace_size(ctypes.byref(bw)) > _abi.SSM_NOALLOC_SCRATCH_BYTES
    assert lib.ssm_scan_bwd_noalloc(ctypes.byref(bw), None) == 7  # SSM_ERR_WORKSPACE
    assert lib.ssm_scan_bwd_noalloc(None, None) == 1


@pytest.mark.gpu
def test_noalloc_backward_matches_regular_backward_twice():
    import torch
    import selective_state_space_34_b200 as ssm
    from selective_state_space_34_b200 import api, workloads as wl
    from gpu_helpers import assert_grad_close, dev_arrays, param_kw, to_np

    w = wl.shaped("mamba130m_fwd", Bt=2, Dn=96, N=16, L=272, backward=True)
    a = wl.generate(w)
    t = dev_arrays(a, "bf16")
    kw = param_kw(t)
    states = ssm.ssm_scan_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], save_states=True,
                              **kw)["chunk_states"]
    ref = ssm.ssm_scan_bwd(t["dout"], t["x"], t["dt"], t["A_log"], t["B"], t["C"],
                           chunk_states=states, **kw)
    torch.cuda.synchronize()
    lib = _abi.load()
    for call in range(2):
        bw = api._bwd_struct(t["dout"], t["x"], t["dt"], t["A_log"], t["B"], t["C"], kw["D"],
                             kw["z"], kw["dt_bias"], kw["conv_w"], kw["conv_b"], True, states)
        assert lib.ssm_bwd_workspace_size(ctypes.byref(bw)) <= _abi.SSM_NOALLOC_SCRATCH_BYTES
        got = {k: torch.full_like(v, float("nan")) for k, v in ref.items()}
        for k, v in got.items():
            setattr(bw, k, v.data_ptr())
        stream = torch.cuda.current_stream().cuda_stream
        assert lib.ssm_scan_bwd_noalloc(ctypes.byref(bw), stream) == 0
        torch.cuda.synchronize()
        for k in ref:
            assert_grad_close("%s (call %d)" % (k, call + 1), to_np(got[k]), to_np(ref[k]).astype(np.float64))


@pytest.mark.gpu
def test_noalloc_backward_at_the_measured_size_twice():
    """4 x 4096 x 16 x 4096 with saved states: the per-tile dB / dC partials alone would need
    256 MiB, so the entry point runs with clusters of 4 CTAs that add those partials on chip
    (65 MiB of scratch). Two calls in a row against the regular backward."""
    import torch
    import selective_state_space_34_b200 as ssm
    from selective_state_space_34_b200 import api, workloads as wl
    from gpu_helpers import assert_grad_close, dev_arrays, param_kw, to_np

    w = wl.WORKLOADS["mamba1p4b_fwdbwd"]
    t = dev_arrays(wl.generate(w), "bf16")
    kw = param_kw(t)
    states = ssm.ssm_scan_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], save_states=True,
                              **kw)["chunk_states"]
    ref = ssm.ssm_scan_bwd(t["dout"], t["x"], t["dt"], t["A_log"], t["B"], t["C"],
                           chunk_states=states, **kw)
    torch.cuda.synchronize()
    ref = {k: to_np(v).astype(np.float64) for k, v in ref.items()}
    lib = _abi.load()
    for call in range(2):
        bw = api._bwd_struct(t["dout"], t["x"], t["dt"], t["A_log"], t["B"], t["C"], kw["D"],
                             kw["z"], kw["dt_bias"], kw["conv_w"], kw["conv_b"], True, states)
        assert lib.ssm_bwd_workspace_size(ctypes.byref(bw)) > _abi.SSM_NOALLOC_SCRATCH_BYTES
        got = {k: torch.full(v.shape, float("nan"), device="cuda") for k, v in ref.items()}
        for k, v in got.items():
            setattr(bw, k, v.data_ptr())
        stream = torch.cuda.current_stream().cuda_stream
        assert lib.ssm_scan_bwd_noalloc(ctypes.byref(bw), stream) == 0
        torch.cuda.synchronize()
        for k in ref:
            assert_grad_close("%s (call %d)" % (k, call + 1), to_np(got[k]), ref[k])
        del got
