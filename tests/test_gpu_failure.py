"""Failure detection without a GPU fault: the bounded device-side waits of the tensor-core path.

The SSD kernels wait for each tensor-core product through an mbarrier, polling a bounded number of
times; on a timeout they set an error word, release their tensor memory and exit, and the host maps
the word to SSM_ERR_TIMEOUT. The self-test runs that wait on an mbarrier that nothing arrives at,
so the timeout path is taken for real, and the context must stay usable afterwards."""
import time

import pytest
import torch

import selective_state_space_34_b200 as ssm
from selective_state_space_34_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _ssd_inputs():
    a = wl.generate_ssd(1, 4, 300, 64, 64, seed=21)
    return {k: torch.from_numpy(v).to("cuda", torch.bfloat16 if k in ("x", "dt", "B", "C") else torch.float32)
            for k, v in a.items()}


def _ssd(t):
    return ssm.ssm_ssd_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], D=t["D"],
                           dt_bias=t["dt_bias"], out_dtype=torch.float32, check=True)


def test_wait_completes_when_the_arrival_comes():
    assert ssm.ssm_wait_selftest(True, polls=1 << 22) is True


def test_wait_runs_out_and_the_context_survives():
    t = _ssd_inputs()
    before = _ssd(t)
    torch.cuda.synchronize()
    # A poll that fails may suspend the thread for a hardware-chosen time, so the bound grows only
    # while the previous one ended quickly.
    for polls in (1, 4096, 1 << 16):
        t0 = time.perf_counter()
        assert ssm.ssm_wait_selftest(False, polls=polls) is False
        dt = time.perf_counter() - t0
        print("timeout after %d polls: %.3f ms" % (polls, dt * 1e3))
        if dt > 0.1:
            break
    # the SSD kernels' bound (2^18 polls) then gives up within a few seconds at most
    assert dt / polls * (1 << 18) < 5.0
    # the context is intact: the tensor-core path runs and reports no timeout, same bits as before
    after = _ssd(t)
    torch.cuda.synchronize()
    assert torch.equal(before, after)
    assert ssm.ssm_wait_selftest(True, polls=1 << 22) is True


def test_ssd_check_reports_success_on_a_normal_run():
    t = _ssd_inputs()
    y = _ssd(t)  # check=True raises SSMError(SSM_ERR_TIMEOUT) if any wait ran out
    assert torch.isfinite(y).all()
