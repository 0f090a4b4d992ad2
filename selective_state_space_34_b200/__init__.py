"""B200-native (sm_100a) Mamba-1 selective scan (S6).

Thin PyTorch-facing binding over the C ABI in include/ssm_scan.h. The functions here only check
and marshal arguments (device pointers, sizes, the current CUDA stream) and allocate outputs with
torch; every step of the computation runs in the library's CUDA kernels. There is no CPU or
PyTorch fallback: without the built library or a CUDA device the calls raise.

    out = ssm_scan_fwd(x, dt, A_log, B, C, D=D, z=z, dt_bias=dt_bias, conv_w=conv_w, conv_b=conv_b)
    grads = ssm_scan_bwd(dout, x, dt, A_log, B, C, ..., chunk_states=states)
    u = ssm_conv1d_silu(x, conv_w, conv_b)
    y_t = ssm_scan_step(x_t, dt_t, A_log, B_t, C_t, h, conv_hist, ...)   # one decode token
    y = ssm_ssd_fwd(x, dt, A_log, B, C, D=D)      # Mamba-2 state-space duality (heads)

Shapes: x, dt, z (Bt, Dn, L); B, C (Bt, N, L); A_log (Dn, N); D, dt_bias, conv_b (Dn,);
conv_w (Dn, K) newest-first taps. Activations are fp32 or bf16 (one dtype for all of them);
parameters are fp32.
"""
from __future__ import annotations

from .api import (ssm_conv1d_silu, ssm_scan_bwd, ssm_scan_fwd, ssm_scan_step, ssm_ssd_fwd,
                  ssm_bwd_workspace_size, ssm_num_state_chunks, ssm_wait_selftest)

__all__ = ["ssm_scan_fwd", "ssm_scan_bwd", "ssm_scan_step", "ssm_ssd_fwd", "ssm_conv1d_silu",
           "ssm_bwd_workspace_size", "ssm_num_state_chunks", "ssm_wait_selftest"]
