"""Shared helpers for the GPU parity tests: move seeded workloads to the device, run the CUDA path
through the binding, run the oracle on the same values, and compare with stated tolerances.

Tolerances (elementwise |gpu - oracle| <= atol + rtol |oracle|):
  * bf16-input forward, fp32 output: rtol 2e-3, atol 1e-4.
  * bf16-input forward, bf16 output: rtol 2e-3 + 2^-8 (one bf16 rounding of the result),
    atol 1e-4.
  * fp32-input forward: rtol 1e-5, atol 1e-6.
  * gradients: rtol 1e-2, atol 1e-4 * max|oracle gradient| of that tensor (fp32 sums of
    thousands of terms have absolute, not relative, error where the sum cancels).
"""
import numpy as np
import torch

import oracle

TOL = {
    ("bf16", "f32"): (2e-3, 1e-4),
    ("bf16", "bf16"): (2e-3 + 2.0 ** -8, 1e-4),
    ("f32", "f32"): (1e-5, 1e-6),
    ("f32", "bf16"): (1e-5 + 2.0 ** -8, 1e-6),
}
GRAD_RTOL, GRAD_ATOL_FRAC = 1e-2, 1e-4


def dev_arrays(a, in_dtype, device="cuda"):
    """numpy workload -> torch tensors on the device; activations in the input dtype."""
    act = torch.bfloat16 if in_dtype == "bf16" else torch.float32
    out = {}
    for k, v in a.items():
        if v is None:
            out[k] = None
        elif k in ("x", "dt", "z", "B", "C", "dout", "conv_hist"):
            out[k] = torch.from_numpy(np.ascontiguousarray(v)).to(device=device, dtype=act)
        else:
            out[k] = torch.from_numpy(np.ascontiguousarray(v)).to(device=device, dtype=torch.float32)
    return out


def param_kw(t, conv=True, gate=True, D=True, bias=True):
    return dict(D=t["D"] if D else None, z=t["z"] if gate else None,
                dt_bias=t["dt_bias"] if bias else None,
                conv_w=t["conv_w"] if conv else None, conv_b=t["conv_b"] if conv else None)


def oracle_kw(a, conv=True, gate=True, D=True, bias=True):
    return dict(D=a["D"] if D else None, z=a["z"] if gate else None,
                dt_bias=a["dt_bias"] if bias else None,
                conv_w=a["conv_w"] if conv else None, conv_b=a["conv_b"] if conv else None)


def assert_close(name, got, ref, rtol, atol):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), name + ": non-finite values"
    err = np.abs(got - ref)
    bad = err > atol + rtol * np.abs(ref)
    if bad.any():
        i = np.unravel_index(np.argmax(err - (atol + rtol * np.abs(ref))), ref.shape)
        raise AssertionError("%s: %d/%d outside tol (rtol %g, atol %g); worst at %s: gpu %r oracle %r"
                             % (name, int(bad.sum()), bad.size, rtol, atol, i, got[i], ref[i]))


def assert_grad_close(name, got, ref):
    ref = np.asarray(ref, dtype=np.float64)
    atol = GRAD_ATOL_FRAC * max(np.abs(ref).max(), 1e-30)
    assert_close(name, got, ref, GRAD_RTOL, atol)


def channel_slice(a, b, d):
    """The inputs of one (batch, channel) pair, as a Bt=1, Dn=1 problem for the oracle."""
    s = {}
    for k, v in a.items():
        if v is None:
            s[k] = None
        elif k in ("x", "dt", "z", "dout"):
            s[k] = v[b:b + 1, d:d + 1]
        elif k in ("B", "C"):
            s[k] = v[b:b + 1]
        elif k in ("A_log", "conv_w"):
            s[k] = v[d:d + 1]
        else:
            s[k] = v[d:d + 1]
    return s


def to_np(t):
    return t.detach().float().cpu().numpy() if t.dtype == torch.bfloat16 else t.detach().cpu().numpy()
