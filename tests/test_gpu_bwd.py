"""Backward parity: every gradient of the CUDA backward against the float64 oracle's VJP on the same
seeded inputs; the finite-difference slice; full-size workloads on sampled channels."""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_34_b200 as ssm
from selective_state_space_34_b200 import workloads as wl
from gpu_helpers import (assert_grad_close, channel_slice, dev_arrays, oracle_kw, param_kw, to_np)

pytestmark = pytest.mark.gpu

GRADS = ["dx", "ddt", "dz", "dA_log", "dB", "dC", "dD", "ddt_bias", "dconv_w", "dconv_b"]


def run_bwd(w, use_saved_states=True, conv=True, gate=True, seed=None):
    a = wl.generate(w, seed=seed)
    if "dout" not in a or a["dout"] is None:
        a["dout"] = wl.generate(wl.shaped(w.name, backward=True, Bt=w.Bt, Dn=w.Dn, N=w.N, L=w.L,
                                          in_dtype=w.in_dtype), seed=seed)["dout"]
    t = dev_arrays(a, w.in_dtype)
    kw = param_kw(t, conv and w.conv, gate and w.gate)
    states = None
    if use_saved_states:
        states = ssm.ssm_scan_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], save_states=True,
                                  **kw)["chunk_states"]
    g = ssm.ssm_scan_bwd(t["dout"], t["x"], t["dt"], t["A_log"], t["B"], t["C"],
                         chunk_states=states, **kw)
    torch.cuda.synchronize()
    ref = oracle.bwd(a["x"], a["dt"], a["A_log"], a["B"], a["C"], a["dout"],
                     **oracle_kw(a, conv and w.conv, gate and w.gate))
    for k in GRADS:
        if k in ref:
            assert_grad_close(k, to_np(g[k]), ref[k])
    return a, g, ref


@pytest.mark.parametrize("Bt,Dn,N,L", [
    (2, 40, 16, 200), (1, 33, 16, 77), (1, 7, 16, 3), (2, 9, 4, 50), (2, 9, 5, 50),
    (2, 9, 32, 50), (2, 9, 64, 50), (1, 5, 16, 16), (1, 5, 16, 17),
])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_shapes(Bt, Dn, N, L, dtype):
    run_bwd(wl.shaped("mamba130m_fwd", Bt=Bt, Dn=Dn, N=N, L=L, in_dtype=dtype, backward=True))


@pytest.mark.parametrize("Bt,Dn", [(2, 4800), (1, 5000)])
def test_wide_lane_layouts(Bt, Dn):
    run_bwd(wl.shaped("mamba130m_fwd", Bt=Bt, Dn=Dn, L=40, backward=True))


def test_tile_sum_paths_agree_bitwise():
    """dB / dC are summed over channel tiles with 16-byte accesses when every buffer allows it and
    one element at a time otherwise (here: outputs starting a float in); both add the tiles in the
    same order, so the results are identical bit for bit."""
    w = wl.shaped("mamba130m_fwd", Bt=2, Dn=200, N=16, L=96, backward=True)
    t = dev_arrays(wl.generate(w), "bf16")
    kw = param_kw(t)
    g1 = ssm.ssm_scan_bwd(t["dout"], t["x"], t["dt"], t["A_log"], t["B"], t["C"], **kw)
    flat = torch.empty(2 * g1["dB"].numel() + 2, device="cuda")
    dB = flat[1:1 + g1["dB"].numel()].view_as(g1["dB"])
    dC = flat[2 + g1["dB"].numel():].view_as(g1["dC"])
    g2 = ssm.ssm_scan_bwd(t["dout"], t["x"], t["dt"], t["A_log"], t["B"], t["C"],
                          grads={"dB": dB, "dC": dC}, **kw)
    torch.cuda.synchronize()
    assert torch.equal(g2["dB"], g1["dB"]) and torch.equal(g2["dC"], g1["dC"])


@pytest.mark.parametrize("subset", [("dA_log", "dD"), ("dB",), ("dC", "ddt_bias", "dconv_w")])
def test_gradient_subsets_match_the_full_set(subset):
    """Asking for some gradients only (the rest null) gives the same bits for those: the tile and
    parameter reductions run as one launch, or the parameters alone when dB and dC are not asked."""
    w = wl.shaped("mamba130m_fwd", Bt=2, Dn=72, N=16, L=96, backward=True)
    t = dev_arrays(wl.generate(w), "bf16")
    kw = param_kw(t)
    g1 = ssm.ssm_scan_bwd(t["dout"], t["x"], t["dt"], t["A_log"], t["B"], t["C"], **kw)
    part = {k: torch.full_like(g1[k], float("nan")) for k in subset}
    g2 = ssm.ssm_scan_bwd(t["dout"], t["x"], t["dt"], t["A_log"], t["B"], t["C"], grads=part, **kw)
    torch.cuda.synchronize()
    for k in subset:
        assert torch.equal(g2[k], g1[k]), k


def test_recomputed_states_match_saved_states():
    w = wl.shaped("mamba130m_fwd", Bt=2, Dn=24, L=100, backward=True)
    run_bwd(w, use_saved_states=False)


@pytest.mark.parametrize("variant", ["no_conv", "no_gate", "bare"])
def test_optional_pieces(variant):
    w = wl.shaped("mamba130m_fwd", Bt=2, Dn=12, L=64, backward=True)
    run_bwd(w, conv=variant not in ("no_conv", "bare"), gate=variant not in ("no_gate", "bare"))


def test_tiny_fp32_workload():
    w = wl.shaped("tiny_fp32", backward=True)
    run_bwd(w)


def test_deterministic():
    w = wl.shaped("mamba130m_fwd", Bt=2, Dn=64, L=96, backward=True)
    a = wl.generate(w)
    t = dev_arrays(a, "bf16")
    kw = param_kw(t)
    g1 = ssm.ssm_scan_bwd(t["dout"], t["x"], t["dt"], t["A_log"], t["B"], t["C"], **kw)
    g2 = ssm.ssm_scan_bwd(t["dout"], t["x"], t["dt"], t["A_log"], t["B"], t["C"], **kw)
    for k in g1:
        assert torch.equal(g1[k], g2[k]), k


def test_finite_difference_slice():
    # 1x8x4x32, fp32: GPU gradients against central differences of the oracle's forward, with the
    # rustytorch tolerance 5e-3 + 5e-2 |fd| on every element of every gradient.
    w = wl.WORKLOADS["fd_slice"]
    a = wl.generate(w)
    t = dev_arrays(a, "f32")
    g = ssm.ssm_scan_bwd(t["dout"], t["x"], t["dt"], t["A_log"], t["B"], t["C"], **param_kw(t))
    torch.cuda.synchronize()
    names = {"x": "dx", "dt": "ddt", "z": "dz", "B": "dB", "C": "dC", "A_log": "dA_log", "D": "dD",
             "dt_bias": "ddt_bias", "conv_w": "dconv_w", "conv_b": "dconv_b"}
    p = {k: np.array(a[k], dtype=np.float64) for k in names}

    def loss():
        out = oracle.fwd(p["x"], p["dt"], p["A_log"], p["B"], p["C"], **oracle_kw(p))
        return float(np.sum(out * a["dout"]))
    h = 1e-6
    checked = 0
    for k, gk in names.items():
        an = to_np(g[gk]).astype(np.float64)
        flat = p[k].reshape(-1)
        fd = np.zeros(flat.size)
        for i in range(flat.size):
            old = flat[i]
            flat[i] = old + h
            lp = loss()
            flat[i] = old - h
            lm = loss()
            flat[i] = old
            fd[i] = (lp - lm) / (2 * h)
        ok = np.abs(an.reshape(-1) - fd) <= 5e-3 + 5e-2 * np.abs(fd)
        assert ok.all(), "%s: %d elements outside the finite-difference tolerance" % (gk, (~ok).sum())
        checked += fd.size
    assert checked >= 30


@pytest.mark.slow
def test_full_fwdbwd_sampled_channels():
    # The forward+backward workload at full size (4 x 4096 x 16 x 4096), in the benchmark's launch
    # configuration. Per-channel gradients are checked on sampled channels; dB and dC (sums over
    # all channels) are checked with a dout that is zero outside the sampled channels, which makes
    # every other channel's contribution exactly zero.
    w = wl.WORKLOADS["mamba1p4b_fwdbwd"]
    a = wl.generate(w)
    picks = wl.sample_channels(w.Bt, w.Dn, 16)
    for masked in (False, True):
        if masked:
            mask = np.zeros((w.Bt, w.Dn, 1), dtype=np.float32)
            for b, d in picks:
                mask[b, d] = 1.0
            a2 = dict(a)
            a2["dout"] = a["dout"] * mask
        else:
            a2 = a
        t = dev_arrays(a2, "bf16")
        kw = param_kw(t)
        st = ssm.ssm_scan_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], save_states=True,
                              **kw)["chunk_states"]
        g = ssm.ssm_scan_bwd(t["dout"], t["x"], t["dt"], t["A_log"], t["B"], t["C"],
                             chunk_states=st, **kw)
        torch.cuda.synchronize()
        got = {k: to_np(v) for k, v in g.items()}
        del g, t, st
        torch.cuda.empty_cache()
        dB_ref = np.zeros((w.Bt, w.N, w.L))
        dC_ref = np.zeros((w.Bt, w.N, w.L))
        for b, d in picks:
            s = channel_slice(a2, b, d)
            r = oracle.bwd(s["x"], s["dt"], s["A_log"], s["B"], s["C"], s["dout"], **oracle_kw(s))
            for k in ("dx", "ddt", "dz"):
                assert_grad_close("%s (b=%d,d=%d)" % (k, b, d), got[k][b:b + 1, d:d + 1], r[k])
            dB_ref[b] += r["dB"][0]
            dC_ref[b] += r["dC"][0]
        if masked:
            assert_grad_close("dB (masked)", got["dB"], dB_ref)
            assert_grad_close("dC (masked)", got["dC"], dC_ref)
    # per-channel parameter gradients sum over the batch: check a few channels d over all b
    ds = sorted(set(int(d) for _, d in picks))[:6]
    # run once more unmasked to get the per-channel parameter gradients
    t = dev_arrays(a, "bf16")
    kw = param_kw(t)
    g = ssm.ssm_scan_bwd(t["dout"], t["x"], t["dt"], t["A_log"], t["B"], t["C"], **kw)
    torch.cuda.synchronize()
    for d in ds:
        acc = None
        for b in range(w.Bt):
            s = channel_slice(a, b, d)
            r = oracle.bwd(s["x"], s["dt"], s["A_log"], s["B"], s["C"], s["dout"], **oracle_kw(s))
            acc = r if acc is None else {k: acc[k] + r[k] for k in acc}
        for k in ("dA_log", "dD", "ddt_bias", "dconv_w", "dconv_b"):
            assert_grad_close("%s (d=%d)" % (k, d), to_np(g[k])[d:d + 1], acc[k])
