"""Parity of the split-L forward (the sequence cut into segments that run in parallel: end states
from a zero start, a carry of the states across segments, then every segment from its carried
start -- "Sequence and state-space models", the chunked scan; "Selective Mamba", runArray) against
the float64 oracle over the whole sequence, and against the one-pass kernel."""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_34_b200 as ssm
from selective_state_space_34_b200 import workloads as wl
from gpu_helpers import TOL, assert_close, dev_arrays, oracle_kw, param_kw, to_np

pytestmark = pytest.mark.gpu


def _setup(Bt, Dn, N, L, dtype, conv=True, gate=True, seed=None):
    w = wl.shaped("mamba130m_fwd", Bt=Bt, Dn=Dn, N=N, L=L, in_dtype=dtype, conv=conv, gate=gate)
    a = wl.generate(w, seed=seed)
    a.update(wl.carried_state(w, seed=seed))
    return w, a, dev_arrays(a, dtype)


@pytest.mark.parametrize("nseg", [2, 3, 5, 16])
@pytest.mark.parametrize("Bt,Dn,L", [(1, 24, 1000), (2, 40, 300), (1, 8, 4113)])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_split_matches_oracle_and_one_pass(nseg, Bt, Dn, L, dtype):
    w, a, t = _setup(Bt, Dn, 16, L, dtype)
    kw = param_kw(t)
    one = ssm.ssm_scan_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], out_dtype=torch.float32,
                           save_states=True, return_u=True, **kw)
    sp = ssm.ssm_scan_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], out_dtype=torch.float32,
                          save_states=True, return_u=True, n_segments=nseg, **kw)
    torch.cuda.synchronize()
    ref = oracle.fwd(a["x"], a["dt"], a["A_log"], a["B"], a["C"], **oracle_kw(a))
    rtol, atol = TOL[(dtype, "f32")]
    assert_close("out", to_np(sp["out"]), ref, rtol, atol)
    # against the one-pass kernel: the carry only reorders fp32 rounding
    assert_close("out vs one pass", to_np(sp["out"]), to_np(one["out"]), rtol, atol)
    assert_close("chunk_states", to_np(sp["chunk_states"]), to_np(one["chunk_states"]), rtol, atol)
    assert torch.equal(sp["u"], one["u"])  # u does not depend on the state


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("euler", [False, True])
def test_split_with_carried_state(dtype, euler):
    w, a, t = _setup(2, 24, 16, 777, dtype)
    disc = "euler" if euler else "zoh"
    r = ssm.ssm_scan_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], out_dtype=torch.float32,
                         h0=t["h0"], conv_hist=t["conv_hist"], return_state=True,
                         discretization=disc, n_segments=4, **param_kw(t))
    torch.cuda.synchronize()
    ref, ex = oracle.fwd(a["x"], a["dt"], a["A_log"], a["B"], a["C"], euler=euler, h0=a["h0"],
                         conv_hist=a["conv_hist"], want_state=True, **oracle_kw(a))
    rtol, atol = TOL[(dtype, "f32")]
    assert_close("out", to_np(r["out"]), ref, rtol, atol)
    assert_close("h_last", to_np(r["h_last"]), ex["h_last"], rtol, atol)
    assert np.array_equal(to_np(r["conv_hist"]), ex["conv_hist"])


@pytest.mark.parametrize("variant", ["no_conv", "no_gate", "bare"])
def test_split_optional_pieces(variant):
    conv, gate = variant not in ("no_conv", "bare"), variant not in ("no_gate", "bare")
    w, a, t = _setup(1, 16, 16, 900, "bf16", conv=conv, gate=gate)
    kw = param_kw(t, conv=conv, gate=gate)
    out = ssm.ssm_scan_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], out_dtype=torch.float32,
                           n_segments=3, **kw)
    torch.cuda.synchronize()
    ref = oracle.fwd(a["x"], a["dt"], a["A_log"], a["B"], a["C"], **oracle_kw(a, conv=conv, gate=gate))
    assert_close("out", to_np(out), ref, *TOL[("bf16", "f32")])


@pytest.mark.parametrize("N", [4, 5, 64])
def test_split_state_sizes(N):
    w, a, t = _setup(1, 12, N, 640, "bf16")
    out = ssm.ssm_scan_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], out_dtype=torch.float32,
                           n_segments=5, **param_kw(t))
    torch.cuda.synchronize()
    ref = oracle.fwd(a["x"], a["dt"], a["A_log"], a["B"], a["C"], **oracle_kw(a))
    assert_close("out", to_np(out), ref, *TOL[("bf16", "f32")])


def test_split_bf16_output_and_auto():
    """Automatic choice on a few-channel long shape (it splits) and on a wide one (it does not)."""
    w, a, t = _setup(1, 64, 16, 8192, "bf16")
    kw = param_kw(t)
    one = ssm.ssm_scan_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], **kw)
    auto = ssm.ssm_scan_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], n_segments=-1, **kw)
    torch.cuda.synchronize()
    rtol, atol = TOL[("bf16", "bf16")]
    assert_close("auto vs one pass", to_np(auto), to_np(one), rtol, atol)
    args, _ = ssm.api._fwd_args(t["x"], t["dt"], t["A_log"], t["B"], t["C"], kw["D"], kw["z"],
                                kw["dt_bias"], kw["conv_w"], kw["conv_b"], True, None)
    import ctypes
    from selective_state_space_34_b200 import _abi
    args.n_segments = -1
    assert _abi.load().ssm_fwd_workspace_size(ctypes.byref(args)) > 0   # it splits
    args.Dn = 32768
    assert _abi.load().ssm_fwd_workspace_size(ctypes.byref(args)) == 0  # a full wave without it


def test_long_few_channels_sampled():
    """1 x 256 channels x 32768 steps in 16 segments: sampled channels against the oracle."""
    w, a, t = _setup(1, 256, 16, 32768, "bf16")
    out = ssm.ssm_scan_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], out_dtype=torch.float32,
                           n_segments=16, **param_kw(t))
    torch.cuda.synchronize()
    got = to_np(out)
    for (b, d) in wl.sample_channels(1, 256, 6):
        s = {k: (None if v is None else (v[b:b + 1, d:d + 1] if k in ("x", "dt", "z") else
                                         (v[b:b + 1] if k in ("B", "C") else v[d:d + 1])))
             for k, v in a.items() if k in ("x", "dt", "z", "B", "C", "A_log", "D", "dt_bias",
                                             "conv_w", "conv_b")}
        ref = oracle.fwd(s["x"], s["dt"], s["A_log"], s["B"], s["C"], **oracle_kw(s))
        assert_close("out[%d,%d]" % (b, d), got[b:b + 1, d:d + 1], ref, *TOL[("bf16", "f32")])


GRADS = ["dx", "ddt", "dz", "dA_log", "dB", "dC", "dD", "ddt_bias", "dconv_w", "dconv_b",
         "dh0", "dconv_hist"]


def _bwd_case(Bt, Dn, N, L, dtype, nseg, conv=True, gate=True, carried=True, euler=False,
              saved=True):
    w = wl.shaped("mamba130m_fwd", Bt=Bt, Dn=Dn, N=N, L=L, in_dtype=dtype, conv=conv, gate=gate,
                  backward=True)
    a = wl.generate(w)
    a.update(wl.carried_state(w))
    if not carried:
        a["h0"] = a["conv_hist"] = a["dh_last"] = None
    t = dev_arrays(a, dtype)
    kw = param_kw(t, conv=conv, gate=gate)
    disc = "euler" if euler else "zoh"
    st = dict(h0=t["h0"], conv_hist=t["conv_hist"] if conv else None, discretization=disc)
    states = None
    if saved:
        states = ssm.ssm_scan_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], save_states=True,
                                  n_segments=nseg, **st, **kw)["chunk_states"]
    g = ssm.ssm_scan_bwd(t["dout"], t["x"], t["dt"], t["A_log"], t["B"], t["C"],
                         chunk_states=states, dh_last=t["dh_last"], state_grads=True,
                         n_segments=nseg, **st, **kw)
    g1 = ssm.ssm_scan_bwd(t["dout"], t["x"], t["dt"], t["A_log"], t["B"], t["C"],
                          chunk_states=states, dh_last=t["dh_last"], state_grads=True, **st, **kw)
    torch.cuda.synchronize()
    ok = oracle_kw(a, conv=conv, gate=gate)
    ref = oracle.bwd(a["x"], a["dt"], a["A_log"], a["B"], a["C"], a["dout"], euler=euler,
                     h0=a["h0"], conv_hist=a["conv_hist"] if conv else None,
                     dh_last=a["dh_last"], **ok)
    from gpu_helpers import assert_grad_close
    for k in GRADS:
        if k in ref and k in g:
            assert_grad_close(k, to_np(g[k]), ref[k])
            assert_grad_close(k + " vs one pass", to_np(g[k]), to_np(g1[k]))


@pytest.mark.parametrize("nseg", [2, 3, 7])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_split_backward(nseg, dtype):
    _bwd_case(2, 24, 16, 1000, dtype, nseg)


@pytest.mark.parametrize("case", ["no_conv", "no_gate", "plain", "euler", "recompute", "N5", "N64"])
def test_split_backward_variants(case):
    kw = dict(conv=case != "no_conv", gate=case != "no_gate", carried=case != "plain",
              euler=case == "euler", saved=case != "recompute")
    N = {"N5": 5, "N64": 64}.get(case, 16)
    _bwd_case(1, 16, N, 777, "bf16", 4, **kw)


def test_split_backward_long_few_channels():
    _bwd_case(1, 32, 16, 8192, "bf16", 16, carried=False)


@pytest.mark.slow
def test_full_few_channel_long_split_sampled():
    """The split-L workload at full size (1 x 512 x 16 x 65536, bf16) in the benchmark's launch
    configuration (automatic split), forward and backward, on sampled channels; dB / dC with a dout
    that is zero outside the sampled channels, so every other channel contributes exactly zero."""
    from gpu_helpers import assert_grad_close, channel_slice
    w = wl.WORKLOADS["long_fewch_fwdbwd"]
    a = wl.generate(w)
    picks = wl.sample_channels(w.Bt, w.Dn, 6)
    mask = np.zeros((w.Bt, w.Dn, 1), dtype=np.float32)
    for b, d in picks:
        mask[b, d] = 1.0
    a["dout"] = a["dout"] * mask
    t = dev_arrays(a, "bf16")
    kw = param_kw(t)
    r = ssm.ssm_scan_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], out_dtype=torch.float32,
                         save_states=True, n_segments=-1, **kw)
    g = ssm.ssm_scan_bwd(t["dout"], t["x"], t["dt"], t["A_log"], t["B"], t["C"],
                         chunk_states=r["chunk_states"], n_segments=-1, **kw)
    torch.cuda.synchronize()
    out = to_np(r["out"])
    got = {k: to_np(v) for k, v in g.items()}
    dB_ref = np.zeros((w.Bt, w.N, w.L))
    dC_ref = np.zeros((w.Bt, w.N, w.L))
    for b, d in picks:
        s = channel_slice(a, b, d)
        ref = oracle.fwd(s["x"], s["dt"], s["A_log"], s["B"], s["C"], **oracle_kw(s))
        assert_close("out (b=%d,d=%d)" % (b, d), out[b:b + 1, d:d + 1], ref, *TOL[("bf16", "f32")])
        rg = oracle.bwd(s["x"], s["dt"], s["A_log"], s["B"], s["C"], s["dout"], **oracle_kw(s))
        for k in ("dx", "ddt", "dz"):
            assert_grad_close("%s (b=%d,d=%d)" % (k, b, d), got[k][b:b + 1, d:d + 1], rg[k])
        for k in ("dA_log", "dD", "ddt_bias", "dconv_w", "dconv_b"):
            assert_grad_close("%s (d=%d)" % (k, d), got[k][d:d + 1], rg[k])   # Bt = 1
        dB_ref[b] += rg["dB"][0]
        dC_ref[b] += rg["dC"][0]
    assert_grad_close("dB (masked)", got["dB"], dB_ref)
    assert_grad_close("dC (masked)", got["dC"], dC_ref)


def test_split_backward_deterministic():
    w = wl.shaped("mamba130m_fwd", Bt=1, Dn=32, N=16, L=2048, backward=True)
    a = wl.generate(w)
    t = dev_arrays(a, "bf16")
    kw = param_kw(t)
    g1 = ssm.ssm_scan_bwd(t["dout"], t["x"], t["dt"], t["A_log"], t["B"], t["C"], n_segments=8, **kw)
    g2 = ssm.ssm_scan_bwd(t["dout"], t["x"], t["dt"], t["A_log"], t["B"], t["C"], n_segments=8, **kw)
    torch.cuda.synchronize()
    for k in g1:
        assert torch.equal(g1[k], g2[k]), k
