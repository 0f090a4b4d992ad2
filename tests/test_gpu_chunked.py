"""The chunked (time-parallel) scan layout of the forward, scan_form="chunked": lanes own consecutive
time steps and each 64-step chunk is scanned by a warp-shuffle scan of (product of A_bar, end state)
pairs ("State-Space Models & Long-Context Sequence Architectures (Mamba)", Lab 3; "state-space
models", "One recurrence, one convolution"). Every output against the float64 oracle with the
forward tolerances, on shapes that cover one lane, one lane group, several chunks and ragged tails,
every optional piece, both input dtypes, the carried state, and the saved states the backward
consumes."""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_34_b200 as ssm
from selective_state_space_34_b200 import workloads as wl
from gpu_helpers import (TOL, assert_close, assert_grad_close, dev_arrays, oracle_kw, param_kw,
                         to_np)

pytestmark = pytest.mark.gpu


def _fwd(w, dtype_out="f32", conv=True, gate=True, D=True, bias=True, softplus=True, euler=False,
         check_u=True):
    a = wl.generate(w)
    t = dev_arrays(a, w.in_dtype)
    tdt = torch.bfloat16 if dtype_out == "bf16" else torch.float32
    res = ssm.ssm_scan_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], delta_softplus=softplus,
                           out_dtype=tdt, return_u=True, scan_form="chunked",
                           discretization="euler" if euler else "zoh",
                           **param_kw(t, conv and w.conv, gate and w.gate, D, bias))
    torch.cuda.synchronize()
    ref, ex = oracle.fwd(a["x"], a["dt"], a["A_log"], a["B"], a["C"], delta_softplus=softplus,
                         want_u=True, euler=euler,
                         **oracle_kw(a, conv and w.conv, gate and w.gate, D, bias))
    rtol, atol = TOL[(w.in_dtype, dtype_out)]
    assert_close("out", to_np(res["out"]), ref, rtol, atol)
    if check_u:
        assert_close("u", to_np(res["u"]), ex["u"], rtol, atol)


@pytest.mark.parametrize("Bt,Dn,N,L", [
    (1, 3, 16, 1), (1, 3, 16, 7), (2, 5, 16, 8), (1, 17, 16, 63), (2, 16, 16, 64), (1, 9, 16, 65),
    (2, 20, 16, 200), (1, 33, 16, 257),            # several chunks, ragged tails, Dn not x16
    (2, 9, 1, 50), (2, 9, 3, 50), (2, 9, 5, 50), (2, 9, 17, 50), (2, 9, 32, 130), (2, 9, 64, 130),
])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_shapes(Bt, Dn, N, L, dtype):
    _fwd(wl.shaped("mamba130m_fwd", Bt=Bt, Dn=Dn, N=N, L=L, in_dtype=dtype))


@pytest.mark.parametrize("variant", ["no_conv", "no_gate", "no_D", "no_bias", "bare", "euler", "bf16_out"])
def test_optional_pieces(variant):
    w = wl.shaped("mamba130m_fwd", Bt=2, Dn=20, L=150)
    if variant == "bare":
        _fwd(w, conv=False, gate=False, D=False, bias=False)
    else:
        _fwd(w, dtype_out="bf16" if variant == "bf16_out" else "f32", conv=variant != "no_conv",
             gate=variant != "no_gate", D=variant != "no_D", bias=variant != "no_bias",
             euler=variant == "euler")


@pytest.mark.parametrize("K", [1, 2, 3])
def test_conv_widths(K):
    _fwd(wl.shaped("mamba130m_fwd", Bt=1, Dn=12, L=140, K=K))


def test_misaligned_rows_take_the_scalar_path():
    # L = 77: rows not 16-byte aligned, every load and store element by element
    _fwd(wl.shaped("mamba130m_fwd", Bt=2, Dn=18, L=77))


@pytest.mark.parametrize("L", [1, 50, 200])
def test_carried_state_in_and_out(L):
    """h0 / conv_hist in, h_last / conv_hist out ("Selective Mamba", State, runArray)."""
    w = wl.shaped("mamba130m_fwd", Bt=2, Dn=10, L=L)
    a = wl.generate(w)
    cs = wl.carried_state(w)
    t = dev_arrays(a, "bf16")
    h0 = torch.from_numpy(cs["h0"]).cuda()
    hist = torch.from_numpy(cs["conv_hist"]).cuda().to(torch.bfloat16)
    res = ssm.ssm_scan_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], out_dtype=torch.float32,
                           h0=h0, conv_hist=hist, return_state=True, scan_form="chunked",
                           **param_kw(t))
    torch.cuda.synchronize()
    ref, ex = oracle.fwd(a["x"], a["dt"], a["A_log"], a["B"], a["C"], h0=cs["h0"],
                         conv_hist=cs["conv_hist"], want_state=True, **oracle_kw(a))
    rtol, atol = TOL[("bf16", "f32")]
    assert_close("out", to_np(res["out"]), ref, rtol, atol)
    assert_close("h_last", res["h_last"].cpu().numpy(), ex["h_last"], rtol, atol)
    assert np.array_equal(to_np(res["conv_hist"]), ex["conv_hist"])  # copied inputs: exact


def test_chunk_chain_equals_one_pass():
    """Consecutive calls carrying the state reproduce the oracle over the whole sequence."""
    w = wl.shaped("mamba130m_fwd", Bt=1, Dn=9, L=300)
    a = wl.generate(w)
    t = dev_arrays(a, "bf16")
    kw = param_kw(t)
    h, hist, outs = None, None, []
    for lo, hi in ((0, 70), (70, 71), (71, 71), (71, 300)):
        sl = {k: t[k][..., lo:hi].contiguous() for k in ("x", "dt", "z", "B", "C")}
        r = ssm.ssm_scan_fwd(sl["x"], sl["dt"], t["A_log"], sl["B"], sl["C"], out_dtype=torch.float32,
                             h0=h, conv_hist=hist, return_state=True, scan_form="chunked",
                             **dict(kw, z=sl["z"]))
        h, hist = r["h_last"], r["conv_hist"]
        outs.append(r["out"])
    torch.cuda.synchronize()
    got = torch.cat(outs, dim=-1).cpu().numpy()
    ref = oracle.fwd(a["x"], a["dt"], a["A_log"], a["B"], a["C"], **oracle_kw(a))
    assert_close("chain", got, ref, *TOL[("bf16", "f32")])


@pytest.mark.parametrize("L", [16, 70, 200])
def test_saved_states_feed_the_backward(L):
    """The states saved every 16 steps match the lane layout's, and the backward run from them
    gives the oracle's gradients."""
    w = wl.shaped("mamba130m_fwd", Bt=2, Dn=24, L=L, backward=True)
    a = wl.generate(w)
    t = dev_arrays(a, "bf16")
    kw = param_kw(t)
    ch = ssm.ssm_scan_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], save_states=True,
                          scan_form="chunked", **kw)
    ln = ssm.ssm_scan_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], save_states=True, **kw)
    g = ssm.ssm_scan_bwd(t["dout"], t["x"], t["dt"], t["A_log"], t["B"], t["C"],
                         chunk_states=ch["chunk_states"], **kw)
    torch.cuda.synchronize()
    # both layouts round differently; each is within the forward tolerance of the true states
    lane_states = ln["chunk_states"].cpu().numpy().astype(np.float64)
    assert_close("states", ch["chunk_states"].cpu().numpy(), lane_states, 2e-3,
                 1e-4 * np.abs(lane_states).max())
    ref = oracle.bwd(a["x"], a["dt"], a["A_log"], a["B"], a["C"], a["dout"], **oracle_kw(a))
    for k in ("dx", "ddt", "dz", "dA_log", "dB", "dC", "dD", "ddt_bias", "dconv_w", "dconv_b"):
        assert_grad_close(k, to_np(g[k]), ref[k])


def test_backward_recomputing_states_with_the_chunked_layout():
    w = wl.shaped("mamba130m_fwd", Bt=1, Dn=20, L=130, backward=True)
    a = wl.generate(w)
    t = dev_arrays(a, "bf16")
    g = ssm.ssm_scan_bwd(t["dout"], t["x"], t["dt"], t["A_log"], t["B"], t["C"], scan_form="chunked",
                         **param_kw(t))
    torch.cuda.synchronize()
    ref = oracle.bwd(a["x"], a["dt"], a["A_log"], a["B"], a["C"], a["dout"], **oracle_kw(a))
    for k in ("dx", "ddt", "dz", "dA_log", "dB", "dC"):
        assert_grad_close(k, to_np(g[k]), ref[k])
