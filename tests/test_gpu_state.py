"""Parity of the carried state ("Selective Mamba", State / step / runArray; the state-space models
page, the selective scan step): a forward that starts from h0 and a conv history and returns the
final state, chained chunks against one pass, the single-token decode step against the oracle run
step by step, the Euler discretisation, and the backward's gradients w.r.t. the carried state."""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_34_b200 as ssm
from selective_state_space_34_b200 import workloads as wl
from gpu_helpers import (TOL, assert_close, assert_grad_close, dev_arrays, oracle_kw, param_kw,
                         to_np)

pytestmark = pytest.mark.gpu

GRADS = ["dx", "ddt", "dz", "dA_log", "dB", "dC", "dD", "ddt_bias", "dconv_w", "dconv_b",
         "dh0", "dconv_hist"]


def _setup(Bt, Dn, N, L, dtype, conv=True, gate=True, backward=False, seed=None):
    w = wl.shaped("mamba130m_fwd", Bt=Bt, Dn=Dn, N=N, L=L, in_dtype=dtype, conv=conv, gate=gate,
                  backward=backward)
    a = wl.generate(w, seed=seed)
    a.update(wl.carried_state(w, seed=seed))
    return w, a, dev_arrays(a, dtype)


@pytest.mark.parametrize("L", [1, 2, 3, 5, 16, 17, 77, 200])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("euler", [False, True])
def test_fwd_from_carried_state(L, dtype, euler):
    w, a, t = _setup(2, 40, 16, L, dtype)
    disc = "euler" if euler else "zoh"
    r = ssm.ssm_scan_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], out_dtype=torch.float32,
                         h0=t["h0"], conv_hist=t["conv_hist"], return_state=True,
                         discretization=disc, **param_kw(t))
    torch.cuda.synchronize()
    ref, ex = oracle.fwd(a["x"], a["dt"], a["A_log"], a["B"], a["C"], euler=euler, h0=a["h0"],
                         conv_hist=a["conv_hist"], want_state=True, **oracle_kw(a))
    rtol, atol = TOL[(dtype, "f32")]
    assert_close("out", to_np(r["out"]), ref, rtol, atol)
    assert_close("h_last", to_np(r["h_last"]), ex["h_last"], rtol, atol)
    # the history is a copy of inputs: exact
    assert np.array_equal(to_np(r["conv_hist"]), ex["conv_hist"])


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_fwd_state_without_conv_or_gate(dtype):
    w, a, t = _setup(1, 24, 8, 50, dtype, conv=False, gate=False)
    r = ssm.ssm_scan_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], out_dtype=torch.float32,
                         h0=t["h0"], return_state=True, **param_kw(t, conv=False, gate=False))
    torch.cuda.synchronize()
    ref, ex = oracle.fwd(a["x"], a["dt"], a["A_log"], a["B"], a["C"], h0=a["h0"], want_state=True,
                         **oracle_kw(a, conv=False, gate=False))
    rtol, atol = TOL[(dtype, "f32")]
    assert_close("out", to_np(r["out"]), ref, rtol, atol)
    assert_close("h_last", to_np(r["h_last"]), ex["h_last"], rtol, atol)
    assert "conv_hist" not in r


def test_zero_state_matches_plain_forward():
    """h0 = 0 and a zero history are the plain forward, bit for bit."""
    w, a, t = _setup(2, 48, 16, 100, "bf16")
    kw = param_kw(t)
    plain = ssm.ssm_scan_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], **kw)
    zs = ssm.ssm_scan_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], **kw,
                          h0=torch.zeros_like(t["h0"]), conv_hist=torch.zeros_like(t["conv_hist"]))
    assert torch.equal(plain, zs)


@pytest.mark.parametrize("cuts", [(0, 37, 37, 100, 160), (1, 2, 3, 64), (50,)])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_chunks_chain_to_one_pass(cuts, dtype):
    """Running the sequence in chunks, each starting from the previous chunk's final state and
    conv history (including empty and one-step chunks), gives the one-pass result."""
    L = 160
    w, a, t = _setup(2, 40, 16, L, dtype)
    kw = param_kw(t)
    bounds = [0] + [c for c in cuts if c <= L] + [L]
    h, hist, outs = t["h0"], t["conv_hist"], []
    for lo, hi in zip(bounds[:-1], bounds[1:]):
        sl = lambda v: v[..., lo:hi].contiguous()
        r = ssm.ssm_scan_fwd(sl(t["x"]), sl(t["dt"]), t["A_log"], sl(t["B"]), sl(t["C"]),
                             **dict(kw, z=sl(t["z"])), out_dtype=torch.float32, h0=h,
                             conv_hist=hist, return_state=True)
        h, hist = r["h_last"], r["conv_hist"]
        outs.append(r["out"])
    torch.cuda.synchronize()
    ref, ex = oracle.fwd(a["x"], a["dt"], a["A_log"], a["B"], a["C"], h0=a["h0"],
                         conv_hist=a["conv_hist"], want_state=True, **oracle_kw(a))
    rtol, atol = TOL[(dtype, "f32")]
    assert_close("out", to_np(torch.cat(outs, dim=-1)), ref, rtol, atol)
    assert_close("h_last", to_np(h), ex["h_last"], rtol, atol)
    assert np.array_equal(to_np(hist), ex["conv_hist"])


def test_empty_chunk_carries_state_through():
    w, a, t = _setup(2, 16, 16, 0, "bf16")
    r = ssm.ssm_scan_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], h0=t["h0"],
                         conv_hist=t["conv_hist"], return_state=True, **param_kw(t))
    r0 = ssm.ssm_scan_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], return_state=True,
                          **param_kw(t))
    torch.cuda.synchronize()
    assert torch.equal(r["h_last"], t["h0"]) and torch.equal(r["conv_hist"], t["conv_hist"])
    assert not r0["h_last"].any() and not r0["conv_hist"].any()


@pytest.mark.parametrize("T", [1, 5, 40])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("euler", [False, True])
def test_decode_steps_match_oracle(T, dtype, euler):
    """T calls of the one-token step from (h0, conv_hist) give the oracle's outputs for the
    T-token sequence and its final state."""
    w, a, t = _setup(3, 72, 16, T, dtype)
    disc = "euler" if euler else "zoh"
    h, hist = t["h0"].clone(), t["conv_hist"].clone()
    outs = []
    for s in range(T):
        col = lambda v: v[..., s].contiguous()
        outs.append(ssm.ssm_scan_step(col(t["x"]), col(t["dt"]), t["A_log"], col(t["B"]),
                                      col(t["C"]), h, hist, D=t["D"], z=col(t["z"]),
                                      dt_bias=t["dt_bias"], conv_w=t["conv_w"],
                                      conv_b=t["conv_b"], out_dtype=torch.float32,
                                      discretization=disc))
    torch.cuda.synchronize()
    ref, ex = oracle.fwd(a["x"], a["dt"], a["A_log"], a["B"], a["C"], euler=euler, h0=a["h0"],
                         conv_hist=a["conv_hist"], want_state=True, **oracle_kw(a))
    rtol, atol = TOL[(dtype, "f32")]
    assert_close("out", to_np(torch.stack(outs, dim=-1)), ref, rtol, atol)
    assert_close("h", to_np(h), ex["h_last"], rtol, atol)
    assert np.array_equal(to_np(hist), ex["conv_hist"])


@pytest.mark.parametrize("N", [1, 4, 16, 24, 32, 33, 64])
def test_decode_step_state_sizes_and_bf16_out(N):
    w, a, t = _setup(2, 33, N, 1, "bf16", gate=False)
    h, hist = t["h0"].clone(), t["conv_hist"].clone()
    col = lambda v: v[..., 0].contiguous()
    y = ssm.ssm_scan_step(col(t["x"]), col(t["dt"]), t["A_log"], col(t["B"]), col(t["C"]), h, hist,
                          D=t["D"], dt_bias=t["dt_bias"], conv_w=t["conv_w"], conv_b=t["conv_b"])
    torch.cuda.synchronize()
    assert y.dtype == torch.bfloat16
    ref, ex = oracle.fwd(a["x"], a["dt"], a["A_log"], a["B"], a["C"], h0=a["h0"],
                         conv_hist=a["conv_hist"], want_state=True, **oracle_kw(a, gate=False))
    rtol, atol = TOL[("bf16", "bf16")]
    assert_close("out", to_np(y), ref[..., 0], rtol, atol)
    assert_close("h", to_np(h), ex["h_last"], *TOL[("bf16", "f32")])


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_decode_step_misaligned_rows_give_the_same_bits(dtype):
    """State, A_log, B and C one element off a 16-byte boundary take the element-by-element path
    of the state passes; the same values in aligned storage take the 16-byte path. Same bits."""
    w, a, t = _setup(3, 45, 16, 1, dtype)
    col = lambda v: v[..., 0].contiguous()

    def shifted(v):  # the same values, starting one element into a fresh buffer
        buf = torch.empty(v.numel() + 1, dtype=v.dtype, device=v.device)
        out = buf[1:].view(v.shape)
        out.copy_(v)
        return out

    kw = dict(D=t["D"], z=col(t["z"]), dt_bias=t["dt_bias"], conv_w=t["conv_w"], conv_b=t["conv_b"],
              out_dtype=torch.float32)
    h1, hist1 = t["h0"].clone(), t["conv_hist"].clone()
    y1 = ssm.ssm_scan_step(col(t["x"]), col(t["dt"]), t["A_log"], col(t["B"]), col(t["C"]), h1, hist1, **kw)
    h2, hist2 = shifted(t["h0"]), t["conv_hist"].clone()
    y2 = ssm.ssm_scan_step(col(t["x"]), col(t["dt"]), shifted(t["A_log"]), shifted(col(t["B"])),
                           shifted(col(t["C"])), h2, hist2, **kw)
    torch.cuda.synchronize()
    assert h2.data_ptr() % 16 != 0
    assert torch.equal(y1, y2) and torch.equal(h1, h2) and torch.equal(hist1, hist2)


def test_scan_then_step_continues_the_scan():
    """A scan over the first L-1 tokens followed by one decode step matches the scan over L."""
    L = 33
    w, a, t = _setup(2, 40, 16, L, "f32")
    kw = param_kw(t)
    full = ssm.ssm_scan_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], **kw)
    sl = lambda v: v[..., :L - 1].contiguous()
    r = ssm.ssm_scan_fwd(sl(t["x"]), sl(t["dt"]), t["A_log"], sl(t["B"]), sl(t["C"]),
                         **dict(kw, z=sl(t["z"])), return_state=True)
    col = lambda v: v[..., L - 1].contiguous()
    y = ssm.ssm_scan_step(col(t["x"]), col(t["dt"]), t["A_log"], col(t["B"]), col(t["C"]),
                          r["h_last"], r["conv_hist"], D=t["D"], z=col(t["z"]),
                          dt_bias=t["dt_bias"], conv_w=t["conv_w"], conv_b=t["conv_b"])
    torch.cuda.synchronize()
    assert_close("last", to_np(y), to_np(full[..., L - 1]), 1e-5, 1e-6)


def _bwd(t, kw, L_slice=None, h0=None, conv_hist=None, dh_last=None, disc="zoh"):
    return ssm.ssm_scan_bwd(t["dout"], t["x"], t["dt"], t["A_log"], t["B"], t["C"], **kw,
                            h0=h0, conv_hist=conv_hist, dh_last=dh_last, discretization=disc,
                            state_grads=True)


@pytest.mark.parametrize("L", [1, 3, 16, 17, 50, 200])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("euler", [False, True])
def test_bwd_with_carried_state(L, dtype, euler):
    w, a, t = _setup(2, 40, 16, L, dtype, backward=True)
    disc = "euler" if euler else "zoh"
    kw = param_kw(t)
    states = ssm.ssm_scan_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], save_states=True,
                              h0=t["h0"], conv_hist=t["conv_hist"], discretization=disc,
                              **kw)["chunk_states"]
    g = ssm.ssm_scan_bwd(t["dout"], t["x"], t["dt"], t["A_log"], t["B"], t["C"], **kw,
                         chunk_states=states, h0=t["h0"], conv_hist=t["conv_hist"],
                         dh_last=t["dh_last"], discretization=disc)
    g2 = _bwd(t, kw, h0=t["h0"], conv_hist=t["conv_hist"], dh_last=t["dh_last"], disc=disc)
    torch.cuda.synchronize()
    ref = oracle.bwd(a["x"], a["dt"], a["A_log"], a["B"], a["C"], a["dout"], euler=euler,
                     h0=a["h0"], conv_hist=a["conv_hist"], dh_last=a["dh_last"], **oracle_kw(a))
    for k in GRADS:
        assert_grad_close(k, to_np(g[k]), ref[k])
        assert_grad_close(k + " (recomputed states)", to_np(g2[k]), ref[k])


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_euler_plain_forward_and_backward(dtype):
    """Euler without any carried state, on a shape spanning several tiles and a ragged tail."""
    w, a, t = _setup(2, 300, 16, 83, dtype, backward=True)
    kw = param_kw(t)
    out = ssm.ssm_scan_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], out_dtype=torch.float32,
                           discretization="euler", **kw)
    g = ssm.ssm_scan_bwd(t["dout"], t["x"], t["dt"], t["A_log"], t["B"], t["C"],
                         discretization="euler", **kw)
    torch.cuda.synchronize()
    ok = oracle_kw(a)
    ref = oracle.fwd(a["x"], a["dt"], a["A_log"], a["B"], a["C"], euler=True, **ok)
    assert_close("out", to_np(out), ref, *TOL[(dtype, "f32")])
    gref = oracle.bwd(a["x"], a["dt"], a["A_log"], a["B"], a["C"], a["dout"], euler=True, **ok)
    for k in GRADS[:10]:
        assert_grad_close(k, to_np(g[k]), gref[k])


def test_bwd_chunks_chain_to_one_pass():
    """Backward over two chunks: the second chunk's dh0 is the first chunk's dh_last, and its
    dconv_hist adds into the first chunk's dx over its last K-1 steps; parameter gradients add."""
    L, cut = 120, 45
    w, a, t = _setup(2, 40, 16, L, "f32", backward=True)
    kw = param_kw(t)
    sl1 = lambda v: v[..., :cut].contiguous()
    sl2 = lambda v: v[..., cut:].contiguous()
    r1 = ssm.ssm_scan_fwd(sl1(t["x"]), sl1(t["dt"]), t["A_log"], sl1(t["B"]), sl1(t["C"]),
                          **dict(kw, z=sl1(t["z"])), h0=t["h0"], conv_hist=t["conv_hist"],
                          return_state=True)
    g2 = ssm.ssm_scan_bwd(sl2(t["dout"]), sl2(t["x"]), sl2(t["dt"]), t["A_log"], sl2(t["B"]),
                          sl2(t["C"]), **dict(kw, z=sl2(t["z"])), h0=r1["h_last"],
                          conv_hist=r1["conv_hist"], state_grads=True)
    g1 = ssm.ssm_scan_bwd(sl1(t["dout"]), sl1(t["x"]), sl1(t["dt"]), t["A_log"], sl1(t["B"]),
                          sl1(t["C"]), **dict(kw, z=sl1(t["z"])), h0=t["h0"],
                          conv_hist=t["conv_hist"], dh_last=g2["dh0"])
    torch.cuda.synchronize()
    ref = oracle.bwd(a["x"], a["dt"], a["A_log"], a["B"], a["C"], a["dout"], h0=a["h0"],
                     conv_hist=a["conv_hist"], **oracle_kw(a))
    K1 = t["conv_w"].shape[1] - 1
    dx1 = g1["dx"].clone()
    # entry j of the history is step cut-1-j of the first chunk
    dx1[..., cut - K1:] += g2["dconv_hist"].flip(-1)
    for k in ("dx", "ddt", "dz", "dB", "dC"):
        assert_grad_close(k, to_np(torch.cat([dx1 if k == "dx" else g1[k], g2[k]], dim=-1)),
                          ref[k])
    for k in ("dA_log", "dD", "ddt_bias", "dconv_w", "dconv_b"):
        assert_grad_close(k, to_np(g1[k] + g2[k]), ref[k])
    assert_grad_close("dh0", to_np(g1["dh0"]), ref["dh0"])
    assert_grad_close("dconv_hist", to_np(g1["dconv_hist"]), ref["dconv_hist"])


def test_bwd_empty_chunk_passes_the_state_gradient():
    w, a, t = _setup(2, 16, 16, 0, "bf16", backward=True)
    g = _bwd(t, param_kw(t), h0=t["h0"], conv_hist=t["conv_hist"], dh_last=t["dh_last"])
    torch.cuda.synchronize()
    assert torch.equal(g["dh0"], t["dh_last"])
    assert not g["dconv_hist"].any() and not g["dA_log"].any() and not g["dconv_w"].any()
