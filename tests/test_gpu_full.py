"""Full-tensor parity on the measured workloads: every element of every result of the CUDA path,
in the benchmark's launch configurations, against the float64 oracle.

Workloads (seeds 1000 + index, distributions of the rustytorch commit log's "canonical S6 init"
and "Selective Mamba", Parameters): the 130M-shaped block 2 x 1536 x 16 x 2048, the 1.4B-shaped
block 4 x 4096 x 16 x 4096 (fp32 and bf16 output), the long-context case 1 x 5120 x 16 x 65536,
and the forward + backward step on the 1.4B shape (out and all ten gradients).

The oracle runs channel blocks of one batch element each, in a thread pool (every call
single-threaded; the C oracle releases the GIL). Channels are independent in the method, so a
block's outputs are the oracle's outputs for those channels. dB and dC are sums over channels and
the per-channel parameter gradients sums over batch elements: the blocks' float64 contributions
are added here, in block order, before the comparison. Every comparison uses the tolerances of the
other parity tests (tests/gpu_helpers.py); for a gradient the absolute part is 1e-4 of the largest
oracle value of that whole tensor.
"""
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import oracle
import selective_state_space_34_b200 as ssm
from selective_state_space_34_b200 import workloads as wl
from gpu_helpers import GRAD_ATOL_FRAC, GRAD_RTOL, TOL, dev_arrays, param_kw

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

THREADS = max(1, os.cpu_count() or 1)


def _blocks(Bt, Dn, per):
    return [(b, lo, min(Dn, lo + per)) for b in range(Bt) for lo in range(0, Dn, per)]


def _slice(a, b, lo, hi):
    """Inputs of channels lo..hi-1 of batch element b, as a Bt = 1 problem."""
    s = slice(lo, hi)
    kw = dict(D=a["D"][s], z=None if a["z"] is None else a["z"][b:b + 1, s],
              dt_bias=a["dt_bias"][s],
              conv_w=None if a["conv_w"] is None else a["conv_w"][s],
              conv_b=None if a["conv_b"] is None else a["conv_b"][s])
    return (a["x"][b:b + 1, s], a["dt"][b:b + 1, s], a["A_log"][s], a["B"][b:b + 1],
            a["C"][b:b + 1], kw)


def _excess(got, ref, rtol):
    """max over elements of |got - ref| - rtol |ref| (the absolute part is compared later)."""
    got = np.asarray(got, dtype=np.float64)
    if not np.all(np.isfinite(got)):
        return np.inf
    return float(np.max(np.abs(got - ref) - rtol * np.abs(ref)))


def _to_host(t):
    return t.float().cpu().numpy() if t.dtype == torch.bfloat16 else t.cpu().numpy()


# ---- forward ------------------------------------------------------------------------------------

def _full_forward(name, out_dtype, n_segments, per=64, scan_form="lanes"):
    w = wl.WORKLOADS[name]
    a = wl.generate(w)
    t = dev_arrays(a, w.in_dtype)
    tdt = torch.bfloat16 if out_dtype == "bf16" else torch.float32
    out = ssm.ssm_scan_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], out_dtype=tdt,
                           n_segments=n_segments, scan_form=scan_form, **param_kw(t, w.conv, w.gate))
    torch.cuda.synchronize()
    got = _to_host(out)
    del out, t
    torch.cuda.empty_cache()
    rtol, atol = TOL[(w.in_dtype, out_dtype)]

    def check(blk):
        b, lo, hi = blk
        x, dt, Al, B, C, kw = _slice(a, b, lo, hi)
        ref = oracle.fwd(x, dt, Al, B, C, n_threads=1, **kw)[0]
        return _excess(got[b, lo:hi], ref, rtol), int(np.sum(
            np.abs(got[b, lo:hi].astype(np.float64) - ref) > atol + rtol * np.abs(ref)))

    with ThreadPoolExecutor(max_workers=THREADS) as ex:
        res = list(ex.map(check, _blocks(w.Bt, w.Dn, per)))
    worst = max(r[0] for r in res)
    n_bad = sum(r[1] for r in res)
    assert worst <= atol and n_bad == 0, (
        "%s (%s out, n_segments %d): %d of %d elements outside rtol %g atol %g (worst excess %g)"
        % (name, out_dtype, n_segments, n_bad, got.size, rtol, atol, worst))


@pytest.mark.parametrize("n_segments", [0, -1])
def test_mamba130m_every_element(n_segments):
    # 2 x 1536 x 16 x 2048: one pass, and the automatic split-L choice (4 segments on B200)
    _full_forward("mamba130m_fwd", "f32", n_segments)


@pytest.mark.parametrize("out_dtype", ["bf16", "f32"])
def test_mamba1p4b_every_element(out_dtype):
    # 4 x 4096 x 16 x 4096, one pass (the automatic choice keeps this shape in one pass)
    _full_forward("mamba1p4b_fwd", out_dtype, 0)


@pytest.mark.parametrize("n_segments", [0, -1])
def test_long_context_every_element(n_segments):
    # 1 x 5120 x 16 x 65536: one pass, and the automatic split (8 segments on B200)
    _full_forward("long_fwd", "bf16", n_segments, per=32)


@pytest.mark.parametrize("name,per", [("mamba1p4b_fwd", 64), ("long_fwd", 32)])
def test_chunked_layout_every_element(name, per):
    # the chunked (time-parallel) scan layout, one pass, bf16 out
    _full_forward(name, "bf16", 0, per=per, scan_form="chunked")


# ---- forward + backward step --------------------------------------------------------------------

GRADS_ACT = ("dx", "ddt", "dz")                       # (Bt, Dn, L): compared block by block
GRADS_PARAM = ("dA_log", "dD", "ddt_bias", "dconv_w", "dconv_b")  # summed over batch elements


def test_fwdbwd_step_every_element():
    """The benchmark's step on 4 x 4096 x 16 x 4096: the forward saving its chunk states (bf16
    output), then the backward from them. Every element of out and of all ten gradients."""
    w = wl.WORKLOADS["mamba1p4b_fwdbwd"]
    a = wl.generate(w)
    t = dev_arrays(a, w.in_dtype)
    kw = param_kw(t, w.conv, w.gate)
    res = ssm.ssm_scan_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], out_dtype=torch.bfloat16,
                           save_states=True, **kw)
    g = ssm.ssm_scan_bwd(t["dout"], t["x"], t["dt"], t["A_log"], t["B"], t["C"],
                         chunk_states=res["chunk_states"], **kw)
    torch.cuda.synchronize()
    got_out = _to_host(res["out"])
    got = {k: v.cpu().numpy() for k, v in g.items()}
    del res, g, t
    torch.cuda.empty_cache()
    rtol_o, atol_o = TOL[(w.in_dtype, "bf16")]

    def run(blk):
        b, lo, hi = blk
        x, dt, Al, B, C, okw = _slice(a, b, lo, hi)
        dout = a["dout"][b:b + 1, lo:hi]
        out = oracle.fwd(x, dt, Al, B, C, n_threads=1, **okw)[0]
        r = oracle.bwd(x, dt, Al, B, C, dout, n_threads=1, **okw)
        st = {"out": (_excess(got_out[b, lo:hi], out, rtol_o), float(np.abs(out).max()))}
        for k in GRADS_ACT:
            st[k] = (_excess(got[k][b, lo:hi], r[k][0], GRAD_RTOL), float(np.abs(r[k]).max()))
        return blk, st, r["dB"][0], r["dC"][0], {k: r[k] for k in GRADS_PARAM}

    dB = np.zeros((w.Bt, w.N, w.L))
    dC = np.zeros((w.Bt, w.N, w.L))
    par = {k: np.zeros(got[k].shape) for k in GRADS_PARAM}
    worst = {k: (-np.inf, 0.0) for k in ("out",) + GRADS_ACT}
    with ThreadPoolExecutor(max_workers=THREADS) as ex:
        for (b, lo, hi), st, rb, rc, rp in ex.map(run, _blocks(w.Bt, w.Dn, 32)):
            for k, (e, m) in st.items():
                worst[k] = (max(worst[k][0], e), max(worst[k][1], m))
            dB[b] += rb
            dC[b] += rc
            for k in GRADS_PARAM:
                par[k][lo:hi] += rp[k]
    e, _ = worst["out"]
    assert e <= atol_o, "out: worst excess %g over atol %g" % (e, atol_o)
    for k in GRADS_ACT:
        e, m = worst[k]
        assert e <= GRAD_ATOL_FRAC * m, "%s: worst excess %g over atol %g" % (k, e, GRAD_ATOL_FRAC * m)
    whole = dict(par, dB=dB, dC=dC)
    for k, ref in whole.items():
        e = _excess(got[k], ref, GRAD_RTOL)
        atol = GRAD_ATOL_FRAC * max(float(np.abs(ref).max()), 1e-30)
        assert e <= atol, "%s: worst excess %g over atol %g" % (k, e, atol)
