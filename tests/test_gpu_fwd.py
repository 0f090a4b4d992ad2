"""Forward parity: the CUDA path (through the C ABI) against the float64 oracle on the same seeded
inputs, element by element; plus full-size workloads in the benchmark's launch configuration on
sampled channels, invariants, and edge cases."""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_34_b200 as ssm
from selective_state_space_34_b200 import workloads as wl
from gpu_helpers import (TOL, assert_close, channel_slice, dev_arrays, oracle_kw, param_kw, to_np)

pytestmark = pytest.mark.gpu


def run_case(w, conv=True, gate=True, D=True, bias=True, softplus=True, out_dtype=None,
             seed=None, check_u=False):
    a = wl.generate(w, seed=seed)
    t = dev_arrays(a, w.in_dtype)
    od = out_dtype or "f32"
    tdt = torch.bfloat16 if od == "bf16" else torch.float32
    res = ssm.ssm_scan_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], delta_softplus=softplus,
                           out_dtype=tdt, return_u=True,
                           **param_kw(t, conv and w.conv, gate and w.gate, D, bias))
    torch.cuda.synchronize()
    ref, ex = oracle.fwd(a["x"], a["dt"], a["A_log"], a["B"], a["C"], delta_softplus=softplus,
                         want_u=True, **oracle_kw(a, conv and w.conv, gate and w.gate, D, bias))
    rtol, atol = TOL[(w.in_dtype, od)]
    assert_close("out", to_np(res["out"]), ref, rtol, atol)
    if check_u:
        assert_close("u", to_np(res["u"]), ex["u"], rtol, atol)
    return a, t, res


def test_tiny_fp32_workload():
    # 1 x 16 x 4 x 64, fp32, scan only (no conv): the oracle's own small case, every element
    run_case(wl.WORKLOADS["tiny_fp32"], check_u=True)


@pytest.mark.parametrize("Bt,Dn,N,L", [
    (2, 40, 16, 200),     # several stages + ragged tail (200 = 6*32 + 8)
    (1, 33, 16, 77),      # L not a multiple of 8: scalar staging path; Dn not a tile multiple
    (3, 5, 16, 32),       # exactly one stage
    (1, 7, 16, 1), (1, 7, 16, 2), (1, 7, 16, 3),   # shorter than the conv
    (2, 9, 1, 50), (2, 9, 3, 50), (2, 9, 4, 50), (2, 9, 5, 50), (2, 9, 8, 50),
    (2, 9, 12, 50), (2, 9, 24, 50), (2, 9, 32, 50), (2, 9, 48, 50), (2, 9, 64, 50),
])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_shapes(Bt, Dn, N, L, dtype):
    w = wl.shaped("mamba130m_fwd", Bt=Bt, Dn=Dn, N=N, L=L, in_dtype=dtype)
    run_case(w, check_u=True)


@pytest.mark.parametrize("Bt,Dn", [(2, 4800), (1, 5000), (1, 3000)])
def test_every_lane_layout(Bt, Dn):
    # channel counts that select 4, 8 and 16 lanes per channel for d_state = 16
    w = wl.shaped("mamba130m_fwd", Bt=Bt, Dn=Dn, L=40)
    run_case(w)


@pytest.mark.parametrize("variant", ["no_conv", "no_gate", "no_D", "no_bias", "raw_delta",
                                     "bare"])
def test_optional_pieces(variant):
    w = wl.shaped("mamba130m_fwd", Bt=2, Dn=20, L=96)
    kw = dict(conv=variant != "no_conv", gate=variant != "no_gate", D=variant != "no_D",
              bias=variant != "no_bias", softplus=variant != "raw_delta")
    if variant == "raw_delta":
        # dt is then Delta itself (plus dt_bias); keep it positive and small
        a = wl.generate(w)
        a["dt"] = wl.round_to_bf16(np.abs(a["dt"]) * 0.05 + 0.001)
        a["dt_bias"] = np.zeros_like(a["dt_bias"])
        t = dev_arrays(a, "bf16")
        out = ssm.ssm_scan_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], delta_softplus=False,
                               out_dtype=torch.float32, **param_kw(t))
        ref = oracle.fwd(a["x"], a["dt"], a["A_log"], a["B"], a["C"], delta_softplus=False,
                         **oracle_kw(a))
        assert_close("out", to_np(out), ref, *TOL[("bf16", "f32")])
        return
    if variant == "bare":
        kw = dict(conv=False, gate=False, D=False, bias=False)
    run_case(w, **kw)


@pytest.mark.parametrize("K", [1, 2, 3, 4])
def test_conv_widths(K):
    w = wl.shaped("mamba130m_fwd", Bt=1, Dn=12, L=70, K=K)
    run_case(w, check_u=True)


def test_bf16_output():
    w = wl.shaped("mamba130m_fwd", Bt=2, Dn=24, L=136)
    run_case(w, out_dtype="bf16", check_u=True)


def test_misaligned_views_take_the_scalar_path():
    w = wl.shaped("mamba130m_fwd", Bt=1, Dn=6, L=64)
    a = wl.generate(w)
    t = dev_arrays(a, "bf16")
    # views starting one element in: 2-byte aligned, not 16-byte aligned
    def shift(v):
        buf = torch.empty(v.numel() + 1, dtype=v.dtype, device=v.device)
        buf[1:] = v.reshape(-1)
        return buf[1:].view(v.shape)
    t2 = dict(t)
    for k in ("x", "dt", "z", "B", "C"):
        t2[k] = shift(t[k])
    out = ssm.ssm_scan_fwd(t2["x"], t2["dt"], t2["A_log"], t2["B"], t2["C"],
                           out_dtype=torch.float32, **param_kw(t2))
    ref = oracle.fwd(a["x"], a["dt"], a["A_log"], a["B"], a["C"], **oracle_kw(a))
    assert_close("out", to_np(out), ref, *TOL[("bf16", "f32")])


@pytest.mark.parametrize("Dn,N", [(4800, 16), (20, 16), (20, 12), (20, 5)])  # 4800: 4 states per lane
def test_saved_states_into_a_misaligned_buffer(Dn, N):
    """A caller's saved-state buffer need only be 4-byte aligned: one starting a float in gives the
    same bits as an aligned one (16-byte stores only where base, row and lane offsets allow them)."""
    import ctypes
    from selective_state_space_34_b200 import _abi, api
    w = wl.shaped("mamba130m_fwd", Bt=2, Dn=Dn, N=N, L=72)
    t = dev_arrays(wl.generate(w), "bf16")
    kw = param_kw(t)
    ref = ssm.ssm_scan_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], save_states=True, **kw)
    flat = torch.full((ref["chunk_states"].numel() + 1,), float("nan"), device="cuda")
    out = torch.empty_like(ref["out"])
    args, _ = api._fwd_args(t["x"], t["dt"], t["A_log"], t["B"], t["C"], kw["D"], kw["z"], kw["dt_bias"],
                            kw["conv_w"], kw["conv_b"], True, ref["out"].dtype)
    args.out, args.chunk_states = out.data_ptr(), flat[1:].data_ptr()
    _abi.check("ssm_scan_fwd", _abi.load().ssm_scan_fwd(ctypes.byref(args), torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    assert torch.equal(flat[1:].view_as(ref["chunk_states"]), ref["chunk_states"])
    assert torch.equal(out, ref["out"])
    # the backward reads such a buffer as well (16-byte loads only where aligned): same gradients
    dout = torch.randn(out.shape, device="cuda", generator=torch.Generator("cuda").manual_seed(2)).to(t["x"].dtype)
    g_al = ssm.ssm_scan_bwd(dout, t["x"], t["dt"], t["A_log"], t["B"], t["C"],
                            chunk_states=ref["chunk_states"], **kw)
    g_mis = ssm.ssm_scan_bwd(dout, t["x"], t["dt"], t["A_log"], t["B"], t["C"],
                             chunk_states=flat[1:].view_as(ref["chunk_states"]), **kw)
    torch.cuda.synchronize()
    for k in g_al:
        assert torch.equal(g_al[k], g_mis[k]), k


def test_empty_problems_leave_outputs_alone():
    x = torch.zeros(2, 4, 0, device="cuda")
    out = ssm.ssm_scan_fwd(x, x, torch.zeros(4, 16, device="cuda"), torch.zeros(2, 16, 0, device="cuda"),
                           torch.zeros(2, 16, 0, device="cuda"))
    assert out.shape == (2, 4, 0)
    x = torch.zeros(0, 4, 8, device="cuda")
    ssm.ssm_scan_fwd(x, x, torch.zeros(4, 16, device="cuda"), torch.zeros(0, 16, 8, device="cuda"),
                     torch.zeros(0, 16, 8, device="cuda"))
    torch.cuda.synchronize()


def test_run_to_run_determinism():
    w = wl.shaped("mamba130m_fwd", Bt=2, Dn=64, L=300)
    a = wl.generate(w)
    t = dev_arrays(a, "bf16")
    o1 = ssm.ssm_scan_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], **param_kw(t))
    o2 = ssm.ssm_scan_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], **param_kw(t))
    assert torch.equal(o1, o2)


def test_causality_on_device():
    w = wl.shaped("mamba130m_fwd", Bt=1, Dn=8, L=128, in_dtype="f32")
    a = wl.generate(w)
    t = dev_arrays(a, "f32")
    base = ssm.ssm_scan_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], **param_kw(t))
    t0 = 77
    for k in ("x", "dt", "B", "C", "z"):
        t2 = dict(t)
        t2[k] = t[k].clone()
        t2[k][..., t0] += 0.5
        pert = ssm.ssm_scan_fwd(t2["x"], t2["dt"], t2["A_log"], t2["B"], t2["C"], **param_kw(t2))
        assert torch.equal(pert[..., :t0], base[..., :t0]), k
        assert not torch.equal(pert[..., t0:], base[..., t0:]), k


def test_chunk_states_are_the_states():
    # With C = e_n, D = 0 and no gate the oracle's output is h_t[n]; compare the saved states.
    w = wl.shaped("mamba130m_fwd", Bt=2, Dn=10, N=8, L=70)
    a = wl.generate(w)
    t = dev_arrays(a, "bf16")
    res = ssm.ssm_scan_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], save_states=True,
                           **param_kw(t))
    st = res["chunk_states"].cpu().numpy()           # (Bt, Dn, n_ck, N)
    ends = [min(16 * (k + 1), 70) - 1 for k in range(st.shape[2])]
    for n in range(w.N):
        Ce = np.zeros_like(a["C"])
        Ce[:, n, :] = 1.0
        h = oracle.fwd(a["x"], a["dt"], a["A_log"], a["B"], Ce, D=None, z=None,
                       dt_bias=a["dt_bias"], conv_w=a["conv_w"], conv_b=a["conv_b"])
        assert_close("state n=%d" % n, st[:, :, :, n], h[:, :, ends], 2e-3, 1e-4)


# ---- full-size workloads in the benchmark's launch configuration --------------------------------

def _sampled_parity(name, out_dtype, k=24, **over):
    w = wl.WORKLOADS[name]
    a = wl.generate(w)
    t = dev_arrays(a, w.in_dtype)
    tdt = torch.bfloat16 if out_dtype == "bf16" else torch.float32
    out = ssm.ssm_scan_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], out_dtype=tdt,
                           **param_kw(t, w.conv, w.gate))
    torch.cuda.synchronize()
    got = to_np(out)
    del out, t
    for b, d in wl.sample_channels(w.Bt, w.Dn, k):
        s = channel_slice(a, b, d)
        ref = oracle.fwd(s["x"], s["dt"], s["A_log"], s["B"], s["C"], **oracle_kw(s, w.conv, w.gate))
        assert_close("%s (b=%d,d=%d)" % (name, b, d), got[b:b + 1, d:d + 1], ref,
                     *TOL[(w.in_dtype, out_dtype)])
    assert np.all(np.isfinite(got))


@pytest.mark.slow
def test_full_mamba130m_sampled():
    _sampled_parity("mamba130m_fwd", "f32")


@pytest.mark.slow
@pytest.mark.parametrize("out_dtype", ["bf16", "f32"])
def test_full_mamba1p4b_sampled(out_dtype):
    _sampled_parity("mamba1p4b_fwd", out_dtype)


@pytest.mark.slow
def test_full_long_context_sampled():
    _sampled_parity("long_fwd", "bf16", k=12)


@pytest.mark.slow
def test_long_context_closed_form_carry():
    # Constant u and B along the sequence: h_t = (B u / |A|)(1 - exp(A * (t+1) * Delta_d)) for the
    # per-channel Delta of the long workload -- checks the carry over 65536 steps with no oracle.
    w = wl.WORKLOADS["long_fwd"]
    Dn, N, L = 256, w.N, w.L
    rng = np.random.default_rng(3)
    lu = rng.uniform(np.log(1e-3), np.log(1e-1), Dn)
    delta = np.exp(lu)
    dt_bias = wl.softplus_inverse(delta).astype(np.float32)
    u = wl.round_to_bf16(rng.uniform(0.5, 1.5, Dn).astype(np.float32))
    Bv = wl.round_to_bf16(rng.standard_normal(N).astype(np.float32) * 0.25)
    Cv = wl.round_to_bf16(rng.standard_normal(N).astype(np.float32) * 0.25)
    A_log = np.tile(np.log(np.arange(1, N + 1, dtype=np.float64)), (Dn, 1)).astype(np.float32)
    dev = "cuda"
    bf = torch.bfloat16
    x = torch.from_numpy(u).to(dev, bf)[None, :, None].expand(1, Dn, L).contiguous()
    dt = torch.zeros(1, Dn, L, device=dev, dtype=bf)
    B = torch.from_numpy(Bv).to(dev, bf)[None, :, None].expand(1, N, L).contiguous()
    C = torch.from_numpy(Cv).to(dev, bf)[None, :, None].expand(1, N, L).contiguous()
    out = ssm.ssm_scan_fwd(x, dt, torch.from_numpy(A_log).to(dev), B, C,
                           dt_bias=torch.from_numpy(dt_bias).to(dev), out_dtype=torch.float32)
    got = out[0].cpu().numpy().astype(np.float64)
    A = -np.exp(A_log.astype(np.float64))
    dlt = np.array([oracle.softplus(v) for v in dt_bias.astype(np.float64)])
    ts = np.arange(L, dtype=np.float64) + 1.0
    for d in range(0, Dn, 37):
        h = (Bv[:, None].astype(np.float64) * u[d] / np.abs(A[d])[:, None]) * \
            (1.0 - np.exp(A[d][:, None] * dlt[d] * ts[None, :]))
        ref = (Cv[:, None].astype(np.float64) * h).sum(axis=0)
        assert_close("closed form d=%d" % d, got[d], ref, 2e-3, 1e-4)
