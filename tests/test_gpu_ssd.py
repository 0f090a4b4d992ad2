"""Parity of the Mamba-2 state-space-duality forward on the tensor cores ("state-space models",
"Mamba-2 and state-space duality") against the float64 recurrence of the oracle, in both forms: the
fused one-launch kernel (form "auto" picks it for P = 64) and the three-pass one ("three_pass";
"auto" picks it for P = 128).

Bound, from the arithmetic. bf16 keeps 8 significant bits, so one round-to-nearest changes a value
by at most 2^-8 of itself. Every output is a sum of terms (C_t . B_s) (decay) beta_s x_s (plus D x_t
and the carried state's terms); the inputs x, B, C are bf16 already, and a term meets at most two
roundings on its way:
  * a term from the same chunk: the masked, decayed score (C_t . B_s) 2^{ct_t - q_s} (with D on its
    diagonal) rounded to bf16 as the operand of G'X -- one rounding;
  * a term from an earlier chunk: the scaled operand of the chunk-state product (e^{cum_end - cum_s}
    beta_s B_s in the three-pass form, the same weight times x_s in the fused form), and the state
    entering the chunk (bf16 operand of C H_in) -- two.
So the bf16 part is at most ((1 + 2^-8)^2 - 1) Y_abs, with Y_abs the oracle run on |x|, |B|, |C|,
|D| (|h0|): an upper bound on the sum of the terms' magnitudes (|C_t . B_s| <= |C_t| . |B_s|; beta,
the decays and the state recursion are non-negative maps of non-negative inputs). The fp32 part:
  * each tensor-core product accumulates at most 128 products in fp32 (<= 2^-16 of their magnitude
    sum, allowing a truncating accumulator), at most three products on a term's path;
  * the carry between chunks, one multiply-add per chunk (<= 2^-20 each, <= 64 chunks here);
  * the exp2 / exp approximations, <= 2^-21 each, at most three factors on a path;
  together below 2^-12 Y_abs; and
  * the exponents: cum_t is a chunk-local running sum of Delta A in fp32 whose partial sums are at
    most M = max over chunks of sum |Delta A|, so each of its ~10 roundings and the conversion to
    base 2 move an exponent by at most about M 2^-24 (log2 e for base 2); a factor 2^e with e off by
    de changes by ln2 de of itself. 16 M 2^-24 Y_abs covers it.
Total: |y - y_ref| <= (2^-7 + 2^-16 + 2^-12 + 16 M 2^-24) Y_abs, plus 2^-8 |y_ref| for a bf16 output.
The final state h_last is carried in fp32 and meets only the scaled-operand rounding:
|h - h_ref| <= (2^-8 + 2^-12 + 16 M 2^-24) H_abs."""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_34_b200 as ssm
from selective_state_space_34_b200 import _abi, workloads as wl

pytestmark = pytest.mark.gpu


def _decay_span(a, softplus=True, Q=128):
    """M of the bound: the largest chunk-local sum of |Delta A| over (batch, head, chunk)."""
    v = a["dt"].astype(np.float64) + a["dt_bias"].astype(np.float64)[None, :, None]
    delta = np.logaddexp(0.0, v) if softplus else v
    A = np.exp(a["A_log"].astype(np.float64))[None, :, None]
    x = np.abs(delta * A)
    L = x.shape[2]
    pad = (-L) % Q
    x = np.concatenate([x, np.zeros(x.shape[:2] + (pad,))], axis=2) if pad else x
    return float(x.reshape(x.shape[0], x.shape[1], -1, Q).sum(axis=3).max()) if x.size else 0.0


def bound_coefs(a, softplus=True):
    """(output coefficient, final-state coefficient) of the derived bound, times Y_abs / H_abs."""
    fp32 = 2.0 ** -12 + 16.0 * _decay_span(a, softplus) * 2.0 ** -24
    return 2.0 ** -7 + 2.0 ** -16 + fp32, 2.0 ** -8 + fp32


def _run(Bt, H, L, P, N, out_dtype=torch.float32, euler=False, softplus=True, carry=False, D=True,
         seed=7, form="auto"):
    a = wl.generate_ssd(Bt, H, L, P, N, seed=seed)
    if not softplus:
        # without softplus dt + dt_bias is Delta itself: a step size, so non-negative
        a["dt"] = wl.round_to_bf16(np.abs(a["dt"]) * np.float32(0.05))
        a["dt_bias"] = np.zeros_like(a["dt_bias"])
    dev = "cuda"
    t = {k: torch.from_numpy(v).to(dev, torch.bfloat16 if k in ("x", "dt", "B", "C") else torch.float32)
         for k, v in a.items()}
    h0 = None
    if carry:
        h0_np = np.random.default_rng(seed).standard_normal((Bt, H, N, P)).astype(np.float32) * 0.3
        h0 = torch.from_numpy(h0_np).to(dev)
    r = ssm.ssm_ssd_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], D=t["D"] if D else None,
                        dt_bias=t["dt_bias"], h0=h0, delta_softplus=softplus, out_dtype=out_dtype,
                        discretization="euler" if euler else "zoh", return_state=carry, form=form)
    torch.cuda.synchronize()
    y = (r[0] if carry else r).float().cpu().numpy()
    kw = dict(dt_bias=a["dt_bias"], delta_softplus=softplus, euler=euler)
    ref = oracle.ssd_fwd(a["x"], a["dt"], a["A_log"], a["B"], a["C"], D=a["D"] if D else None,
                         h0=None if h0 is None else h0.cpu().numpy(), want_state=carry, **kw)
    yref = ref[0] if carry else ref
    yabs = oracle.ssd_fwd(np.abs(a["x"]), a["dt"], a["A_log"], np.abs(a["B"]), np.abs(a["C"]),
                          D=np.abs(a["D"]) if D else None,
                          h0=None if h0 is None else np.abs(h0.cpu().numpy()), **kw)
    cy, ch = bound_coefs(a, softplus)
    tol = cy * yabs + (2.0 ** -8 * np.abs(yref) if out_dtype == torch.bfloat16 else 0.0)
    err = np.abs(y - yref)
    bad = err > tol
    assert np.all(np.isfinite(y))
    if bad.any():
        i = np.unravel_index(np.argmax(err - tol), err.shape)
        raise AssertionError("%d/%d outside the bound; worst at %s: gpu %r oracle %r bound %r"
                             % (bad.sum(), bad.size, i, y[i], yref[i], tol[i]))
    if carry:
        hl = r[1].cpu().numpy()
        # the final state is fp32 throughout except the chunk-state products' bf16 operands
        habs = oracle.ssd_fwd(np.abs(a["x"]), a["dt"], a["A_log"], np.abs(a["B"]), np.abs(a["C"]),
                              h0=np.abs(h0.cpu().numpy()), want_state=True, **kw)[1]
        herr = np.abs(hl - ref[1]) - ch * habs
        assert herr.max() <= 0, "final state: worst excess %g over the bound" % herr.max()
    return y, yref


FORMS = ["auto", "three_pass"]


@pytest.mark.parametrize("form", FORMS)
@pytest.mark.parametrize("P,N", [(64, 128), (64, 64), (128, 128), (128, 64)])
@pytest.mark.parametrize("L", [128, 300, 1, 129, 8])
def test_ssd_shapes(P, N, L, form):
    _run(2, 3, L, P, N, form=form)


@pytest.mark.parametrize("Bt,H,L,P,N,out", [
    (1, 8, 300, 128, 128, torch.float32),   # 8 heads per CTA; fp32 rows of 512 B leave in two passes
    (2, 4, 200, 128, 64, torch.bfloat16),   # 4 heads per CTA
    (1, 8, 130, 64, 64, torch.float32),     # 8 heads, N = 64 (half the C H_in slices), ragged tail
    (1, 6, 257, 64, 128, torch.bfloat16),   # 2 heads per CTA
])
@pytest.mark.parametrize("form", FORMS)
def test_ssd_head_groups(Bt, H, L, P, N, out, form):
    _run(Bt, H, L, P, N, out_dtype=out, carry=True, form=form)


@pytest.mark.parametrize("form", FORMS)
@pytest.mark.parametrize("variant", ["euler", "no_softplus", "bf16_out", "no_D", "carried_state"])
def test_ssd_variants(variant, form):
    _run(1, 2, 257, 64, 128, euler=variant == "euler", softplus=variant != "no_softplus",
         out_dtype=torch.bfloat16 if variant == "bf16_out" else torch.float32,
         D=variant != "no_D", carry=variant == "carried_state", form=form)


@pytest.mark.parametrize("form", FORMS)
def test_ssd_longer_sequence(form):
    """16 chunks: the carried state crosses many chunk boundaries."""
    _run(1, 4, 2048, 64, 128, form=form)


def test_ssd_fused_form_needs_head_dim_64():
    a = wl.generate_ssd(1, 2, 64, 128, 64, seed=2)
    t = {k: torch.from_numpy(v).to("cuda", torch.bfloat16 if k in ("x", "dt", "B", "C") else torch.float32)
         for k, v in a.items()}
    with pytest.raises(_abi.SSMError) as e:
        ssm.ssm_ssd_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], form="fused")
    assert e.value.code == 5  # SSM_ERR_UNSUPPORTED


def test_ssd_matches_selective_scan_for_one_channel_semantics():
    """Cross-check of the two CUDA paths' shared discretisation: with one head, the SSD of a
    sequence whose x is the same in all P channels equals P copies of the per-channel result, and
    the result is linear in x (doubling x doubles y)."""
    a = wl.generate_ssd(1, 2, 200, 64, 64, seed=3)
    x1 = a["x"].copy()
    x1[...] = a["x"][..., :1]
    t = {k: torch.from_numpy(v).to("cuda", torch.bfloat16 if k in ("x", "dt", "B", "C") else torch.float32)
         for k, v in a.items()}
    xs = torch.from_numpy(x1).to("cuda", torch.bfloat16)
    y = ssm.ssm_ssd_fwd(xs, t["dt"], t["A_log"], t["B"], t["C"], D=t["D"], dt_bias=t["dt_bias"],
                        out_dtype=torch.float32)
    y2 = ssm.ssm_ssd_fwd(xs * 2, t["dt"], t["A_log"], t["B"], t["C"], D=t["D"], dt_bias=t["dt_bias"],
                         out_dtype=torch.float32)
    torch.cuda.synchronize()
    torch.testing.assert_close(y, y[..., :1].expand_as(y), rtol=1e-6, atol=1e-7)  # same per channel
    assert torch.equal(y2, 2 * y)     # exact: scaling by 2 commutes with every rounding on the way


@pytest.mark.slow
@pytest.mark.parametrize("form", FORMS)
def test_full_ssd_layer_sampled_heads(form):
    """The benchmarked SSD layer at full size (4 x 64 heads x 64 x 4096, N = 128, bf16 out), on
    sampled (batch, head) pairs over the whole sequence, within the derived bound."""
    cfg = wl.SSD_WORKLOADS["ssd_fwd"]
    Bt, H, L, P, N = cfg["Bt"], cfg["H"], cfg["L"], cfg["P"], cfg["N"]
    a = wl.generate_ssd(Bt, H, L, P, N, seed=cfg["seed"])
    t = {k: torch.from_numpy(v).to("cuda", torch.bfloat16 if k in ("x", "dt", "B", "C") else torch.float32)
         for k, v in a.items()}
    y = ssm.ssm_ssd_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], D=t["D"], dt_bias=t["dt_bias"],
                        form=form)
    torch.cuda.synchronize()
    y = y.float().cpu().numpy()
    for (b, h) in wl.sample_channels(Bt, H, 8):
        sl = dict(x=a["x"][b:b + 1, h:h + 1], dt=a["dt"][b:b + 1, h:h + 1], B=a["B"][b:b + 1],
                  C=a["C"][b:b + 1], A_log=a["A_log"][h:h + 1], D=a["D"][h:h + 1],
                  dt_bias=a["dt_bias"][h:h + 1])
        ref = oracle.ssd_fwd(sl["x"], sl["dt"], sl["A_log"], sl["B"], sl["C"], D=sl["D"], dt_bias=sl["dt_bias"])
        yabs = oracle.ssd_fwd(np.abs(sl["x"]), sl["dt"], sl["A_log"], np.abs(sl["B"]), np.abs(sl["C"]),
                              D=np.abs(sl["D"]), dt_bias=sl["dt_bias"])
        got = y[b:b + 1, h:h + 1]
        tol = bound_coefs(sl)[0] * yabs + 2.0 ** -8 * np.abs(ref)
        assert np.all(np.abs(got - ref) <= tol), "head (%d, %d): worst excess %g" % (b, h, (np.abs(got - ref) - tol).max())


@pytest.mark.parametrize("form", FORMS)
def test_ssd_deterministic_and_empty(form):
    a = wl.generate_ssd(2, 8, 300, 64, 128, seed=11)
    t = {k: torch.from_numpy(v).to("cuda", torch.bfloat16 if k in ("x", "dt", "B", "C") else torch.float32)
         for k, v in a.items()}
    kw = dict(D=t["D"], dt_bias=t["dt_bias"], return_state=True, form=form)
    y1, h1 = ssm.ssm_ssd_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], **kw)
    y2, h2 = ssm.ssm_ssd_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], **kw)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2) and torch.equal(h1, h2)   # no atomics: bitwise run to run
    # an empty sequence hands the state through
    h0 = torch.randn(2, 8, 128, 64, device="cuda")
    e = lambda v, shape: torch.empty(shape, dtype=v.dtype, device="cuda")
    y0, hl = ssm.ssm_ssd_fwd(e(t["x"], (2, 8, 0, 64)), e(t["dt"], (2, 8, 0)), t["A_log"],
                             e(t["B"], (2, 0, 128)), e(t["C"], (2, 0, 128)), h0=h0, **kw)
    torch.cuda.synchronize()
    assert y0.numel() == 0 and torch.equal(hl, h0)


@pytest.mark.parametrize("form", FORMS)
def test_ssd_timing_events_bracket_the_output_kernel(form):
    """The optional event pair is recorded around the fused kernel, or the output kernel of the
    three-pass form: its interval is positive and shorter than the whole call."""
    a = wl.generate_ssd(2, 16, 1024, 64, 128, seed=5)
    t = {k: torch.from_numpy(v).to("cuda", torch.bfloat16 if k in ("x", "dt", "B", "C") else torch.float32)
         for k, v in a.items()}
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    for e in ev[:2]:
        e.record()  # the handles exist before they are passed down
    torch.cuda.synchronize()
    ev[2].record()
    y = ssm.ssm_ssd_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], D=t["D"], dt_bias=t["dt_bias"],
                        timing_events=ev[:2], form=form)
    ev[3].record()
    torch.cuda.synchronize()
    kernel_ms, call_ms = ev[0].elapsed_time(ev[1]), ev[2].elapsed_time(ev[3])
    assert 0.0 < kernel_ms < call_ms
    y2 = ssm.ssm_ssd_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], D=t["D"], dt_bias=t["dt_bias"],
                         form=form)
    torch.cuda.synchronize()
    assert torch.equal(y, y2)  # recording changes nothing in the result
