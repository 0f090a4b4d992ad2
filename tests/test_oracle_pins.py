"""Pins for the float64 oracle: values and identities fixed by the pages and by mathematics,
none of which is a re-typing of the oracle's own formulas.

Pages cited (title, section):
  "Sequence and state-space models" (docs.algenta.ai), `state_space_models` worked example;
  "state-space models" (aarnphm.xyz), "From continuous time to tokens", "One recurrence, one
  convolution"; "State-Space Models & Long-Context Sequence Architectures (Mamba)", Lab 1
  (dense ZOH via expm), Lab 2 (stable softplus), Lab 3 (associative scan);
  "Selective Mamba" (TorchLean), Parameters / State; rustytorch commit log (liveness,
  causality, determinism, finite-difference gradient check).
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.linalg

import oracle
from selective_state_space_34_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "scalar_ssm_worked_values.json")


@pytest.fixture(scope="module")
def gold():
    with open(GOLDEN) as f:
        return json.load(f)


def _single(x, dt, A_log, B, C, D=0.0, z=None, dt_bias=None, softplus=False, conv_w=None):
    """One channel, one batch element: x, dt, z are (L,), B, C are (N, L), A_log is (N,)."""
    L = len(x)
    N = len(A_log)
    out = oracle.fwd(np.asarray(x, float).reshape(1, 1, L), np.asarray(dt, float).reshape(1, 1, L),
                     np.asarray(A_log, float).reshape(1, N), np.asarray(B, float).reshape(1, N, L),
                     np.asarray(C, float).reshape(1, N, L), D=np.array([D], float),
                     z=None if z is None else np.asarray(z, float).reshape(1, 1, L),
                     dt_bias=None if dt_bias is None else np.array([dt_bias], float),
                     conv_w=conv_w, delta_softplus=softplus)
    return out[0, 0]


# ---- worked values printed on "Sequence and state-space models" -------------------------------

def test_softplus_worked_values(gold):
    assert oracle.softplus(gold["softplus_0"]["v"]) == gold["softplus_0"]["value"]
    assert oracle.softplus(gold["softplus_1"]["v"]) == gold["softplus_1"]["value"]


def test_zoh_worked_values(gold):
    ab, bb = oracle.zoh(gold["zoh_B_bar"]["A"], gold["zoh_B_bar"]["B"], gold["zoh_B_bar"]["delta"])
    assert ab == pytest.approx(gold["zoh_A_bar"]["value"], rel=1e-15, abs=0)
    assert bb == pytest.approx(gold["zoh_B_bar"]["value"], rel=1e-15, abs=0)


def test_first_step_of_full_forward_matches_worked_h1(gold):
    # a = -1 (A_log = 0), delta = 0.5 given directly, b = 2, x = 1, C = 1, D = 0: y_0 = h_1.
    y = _single([1.0], [0.5], [0.0], [[2.0]], [[1.0]], D=0.0, softplus=False)
    assert y[0] == pytest.approx(gold["recurrence_h1"]["value"], rel=1e-15, abs=0)


def test_exact_zoh_is_not_the_euler_step(gold):
    # The page puts Mamba's first-order B-bar = delta*B about 27% away from the exact value.
    y = _single([1.0], [0.5], [0.0], [[2.0]], [[1.0]], softplus=False)[0]
    euler = gold["euler_h1"]["delta"] * gold["euler_h1"]["B"] * gold["euler_h1"]["x"]
    assert euler == gold["euler_h1"]["value"]
    gap = (euler - y) / y
    assert abs(gap - gold["exact_vs_euler_gap"]["approx_fraction"]) < 0.005


def test_s4_kernel_lag2_via_impulse_response(gold):
    # Impulse response at lag 2 is C * A_bar^2 * B_bar; choose B so that B_bar = 2 at delta = 0.5.
    g = gold["s4_kernel_lag2"]
    delta, A = 0.5, -1.0
    B = g["B_bar"] * A / math.expm1(delta * A)
    y = _single([1.0, 0.0, 0.0], [delta] * 3, [0.0], [[B] * 3], [[g["C"]] * 3], softplus=False)
    assert y[2] == pytest.approx(g["value"], rel=1e-14, abs=0)
    assert math.exp(2 * delta * A) == pytest.approx(g["A_bar_squared"], rel=1e-15)


# ---- closed forms and identities ----------------------------------------------------------------

def test_halving_scalar_case_is_exact():
    # A = -1, B = C = 1, delta = softplus(0) = log 2: every step keeps exactly half the state and
    # adds half the input ("state-space models", "From continuous time to tokens").
    L = 40
    x = np.zeros(L)
    x[0] = 1.0
    y = _single(x, np.zeros(L), [0.0], [np.ones(L)], [np.ones(L)], D=0.0, dt_bias=0.0, softplus=True)
    expect = 2.0 ** -(np.arange(L) + 1.0)
    assert np.array_equal(y, expect)
    # and with a general input the state is the half-blend h_t = h_{t-1}/2 + x_t/2
    rng = np.random.default_rng(3)
    x = rng.standard_normal(L)
    y = _single(x, np.zeros(L), [0.0], [np.ones(L)], [np.ones(L)], dt_bias=0.0, softplus=True)
    h, ref = 0.0, []
    for v in x:
        h = 0.5 * h + 0.5 * v
        ref.append(h)
    np.testing.assert_allclose(y, ref, rtol=1e-14, atol=1e-16)


def test_fixed_coefficients_equal_brute_force_causal_convolution():
    # Constant delta, B, C: y_t = sum_j K_{t-j} x_j + D x_t with K_k = C A_bar^k B_bar
    # ("state-space models", "One recurrence, one convolution"). A_bar and B_bar come from the
    # dense zero-order hold with a matrix exponential (glossary Lab 1) on a diagonal A.
    rng = np.random.default_rng(11)
    N, L = 5, 48
    A_log = rng.uniform(-1.0, 1.5, N)
    A = -np.exp(A_log)
    delta = 0.37
    Bv, Cv = rng.standard_normal(N), rng.standard_normal(N)
    x = rng.standard_normal(L)
    Dd = 0.7
    Ad = scipy.linalg.expm(delta * np.diag(A))
    Bd = np.linalg.inv(delta * np.diag(A)) @ (Ad - np.eye(N)) @ (delta * Bv)
    K = np.array([Cv @ np.linalg.matrix_power(Ad, k) @ Bd for k in range(L)])
    ref = np.array([sum(K[t - j] * x[j] for j in range(t + 1)) + Dd * x[t] for t in range(L)])
    y = _single(x, np.full(L, delta), A_log, np.tile(Bv[:, None], L), np.tile(Cv[:, None], L),
                D=Dd, softplus=False)
    np.testing.assert_allclose(y, ref, rtol=1e-11, atol=1e-12)


def test_constant_input_closed_form_with_time_varying_delta():
    # Constant u and B over t: each exact-ZOH step is a convex blend towards B u / |A|, so
    # h_t[n] = (B_n u / |A_n|) (1 - exp(A_n * sum_{s<=t} delta_s)) for any delta sequence.
    rng = np.random.default_rng(5)
    N, L = 6, 300
    A_log = np.log(np.arange(1, N + 1) * 0.5)
    A = -np.exp(A_log)
    dt = rng.standard_normal(L) * 0.8
    bias = -3.0
    Bv = rng.standard_normal(N)
    C = rng.standard_normal((N, L))
    u = 0.8
    S = np.cumsum([oracle.softplus(v + bias) for v in dt])
    h = (Bv[:, None] * u / np.abs(A)[:, None]) * (1.0 - np.exp(A[:, None] * S[None, :]))
    ref = (C * h).sum(axis=0) + 0.25 * u
    y = _single(np.full(L, u), dt, A_log, np.tile(Bv[:, None], L), C, D=0.25, dt_bias=bias,
                softplus=True)
    np.testing.assert_allclose(y, ref, rtol=1e-11, atol=1e-13)


def test_associative_chunked_scan_equals_sequential():
    # The combine (A1, b1) o (A2, b2) = (A2 A1, A2 b1 + b2) scanned chunk by chunk with a carry
    # equals the sequential recurrence (glossary Lab 3, max difference < 1e-8), and both equal
    # the oracle's output for the same discretised pairs.
    rng = np.random.default_rng(2)
    N, L, chunk = 4, 200, 16
    A_log = rng.uniform(-0.5, 1.0, N)
    A = -np.exp(A_log)
    delta = rng.uniform(0.01, 0.5, L)
    Bm, Cm = rng.standard_normal((N, L)), rng.standard_normal((N, L))
    u = rng.standard_normal(L)
    a = np.exp(delta[None, :] * A[:, None])
    b = np.expm1(delta[None, :] * A[:, None]) / A[:, None] * Bm * u[None, :]
    seq = np.zeros((N, L))
    h = np.zeros(N)
    for t in range(L):
        h = a[:, t] * h + b[:, t]
        seq[:, t] = h
    par = np.zeros((N, L))
    carry = np.zeros(N)
    for c0 in range(0, L, chunk):
        # inclusive tree scan inside the chunk (Hillis-Steele), then apply the carry
        P, Q = a[:, c0:c0 + chunk].copy(), b[:, c0:c0 + chunk].copy()
        step = 1
        while step < P.shape[1]:
            P2, Q2 = P.copy(), Q.copy()
            P2[:, step:] = P[:, step:] * P[:, :-step]
            Q2[:, step:] = P[:, step:] * Q[:, :-step] + Q[:, step:]
            P, Q = P2, Q2
            step *= 2
        par[:, c0:c0 + chunk] = P * carry[:, None] + Q
        carry = par[:, c0 + P.shape[1] - 1]
    assert np.max(np.abs(seq - par)) < 1e-8
    y = _single(u, delta, A_log, Bm, Cm, softplus=False)
    np.testing.assert_allclose(y, (Cm * seq).sum(axis=0), rtol=1e-11, atol=1e-12)


def test_zoh_matches_dense_matrix_exponential():
    # Diagonal special case of the dense ZOH (glossary Lab 1): expm and an inverse.
    rng = np.random.default_rng(8)
    for _ in range(20):
        A = -math.exp(rng.uniform(-3, 3))
        B = rng.standard_normal()
        delta = math.exp(rng.uniform(-7, 1))
        ab, bb = oracle.zoh(A, B, delta)
        Ad = scipy.linalg.expm(np.array([[delta * A]]))[0, 0]
        Bd = (1.0 / (delta * A)) * (Ad - 1.0) * delta * B
        assert ab == pytest.approx(Ad, rel=1e-14)
        assert bb == pytest.approx(Bd, rel=1e-8)  # Ad - 1 cancels for tiny delta*A; oracle uses expm1


def test_softplus_stable_form_and_sigmoid():
    for v in [-30.0, -5.0, -0.3, 0.0, 0.7, 4.0, 25.0]:
        assert oracle.softplus(v) == pytest.approx(math.log1p(math.exp(v)), rel=1e-14)
    assert oracle.softplus(800.0) == 800.0            # no overflow in the stable form
    assert oracle.softplus(-800.0) == 0.0
    for v in [-40.0, -2.0, 0.0, 3.0, 40.0]:
        assert oracle.sigmoid(v) + oracle.sigmoid(-v) == pytest.approx(1.0, rel=1e-15)
        assert oracle.silu(v) == pytest.approx(v / (1.0 + math.exp(-v)), rel=1e-14)


# ---- conv orientation, zero weights, causality, determinism -------------------------------------

def test_conv_tap_zero_is_the_current_token():
    # "Selective Mamba": convKernel row zero multiplies the current projected token; history is
    # newest-first and zero-padded; the bias is added before the SiLU.
    rng = np.random.default_rng(4)
    x = rng.standard_normal((1, 2, 10))
    for k in range(4):
        w = np.zeros((2, 4))
        w[:, k] = 1.0
        u = oracle.conv1d_silu(x, w, np.zeros(2))
        shifted = np.zeros_like(x)
        shifted[..., k:] = x[..., :10 - k]
        expect = np.vectorize(oracle.silu)(shifted)
        assert np.array_equal(u, expect)


def test_zero_weights_return_the_bias():
    # Zero taps: conv output is the bias, u = SiLU(bias). B = 0: y = D u. D = 0 as well: out = 0.
    w = wl.shaped("fd_slice", Dn=3, L=12)
    a = wl.generate(w)
    conv_b = np.array([0.3, -1.2, 2.0])
    zeros_w = np.zeros_like(a["conv_w"])
    out, ex = oracle.fwd(a["x"], a["dt"], a["A_log"], np.zeros_like(a["B"]), a["C"], D=a["D"],
                         z=a["z"], dt_bias=a["dt_bias"], conv_w=zeros_w, conv_b=conv_b,
                         want_u=True, want_y=True)
    su = np.array([oracle.silu(v) for v in conv_b])
    assert np.array_equal(ex["u"], np.broadcast_to(su[None, :, None], ex["u"].shape))
    assert np.array_equal(ex["y"], a["D"][None, :, None] * ex["u"])
    out0 = oracle.fwd(a["x"], a["dt"], a["A_log"], np.zeros_like(a["B"]), a["C"],
                      D=np.zeros(3), z=a["z"], dt_bias=a["dt_bias"], conv_w=zeros_w, conv_b=conv_b)
    assert np.all(out0 == 0.0)


def test_causality_no_future_leakage():
    w = wl.shaped("fd_slice", Dn=4, L=40)
    a = wl.generate(w)
    kw = dict(D=a["D"], z=a["z"], dt_bias=a["dt_bias"], conv_w=a["conv_w"], conv_b=a["conv_b"])
    base = oracle.fwd(a["x"], a["dt"], a["A_log"], a["B"], a["C"], **kw)
    t0 = 23
    for name in ["x", "dt", "B", "C", "z"]:
        b = {k: (None if v is None else np.array(v, dtype=np.float64)) for k, v in a.items()}
        b[name][..., t0] += 0.5
        kw2 = dict(D=b["D"], z=b["z"], dt_bias=b["dt_bias"], conv_w=b["conv_w"], conv_b=b["conv_b"])
        pert = oracle.fwd(b["x"], b["dt"], b["A_log"], b["B"], b["C"], **kw2)
        assert np.array_equal(pert[..., :t0], base[..., :t0]), name
        assert not np.array_equal(pert[..., t0:], base[..., t0:]), name


def test_seeded_determinism():
    w = wl.shaped("mamba130m_fwd", Bt=1, Dn=6, L=50)
    a1, a2 = wl.generate(w), wl.generate(w)
    for k in a1:
        if a1[k] is None:
            assert a2[k] is None
        else:
            assert np.array_equal(a1[k], a2[k]), k
    kw = dict(D=a1["D"], z=a1["z"], dt_bias=a1["dt_bias"], conv_w=a1["conv_w"], conv_b=a1["conv_b"])
    o1 = oracle.fwd(a1["x"], a1["dt"], a1["A_log"], a1["B"], a1["C"], **kw)
    o2 = oracle.fwd(a1["x"], a1["dt"], a1["A_log"], a1["B"], a1["C"], n_threads=3, **kw)
    assert np.array_equal(o1, o2)
    a3 = wl.generate(w, seed=w.seed + 1)
    assert not np.array_equal(a1["x"], a3["x"])


def test_bf16_rounding_is_round_to_nearest_even():
    v = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -9, -2.5, 3.14159], np.float32)
    r = wl.round_to_bf16(v)
    assert r[0] == 1.0 and r[1] == 1.0 and r[2] == 1.0 + 2 ** -6 and r[3] == 1.0
    assert r[4] == -2.5 and abs(r[5] - 3.140625) == 0.0
    assert np.all((r.view(np.uint32) & 0xFFFF) == 0)


# ---- gradients: central finite differences of the oracle's own forward --------------------------

def _loss_and_inputs(a):
    names = ["x", "dt", "z", "B", "C", "A_log", "D", "dt_bias", "conv_w", "conv_b"]
    p = {k: np.array(a[k], dtype=np.float64) for k in names}

    def loss(q):
        out = oracle.fwd(q["x"], q["dt"], q["A_log"], q["B"], q["C"], D=q["D"], z=q["z"],
                         dt_bias=q["dt_bias"], conv_w=q["conv_w"], conv_b=q["conv_b"])
        return float(np.sum(out * a["dout"]))
    return p, loss


def test_backward_matches_central_finite_differences():
    # The analytic VJP against central differences on the 1x8x4x32 slice, every element, with the
    # rustytorch tolerance (5e-3 + 5e-2 |fd|) as the outer bound and a float64-tight inner bound.
    w = wl.WORKLOADS["fd_slice"]
    a = wl.generate(w)
    p, loss = _loss_and_inputs(a)
    g = oracle.bwd(p["x"], p["dt"], p["A_log"], p["B"], p["C"], a["dout"], D=p["D"], z=p["z"],
                   dt_bias=p["dt_bias"], conv_w=p["conv_w"], conv_b=p["conv_b"])
    gmap = {"x": "dx", "dt": "ddt", "z": "dz", "B": "dB", "C": "dC", "A_log": "dA_log",
            "D": "dD", "dt_bias": "ddt_bias", "conv_w": "dconv_w", "conv_b": "dconv_b"}
    h = 1e-6
    checked = 0
    for name, gname in gmap.items():
        an = g[gname]
        fd = np.zeros_like(an)
        flat = p[name].reshape(-1)
        for i in range(flat.size):
            old = flat[i]
            flat[i] = old + h
            lp = loss(p)
            flat[i] = old - h
            lm = loss(p)
            flat[i] = old
            fd.reshape(-1)[i] = (lp - lm) / (2 * h)
        scale = max(1.0, np.max(np.abs(fd)))
        assert np.all(np.abs(an - fd) <= 5e-3 + 5e-2 * np.abs(fd)), name
        np.testing.assert_allclose(an, fd, rtol=1e-6, atol=1e-7 * scale, err_msg=name)
        checked += fd.size
    assert checked >= 30


def test_every_parameter_is_live():
    # rustytorch liveness: on a generic seed every gradient has non-zero entries.
    w = wl.WORKLOADS["fd_slice"]
    a = wl.generate(w)
    g = oracle.bwd(a["x"], a["dt"], a["A_log"], a["B"], a["C"], a["dout"], D=a["D"], z=a["z"],
                   dt_bias=a["dt_bias"], conv_w=a["conv_w"], conv_b=a["conv_b"])
    for k, v in g.items():
        assert np.count_nonzero(v) > 0.9 * v.size, k


def test_backward_without_conv_and_gate_and_multibatch():
    # dx = du without a conv; dout = dy without a gate; per-channel grads sum over batch.
    rng = np.random.default_rng(21)
    Bt, Dn, N, L = 3, 2, 3, 9
    x, dt = rng.standard_normal((Bt, Dn, L)), rng.standard_normal((Bt, Dn, L)) * 0.5
    A_log = rng.uniform(-0.5, 0.5, (Dn, N))
    B, C = rng.standard_normal((Bt, N, L)), rng.standard_normal((Bt, N, L))
    D, bias = rng.standard_normal(Dn), np.full(Dn, -1.0)
    dout = rng.standard_normal((Bt, Dn, L))
    g = oracle.bwd(x, dt, A_log, B, C, dout, D=D, dt_bias=bias)
    parts = [oracle.bwd(x[i:i + 1], dt[i:i + 1], A_log, B[i:i + 1], C[i:i + 1], dout[i:i + 1],
                        D=D, dt_bias=bias) for i in range(Bt)]
    np.testing.assert_allclose(g["dA_log"], sum(p["dA_log"] for p in parts), rtol=1e-13)
    np.testing.assert_allclose(g["dD"], sum(p["dD"] for p in parts), rtol=1e-13)
    np.testing.assert_allclose(g["dB"], np.concatenate([p["dB"] for p in parts]), rtol=1e-13)

    def loss(xx):
        return float(np.sum(oracle.fwd(xx, dt, A_log, B, C, D=D, dt_bias=bias) * dout))
    fd = np.zeros_like(x)
    for i in range(x.size):
        xp, xm = x.copy(), x.copy()
        xp.reshape(-1)[i] += 1e-6
        xm.reshape(-1)[i] -= 1e-6
        fd.reshape(-1)[i] = (loss(xp) - loss(xm)) / 2e-6
    np.testing.assert_allclose(g["dx"], fd, rtol=1e-6, atol=1e-8)


# ---- state carry across chunks ("Selective Mamba": State, step, runArray) and the Euler step ----

def _carry_case(L=37, Dn=3, N=4, K=4, seed=31, euler=False):
    w = wl.shaped("fd_slice", Dn=Dn, N=N, L=L, K=K, seed=seed)
    a = wl.generate(w)
    kw = dict(D=a["D"], z=a["z"], dt_bias=a["dt_bias"], conv_w=a["conv_w"], conv_b=a["conv_b"],
              euler=euler)
    return a, kw


@pytest.mark.parametrize("split", [0, 1, 2, 3, 16, 36, 37])
@pytest.mark.parametrize("euler", [False, True])
def test_chunked_continuation_equals_one_pass(split, euler):
    # runArray: a chunk returns the hidden state and the conv history the next chunk needs; chunk
    # boundaries change nothing, so two chunks reproduce one pass exactly.
    a, kw = _carry_case(euler=euler)
    whole, ex = oracle.fwd(a["x"], a["dt"], a["A_log"], a["B"], a["C"], want_state=True, **kw)
    s1 = slice(0, split)
    s2 = slice(split, None)
    o1, e1 = oracle.fwd(a["x"][..., s1], a["dt"][..., s1], a["A_log"], a["B"][..., s1],
                        a["C"][..., s1], want_state=True, **dict(kw, z=a["z"][..., s1]))
    o2, e2 = oracle.fwd(a["x"][..., s2], a["dt"][..., s2], a["A_log"], a["B"][..., s2],
                        a["C"][..., s2], want_state=True, h0=e1["h_last"], conv_hist=e1["conv_hist"],
                        **dict(kw, z=a["z"][..., s2]))
    assert np.array_equal(np.concatenate([o1, o2], axis=-1), whole)
    assert np.array_equal(e2["h_last"], ex["h_last"])
    assert np.array_equal(e2["conv_hist"], ex["conv_hist"])


def test_empty_chunk_preserves_state():
    a, kw = _carry_case()
    rng = np.random.default_rng(4)
    h0 = rng.standard_normal((1, 3, 4))
    hist = rng.standard_normal((1, 3, 3))
    e = a["x"][..., :0]
    _, ex = oracle.fwd(e, e, a["A_log"], a["B"][..., :0], a["C"][..., :0], want_state=True,
                       h0=h0, conv_hist=hist, **dict(kw, z=e))
    assert np.array_equal(ex["h_last"], h0)
    assert np.array_equal(ex["conv_hist"], hist)


def test_single_token_steps_equal_one_pass():
    # step: one token at a time with the carried state reproduces the sequence.
    a, kw = _carry_case(L=12)
    whole = oracle.fwd(a["x"], a["dt"], a["A_log"], a["B"], a["C"], **kw)
    h, hist, outs = None, None, []
    for t in range(12):
        s = slice(t, t + 1)
        o, ex = oracle.fwd(a["x"][..., s], a["dt"][..., s], a["A_log"], a["B"][..., s],
                           a["C"][..., s], want_state=True, h0=h, conv_hist=hist,
                           **dict(kw, z=a["z"][..., s]))
        h, hist = ex["h_last"], ex["conv_hist"]
        outs.append(o)
    assert np.array_equal(np.concatenate(outs, axis=-1), whole)


def test_euler_first_step_worked_value(gold):
    # "Sequence and state-space models": mamba_selective_scan_step gives h_1 = 1.0 exactly.
    g = gold["euler_h1"]
    y = oracle.fwd(np.array([[[g["x"]]]]), np.array([[[g["delta"]]]]), np.zeros((1, 1)),
                   np.array([[[g["B"]]]]), np.ones((1, 1, 1)), D=np.zeros(1), delta_softplus=False,
                   euler=True)
    assert y[0, 0, 0] == g["value"]


def test_euler_approaches_exact_zoh_for_small_steps():
    # (A-bar - 1)/A = Delta (1 + Delta A / 2 + ...): the two discretisations agree to O(Delta A).
    for delta in [1e-1, 1e-2, 1e-3]:
        ye = oracle.fwd(np.ones((1, 1, 1)), np.full((1, 1, 1), delta), np.zeros((1, 1)),
                        np.ones((1, 1, 1)), np.ones((1, 1, 1)), delta_softplus=False, euler=True)
        yz = oracle.fwd(np.ones((1, 1, 1)), np.full((1, 1, 1), delta), np.zeros((1, 1)),
                        np.ones((1, 1, 1)), np.ones((1, 1, 1)), delta_softplus=False)
        rel = (ye - yz)[0, 0, 0] / yz[0, 0, 0]
        assert abs(rel - delta / 2) < delta * delta


@pytest.mark.parametrize("euler", [False, True])
def test_carried_state_gradients_match_finite_differences(euler):
    # gradients of every input including h0, the conv history, and an incoming dh_last
    a, kw = _carry_case(L=9, Dn=2, N=3, euler=euler)
    rng = np.random.default_rng(9)
    h0 = rng.standard_normal((1, 2, 3))
    hist = rng.standard_normal((1, 2, 3))
    dout = rng.standard_normal(a["x"].shape)
    dhl = rng.standard_normal((1, 2, 3))
    p = {"x": np.array(a["x"], float), "dt": np.array(a["dt"], float), "B": np.array(a["B"], float),
         "C": np.array(a["C"], float), "A_log": np.array(a["A_log"], float),
         "conv_w": np.array(a["conv_w"], float), "h0": h0.copy(), "conv_hist": hist.copy()}

    def loss():
        o, ex = oracle.fwd(p["x"], p["dt"], p["A_log"], p["B"], p["C"], want_state=True,
                           h0=p["h0"], conv_hist=p["conv_hist"],
                           **dict(kw, conv_w=p["conv_w"]))
        return float(np.sum(o * dout) + np.sum(ex["h_last"] * dhl))
    g = oracle.bwd(p["x"], p["dt"], p["A_log"], p["B"], p["C"], dout, h0=h0, conv_hist=hist,
                   dh_last=dhl, **dict(kw, conv_w=p["conv_w"]))
    names = {"x": "dx", "dt": "ddt", "B": "dB", "C": "dC", "A_log": "dA_log", "conv_w": "dconv_w",
             "h0": "dh0", "conv_hist": "dconv_hist"}
    for k, gk in names.items():
        flat = p[k].reshape(-1)
        fd = np.zeros(flat.size)
        for i in range(flat.size):
            old = flat[i]
            flat[i] = old + 1e-6
            lp = loss()
            flat[i] = old - 1e-6
            lm = loss()
            flat[i] = old
            fd[i] = (lp - lm) / 2e-6
        np.testing.assert_allclose(g[gk].reshape(-1), fd, rtol=1e-6, atol=1e-7 * max(1, np.abs(fd).max()),
                                   err_msg=gk)
