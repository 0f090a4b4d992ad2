"""Pins of the Mamba-2 state-space-duality (SSD) oracle ("state-space models", "Mamba-2 and
state-space duality") against things other than itself: the page's unrolled sum computed by brute
force, the page's matrix form Y = (L o Q K^T) V, the selective-scan oracle it reduces to when a
head has one channel, the worked scalar values printed on "Sequence and state-space models", the
causal linear attention it becomes when the decay is 1, and the chunked algorithm (matrix products
within chunks, states carried between them) that the GPU kernels use."""
import json
import os

import numpy as np
import pytest

import oracle

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "scalar_ssm_worked_values.json")))


def _case(Bt=2, H=3, L=11, P=4, N=5, seed=0):
    rng = np.random.default_rng(seed)
    return dict(x=rng.standard_normal((Bt, H, L, P)), dt=rng.standard_normal((Bt, H, L)),
                B=rng.standard_normal((Bt, L, N)) * 0.5, C=rng.standard_normal((Bt, L, N)) * 0.5,
                A_log=rng.uniform(-1.0, 1.0, H), D=rng.standard_normal(H),
                dt_bias=rng.uniform(-2.0, 0.5, H))


def _discretise(c, euler=False):
    """Delta, a and beta per (b, h, t) written out from the definitions (not the oracle's code)."""
    v = c["dt"] + c["dt_bias"][None, :, None]
    delta = np.logaddexp(0.0, v)                      # softplus
    A = -np.exp(c["A_log"])[None, :, None]
    a = np.exp(delta * A)
    beta = delta if euler else np.expm1(delta * A) / A
    return delta, a, beta


@pytest.mark.parametrize("euler", [False, True])
def test_unrolled_sum_by_brute_force(euler):
    c = _case()
    _, a, beta = _discretise(c, euler)
    Bt, H, L, P = c["x"].shape
    want = np.zeros_like(c["x"])
    for b in range(Bt):
        for h in range(H):
            for t in range(L):
                acc = np.zeros(P)
                for s in range(t + 1):
                    decay = np.prod(a[b, h, s + 1:t + 1])           # empty product = 1
                    acc += (c["C"][b, t] @ (beta[b, h, s] * c["B"][b, s])) * decay * c["x"][b, h, s]
                want[b, h, t] = acc + c["D"][h] * c["x"][b, h, t]
    got = oracle.ssd_fwd(c["x"], c["dt"], c["A_log"], c["B"], c["C"], D=c["D"], dt_bias=c["dt_bias"],
                         euler=euler)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


def test_matrix_form_masked_attention():
    """Y = (L o Q K^T) V with Q = C rows, K = B-bar rows, V = x, L_ts = prod_{k=s+1..t} a_k."""
    c = _case(seed=1)
    _, a, beta = _discretise(c)
    Bt, H, L, P = c["x"].shape
    got = oracle.ssd_fwd(c["x"], c["dt"], c["A_log"], c["B"], c["C"], D=None, dt_bias=c["dt_bias"])
    for b in range(Bt):
        for h in range(H):
            la = np.log(a[b, h])
            cum = np.cumsum(la)
            Lm = np.tril(np.exp(cum[:, None] - cum[None, :]))     # prod over k = s+1..t
            Q = c["C"][b]
            K = beta[b, h][:, None] * c["B"][b]
            Y = (Lm * (Q @ K.T)) @ c["x"][b, h]
            np.testing.assert_allclose(got[b, h], Y, rtol=1e-11, atol=1e-11)


@pytest.mark.parametrize("euler", [False, True])
def test_one_channel_heads_are_the_selective_scan(euler):
    """P = 1: head h is a selective-scan channel whose N states share one A (the selective-scan
    oracle, a separate function, with A_log[d, n] = A_log[h] for every n, no conv, no gate)."""
    c = _case(Bt=2, H=4, L=13, P=1, N=3, seed=2)
    got = oracle.ssd_fwd(c["x"], c["dt"], c["A_log"], c["B"], c["C"], D=c["D"], dt_bias=c["dt_bias"],
                         euler=euler)
    x = c["x"][..., 0]                                      # (Bt, Dn=H, L)
    A_log = np.repeat(c["A_log"][:, None], 3, axis=1)
    ref = oracle.fwd(x, c["dt"], A_log, c["B"].transpose(0, 2, 1), c["C"].transpose(0, 2, 1),
                     D=c["D"], dt_bias=c["dt_bias"], euler=euler)
    np.testing.assert_allclose(got[..., 0], ref, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("euler", [False, True])
def test_worked_scalar_values(euler):
    """The page's scalar example: A = -1, Delta = 0.5, B = 2, x = 1, C = 1, h_prev = 0."""
    x = np.ones((1, 1, 1, 1))
    y = oracle.ssd_fwd(x, np.full((1, 1, 1), 0.5), np.zeros(1), np.full((1, 1, 1), 2.0),
                       np.ones((1, 1, 1)), delta_softplus=False, euler=euler)
    want = GOLDEN["euler_h1"]["value"] if euler else GOLDEN["recurrence_h1"]["value"]
    assert y[0, 0, 0, 0] == pytest.approx(want, rel=1e-15)
    # a second step with x = 0 decays it by A_bar = exp(-0.5)
    y2 = oracle.ssd_fwd(np.array([[[[1.0], [0.0]]]]), np.full((1, 1, 2), 0.5), np.zeros(1),
                        np.full((1, 2, 1), 2.0), np.ones((1, 2, 1)), delta_softplus=False, euler=euler)
    assert y2[0, 0, 1, 0] == pytest.approx(want * GOLDEN["zoh_A_bar"]["value"], rel=1e-15)


def test_unit_decay_is_causal_linear_attention():
    """A -> 0 makes every a_t = 1; with the Euler input, y_t = sum_{s<=t} (C_t . B_s) Delta_s x_s."""
    c = _case(seed=3)
    c["A_log"] = np.full(3, -60.0)
    delta, _, _ = _discretise(c, euler=True)
    got = oracle.ssd_fwd(c["x"], c["dt"], c["A_log"], c["B"], c["C"], dt_bias=c["dt_bias"], euler=True)
    Bt, H, L, P = c["x"].shape
    for b in range(Bt):
        for h in range(H):
            kv = np.cumsum((delta[b, h][:, None, None] * c["B"][b][:, :, None]) * c["x"][b, h][:, None, :], axis=0)
            y = np.einsum("tn,tnp->tp", c["C"][b], kv)
            np.testing.assert_allclose(got[b, h], y, rtol=1e-10, atol=1e-10)


@pytest.mark.parametrize("Q", [1, 4, 5, 16])
def test_chunked_algorithm(Q):
    """Matrix products within chunks of Q steps plus states carried between chunks (the form the
    GPU computes) give the recurrence: Y_c = (L_c o C_c Bbar_c^T) X_c + diag(e^{cum}) C_c H_{c-1},
    H_c = e^{cum_end} H_{c-1} + Bbar_c^T diag(e^{cum_end - cum}) X_c."""
    c = _case(L=23, seed=4)
    _, a, beta = _discretise(c)
    Bt, H, L, P = c["x"].shape
    N = c["B"].shape[2]
    got = oracle.ssd_fwd(c["x"], c["dt"], c["A_log"], c["B"], c["C"], D=c["D"], dt_bias=c["dt_bias"])
    for b in range(Bt):
        for h in range(H):
            state = np.zeros((N, P))
            out = np.zeros((L, P))
            for c0 in range(0, L, Q):
                sl = slice(c0, min(L, c0 + Q))
                cum = np.cumsum(np.log(a[b, h, sl]))
                Bb = beta[b, h, sl][:, None] * c["B"][b, sl]
                Cc, X = c["C"][b, sl], c["x"][b, h, sl]
                Lm = np.tril(np.exp(cum[:, None] - cum[None, :]))
                out[sl] = (Lm * (Cc @ Bb.T)) @ X + np.exp(cum)[:, None] * (Cc @ state)
                state = np.exp(cum[-1]) * state + Bb.T @ (np.exp(cum[-1] - cum)[:, None] * X)
            out += c["D"][h] * c["x"][b, h]
            np.testing.assert_allclose(got[b, h], out, rtol=1e-10, atol=1e-10)


def test_state_carry_splits_the_sequence():
    c = _case(L=17, seed=5)
    kw = dict(D=c["D"], dt_bias=c["dt_bias"])
    full, hl = oracle.ssd_fwd(c["x"], c["dt"], c["A_log"], c["B"], c["C"], want_state=True, **kw)
    y1, h1 = oracle.ssd_fwd(c["x"][:, :, :9], c["dt"][:, :, :9], c["A_log"], c["B"][:, :9],
                            c["C"][:, :9], want_state=True, **kw)
    y2, h2 = oracle.ssd_fwd(c["x"][:, :, 9:], c["dt"][:, :, 9:], c["A_log"], c["B"][:, 9:],
                            c["C"][:, 9:], h0=h1, want_state=True, **kw)
    np.testing.assert_allclose(np.concatenate([y1, y2], axis=2), full, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(h2, hl, rtol=1e-13, atol=1e-13)
