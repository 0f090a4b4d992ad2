"""Out-of-bounds writes and reads of uninitialised memory, detected without a sanitizer.

Every buffer the binding allocates for a call (outputs, saved states, workspaces) is carved out of
a larger allocation whose bytes are all set to a fill pattern, leaving guard bands of 4 KiB on
both sides. After the call:
  * both guard bands still hold the pattern (no write past either end of any buffer);
  * no element of an output still holds the pattern (every output element was written);
  * the results are bit-identical to the same call with another fill pattern (nothing reads
    memory the library did not write first, workspace included).
The inputs are copied into guarded buffers as well, so the last comparison also shows that nothing
outside an input buffer reaches a result. The shapes are ragged in every tiled axis (channels,
steps, heads) so that tails are exercised."""
import math

import numpy as np
import pytest
import torch

import selective_state_space_34_b200 as ssm
from selective_state_space_34_b200 import api
from selective_state_space_34_b200 import workloads as wl
from gpu_helpers import dev_arrays, param_kw

pytestmark = pytest.mark.gpu

GUARD = 4096


class GuardedTorch:
    """Stands in for the torch module inside the binding; empty() hands out guarded views."""

    def __init__(self, fill):
        self.fill = fill
        self.allocs = []

    def __getattr__(self, name):
        return getattr(torch, name)

    def empty(self, *size, dtype=None, device=None, **kw):
        shape = tuple(size[0]) if len(size) == 1 and isinstance(size[0], (tuple, list, torch.Size)) \
            else tuple(int(s) for s in size)
        dtype = dtype or torch.get_default_dtype()
        nbytes = math.prod(shape) * torch.empty((), dtype=dtype).element_size()
        raw = torch.full((2 * GUARD + nbytes,), self.fill, dtype=torch.uint8, device=device)
        t = raw[GUARD:GUARD + nbytes].view(dtype).view(shape)
        self.allocs.append((raw, nbytes, dtype))
        return t

    def check(self):
        for raw, nbytes, dtype in self.allocs:
            band = torch.cat([raw[:GUARD], raw[GUARD + nbytes:]])
            assert bool((band == self.fill).all()), "guard band written (%s, %d bytes)" % (dtype, nbytes)
            if dtype != torch.uint8 and nbytes:
                body = raw[GUARD:GUARD + nbytes].view(-1, torch.empty((), dtype=dtype).element_size())
                untouched = (body == self.fill).all(dim=1)
                assert not bool(untouched.any()), \
                    "%d of %d elements never written (%s)" % (int(untouched.sum()), body.shape[0], dtype)


def _inputs(g, t):
    """Copies of the input tensors in guarded buffers of g."""
    out = {}
    for k, v in t.items():
        if v is None:
            out[k] = None
        else:
            out[k] = g.empty(tuple(v.shape), dtype=v.dtype, device=v.device)
            out[k].copy_(v)
    return out


def _guarded(monkeypatch, fn):
    """Run fn() twice under two fill patterns; check guards and return both results."""
    outs = []
    for fill in (0xA5, 0x5A):
        g = GuardedTorch(fill)
        monkeypatch.setattr(api, "torch", g)
        try:
            r = fn(g)
            torch.cuda.synchronize()
        finally:
            monkeypatch.setattr(api, "torch", torch)
        g.check()
        outs.append(r)
    return outs


def _flat(r):
    if isinstance(r, torch.Tensor):
        return {"": r}
    if isinstance(r, (tuple, list)):
        return {str(i): v for i, v in enumerate(r) if v is not None}
    return dict(r)


def _same(a, b):
    fa, fb = _flat(a), _flat(b)
    assert fa.keys() == fb.keys()
    for k in fa:
        x, y = fa[k].contiguous().view(torch.uint8), fb[k].contiguous().view(torch.uint8)
        assert torch.equal(x, y), "result %r depends on the initial memory contents" % k


def _setup(Bt, Dn, N, L, dtype, backward=False, seed=11):
    w = wl.shaped("mamba130m_fwd", Bt=Bt, Dn=Dn, N=N, L=L, in_dtype=dtype, conv=True, gate=True,
                  backward=backward)
    a = wl.generate(w, seed=seed)
    a.update(wl.carried_state(w, seed=seed))
    return dev_arrays(a, dtype)


@pytest.mark.parametrize("dtype,N,L,nseg", [("bf16", 16, 333, 0), ("bf16", 16, 333, 3),
                                            ("f32", 64, 100, 0), ("bf16", 4, 77, 2)])
def test_fwd_guards(monkeypatch, dtype, N, L, nseg):
    t = _setup(2, 70, N, L, dtype)
    od = torch.bfloat16 if dtype == "bf16" else torch.float32

    def run(g):
        i = _inputs(g, t)
        return ssm.ssm_scan_fwd(i["x"], i["dt"], i["A_log"], i["B"], i["C"], out_dtype=od,
                                save_states=True, return_u=True, return_state=True, h0=i["h0"],
                                conv_hist=i["conv_hist"], n_segments=nseg, **param_kw(i))

    a, b = _guarded(monkeypatch, run)
    _same(a, b)


@pytest.mark.parametrize("dtype,N,L", [("bf16", 16, 333), ("f32", 64, 100), ("bf16", 5, 77), ("f32", 16, 64)])
def test_chunked_fwd_guards(monkeypatch, dtype, N, L):
    """The chunked (time-parallel) forward: every output, saved state and carried state."""
    t = _setup(2, 70, N, L, dtype)
    od = torch.bfloat16 if dtype == "bf16" else torch.float32

    def run(g):
        i = _inputs(g, t)
        return ssm.ssm_scan_fwd(i["x"], i["dt"], i["A_log"], i["B"], i["C"], out_dtype=od,
                                save_states=True, return_u=True, return_state=True, h0=i["h0"],
                                conv_hist=i["conv_hist"], scan_form="chunked", **param_kw(i))

    a, b = _guarded(monkeypatch, run)
    _same(a, b)


@pytest.mark.parametrize("dtype,N,L,nseg,saved", [("bf16", 16, 333, 0, False), ("bf16", 16, 333, 3, False),
                                                  ("f32", 64, 100, 0, True), ("bf16", 16, 130, 2, True)])
def test_bwd_guards(monkeypatch, dtype, N, L, nseg, saved):
    t = _setup(2, 70, N, L, dtype, backward=True)
    st = None
    if saved:
        st = ssm.ssm_scan_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], save_states=True,
                              h0=t["h0"], conv_hist=t["conv_hist"], **param_kw(t))["chunk_states"]
    dh_last = torch.randn(2, 70, N, device="cuda", generator=torch.Generator("cuda").manual_seed(3))

    def run(g):
        i = _inputs(g, dict(t, st=st, dh_last=dh_last))
        return ssm.ssm_scan_bwd(i["dout"], i["x"], i["dt"], i["A_log"], i["B"], i["C"],
                                chunk_states=i["st"], h0=i["h0"], conv_hist=i["conv_hist"],
                                dh_last=i["dh_last"], state_grads=True, n_segments=nseg,
                                **param_kw(i))

    a, b = _guarded(monkeypatch, run)
    assert {"dx", "ddt", "dz", "dA_log", "dB", "dC", "dD", "ddt_bias", "dconv_w", "dconv_b", "dh0",
            "dconv_hist"} <= set(a)
    _same(a, b)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_step_guards(monkeypatch, dtype):
    Bt, Dn, N, K = 3, 70, 16, 4
    gen = torch.Generator("cuda").manual_seed(5)
    act = torch.bfloat16 if dtype == "bf16" else torch.float32
    rnd = lambda *s, dt=act: torch.randn(*s, device="cuda", generator=gen).to(dt)
    x, dt_, z = rnd(Bt, Dn), rnd(Bt, Dn) * 0.5, rnd(Bt, Dn)
    B, C = rnd(Bt, N), rnd(Bt, N)
    A_log = torch.log(torch.arange(1, N + 1, device="cuda", dtype=torch.float32)).repeat(Dn, 1)
    conv_w, conv_b = rnd(Dn, K, dt=torch.float32) * 0.3, rnd(Dn, dt=torch.float32) * 0.1
    h_init, hist_init = rnd(Bt, Dn, N, dt=torch.float32), rnd(Bt, Dn, K - 1)

    def run(g):
        h = g.empty((Bt, Dn, N), dtype=torch.float32, device="cuda")
        hist = g.empty((Bt, Dn, K - 1), dtype=act, device="cuda")
        h.copy_(h_init)
        hist.copy_(hist_init)
        i = _inputs(g, dict(x=x, dt=dt_, z=z, B=B, C=C, A_log=A_log, w=conv_w, b=conv_b))
        y = ssm.ssm_scan_step(i["x"], i["dt"], i["A_log"], i["B"], i["C"], h, conv_hist=hist,
                              z=i["z"], conv_w=i["w"], conv_b=i["b"], D=i["b"], dt_bias=i["b"])
        return {"y": y, "h": h, "hist": hist}

    a, b = _guarded(monkeypatch, run)
    _same(a, b)


@pytest.mark.parametrize("form", ["auto", "three_pass"])
@pytest.mark.parametrize("H,L,P,N,od", [(3, 200, 64, 64, torch.bfloat16), (2, 130, 128, 128, torch.float32),
                                        (8, 385, 64, 128, torch.bfloat16), (2, 77, 64, 128, torch.float32)])
def test_ssd_guards(monkeypatch, H, L, P, N, od, form):
    Bt = 2
    a = wl.generate_ssd(Bt, H, L, P, N, seed=9)
    t = {k: torch.from_numpy(v).to("cuda", torch.bfloat16 if k in ("x", "dt", "B", "C") else torch.float32)
         for k, v in a.items()}
    h0 = torch.randn(Bt, H, N, P, device="cuda", generator=torch.Generator("cuda").manual_seed(1)) * 0.3

    def run(g):
        i = _inputs(g, dict(t, h0=h0))
        return ssm.ssm_ssd_fwd(i["x"], i["dt"], i["A_log"], i["B"], i["C"], D=i["D"],
                               dt_bias=i["dt_bias"], h0=i["h0"], out_dtype=od, return_state=True,
                               check=True, form=form)

    a, b = _guarded(monkeypatch, run)
    _same(a, b)


@pytest.mark.parametrize("L", [333, 336])
@pytest.mark.parametrize("K", [1, 3, 4])
def test_conv_guards(monkeypatch, K, L):
    # L = 336: rows of whole 16-byte vectors (the vector path); 333: element by element
    gen = torch.Generator("cuda").manual_seed(K)
    x = torch.randn(2, 70, L, device="cuda", generator=gen).to(torch.bfloat16)
    w = torch.randn(70, K, device="cuda", generator=gen) * 0.3
    b = torch.randn(70, device="cuda", generator=gen) * 0.1

    def run(g):
        i = _inputs(g, dict(x=x, w=w, b=b))
        return ssm.ssm_conv1d_silu(i["x"], i["w"], i["b"], out_dtype=torch.float32)

    a, b2 = _guarded(monkeypatch, run)
    _same(a, b2)


def test_guard_detects_a_planted_overrun(monkeypatch):
    """The checker itself: a write one element past a guarded buffer is reported."""
    g = GuardedTorch(0xA5)
    t = g.empty((5, 3), dtype=torch.float32, device="cuda")
    t.fill_(1.0)
    g.check()
    raw = g.allocs[0][0]
    raw[GUARD + 60:GUARD + 64] = 0
    with pytest.raises(AssertionError, match="guard band"):
        g.check()
    g2 = GuardedTorch(0xA5)
    t2 = g2.empty((4,), dtype=torch.float32, device="cuda")
    t2[:3] = 2.0
    with pytest.raises(AssertionError, match="never written"):
        g2.check()
