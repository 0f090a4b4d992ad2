"""bench.py's parity report on CPU: the errors it prints for the timed steps' sampled results are
zero when the results are the oracle's own, and its verdict flips when one element is off by more
than the stated tolerance."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import oracle  # noqa: E402
from selective_state_space_34_b200 import workloads as wl  # noqa: E402


def _picks(w, a):
    picks = []
    for b, d in ((0, 0), (0, 7)):
        x, dt, Al, B, C, dout, kw = bench._channel_slice(a, b, d, d + 4)
        out = oracle.fwd(x, dt, Al, B, C, **kw)[0]
        dx = oracle.bwd(x, dt, Al, B, C, dout, **kw)["dx"][0] if w.backward else None
        picks.append((b, d, out, dx))
    return picks


def test_parity_report_of_exact_results():
    w = wl.shaped("mamba130m_fwd", Bt=1, Dn=12, N=4, L=40, in_dtype="f32", backward=True)
    a = wl.generate(w, seed=5)
    r = bench.oracle_parity(w, a, _picks(w, a), out_bf16=False)
    assert r["ok"] and r["out"]["max_abs_err"] == 0.0 and r["dx"]["tol_ratio"] == 0.0
    assert r["channels"] == ["b0:d0-4", "b0:d7-11"]


def test_parity_report_flags_a_wrong_element():
    w = wl.shaped("mamba130m_fwd", Bt=1, Dn=12, N=4, L=40, in_dtype="f32", backward=True)
    a = wl.generate(w, seed=5)
    picks = _picks(w, a)
    b, d, out, dx = picks[1]
    out = out.copy()
    out[2, 17] += 1e-3 + 1e-4 * abs(out[2, 17])
    picks[1] = (b, d, out, dx)
    r = bench.oracle_parity(w, a, picks, out_bf16=False)
    assert not r["ok"] and r["out"]["tol_ratio"] > 1.0 and r["dx"]["tol_ratio"] == 0.0
