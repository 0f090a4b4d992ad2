"""bench.py's parity report on CPU: run over every element of results that are the oracle's own
(whole-tensor calls, against the report's blocks of 32 channels), it passes with float64-rounding
errors; one element off by more than the stated tolerance, in an output, in a gradient summed over
channels (dB) or in one summed over batch elements (dconv_w), fails that tensor alone."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import oracle  # noqa: E402
from selective_state_space_34_b200 import workloads as wl  # noqa: E402


def _exact(w, a):
    kw = dict(D=a["D"], z=a["z"], dt_bias=a["dt_bias"], conv_w=a["conv_w"], conv_b=a["conv_b"])
    got = {"out": oracle.fwd(a["x"], a["dt"], a["A_log"], a["B"], a["C"], **kw)}
    got.update(oracle.bwd(a["x"], a["dt"], a["A_log"], a["B"], a["C"], a["dout"], **kw))
    return got


W = wl.shaped("mamba130m_fwd", Bt=2, Dn=70, N=4, L=40, in_dtype="f32", backward=True)


def test_parity_report_of_exact_results():
    a = wl.generate(W, seed=5)
    r = bench.oracle_parity(W, a, _exact(W, a), out_bf16=False, threads=4)
    assert r["ok"], r
    assert set(r) == {"elements", "ok", "out", "dx", "ddt", "dz", "dA_log", "dB", "dC", "dD",
                      "ddt_bias", "dconv_w", "dconv_b"}
    assert r["out"]["n"] == 2 * 70 * 40 and r["dB"]["n"] == 2 * 4 * 40
    for k in ("out", "dx", "ddt", "dz"):
        assert r[k]["max_abs_err"] == 0.0, k          # the same per-channel arithmetic
    for k in ("dB", "dC", "dA_log", "dconv_w"):       # sums re-associated in float64 only
        assert r[k]["max_abs_err"] <= 1e-12 * max(1.0, r[k]["atol"] * 1e4), k


def test_parity_report_flags_a_wrong_element():
    a = wl.generate(W, seed=5)
    for key, idx in (("out", (1, 65, 17)), ("dB", (0, 2, 9)), ("dconv_w", (33, 1))):
        got = _exact(W, a)
        ref = got[key][idx]
        tol = (1e-5 * abs(ref) + 1e-6) if key == "out" else (1e-2 * abs(ref) + bench_atol(got[key]))
        got[key] = got[key].copy()
        got[key][idx] += 1.5 * tol
        r = bench.oracle_parity(W, a, got, out_bf16=False, threads=4)
        assert not r["ok"] and not r[key]["ok"], key
        assert all(v["ok"] for k, v in r.items() if isinstance(v, dict) and k != key), key


def bench_atol(ref):
    return 1e-4 * abs(ref).max()


def test_measured_traffic_is_attached_only_to_its_workload_and_source(tmp_path, monkeypatch):
    """A stored ncu capture counts for the workloads its entry lists and only while the kernel's
    source file is the one it was taken on."""
    import hashlib
    import json
    src = tmp_path / "selective_state_space_34_b200" / "csrc"
    src.mkdir(parents=True)
    (src / "k.cu").write_text("// kernel source\n")
    sha = hashlib.sha256(b"// kernel source\n").hexdigest()[:16]
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "ncu_traffic.json").write_text(json.dumps({"kernels": {"k": {
        "source": "k.cu", "source_sha256_16": sha, "dram_bytes_per_launch": 1234,
        "workloads": ["shape_a"]}}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.ncu_traffic("k", "k.cu", "shape_a") == 1234
    assert bench.ncu_traffic("k", "k.cu", "shape_b") is None      # another workload
    assert bench.ncu_traffic("other", "k.cu", "shape_a") is None  # no entry
    (src / "k.cu").write_text("// kernel source, edited\n")
    assert bench.ncu_traffic("k", "k.cu", "shape_a") is None      # the source changed
