"""Plants plausible mistakes into a copy of the oracle's C source (on the CPU, in a temporary
directory) and checks that at least one pin of test_oracle_pins.py fails for each of them.
This shows the pins constrain every part of the oracle, not just the parts they name."""
import ctypes
import json
import os
import shutil
import subprocess
import tempfile

import pytest

import oracle
import test_oracle_pins as pins
import test_oracle_ssd as ssd_pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "ssm_oracle.c")

# (name, text in ssm_oracle.c, replacement): one plausible slip each.
MUTATIONS = [
    ("euler_bbar", "expm1(delta * A) / A * B;", "delta * B;"),
    ("dropped_D_skip", "y += (D ? D[d] : 0.0) * u[t];", "y += 0.0 * u[t];"),
    ("reversed_taps", "acc += w[k] * x[t - k];", "acc += w[K - 1 - k] * x[t - k];"),
    ("gate_sigmoid_not_silu", "y * ssm_oracle_silu(z[off + t])", "y * ssm_oracle_sigmoid(z[off + t])"),
    ("softplus_dropped_max", "log1p(exp(-fabs(v))) + (v > 0.0 ? v : 0.0)", "log1p(exp(-fabs(v)))"),
    ("input_inside_decay", "h[n] = Abar * h[n] + Bbar * u[t];", "h[n] = Abar * (h[n] + Bbar * u[t]);"),
    ("A_sign", "const double A = -exp(A_log[d * N + n]);", "const double A = -exp(-A_log[d * N + n]);"),
    ("dropped_conv_bias", "double acc = b;", "double acc = 0.0 * b;"),
    ("bwd_lambda_same_step", "lam[n] = dy[t] * Cb[n * L + t] + anext * lam[n];",
     "lam[n] = dy[t] * Cb[n * L + t] + a[i] * lam[n];"),
    ("bwd_dA_dropped_input_term", "u[t] * Bt_n * (xx * a[i] - em1[i]) / (A[n] * A[n]));", "0.0);"),
    ("bwd_dB_euler", "dBb[n * L + t] += lam[n] * u[t] * em1[i] / A[n];",
     "dBb[n * L + t] += lam[n] * u[t] * dl[t];"),
    ("bwd_gate_derivative", "s * (1.0 + zz * (1.0 - s))", "s"),
    ("bwd_conv_dx_taps", "acc += w[k] * dc[j + k];", "acc += w[K - 1 - k] * dc[j + k];"),
    ("bwd_dAlog_chain", "= dA[n] * A[n];", "= dA[n];"),
    ("history_off_by_one", "acc += w[k] * hist[k - t - 1];", "acc += w[k] * hist[k - t];"),
    ("euler_missing_delta", "if (euler) Bbar = delta * Bb[n * L + t];", "if (euler) Bbar = Bb[n * L + t];"),
    ("dh0_missing_decay", "? a[(size_t)n] * lam[n] : lam[n];", "? lam[n] : lam[n];"),
    ("dh_last_decayed", "a[i + (size_t)N] : 1.0;", "a[i + (size_t)N] : 0.0;"),
    ("bwd_euler_dB", "dBb[n * L + t] += lam[n] * u[t] * dl[t];", "dBb[n * L + t] += lam[n] * u[t];"),
    # the state-space-duality recurrence
    ("ssd_dropped_decay", "st[n * P + p] = a * st[n * P + p] + beta * Bt_[n] * xt[p];",
     "st[n * P + p] = st[n * P + p] + beta * Bt_[n] * xt[p];"),
    ("ssd_euler_ignored", "const double beta = euler ? delta : expm1(delta * A) / A;",
     "const double beta = expm1(delta * A) / A;"),
    ("ssd_zoh_as_euler", "const double beta = euler ? delta : expm1(delta * A) / A;",
     "const double beta = delta;"),
    ("ssd_readout_with_B", "acc += Ct[n] * st[n * P + p];", "acc += Bt_[n] * st[n * P + p];"),
    ("ssd_dropped_skip", "yt[p] = acc + Dh * xt[p];", "yt[p] = acc;"),
    ("ssd_bias_ignored", "const double bias = dt_bias ? dt_bias[hd] : 0.0;", "const double bias = 0.0;"),
    ("ssd_A_sign", "const double A = -exp(A_log[hd]);", "const double A = -exp(-A_log[hd]);"),
    ("ssd_h0_ignored", "st[i] = h0 ? h0[bh * N * P + i] : 0.0;", "st[i] = 0.0;"),
]


def _pin_functions():
    return ([getattr(pins, n) for n in dir(pins) if n.startswith("test_")] +
            [getattr(ssd_pins, n) for n in dir(ssd_pins) if n.startswith("test_")])


def _param_sets(fn):
    """Expand a pin's @pytest.mark.parametrize marks into keyword-argument dicts."""
    import itertools
    sets = [{}]
    for m in getattr(fn, "pytestmark", []):
        if m.name != "parametrize":
            continue
        names = [n.strip() for n in m.args[0].split(",")] if isinstance(m.args[0], str) else list(m.args[0])
        values = [v if len(names) > 1 else (v,) for v in m.args[1]]
        sets = [dict(s, **dict(zip(names, v))) for s, v in itertools.product(sets, values)]
    return sets


def _run_pins(gold):
    failed = []
    for fn in _pin_functions():
        for kw in _param_sets(fn):
            if "gold" in fn.__code__.co_varnames[:fn.__code__.co_argcount]:
                kw = dict(kw, gold=gold)
            try:
                fn(**kw)
            except AssertionError:
                failed.append(fn.__name__)
            except Exception:
                failed.append(fn.__name__ + "(error)")
    return failed


@pytest.fixture(scope="module")
def gold():
    with open(pins.GOLDEN) as f:
        return json.load(f)


@pytest.fixture(scope="module")
def workdir():
    d = tempfile.mkdtemp(prefix="oracle_mut_")
    yield d
    shutil.rmtree(d, ignore_errors=True)


def test_unmutated_oracle_passes_every_pin(gold):
    assert _run_pins(gold) == []


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_mutation_is_caught(name, old, new, gold, workdir):
    src = open(SRC).read()
    assert src.count(old) >= 1, "mutation anchor not found: " + name
    mutated = src.replace(old, new)
    cpath = os.path.join(workdir, name + ".c")
    sopath = os.path.join(workdir, "lib" + name + ".so")
    with open(cpath, "w") as f:
        f.write(mutated)
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-w", "-o", sopath,
                    cpath, "-lm"], check=True)
    saved = oracle._lib
    oracle._lib = oracle.bind(ctypes.CDLL(sopath))
    try:
        failed = _run_pins(gold)
    finally:
        oracle._lib = saved
    assert failed, "no pin caught mutation " + name
