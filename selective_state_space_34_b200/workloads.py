"""Seeded synthetic workloads for the selective scan: shapes, value distributions and seeds.

This module only draws random numbers. It holds none of the scan's arithmetic, imports neither
the CUDA binding nor the oracle, and is the one piece that the tests, the benchmark and the
oracle-side checks share.

Distributions follow the Mamba block shapes the scan is measured on (standard deviations, not
variances): inputs x, z ~ N(0, 1); conv taps ~ N(0, 1/sqrt(4)); B, C ~ N(0, 1/sqrt(16)); the
canonical S6 init A_log[d, n] = ln(n + 1), D = 1, zero conv bias, and dt_bias such that
softplus(dt_bias) is a small step (rustytorch commit log, "canonical S6 init").

Values that the GPU reads in bf16 are rounded to bf16 here (round-to-nearest-even) and returned
as float32 arrays holding exactly those bf16 values, so the oracle sees bit-identical inputs.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace
from typing import Dict, Optional

import numpy as np


@dataclass(frozen=True)
class Workload:
    name: str
    Bt: int
    Dn: int
    N: int
    L: int
    in_dtype: str = "bf16"          # "f32" or "bf16": dtype of x, dt, z, B, C (and dout)
    conv: bool = True               # causal depthwise conv1d (K taps) + SiLU in front
    K: int = 4
    gate: bool = True               # SiLU(z) output gate
    dt_std: float = 1.0
    delta0: float = 0.01            # dt_bias = softplus^{-1}(delta0) for every channel
    delta_loguniform: Optional[tuple] = None  # per-channel Delta_d ~ log-uniform[lo, hi], dt = 0
    bc_std: float = 0.25
    backward: bool = False          # also draw dout
    seed: int = 1000
    note: str = ""

    @property
    def elem_states(self) -> int:
        return self.Bt * self.Dn * self.L * self.N


# The five measured workloads (seeds 1000 + index), the finite-difference slice and the
# few-channel long-context case.
WORKLOADS: Dict[str, Workload] = {
    "tiny_fp32": Workload("tiny_fp32", 1, 16, 4, 64, in_dtype="f32", conv=False, gate=True,
                          dt_std=0.5, delta0=0.05, bc_std=1.0, seed=1000,
                          note="tiny forward, fp32, scan only"),
    "mamba130m_fwd": Workload("mamba130m_fwd", 2, 1536, 16, 2048, seed=1001,
                              note="Mamba-130M-shaped block forward, bf16 in"),
    "mamba1p4b_fwd": Workload("mamba1p4b_fwd", 4, 4096, 16, 4096, seed=1002,
                              note="Mamba-1.4B-shaped fused forward, bf16 in"),
    "long_fwd": Workload("long_fwd", 1, 5120, 16, 65536, seed=1003,
                         delta_loguniform=(1e-3, 1e-1),
                         note="long-context forward, per-channel log-uniform Delta"),
    "mamba1p4b_fwdbwd": Workload("mamba1p4b_fwdbwd", 4, 4096, 16, 4096, backward=True,
                                 seed=1004, note="forward + backward, bf16 in, fp32 grads"),
    "fd_slice": Workload("fd_slice", 1, 8, 4, 32, in_dtype="f32", backward=True, seed=1005,
                         note="finite-difference slice, fp32"),
    # the long-context workload's length and Delta distribution with few channels: the shape
    # class split-L serves (a decode-like batch over a long prompt)
    "long_fewch_fwd": Workload("long_fewch_fwd", 1, 512, 16, 65536, seed=1006,
                               delta_loguniform=(1e-3, 1e-1),
                               note="long-context forward, 512 channels (split-L case)"),
    "long_fewch_fwdbwd": Workload("long_fewch_fwdbwd", 1, 512, 16, 65536, seed=1007,
                                  delta_loguniform=(1e-3, 1e-1), backward=True,
                                  note="long-context forward + backward, 512 channels (split-L)"),
}


def softplus_inverse(delta: np.ndarray) -> np.ndarray:
    """dt_bias value whose softplus is ``delta`` (log(expm1(delta))), used to draw parameters."""
    return np.log(np.expm1(np.asarray(delta, dtype=np.float64)))


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns float32 holding them."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    bits = a.view(np.uint32)
    bias = ((bits >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    out = (bits + bias) & np.uint32(0xFFFF0000)
    return out.view(np.float32)


def _rng(seed: int, stream: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([int(seed), int(stream)]))


def _normal(seed: int, stream: int, shape, std: float) -> np.ndarray:
    a = _rng(seed, stream).standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return a


def generate(w: Workload, seed: Optional[int] = None) -> Dict[str, np.ndarray]:
    """Draw every array of workload ``w``. Keys: x, dt, z (or None), B, C, A_log, D, dt_bias,
    conv_w / conv_b (or None), dout (backward workloads only). Arrays read by the kernels in the
    input dtype are rounded to it; parameters are float32."""
    s = w.seed if seed is None else int(seed)
    Bt, Dn, N, L = w.Bt, w.Dn, w.N, w.L
    rnd = round_to_bf16 if w.in_dtype == "bf16" else (lambda a: a)
    out: Dict[str, Optional[np.ndarray]] = {}
    out["x"] = rnd(_normal(s, 1, (Bt, Dn, L), 1.0))
    if w.delta_loguniform is not None:
        lo, hi = w.delta_loguniform
        lu = _rng(s, 2).uniform(math.log(lo), math.log(hi), size=Dn)
        out["dt"] = np.zeros((Bt, Dn, L), dtype=np.float32)
        out["dt_bias"] = softplus_inverse(np.exp(lu)).astype(np.float32)
    else:
        out["dt"] = rnd(_normal(s, 2, (Bt, Dn, L), w.dt_std))
        out["dt_bias"] = np.full(Dn, softplus_inverse(w.delta0), dtype=np.float32)
    out["z"] = rnd(_normal(s, 3, (Bt, Dn, L), 1.0)) if w.gate else None
    out["B"] = rnd(_normal(s, 4, (Bt, N, L), w.bc_std))
    out["C"] = rnd(_normal(s, 5, (Bt, N, L), w.bc_std))
    out["A_log"] = np.tile(np.log(np.arange(1, N + 1, dtype=np.float64)), (Dn, 1)).astype(np.float32)
    out["D"] = np.ones(Dn, dtype=np.float32)
    if w.conv:
        out["conv_w"] = _normal(s, 6, (Dn, w.K), 1.0 / math.sqrt(w.K))
        out["conv_b"] = np.zeros(Dn, dtype=np.float32)
    else:
        out["conv_w"] = None
        out["conv_b"] = None
    if w.backward:
        out["dout"] = rnd(_normal(s, 7, (Bt, Dn, L), 1.0))
    return out


def carried_state(w: Workload, seed: Optional[int] = None) -> Dict[str, Optional[np.ndarray]]:
    """State carried in from a previous chunk and the gradient arriving at the final state:
    h0 ~ N(0, 0.5) and dh_last ~ N(0, 0.1), both (Bt, Dn, N) float32; conv_hist ~ N(0, 1),
    (Bt, Dn, K-1) in the input dtype (None without a conv)."""
    s = (w.seed if seed is None else int(seed)) + 7919
    rnd = round_to_bf16 if w.in_dtype == "bf16" else (lambda a: a)
    return {
        "h0": _normal(s, 11, (w.Bt, w.Dn, w.N), 0.5),
        "conv_hist": rnd(_normal(s, 12, (w.Bt, w.Dn, w.K - 1), 1.0)) if w.conv else None,
        "dh_last": _normal(s, 13, (w.Bt, w.Dn, w.N), 0.1),
    }


def generate_ssd(Bt: int, H: int, L: int, P: int, N: int, seed: int = 1008) -> Dict[str, np.ndarray]:
    """Inputs of a Mamba-2 state-space-duality layer (the pages give no SSD shapes or
    distributions; these follow the selective-scan workloads): x ~ N(0, 1) (Bt, H, L, P),
    dt ~ N(0, 1) (Bt, H, L), B, C ~ N(0, 1/sqrt(N)) (Bt, L, N), all bf16-rounded; per head
    A_log = ln(1..H spread over [1, 16]), dt_bias = softplus^-1 of a log-uniform step in
    [1e-3, 1e-1], D = 1."""
    out: Dict[str, np.ndarray] = {}
    out["x"] = round_to_bf16(_normal(seed, 21, (Bt, H, L, P), 1.0))
    out["dt"] = round_to_bf16(_normal(seed, 22, (Bt, H, L), 1.0))
    std = 1.0 / math.sqrt(N)
    out["B"] = round_to_bf16(_normal(seed, 23, (Bt, L, N), std))
    out["C"] = round_to_bf16(_normal(seed, 24, (Bt, L, N), std))
    out["A_log"] = np.log(np.linspace(1.0, 16.0, H)).astype(np.float32)
    lu = _rng(seed, 25).uniform(math.log(1e-3), math.log(1e-1), size=H)
    out["dt_bias"] = softplus_inverse(np.exp(lu)).astype(np.float32)
    out["D"] = np.ones(H, dtype=np.float32)
    return out


# Mamba-2-style layer on the 1.4B-shaped block: d_inner 4096 as 64 heads of 64, d_state 128.
SSD_WORKLOADS = {"ssd_fwd": dict(Bt=4, H=64, L=4096, P=64, N=128, seed=1008)}

# Token-by-token decode on the 1.4B-shaped block: 64 sequences x d_inner 4096, d_state 16, conv
# width 4, 256 tokens (one decode step each); the token inputs are the columns of a scan workload
# of that shape, so their distributions are the scan workloads'.
DECODE_WORKLOADS = {"decode_1p4b": Workload("decode_1p4b", 64, 4096, 16, 256, seed=1009)}

# The standalone causal conv1d + SiLU over the 1.4B-shaped activations (x only is used).
CONV_WORKLOADS = {"conv_1p4b": Workload("conv_1p4b", 4, 4096, 16, 4096, seed=1010)}


def shaped(base: str, **overrides) -> Workload:
    """A named workload with some fields replaced (e.g. smaller Bt/Dn/L for a parity case)."""
    return replace(WORKLOADS[base], **overrides)


def sample_channels(Bt: int, Dn: int, k: int, seed: int = 7) -> np.ndarray:
    """k distinct (b, d) channel pairs, always including the first and the last channel."""
    rng = _rng(seed, 99)
    total = Bt * Dn
    k = min(k, total)
    picks = set([0, total - 1])
    while len(picks) < k:
        picks.add(int(rng.integers(0, total)))
    flat = np.array(sorted(picks), dtype=np.int64)
    return np.stack([flat // Dn, flat % Dn], axis=1)
