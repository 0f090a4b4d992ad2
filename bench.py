#!/usr/bin/env python
"""Benchmark of the fused selective scan (Mamba-1 S6) on B200: one JSON line on rank 0.

A step is one pass of the whole hot path over one batch of synthetic input: the fused forward
(conv1d + SiLU -> softplus Delta -> exact-ZOH scan -> D skip -> SiLU(z) gate, saving the chunk
states) followed by the backward (all gradients), on the 4 x 4096 x 16 x 4096 Mamba-1.4B-shaped
workload with bf16 activations, fp32 state and fp32 gradients. The forward alone on the same shape
(the HBM-headline case) is timed in the same run and reported under "forward".

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Multi-GPU (launched with torch.distributed.run): every rank runs its own batch (weak scaling);
the data path has no collective. Timing is on the device (CUDA events), max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = ("selective-scan fwd/bwd (batch·d_inner·L·d_state)/s and HBM GB/s vs peak, "
          "1×B200")
UNIT = "elem_states/s"
# Measured on this machine's B200s (copy bandwidth, bf16 GEMM); used when the per-pod file is absent.
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "source": "fallback"}
# sm_100a pipe rates per SM per clock (FP32 FMA lanes, MUFU ex2), used for the ALU ceiling.
FMA_LANES, MUFU_LANES, N_SM = 128, 16, 148


# ---- rank plumbing (host only; covered by world-size-2 gloo tests on CPU) -----------------------

def rank_env():
    """(world, rank, local_rank) from the launcher's environment; a plain run is rank 0 of 1."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def rank_seed(w, rank):
    """Every rank draws its own batch of the same workload (weak scaling): seed + rank."""
    return w.seed + rank


def max_over_ranks(x, world, device):
    """The slowest rank's value of x (a device time in ms); a no-op on one rank."""
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank, world, steps, max_ms):
    """Whole-job rate: the units every rank processed in `steps` steps over the slowest time."""
    return units_per_rank * world * steps / (max_ms * 1e-3)


def ncu_traffic(kernel, source, workload):
    """DRAM bytes per launch of `kernel` (dram__bytes_read.sum + dram__bytes_write.sum from one ncu
    capture, stored in profiles/ncu_traffic.json with the command that took it), or None when the
    capture was taken on another workload (the entry lists the workloads that launch the kernel
    on the captured shape and dtypes) or on a different version of the kernel's source file."""
    import hashlib
    try:
        sha = hashlib.sha256(open(os.path.join(ROOT, "selective_state_space_34_b200", "csrc", source),
                                  "rb").read()).hexdigest()[:16]
        with open(os.path.join(ROOT, "profiles", "ncu_traffic.json")) as f:
            rec = json.load(f)["kernels"].get(kernel)
        if rec and rec.get("source_sha256_16") == sha and workload in rec.get("workloads", []):
            return int(rec["dram_bytes_per_launch"])
    except Exception:
        return None
    return None


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    except Exception:
        return dict(FALLBACK_PEAKS)


# ---- algorithmic bytes (the minimum the method must move; intermediates never touch HBM) -------

def fwd_bytes(Bt, Dn, N, L, s_in, s_out, n_states=0):
    """The forward's algorithmic bytes (x, dt, z, B, C and the parameters in, out out), plus the
    n_states saved chunk states per channel when the step saves them for the backward."""
    elems = Bt * Dn * L
    b = elems * (3 * s_in + s_out)              # x, dt, z in; out
    b += Bt * N * L * 2 * s_in                  # B, C (shared by all channels)
    b += Dn * (N + 4 + 4) * 4                   # A_log, D, dt_bias, conv taps + bias
    b += Bt * Dn * n_states * N * 4             # chunk states for the backward
    return b


def bwd_bytes(Bt, Dn, N, L, s_in):
    """The backward's algorithmic bytes: x, dt, z, dout, B, C and the parameters in; dx, ddt, dz,
    dB, dC and the parameter gradients out. The saved states and the per-tile dB / dC partials
    are this implementation's own traffic (see bwd_overhead_bytes), not the method's."""
    elems = Bt * Dn * L
    b = elems * (4 * s_in + 3 * 4)              # x, dt, z, dout in; dx, ddt, dz out (fp32)
    b += Bt * N * L * (2 * s_in + 2 * 4)        # B, C in; dB, dC out (fp32)
    b += Dn * (N + 8) * 4 * 2                   # parameters in, parameter grads out
    return b


def bwd_overhead_bytes(Bt, Dn, N, n_states):
    """Traffic of the backward kernel beyond the algorithmic bytes that follows from the interface:
    the saved chunk states it reads (n_states per channel). Its scratch traffic (partial sums)
    shows in the measured `traffic` against `algorithmic_bytes`."""
    return {"saved_states_read": Bt * Dn * n_states * N * 4}


# ---- clocks during the timed region -------------------------------------------------------------

class ClockSampler:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.Q,
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.th = threading.Thread(target=self._read, daemon=True)
            self.th.start()
        except Exception:
            self.proc = None

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append(ln.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.12)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 8:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---- CPU baseline: the float64 oracle on a bounded sample of the same workload ------------------

def _channel_slice(a, b, lo, hi):
    """Inputs of channels lo..hi-1 of batch element b (the oracle runs channels independently;
    B and C are the batch element's own)."""
    sl = slice(lo, hi)
    kw = dict(D=a["D"][sl], z=None if a["z"] is None else a["z"][b:b + 1, sl],
              dt_bias=a["dt_bias"][sl], conv_w=None if a["conv_w"] is None else a["conv_w"][sl],
              conv_b=None if a["conv_b"] is None else a["conv_b"][sl])
    dout = a["dout"][b:b + 1, sl] if a.get("dout") is not None else None
    return (a["x"][b:b + 1, sl], a["dt"][b:b + 1, sl], a["A_log"][sl], a["B"][b:b + 1],
            a["C"][b:b + 1], dout, kw)


def oracle_parity(w, a, got, out_bf16, threads):
    """Every element of the timed steps' own results against the oracle, with the parity tests'
    tolerances: the output rtol 2e-3 (+2^-8 for a bf16 output) with atol 1e-4 for bf16 inputs
    (1e-5 / 1e-6 for fp32); a gradient rtol 1e-2 with atol 1e-4 of the largest oracle value of that
    whole tensor. `got` holds "out" and, after a backward, all ten gradients (host float arrays).

    The oracle runs blocks of 32 channels of one batch element, single-threaded each, in a thread
    pool (channels are independent in the method). dB and dC sum over channels and the per-channel
    parameter gradients over batch elements: the blocks' float64 contributions are added in block
    order before those tensors are compared. tol_ratio = max |err| / (atol + rtol |ref|) <= 1 passes."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    rtol_o, atol_o = (2e-3, 1e-4) if w.in_dtype == "bf16" else (1e-5, 1e-6)
    if out_bf16:
        rtol_o += 2.0 ** -8
    act = [k for k in ("dx", "ddt", "dz") if k in got]
    param = [k for k in ("dA_log", "dD", "ddt_bias", "dconv_w", "dconv_b") if k in got]

    def block(blk):
        b, lo, hi = blk
        x, dt, Al, B, C, dout, kw = _channel_slice(a, b, lo, hi)
        ref = {"out": oracle.fwd(x, dt, Al, B, C, n_threads=1, **kw)[0]}
        r = oracle.bwd(x, dt, Al, B, C, dout, n_threads=1, **kw) if act else {}
        st = {}
        for k in ["out"] + act:
            rk = ref[k] if k == "out" else r[k][0]
            e = np.abs(np.asarray(got[k][b, lo:hi], dtype=np.float64) - rk)
            # per block: max |err|, max |ref|, max |err| - rtol |ref|, count of elements
            rt = rtol_o if k == "out" else 1e-2
            st[k] = (float(e.max()), float(np.abs(rk).max()), float(np.max(e - rt * np.abs(rk))), e.size,
                     bool(np.all(np.isfinite(got[k][b, lo:hi]))))
        return blk, st, r

    blocks = [(b, lo, min(w.Dn, lo + 32)) for b in range(w.Bt) for lo in range(0, w.Dn, 32)]
    agg = {}
    sums = {"dB": np.zeros((w.Bt, w.N, w.L)), "dC": np.zeros((w.Bt, w.N, w.L))} if act else {}
    sums.update({k: np.zeros(got[k].shape) for k in param})
    with ThreadPoolExecutor(max_workers=threads) as ex:
        for (b, lo, hi), st, r in ex.map(block, blocks):
            for k, (emax, rmax, excess, n, finite) in st.items():
                m = agg.setdefault(k, [0.0, 0.0, -np.inf, 0, True])
                agg[k] = [max(m[0], emax), max(m[1], rmax), max(m[2], excess), m[3] + n, m[4] and finite]
            if act:
                sums["dB"][b] += r["dB"][0]
                sums["dC"][b] += r["dC"][0]
                for k in param:
                    sums[k][lo:hi] += r[k]
    res = {"elements": "every element of out%s (%d blocks of <= 32 channels)"
                       % (" and of all ten gradients" if act else "", len(blocks))}
    for k, (emax, rmax, excess, n, finite) in agg.items():
        rt, at = (rtol_o, atol_o) if k == "out" else (1e-2, 1e-4 * max(rmax, 1e-30))
        # excess <= atol is the elementwise test |err| <= atol + rtol |ref| over the whole tensor
        res[k] = {"n": n, "max_abs_err": emax, "rtol": rt, "atol": at,
                  "ok": bool(finite and excess <= at)}
    for k, ref in sums.items():
        g = np.asarray(got[k], dtype=np.float64)
        err = np.abs(g - ref)
        at = 1e-4 * max(float(np.abs(ref).max()), 1e-30)
        res[k] = {"n": int(ref.size), "max_abs_err": float(err.max()), "rtol": 1e-2, "atol": at,
                  "ok": bool(np.all(np.isfinite(g)) and np.all(err <= at + 1e-2 * np.abs(ref)))}
    res["ok"] = all(v["ok"] for v in res.values() if isinstance(v, dict))
    return res


def oracle_sample(w, a, n_channels, threads):
    """Run the oracle's forward + backward on n_channels channels of the workload, spread over a
    thread pool (the C oracle releases the GIL); returns (seconds, elem_states)."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    per = max(1, min(16, n_channels // max(1, threads)))
    # contiguous channel runs of one batch element each, wrapping over (batch, channel) when the
    # sample is larger than the workload
    total, groups, i = w.Bt * w.Dn, [], 0
    while i < n_channels:
        b, d = divmod(i % total, w.Dn)
        n = min(per, w.Dn - d, n_channels - i)
        groups.append((b, d, d + n))
        i += n

    def run(group):
        b, lo, hi = group
        x, dt, Al, B, C, dout, kw = _channel_slice(a, b, lo, hi)
        oracle.fwd(x, dt, Al, B, C, n_threads=1, **kw)
        if w.backward:
            oracle.bwd(x, dt, Al, B, C, dout, n_threads=1, **kw)
        return (hi - lo) * w.L * w.N

    oracle.build()
    t0 = time.perf_counter()
    with ThreadPoolExecutor(max_workers=threads) as ex:
        done = sum(ex.map(run, groups))
    return time.perf_counter() - t0, done


def reference_arm(args, w):
    """--impl reference: the float64 oracle timed on the host cores, on bounded samples. Under a
    multi-rank launch rank 0 alone runs it; the other ranks return without work."""
    _, rank, _ = rank_env()
    if rank != 0:
        return 0
    from selective_state_space_34_b200 import workloads as wl
    a = wl.generate(w)
    threads = os.cpu_count() or 1
    n_ch = max(threads * 4, 64)
    times, work = [], 0
    for i in range(args.warmup + args.steps):
        dt_s, es = oracle_sample(w, a, n_ch, threads)
        if i >= args.warmup:
            times.append(dt_s)
            work += es
    total = sum(times)
    value = work / total
    sample = "%d channels x L=%d x N=%d per step (fwd%s), float64, %d host threads" % (
        n_ch, w.L, w.N, "+bwd" if w.backward else "", threads)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "Bt": w.Bt, "Dn": w.Dn, "N": w.N, "L": w.L,
                   "in_dtype": w.in_dtype, "sampled": True},
        "impl": "reference",
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---- the state-space-duality leg (Mamba-2 heads, tensor cores) ---------------------------------

def ssd_bench(args, cfg, name):
    """The Mamba-2 state-space-duality layer through the C ABI: the fused form (one launch per step,
    timed on its own by the library's timing events) or the three-pass form (three launches, the
    output kernel -- the dominant one -- timed on its own)."""
    import ctypes
    import torch
    from selective_state_space_34_b200 import _abi
    from selective_state_space_34_b200 import workloads as wl
    world, rank, local = rank_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    Bt, H, L, P, N = cfg["Bt"], cfg["H"], cfg["L"], cfg["P"], cfg["N"]
    a = wl.generate_ssd(Bt, H, L, P, N, seed=cfg["seed"] + rank)
    T = {k: torch.from_numpy(v).to(dev, torch.bfloat16 if k in ("x", "dt", "B", "C") else torch.float32)
         for k, v in a.items()}
    y = torch.empty((Bt, H, L, P), dtype=torch.bfloat16, device=dev)
    sa = _abi.SsdArgs()
    sa.x, sa.dt, sa.dt_bias, sa.A_log = T["x"].data_ptr(), T["dt"].data_ptr(), T["dt_bias"].data_ptr(), T["A_log"].data_ptr()
    sa.B, sa.C, sa.D, sa.y = T["B"].data_ptr(), T["C"].data_ptr(), T["D"].data_ptr(), y.data_ptr()
    sa.Bt, sa.H, sa.L, sa.P, sa.N = Bt, H, L, P, N
    sa.in_dtype, sa.out_dtype, sa.delta_softplus, sa.discretization = _abi.SSM_BF16, _abi.SSM_BF16, 1, _abi.SSM_ZOH
    fused = args.ssd_form == "fused" or (args.ssd_form == "auto" and P == 64)
    sa.form = _abi.SSM_SSD_FUSED if fused else _abi.SSM_SSD_THREE_PASS
    lib = _abi.load()
    need = int(lib.ssm_ssd_workspace_size(ctypes.byref(sa)))
    ws = torch.empty(need + 256, dtype=torch.uint8, device=dev)
    sa.workspace, sa.workspace_bytes = (ws.data_ptr() + 255) & ~255, need
    s = torch.cuda.current_stream(dev)
    E = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    ev0 = [E() for _ in range(args.steps)]
    ev_k = [[E(), E()] for _ in range(args.steps)]
    ev_ptr = []
    for pair in ev_k:
        for e in pair:
            e.record(s)  # creates the cudaEvent_t handles before they are passed down
        ev_ptr.append((ctypes.c_void_p * 2)(pair[0].cuda_event, pair[1].cuda_event))
    torch.cuda.synchronize()

    def run(i=None):
        if i is not None:
            ev0[i].record(s)
        sa.timing_events = ctypes.cast(ev_ptr[i], ctypes.c_void_p) if i is not None else None
        _abi.check("ssm_ssd_fwd", lib.ssm_ssd_fwd(ctypes.byref(sa), s.cuda_stream))

    for _ in range(args.warmup):
        run()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.15)
    if world > 1:
        dist.barrier(device_ids=[local])
    torch.cuda.synchronize()
    s0, s1 = E(), E()
    s0.record(s)
    for i in range(args.steps):
        run(i)
    s1.record(s)
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = max_over_ranks(s0.elapsed_time(s1), world, dev) / args.steps
    out_ms = float(np.mean([ev_k[i][0].elapsed_time(ev_k[i][1]) for i in range(args.steps)]))
    per_step = np.array([ev0[i].elapsed_time(ev_k[i][1]) for i in range(args.steps)])
    es = Bt * H * P * L * N
    nC = (L + 127) // 128
    # layer: x, dt, B, C in, y out (bf16); the chunk states are intermediates
    ab = Bt * H * L * P * 2 * 2 + Bt * H * L * 2 + 2 * Bt * L * N * 2
    # output kernel: x, dt, B, C and the entering states (bf16) in, y out
    ob = Bt * H * L * P * 2 + Bt * H * L * 2 + 2 * Bt * L * N * 2 + Bt * H * nC * N * P * 2 + Bt * H * L * P * 2
    # output kernel's tensor work as issued: C B^T once per 8-head group (K = 128), G'X (K = Q) and
    # C H_in (K = N) per head
    hg = 8 if H % 8 == 0 else (4 if H % 4 == 0 else (2 if H % 2 == 0 else 1))
    oflops = 2 * Bt * nC * ((H // hg) * 128 * 128 * 128 + H * (128 * P * 128 + 128 * P * N))
    if fused:
        # the one launch is the layer: its bytes are the layer's; tensor work per (batch, head,
        # chunk) as issued: C B^T (K = N), G'X and the state product (K = Q), C H (K = N)
        kname, ksrc, ob = "ssd_fused_kernel", "ssm_ssd_fused.cu", ab
        oflops = 2 * Bt * H * nC * (128 * 128 * N + 2 * 128 * P * 128 + 128 * P * N)
    else:
        kname, ksrc = "ssd_out_kernel", "ssm_ssd.cu"
    peaks = load_peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    bf16 = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    line = {
        "metric": METRIC, "value": job_throughput(es, world, 1, ms), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "step_ms": {"median": float(np.median(per_step)), "p10": float(np.percentile(per_step, 10)),
                    "p90": float(np.percentile(per_step, 90)), "of": "rank 0, CUDA events around each timed step"},
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": name, "Bt": Bt, "H": H, "P": P, "N": N, "L": L, "chunk": 128,
                   "step": "ssd forward (1 launch, fused)" if fused else "ssd forward (3 launches)",
                   "form": "fused" if fused else "three_pass", "l2": "inputs larger than L2"},
        "roofline": {"bound": "hbm", "achieved": ob / (out_ms * 1e-3) / 1e9, "peak": hbm, "unit": "GB/s",
                     "frac": ob / (out_ms * 1e-3) / 1e9 / hbm, "traffic": ncu_traffic(kname, ksrc, name),
                     "algorithmic_bytes": ob, "kernel": kname, "ms": out_ms,
                     "peak_source": peaks.get("source")},
        "tensor": {"achieved": oflops / (out_ms * 1e-3) / 1e12, "peak": bf16, "unit": "TFLOP/s",
                   "frac": oflops / (out_ms * 1e-3) / 1e12 / bf16, "kernel": kname, "flops": oflops},
        "layer": {"ms": ms, "hbm_gbs": ab / (ms * 1e-3) / 1e9, "hbm_frac": ab / (ms * 1e-3) / 1e9 / hbm,
                  "algorithmic_bytes": ab},
        "gpu_launches": (1 if fused else 3) * args.steps, "clocks": clk,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def decode_bench(args, w):
    """Token-by-token decode through the C ABI (ssm_scan_step, one launch per token): T tokens of
    Bt sequences, each token's x, dt, z, B, C its own resident arrays, the state and conv history
    carried in place. Timed as replays of one CUDA graph holding the T launches (the way a decode
    loop runs them), and as T plain launches from the host."""
    import ctypes
    import torch
    from selective_state_space_34_b200 import _abi
    from selective_state_space_34_b200 import workloads as wl
    world, rank, local = rank_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    Bt, Dn, N, T, K = w.Bt, w.Dn, w.N, w.L, w.K
    a = wl.generate(w, seed=w.seed + rank)
    bf = torch.bfloat16
    # token-major copies: token t's x / dt / z are (Bt, Dn), its B / C (Bt, N)
    tok = {k: torch.from_numpy(np.ascontiguousarray(np.moveaxis(a[k], -1, 0))).to(dev, bf) for k in ("x", "dt", "z", "B", "C")}
    par = {k: torch.from_numpy(a[k]).to(dev, torch.float32) for k in ("A_log", "D", "dt_bias", "conv_w", "conv_b")}
    h = torch.zeros((Bt, Dn, N), dtype=torch.float32, device=dev)
    hist = torch.zeros((Bt, Dn, K - 1), dtype=bf, device=dev)
    out = torch.empty((T, Bt, Dn), dtype=bf, device=dev)
    lib = _abi.load()
    steps = []
    for t in range(T):
        sa = _abi.StepArgs()
        sa.x, sa.dt, sa.z = tok["x"][t].data_ptr(), tok["dt"][t].data_ptr(), tok["z"][t].data_ptr()
        sa.B, sa.C = tok["B"][t].data_ptr(), tok["C"][t].data_ptr()
        sa.A_log, sa.D, sa.dt_bias = par["A_log"].data_ptr(), par["D"].data_ptr(), par["dt_bias"].data_ptr()
        sa.conv_w, sa.conv_b = par["conv_w"].data_ptr(), par["conv_b"].data_ptr()
        sa.h, sa.conv_hist, sa.out = h.data_ptr(), hist.data_ptr(), out[t].data_ptr()
        sa.Bt, sa.Dn, sa.N, sa.K = Bt, Dn, N, K
        sa.in_dtype, sa.out_dtype, sa.delta_softplus, sa.discretization = _abi.SSM_BF16, _abi.SSM_BF16, 1, _abi.SSM_ZOH
        steps.append(sa)
    s = torch.cuda.Stream(dev)

    def run_tokens():
        for sa in steps:
            _abi.check("ssm_scan_step", lib.ssm_scan_step(ctypes.byref(sa), s.cuda_stream))

    with torch.cuda.stream(s):
        for _ in range(2):
            run_tokens()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        run_tokens()
    torch.cuda.synchronize()
    E = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    for _ in range(args.warmup):
        g.replay()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.15)
    if world > 1:
        dist.barrier(device_ids=[local])
    torch.cuda.synchronize()
    e0, e1 = E(), E()
    e0.record(s)
    with torch.cuda.stream(s):
        for _ in range(args.steps):
            g.replay()
    e1.record(s)
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev) / args.steps  # per replay of T tokens
    # the same T tokens as plain launches from the host
    f0, f1 = E(), E()
    f0.record(s)
    with torch.cuda.stream(s):
        run_tokens()
    f1.record(s)
    torch.cuda.synchronize()
    eager_ms = f0.elapsed_time(f1)
    us_tok = ms * 1e3 / T
    # algorithmic bytes of one token step: per (sequence, channel) the state read and written
    # (N fp32 each way), the conv history read and written ((K-1) bf16 each way), x, dt, z in and
    # the output (bf16); per sequence B and C (bf16); the parameters once
    bytes_step = (Bt * Dn * (N * 4 * 2 + (K - 1) * 2 * 2 + 3 * 2 + 2) + Bt * N * 2 * 2
                  + Dn * (N + 3 + K) * 4)
    peaks = load_peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    gbs = bytes_step / (us_tok * 1e-6) / 1e9
    line = {
        "metric": "decode tokens/s (sequences x tokens per second), 1xB200", "value": Bt * T * world / (ms * 1e-3),
        "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "Bt": Bt, "Dn": Dn, "N": N, "K": K, "tokens_per_step": T,
                   "step": "%d decode steps (one launch each) replayed as one CUDA graph" % T,
                   "state": "%.1f MB of state and conv history, resident in L2 across tokens"
                            % ((Bt * Dn * (N * 4 + (K - 1) * 2)) / 1e6)},
        "us_per_token_step": us_tok,
        "eager_us_per_token_step": eager_ms * 1e3 / T,
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                     "algorithmic_bytes": bytes_step, "kernel": "ssm_step_kernel",
                     "traffic": ncu_traffic("ssm_step_kernel", "ssm_step.cu", w.name), "peak_source": peaks.get("source")},
        "gpu_launches": T * args.steps, "clocks": clk,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    del g
    if world > 1:
        dist.destroy_process_group()
    return 0


def conv_bench(args, w):
    """The standalone causal conv1d + SiLU (ssm_conv1d_silu) through the C ABI: bf16 x in, bf16 u
    out, inputs larger than L2; a pure stream, so the roofline is HBM."""
    import ctypes
    import torch
    from selective_state_space_34_b200 import _abi
    from selective_state_space_34_b200 import workloads as wl
    world, rank, local = rank_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    a = wl.generate(w, seed=w.seed + rank)
    x = torch.from_numpy(a["x"]).to(dev, torch.bfloat16)
    cw = torch.from_numpy(a["conv_w"]).to(dev, torch.float32)
    cb = torch.from_numpy(a["conv_b"]).to(dev, torch.float32)
    u = torch.empty_like(x)
    lib = _abi.load()
    s = torch.cuda.current_stream(dev)

    def run():
        _abi.check("ssm_conv1d_silu", lib.ssm_conv1d_silu(
            x.data_ptr(), u.data_ptr(), cw.data_ptr(), cb.data_ptr(), w.Bt, w.Dn, w.L, w.K,
            _abi.SSM_BF16, _abi.SSM_BF16, s.cuda_stream))

    for _ in range(args.warmup):
        run()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.15)
    if world > 1:
        dist.barrier(device_ids=[local])
    torch.cuda.synchronize()
    E = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    e0, e1 = E(), E()
    e0.record(s)
    for _ in range(args.steps):
        run()
    e1.record(s)
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev) / args.steps
    nbytes = w.Bt * w.Dn * w.L * 2 * 2 + w.Dn * (w.K + 1) * 4  # x in, u out (bf16), taps and bias
    peaks = load_peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    gbs = nbytes / (ms * 1e-3) / 1e9
    line = {
        "metric": "causal conv1d + SiLU elements/s, 1xB200", "value": w.Bt * w.Dn * w.L * world / (ms * 1e-3),
        "unit": "elements/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "Bt": w.Bt, "Dn": w.Dn, "L": w.L, "K": w.K,
                   "l2": "inputs larger than L2 (%.0f MB per call)" % (nbytes / 1e6)},
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                     "algorithmic_bytes": nbytes, "kernel": "conv1d_silu_vec_kernel",
                     "traffic": ncu_traffic("conv1d_silu_vec_kernel", "ssm_conv.cu", w.name), "peak_source": peaks.get("source")},
        "gpu_launches": args.steps, "clocks": clk,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


# ---- our arm ----------------------------------------------------------------------------------

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="mamba1p4b_fwdbwd")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--out-dtype", default="bf16", choices=["bf16", "f32"])
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--n-segments", type=int, default=0,
                    help="split-L for the forward: 0 one pass, k up to k segments, -1 automatic")
    ap.add_argument("--scan-form", default="lanes", choices=["lanes", "chunked"],
                    help="layout of a one-pass forward scan: states over lanes, or chunked in time")
    ap.add_argument("--ssd-form", default="auto", choices=["auto", "fused", "three_pass"],
                    help="state-space-duality workloads: one fused launch, or three passes")
    args = ap.parse_args()
    assert args.warmup >= 3, "at least 3 warm-up steps"

    from selective_state_space_34_b200 import workloads as wl
    if args.workload in wl.CONV_WORKLOADS:
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable": "the conv leg has no CPU reference "
                              "arm; its parity is in tests/test_gpu_conv.py"}))
            return 0
        return conv_bench(args, wl.CONV_WORKLOADS[args.workload])
    if args.workload in wl.DECODE_WORKLOADS:
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable": "the decode leg has no CPU reference "
                              "arm; its parity is in tests/test_gpu_state.py"}))
            return 0
        return decode_bench(args, wl.DECODE_WORKLOADS[args.workload])
    if args.workload in wl.SSD_WORKLOADS:
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable": "the state-space-duality leg has no "
                              "CPU reference arm; its parity is in tests/test_gpu_ssd.py"}))
            return 0
        return ssd_bench(args, wl.SSD_WORKLOADS[args.workload], args.workload)
    w = wl.WORKLOADS[args.workload]
    if args.impl == "reference":
        return reference_arm(args, w)

    import torch
    import torch.distributed as dist
    import selective_state_space_34_b200 as ssm

    world, rank, local = rank_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    # each rank draws its own batch (weak scaling)
    a = wl.generate(w, seed=rank_seed(w, rank))
    act = torch.bfloat16 if w.in_dtype == "bf16" else torch.float32
    odt = torch.bfloat16 if args.out_dtype == "bf16" else torch.float32

    def todev(k, dtype):
        return None if a.get(k) is None else torch.from_numpy(a[k]).to(dev, dtype)
    T = {k: todev(k, act) for k in ("x", "dt", "z", "B", "C", "dout")}
    T.update({k: todev(k, torch.float32) for k in ("A_log", "D", "dt_bias", "conv_w", "conv_b")})
    kw = dict(D=T["D"], z=T["z"], dt_bias=T["dt_bias"], conv_w=T["conv_w"], conv_b=T["conv_b"])
    Bt, Dn, N, L = w.Bt, w.Dn, w.N, w.L
    s_in = 2 if act == torch.bfloat16 else 4
    s_out = 2 if odt == torch.bfloat16 else 4
    es = w.elem_states
    backward = w.backward

    out = torch.empty((Bt, Dn, L), dtype=odt, device=dev)
    n_ck = ssm.ssm_num_state_chunks(L)
    states = torch.empty((Bt, Dn, n_ck, N), dtype=torch.float32, device=dev)
    grads = None
    ws = None
    need = 0
    if backward:
        f32 = dict(dtype=torch.float32, device=dev)
        grads = {"dx": torch.empty((Bt, Dn, L), **f32), "ddt": torch.empty((Bt, Dn, L), **f32),
                 "dz": torch.empty((Bt, Dn, L), **f32), "dA_log": torch.empty((Dn, N), **f32),
                 "dB": torch.empty((Bt, N, L), **f32), "dC": torch.empty((Bt, N, L), **f32),
                 "dD": torch.empty((Dn,), **f32), "ddt_bias": torch.empty((Dn,), **f32),
                 "dconv_w": torch.empty(tuple(T["conv_w"].shape), **f32),
                 "dconv_b": torch.empty((Dn,), **f32)}
        need = ssm.ssm_bwd_workspace_size(T["dout"], T["x"], T["dt"], T["A_log"], T["B"], T["C"],
                                          chunk_states=states, n_segments=args.n_segments, **kw)
        ws = torch.empty(need + 256, dtype=torch.uint8, device=dev)

    import ctypes
    from selective_state_space_34_b200 import _abi, api
    lib = _abi.load()
    s = torch.cuda.current_stream(dev)

    # argument structs built once; each step is then plain C-ABI calls on the current stream
    fwd_args, _ = api._fwd_args(T["x"], T["dt"], T["A_log"], T["B"], T["C"], kw["D"], kw["z"],
                                kw["dt_bias"], kw["conv_w"], kw["conv_b"], True, odt,
                                scan_form=args.scan_form)
    fwd_args.out = out.data_ptr()
    fwd_args.chunk_states = states.data_ptr() if backward else None
    ws_f = None
    if args.n_segments:
        fwd_args.n_segments = args.n_segments
        need_f = lib.ssm_fwd_workspace_size(ctypes.byref(fwd_args))
        if need_f:
            ws_f = torch.empty(need_f + 256, dtype=torch.uint8, device=dev)
            fwd_args.workspace = (ws_f.data_ptr() + 255) & ~255
            fwd_args.workspace_bytes = need_f
    fwd_args_fo = _abi.FwdArgs.from_buffer_copy(fwd_args)
    fwd_args_fo.chunk_states = None
    if backward:
        bw_args = api._bwd_struct(T["dout"], T["x"], T["dt"], T["A_log"], T["B"], T["C"], kw["D"],
                                  kw["z"], kw["dt_bias"], kw["conv_w"], kw["conv_b"], True, states)
        for k, v in grads.items():
            setattr(bw_args, k, v.data_ptr())
        bw_args.workspace = (ws.data_ptr() + 255) & ~255
        bw_args.workspace_bytes = need
        bw_args.fwd.n_segments = args.n_segments

    E = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    n_rec = args.steps
    ev_f0 = [E() for _ in range(n_rec)]
    ev_f1 = [E() for _ in range(n_rec)]
    ev_b = [[E(), E()] for _ in range(n_rec)] if backward else None
    ev_b1 = [E() for _ in range(n_rec)] if backward else None
    ev_ptr = []
    for evs in (ev_b or []):
        for e in evs:
            e.record(s)  # creates the underlying cudaEvent_t handles before they are passed down
        ev_ptr.append((ctypes.c_void_p * 2)(evs[0].cuda_event, evs[1].cuda_event))
    torch.cuda.synchronize()

    def step(i=None, timed=False):
        if timed:
            ev_f0[i].record(s)
        _abi.check("ssm_scan_fwd", lib.ssm_scan_fwd(ctypes.byref(fwd_args), s.cuda_stream))
        if timed:
            ev_f1[i].record(s)
        if backward:
            bw_args.timing_events = ctypes.cast(ev_ptr[i], ctypes.c_void_p) if timed else None
            _abi.check("ssm_scan_bwd", lib.ssm_scan_bwd(ctypes.byref(bw_args), s.cuda_stream))
            if timed:
                ev_b1[i].record(s)

    def fwd_only():
        _abi.check("ssm_scan_fwd", lib.ssm_scan_fwd(ctypes.byref(fwd_args_fo), s.cuda_stream))

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])

    # ---- device-resident timing of K steps ----
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.15)
    barrier()
    torch.cuda.synchronize()
    t_start, t_end = E(), E()
    t_start.record(s)
    for i in range(args.steps):
        step(i, timed=True)
    t_end.record(s)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    max_ms = max_over_ranks(t_start.elapsed_time(t_end), world, dev)
    ms_step = max_ms / args.steps
    value = job_throughput(es, world, args.steps, max_ms)

    step_end = ev_b1 if backward else ev_f1
    per_step = np.array([ev_f0[i].elapsed_time(step_end[i]) for i in range(args.steps)])
    step_dist = {"median": float(np.median(per_step)), "p10": float(np.percentile(per_step, 10)),
                 "p90": float(np.percentile(per_step, 90)),
                 "of": "rank 0, CUDA events around each timed step"}
    # the timed steps' own results, kept on the host for the parity check below
    got = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        got = {"out": out.float().cpu().numpy()}
        if backward:
            got.update({k: v.cpu().numpy() for k, v in grads.items()})
    fwd_ms = float(np.mean([ev_f0[i].elapsed_time(ev_f1[i]) for i in range(args.steps)]))
    kern = {"ssm_fwd_kernel": fwd_ms}
    if backward:
        kern["ssm_bwd_kernel"] = float(np.mean([ev_b[i][0].elapsed_time(ev_b[i][1]) for i in range(args.steps)]))
        kern["bwd_reductions"] = float(np.mean([ev_b[i][1].elapsed_time(ev_b1[i]) for i in range(args.steps)]))

    # ---- forward alone on the same shape (no state saving): the HBM-headline case ----
    for _ in range(3):
        fwd_only()
    torch.cuda.synchronize()
    barrier()
    f0, f1 = E(), E()
    nf = max(args.steps, 20)
    f0.record(s)
    for _ in range(nf):
        fwd_only()
    f1.record(s)
    torch.cuda.synchronize()
    fo_ms = max_over_ranks(f0.elapsed_time(f1) / nf, world, dev)

    peaks = load_peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    fb = fwd_bytes(Bt, Dn, N, L, s_in, s_out)
    fwd_roof = {"bound": "hbm", "achieved": fb / (fo_ms * 1e-3) / 1e9, "peak": hbm, "unit": "GB/s",
                "frac": fb / (fo_ms * 1e-3) / 1e9 / hbm,
                "traffic": ncu_traffic("ssm_fwd_kernel", "ssm_fwd.cu", w.name) if (s_out == 2 and s_in == 2) else None,
                "algorithmic_bytes": fb, "kernel": "ssm_fwd_kernel", "ms": fo_ms,
                "peak_source": peaks.get("source")}
    sm_hz = (clk["sm_mhz"] or peaks.get("sm_max_mhz", 1965.0)) * 1e6
    mufu_peak = MUFU_LANES * N_SM * sm_hz / 1e9  # Gexp2/s at the sampled SM clock

    def alu_roof(kernel, ms):
        # the irreducible exp of the method: one A_bar = exp(Delta A) per element-state, against
        # the exp unit's rate (16 results/clk/SM x 148 SMs x sampled clock)
        ach = es / (ms * 1e-3) / 1e9
        return {"bound": "alu", "achieved": ach, "peak": mufu_peak, "unit": "Gexp/s",
                "frac": ach / mufu_peak, "kernel": kernel,
                "peak_source": "16 MUFU ex2 lanes/clk/SM x 148 SMs x sampled SM clock"}
    forward = {"ms": fo_ms, "value": job_throughput(es, world, 1, fo_ms), "unit": UNIT,
               "out_dtype": args.out_dtype, "roofline": fwd_roof,
               "alu_roofline": alu_roof("ssm_fwd_kernel", fo_ms)}

    if backward:
        bms = kern["ssm_bwd_kernel"]
        bb = bwd_bytes(Bt, Dn, N, L, s_in)
        roof = {"bound": "hbm", "achieved": bb / (bms * 1e-3) / 1e9, "peak": hbm, "unit": "GB/s",
                "frac": bb / (bms * 1e-3) / 1e9 / hbm,
                "traffic": ncu_traffic("ssm_bwd_kernel", "ssm_bwd.cu", w.name) if s_in == 2 else None,
                "algorithmic_bytes": bb, "kernel": "ssm_bwd_kernel", "ms": bms,
                "peak_source": peaks.get("source"),
                "overhead_bytes": bwd_overhead_bytes(Bt, Dn, N, n_ck)}
    else:
        roof = dict(fwd_roof)
    # a split forward is three launches (segment summaries, carry, segments); the backward is its
    # kernel and one reduction launch (dB / dC tiles and per-channel parameters, rows of whole
    # 16-byte vectors as here), and a split backward adds the adjoint summaries, their carry and
    # the dx fix-up
    split = ws_f is not None
    launches_per_step = (3 if split else 1) + ((5 if split else 2) if backward else 0)

    # ---- end to end through the C ABI with host buffers: H2D inputs, compute, D2H results ----
    # Every step copies its inputs from pinned host memory and reads all of its results back (the
    # output and, with the backward, every gradient). Copies in and out run on their own streams,
    # so a step costs the slowest of the three.
    names_in = [k for k in ("x", "dt", "z", "B", "C") + (("dout",) if backward else ()) if T[k] is not None]
    host = {k: torch.empty(T[k].shape, dtype=T[k].dtype, pin_memory=True) for k in names_in}
    for k in names_in:
        host[k].copy_(T[k].cpu())
    h2d = sum(host[k].numel() * host[k].element_size() for k in names_in)
    res_names = (["dx", "ddt", "dz", "dA_log", "dB", "dC", "dD", "ddt_bias", "dconv_w", "dconv_b"]
                 if backward else [])
    host_out = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    host_res = {k: torch.empty(grads[k].shape, dtype=torch.float32, pin_memory=True) for k in res_names}
    d2h = host_out.numel() * host_out.element_size() + sum(v.numel() * 4 for v in host_res.values())

    # two device sets of inputs and of results: while step i computes, step i+1's inputs arrive
    # and step i-1's results leave
    T2 = {k: torch.empty_like(T[k]) for k in names_in}
    out2 = torch.empty_like(out)
    grads2 = {k: torch.empty_like(v) for k, v in grads.items()} if backward else None
    fa2 = _abi.FwdArgs.from_buffer_copy(fwd_args)
    for k in ("x", "dt", "z", "B", "C"):
        if k in T2:
            setattr(fa2, k, T2[k].data_ptr())
    fa2.out = out2.data_ptr()
    ba2 = None
    if backward:
        ba2 = _abi.BwdArgs.from_buffer_copy(bw_args)
        for k in ("x", "dt", "z", "B", "C"):
            if k in T2:
                setattr(ba2.fwd, k, T2[k].data_ptr())
        ba2.dout = T2["dout"].data_ptr()
        for k, v in grads2.items():
            setattr(ba2, k, v.data_ptr())
    sets = [(T, fwd_args, bw_args if backward else None, out, grads), (T2, fa2, ba2, out2, grads2)]
    h2d_s, d2h_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_ready, ev_done, ev_back = [E(), E()], [E(), E()], [E(), E()]

    def run_step(fa, ba):
        _abi.check("ssm_scan_fwd", lib.ssm_scan_fwd(ctypes.byref(fa), s.cuda_stream))
        if backward:
            ba.timing_events = None
            _abi.check("ssm_scan_bwd", lib.ssm_scan_bwd(ctypes.byref(ba), s.cuda_stream))

    def e2e_run(n):
        for j in range(2):
            ev_done[j].record(s)
            ev_back[j].record(s)
        for i in range(n):
            Tk, fa, ba, ok, gk = sets[i % 2]
            h2d_s.wait_event(ev_done[i % 2])          # step i-2 is done with this input set
            with torch.cuda.stream(h2d_s):
                for k in names_in:
                    Tk[k].copy_(host[k], non_blocking=True)
            ev_ready[i % 2].record(h2d_s)
            s.wait_event(ev_ready[i % 2])
            s.wait_event(ev_back[i % 2])              # step i-2's results have been read out
            run_step(fa, ba)
            ev_done[i % 2].record(s)
            d2h_s.wait_event(ev_done[i % 2])
            with torch.cuda.stream(d2h_s):
                host_out.copy_(ok, non_blocking=True)
                for k in res_names:
                    host_res[k].copy_(gk[k], non_blocking=True)
            ev_back[i % 2].record(d2h_s)
        for j in range(2):
            s.wait_event(ev_back[j])

    e2e_run(3)
    torch.cuda.synchronize()
    barrier()
    e0, e1 = E(), E()
    e0.record(s)
    e2e_run(args.e2e_steps)
    e1.record(s)
    torch.cuda.synchronize()
    e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    e2e = {"value": job_throughput(es, world, args.e2e_steps, e_ms), "unit": UNIT,
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
           "ms_per_step": e_ms / args.e2e_steps,
           "overlap": "two device sets of inputs and results: step i+1's inputs copied in and step "
                      "i-1's results (out and every gradient) copied out while step i computes"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        threads = os.cpu_count() or 1
        # a short calibration sample sizes the measured one to about 12 s of host work
        c_secs, c_done = oracle_sample(w, a, 16 * threads, threads)
        per_ch = c_secs / (16 * threads)
        n_ch = int(min(4 * w.Bt * w.Dn, max(16 * threads, 12.0 / max(per_ch, 1e-9))))
        secs, done = oracle_sample(w, a, n_ch, threads)
        cpu = {"value": done / secs, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": "%d channels (wrapping over the %d of the workload) x L=%d x N=%d (fwd%s), "
                         "float64, %.1f s" % (n_ch, w.Bt * w.Dn, L, N, "+bwd" if backward else "", secs),
               "parity": oracle_parity(w, a, got, odt == torch.bfloat16, threads)}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "step_ms": step_dist,
            "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": w.name, "Bt": Bt, "Dn": Dn, "N": N, "L": L,
                       "in_dtype": w.in_dtype, "out_dtype": args.out_dtype,
                       "step": "fwd(save states)+bwd" if backward else "fwd",
                       "l2": "inputs larger than L2 (per-step working set %.2f GB)"
                             % ((fwd_bytes(Bt, Dn, N, L, s_in, s_out, n_ck if backward else 0)
                                 + (bwd_bytes(Bt, Dn, N, L, s_in) if backward else 0)) / 1e9),
                       "parallelism": "replica per GPU" if world > 1 else "single GPU",
                       "n_segments": args.n_segments, "scan_form": args.scan_form},
            "roofline": roof,
            "alu_roofline": alu_roof("ssm_bwd_kernel" if backward else "ssm_fwd_kernel",
                                     kern["ssm_bwd_kernel"] if backward else fo_ms),
            "kernels_ms": kern,
            "forward": forward,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
