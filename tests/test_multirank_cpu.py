"""The multi-rank plumbing of bench.py on CPU: two gloo ranks, launched the way torchrun launches
them (WORLD_SIZE / RANK / LOCAL_RANK / MASTER_* in the environment). Checks that each rank draws
its own batch, that timings are combined as the max over ranks on every rank, that the whole-job
rate counts every rank's units over the slowest time, and that the reference arm runs on rank 0
alone. No GPU and no data-path collective are involved."""
import io
import json
import os
import socket
import sys
import types
from contextlib import redirect_stdout

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, outdir):
    os.environ.update({"WORLD_SIZE": str(world), "RANK": str(rank), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    from datetime import timedelta
    import torch.distributed as dist
    import bench
    from selective_state_space_34_b200 import workloads as wl
    dist.init_process_group("gloo", timeout=timedelta(seconds=60))
    try:
        res = {}
        res["env"] = list(bench.rank_env())
        w = wl.WORKLOADS["tiny_fp32"]
        res["seed"] = bench.rank_seed(w, rank)
        a = wl.generate(w, seed=res["seed"])
        res["x_sum"] = float(np.float64(a["x"]).sum())
        # a per-rank device time; every rank must see the slowest one
        res["max_ms"] = bench.max_over_ranks(10.0 + 7.5 * rank, world, "cpu")
        res["rate"] = bench.job_throughput(w.elem_states, world, 4, res["max_ms"])
        buf = io.StringIO()
        args = types.SimpleNamespace(gpus=world, steps=2, warmup=1)
        with redirect_stdout(buf):
            res["ref_rc"] = bench.reference_arm(args, w)
        res["ref_out"] = buf.getvalue()
        dist.barrier()
        with open(os.path.join(outdir, "rank%d.json" % rank), "w") as f:
            json.dump(res, f)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    r = [json.load(open(tmp_path / ("rank%d.json" % i))) for i in range(world)]
    assert [x["env"] for x in r] == [[2, 0, 0], [2, 1, 1]]
    assert r[0]["seed"] != r[1]["seed"] and r[0]["x_sum"] != r[1]["x_sum"]
    assert r[0]["max_ms"] == r[1]["max_ms"] == 17.5
    from selective_state_space_34_b200 import workloads as wl
    es = wl.WORKLOADS["tiny_fp32"].elem_states
    assert r[0]["rate"] == pytest.approx(es * 2 * 4 / 17.5e-3)
    assert r[0]["ref_rc"] == 0 and r[1]["ref_rc"] == 0
    assert r[1]["ref_out"] == ""
    line = json.loads(r[0]["ref_out"].strip())
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"


def test_single_rank_defaults(monkeypatch):
    import bench
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert bench.rank_env() == (1, 0, 0)
    assert bench.max_over_ranks(3.25, 1, "cpu") == 3.25
    assert bench.job_throughput(1000, 1, 10, 2.0) == pytest.approx(1000 * 10 / 2e-3)


def test_oracle_sample_counts_every_sampled_channel():
    """The CPU baseline's sample wraps over (batch, channel) and counts what it ran."""
    import bench
    from selective_state_space_34_b200 import workloads as wl
    w = wl.shaped("tiny_fp32", Bt=2, Dn=6, L=16)
    a = wl.generate(w)
    for n_ch, threads in ((40, 3), (5, 2), (12, 12)):
        _, done = bench.oracle_sample(w, a, n_ch, threads)
        assert done == n_ch * w.L * w.N
