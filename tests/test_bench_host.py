"""Host-side logic of bench.py's multi-rank path, run as world-size-2 gloo
ranks on the CPU: per-rank workloads, max-over-ranks timing and the
whole-job value. No GPU and no CUDA call is involved."""
import importlib.util
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _load_bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import torch.distributed as dist

    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench = _load_bench()
        from dequant_gemv_q4_b200 import synth

        wl = bench.rank_workload(synth.WORKLOADS["q8_0_gemv_1024x1024"], rank, world)
        inp = synth.make_inputs(wl)
        # each rank reports a different step time; every rank must see the slowest
        ms = bench.max_over_ranks(0.25 + 0.5 * rank, world)
        value = bench.job_gbps(bench.algorithmic_bytes(wl), world, ms)
        res = {
            "seed": wl.seed, "N": wl.N, "K": wl.K,
            "x_head": [float(v) for v in np.asarray(inp["x"]).ravel()[:8]],
            "w_sum": int(np.asarray(inp["w"]).astype(np.int64).sum()),
            "ms": ms, "value": value,
        }
        with open(os.path.join(out_dir, "rank%d.json" % rank), "w") as f:
            json.dump(res, f)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_share_max_time_and_run_distinct_problems(tmp_path):
    import torch.multiprocessing as tmp

    world = 2
    tmp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                        join=True, start_method="spawn")
    r = [json.load(open(tmp_path / ("rank%d.json" % i))) for i in range(world)]

    # max over ranks: both ranks hold the slower rank's time
    assert r[0]["ms"] == r[1]["ms"] == pytest.approx(0.75)
    # same shape, different seed and different data on each rank
    assert (r[0]["N"], r[0]["K"]) == (r[1]["N"], r[1]["K"])
    assert r[0]["seed"] != r[1]["seed"]
    assert r[0]["x_head"] != r[1]["x_head"] or r[0]["w_sum"] != r[1]["w_sum"]
    # whole-job value: both ranks' bytes over the common (slowest) step time
    bench = _load_bench()
    from dequant_gemv_q4_b200 import synth
    nbytes = bench.algorithmic_bytes(synth.WORKLOADS["q8_0_gemv_1024x1024"])
    assert r[0]["value"] == r[1]["value"] == pytest.approx(2 * nbytes / 0.75e-3 / 1e9)


def test_single_rank_helpers_need_no_process_group():
    bench = _load_bench()
    from dequant_gemv_q4_b200 import synth

    wl = synth.WORKLOADS["q4k_lmhead_248320x4096"]
    assert bench.rank_workload(wl, 0, 1) is wl
    assert bench.max_over_ranks(1.5, 1) == 1.5
    assert bench.job_gbps(1_000_000_000, 1, 1000.0) == pytest.approx(1.0)
    assert bench.job_gbps(1_000_000_000, 4, 1000.0) == pytest.approx(4.0)
    # seeds stay distinct across ranks of a larger job
    seeds = {bench.rank_workload(wl, r, 8).seed for r in range(8)}
    assert len(seeds) == 8


def test_reference_arm_runs_on_rank_zero_only():
    bench = _load_bench()

    class A:
        workload = "q8_0_gemv_1024x1024"
        steps = 1
        warmup = 0
        gpus = 2

    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.run_reference(A, 1, 2)
    assert buf.getvalue() == ""

    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.run_reference(A, 0, 2)
    line = json.loads(buf.getvalue().strip())
    assert line["impl"] == "reference"
    assert line["n_gpus"] == 2 and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
