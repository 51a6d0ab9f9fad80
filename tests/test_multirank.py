"""N > 1 host logic of the bench on CPU: world-size-2 gloo ranks (replicas only, no data-path collective)."""

import os
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, q):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, torch.device("cpu"))
        w, r, l = bench._dist()
        # the reference arm runs on rank 0 only; other ranks exit without work
        args = bench.parse_args(["--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "3",
                                 "--cpu-seconds", "0.2"])
        ref = bench.run_reference(args, w, r)
        q.put((rank, ms, (w, r, l), ref is None))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_time_and_only_rank0_runs_reference():
    import socket
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=300) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [o[1] for o in out] == [15.0, 15.0]            # both ranks see the slowest rank's time
    assert [o[2] for o in out] == [(2, 0, 0), (2, 1, 1)]
    assert [o[3] for o in out] == [False, True]            # rank 0 produced the reference line


def test_whole_job_value_is_sum_of_replicas_over_max_time():
    sys.path.insert(0, ROOT)
    import bench
    one = bench.whole_job_tflops(1, 10, 1e12, 1000.0)
    two = bench.whole_job_tflops(2, 10, 1e12, 1000.0)
    assert one == pytest.approx(10.0) and two == pytest.approx(20.0)


def test_reference_line_keeps_the_contract():
    """The reference arm (the oracle on the host cores) prints the bench's metric, unit,
    direction and config, with its own cpu_baseline and a zero-copy e2e."""
    sys.path.insert(0, ROOT)
    import bench
    from synth import make_workload
    args = bench.parse_args(["--impl", "reference", "--workload", "tiny", "--steps", "2", "--warmup", "3",
                             "--cpu-seconds", "0.5"])
    line = bench.run_reference(args, 1, 0)
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC and line["unit"] == "TFLOP/s"
    assert line["higher_is_better"] is True and line["steps"] == 2 and line["warmup"] == 3
    w = make_workload("tiny", with_grad=True)
    assert line["config"] == bench.bench_config(args, w, *bench._workers(args), 1)
    assert line["value"] > 0 and line["cpu_baseline"]["value"] == line["value"]
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"] == {"value": line["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    import json
    json.dumps(line)


def test_cpu_baseline_reports_all_cores_and_one_thread():
    sys.path.insert(0, ROOT)
    import bench
    from synth import make_workload
    r = bench.cpu_baseline(make_workload("tiny", with_grad=True), budget_s=0.6)
    assert r["kind"] == "oracle" and r["unit"] == "TFLOP/s" and r["cores"] >= 1
    assert r["value"] > 0 and r["value_one_thread"] > 0
    assert "1 BLAS thread" in r["sample_one_thread"]


def test_seed_option_reaches_the_config():
    sys.path.insert(0, ROOT)
    import bench
    from synth import make_workload
    args = bench.parse_args(["--impl", "reference", "--workload", "tiny", "--seed", "7"])
    w = make_workload("tiny", seed=7, with_grad=True)
    assert bench.bench_config(args, w, 148, 148, 1)["seed"] == 7
    args = bench.parse_args(["--workload", "tiny"])
    assert bench.bench_config(args, w, 148, 148, 1)["seed"] == 1000 + w.config.index


def test_rank_emulation_option():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.parse_args([]).emulate_ranks == 0                 # not part of the default run
    assert bench.parse_args(["--emulate-ranks", "4"]).emulate_ranks == 4
    assert callable(bench.rank_emulation_report)
    a = bench.parse_args(["--split-kv", "--schedule", "contiguous"])
    assert a.split_kv and a.dynamic_claim                           # contiguous names the rank ownership there
    assert not bench.parse_args(["--schedule", "contiguous"]).dynamic_claim
    assert callable(bench.run_split_kv)
    assert bench.parse_args(["--split-kv", "--exchange", "p2p"]).exchange == "p2p"


def test_cpu_baseline_reports_the_error_on_its_sample():
    """With the GPU's rows supplied, the oracle leg also reports their error on the blocks
    it computed (here: the oracle's own rows, exact, then a copy off by 0.5 in dq)."""
    sys.path.insert(0, ROOT)
    import numpy as np
    import bench
    from oracle import attention as oatt
    from synth import make_workload
    w = make_workload("tiny", with_grad=True)
    f = {n: w.f64(n) for n in ("q", "k", "v", "kb", "vb", "dout")}
    O, L = oatt.attention_fwd(f["q"], f["k"], f["v"], f["kb"], f["vb"], w.sample_lens, w.anchors, w.block_size,
                              w.scale)
    g = oatt.attention_bwd(f["q"], f["k"], f["v"], f["kb"], f["vb"], f["dout"], w.sample_lens, w.anchors,
                           w.block_size, w.scale)
    full = {"o": O, "lse": L, "dq": g["dq"], "dkb": g["dkb"], "dvb": g["dvb"]}
    exact = bench.cpu_baseline(w, budget_s=0.2, gpu_rows=lambda rows: {n: x[rows] for n, x in full.items()})
    ps = exact["parity_sample"]
    assert ps["blocks"] >= 1 and all(v < 1e-12 for v in ps["max_abs"].values())
    off = dict(full, dq=full["dq"] + 0.5)
    bad = bench.cpu_baseline(w, budget_s=0.2, gpu_rows=lambda rows: {n: x[rows] for n, x in off.items()})
    assert abs(bad["parity_sample"]["max_abs"]["dq"] - 0.5) < 1e-9
    assert bad["parity_sample"]["max_abs"]["o"] < 1e-12
