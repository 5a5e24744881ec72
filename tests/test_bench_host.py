"""Host-side logic of bench.py (CPU only): the max-over-ranks reduction on
two gloo ranks, the whole-job throughput arithmetic and the reference arm's
JSON line."""
import json
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import workloads


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}",
                            rank=rank, world_size=world)
    try:
        bench.barrier(world)
        local_ms = 10.0 + 5.0 * rank          # rank 1 is the slow one
        max_ms = bench.reduce_max(local_ms, world)
        value = bench.whole_job_gbs(1_000_000_000, 4, world, max_ms)
        with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
            json.dump({"max_ms": max_ms, "value": value}, f)
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_on_two_gloo_ranks(tmp_path):
    port = _free_port()
    mp.spawn(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True)
    res = [json.load(open(tmp_path / f"r{r}.json")) for r in range(2)]
    for r in res:
        assert r["max_ms"] == 15.0
        # 2 ranks x 4 steps x 1 GB in 15 ms
        assert abs(r["value"] - 2 * 4 * 1.0 / 0.015) < 1e-6


def test_whole_job_throughput_single_rank():
    assert bench.reduce_max(3.5, 1) == 3.5
    assert abs(bench.whole_job_gbs(252_817_408, 10, 1, 2.0) - 1264.08704) < 1e-6


def test_bench_workload_bytes_match_the_roofline_table():
    """The default line is the 1.4B-shaped layer: u, delta, z in bf16 and y
    in fp32 per (b, d, t), B and C in bf16 per (b, n, t), A, D, delta_bias
    in fp32."""
    w = workloads.BY_NAME[bench.DEFAULT_WORKLOAD]
    assert w.name == "mamba1.4b-layer"
    bdl = 4 * 4096 * 4096
    assert w.algorithmic_bytes() == bdl * (3 * 2 + 4) + 2 * 4 * 16 * 4096 * 2 + \
        4096 * 16 * 4 + 4096 * 4 * 2 == 672_432_128
    assert w.state_updates == bdl * 16 == 1_073_741_824
    w1 = workloads.BY_NAME["mamba130m-layer"]
    assert w1.algorithmic_bytes() == 252_817_408 and w1.state_updates == 402_653_184


def test_exp_unit_bound_by_hand():
    """One ex2 per state update plus softplus (1) and silu (2) per (b, d, t),
    against 16 per clock per SM x 148 SMs."""
    w = workloads.BY_NAME["mamba130m-layer"]
    b = bench.exp_unit_bound(w, 0.1, 2000.0)
    ops = 402_653_184 + 3 * 8 * 1536 * 2048
    assert b["algorithmic_ops_per_launch"] == ops
    assert abs(b["peak"] - 16 * 148 * 2e9 / 1e12) < 1e-9
    assert abs(b["frac"] - ops / 1e-4 / (16 * 148 * 2e9)) < 1e-9
    assert abs(b["frac_of_exp_mix"] - 402_653_184 / 1e-4 / (20.5 * 148 * 2e9)) < 1e-9


def test_all_elements_error_on_cpu():
    """The bench's every-element parity: the oracle's own output gives only
    the fp32 rounding of y; one perturbed element shows up exactly."""
    import numpy as np
    import oracle
    w = workloads.custom(2, 40, 4, 50, in_dtype="bf16", has_z=True)
    inp = workloads.make_inputs(w, seed=9)
    h = workloads.to_numpy_f64(inp)
    ref = oracle.selective_scan(h["u"], h["delta"], h["A"], h["B"], h["C"], D=h["D"],
                                z=h["z"], delta_bias=h["delta_bias"])
    y = torch.from_numpy(ref.copy()).float()
    st = bench.all_elements_error(y, inp, w, block=16)
    assert st["elements"] == 2 * 40 * 50 and st["max_norm_err"] <= 2.0 ** -24
    y[1, 33, 7] += 0.25
    st = bench.all_elements_error(y, inp, w, block=16)
    assert abs(st["max_norm_err"] - 0.25 / np.abs(ref).max()) <= 2.0 ** -22


def test_single_thread_oracle_timing_reports_one_core():
    res = bench.single_thread_oracle(seconds=0.2)
    assert set(res) == {"tiny-fp32", "mamba130m-layer"}
    for r in res.values():
        assert r["cores"] == 1 and r["value"] > 0


def test_reference_arm_prints_the_contract_line(capsys):
    rc = bench.main(["--impl", "reference", "--workload", "tiny-fp32",
                     "--steps", "2", "--warmup", "1", "--ref-seconds", "0.5"])
    assert rc == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup",
                "ms_per_step", "higher_is_better", "scaling", "vs_baseline",
                "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["metric"] == bench.METRIC and line["unit"] == "GB/s"
    assert line["config"]["workload"] == "tiny-fp32"
    assert line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["value"] > 0


def test_ssd_workload_bytes_and_flops_by_hand():
    """2.7B-shaped layer: x read and y (fp32) written per (b, t, h, p), dt per
    (b, t, h), B and C per (b, t, n), three fp32 vectors per head; scores
    once per (b, chunk, group), the other three products per (b, chunk, head)."""
    w = workloads.SSD_BY_NAME["mamba2-2.7b-layer"]
    btp = 8 * 2048 * 80 * 64
    want = btp * (2 + 4) + 8 * 2048 * 80 * 2 + 2 * 8 * 2048 * 128 * 2 + 80 * 4 * 3
    assert w.algorithmic_bytes(4) == want == 514327488
    assert w.algorithmic_bytes(2) == want - btp * 2
    chunks = 2048 // 128
    scores = 8 * chunks * 2 * 128 * 128 * 128
    per_head = 8 * chunks * 80 * (2 * 128 * 128 * 64 + 2 * 2 * 128 * 128 * 64)
    assert w.chunk_flops() == scores + per_head == 64961380352


def test_ssd_oracle_sample_timing_on_cpu():
    """The SSD CPU baseline samples whole groups of heads and reports a
    positive rate (inputs on the CPU here; on the GPU machine they are copied)."""
    w = workloads.SSD_BY_NAME["ssd-small"]
    inp = workloads.make_ssd_inputs(w, seed=3)
    groups = bench._ssd_sample(inp, w, 3)
    assert sum(g["x"].shape[2] for g in groups) == 2  # rounded to whole groups
    assert all(g["B"].shape[2] * 2 == g["x"].shape[2] for g in groups)
    gbs, heads, threads, secs = bench.ssd_oracle_timing(inp, w, 0.05)
    assert gbs > 0 and heads % 2 == 0 and 2 <= heads <= w.batch * w.nheads
    assert threads >= 1 and secs > 0


def test_sampled_parity_helpers_on_cpu():
    """The bench's parity samples: the oracle's own output gives only the
    rounding of y to fp32 (the GPU's output dtype), a perturbed one the
    perturbation relative to max |y|."""
    import numpy as np
    import oracle
    w = workloads.custom(2, 8, 4, 40, in_dtype="f32", has_z=True)
    inp = workloads.make_inputs(w, seed=4)
    h = workloads.to_numpy_f64(inp)
    ref = oracle.selective_scan(h["u"], h["delta"], h["A"], h["B"], h["C"], D=h["D"],
                                z=h["z"], delta_bias=h["delta_bias"])
    y = torch.from_numpy(ref.copy())
    assert bench.sample_max_norm_err(y, inp, w, 12) <= 2.0 ** -24
    y[0, 3, 7] += 0.5
    scale = float(np.abs(ref[:1]).max())
    assert abs(bench.sample_max_norm_err(y, inp, w, 8) - 0.5 / scale) <= 2.0 ** -23

    ws = workloads.SSD_BY_NAME["ssd-small"]
    si = workloads.make_ssd_inputs(ws, seed=5)
    hs = workloads.to_numpy_f64(si)
    yref = oracle.ssd_scan(hs["x"], hs["dt"], hs["A"], hs["B"], hs["C"], D=hs["D"],
                           z=hs["z"], dt_bias=hs["dt_bias"])
    assert bench.ssd_sample_max_norm_err(torch.from_numpy(yref.copy()), si, ws) <= 2.0 ** -24


def test_reference_arm_for_the_ssd_pass(capsys):
    """--impl reference --pass ssd times the SSD oracle on the SSD workload,
    with the SSD line's metric, unit and config."""
    rc = bench.main(["--impl", "reference", "--pass", "ssd", "--ssd-workload", "ssd-small",
                     "--steps", "2", "--warmup", "1", "--ref-seconds", "0.3"])
    assert rc == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["metric"] == bench.SSD_METRIC
    assert line["unit"] == "GB/s" and line["value"] > 0
    assert line["config"] == bench.ssd_config(workloads.SSD_BY_NAME["ssd-small"], "f32")
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0
