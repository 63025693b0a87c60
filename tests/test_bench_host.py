"""Host-side logic of the benchmark on CPU: two gloo ranks agree on the slowest
rank's time, and the workload accounting counts only algorithmic bytes and
FLOPs."""
import math
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from moe_inputs import CONFIGS


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dev = torch.device("cpu")
        bench.barrier(dev)
        t = bench.max_over_ranks(1.5 + rank, dev)
        again = bench.max_over_ranks(10.0 - rank, dev)
        out[rank] = (t, again, bench.dist_env())
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for rank in range(world):
        t, again, env = res[rank]
        assert t == 2.5 and again == 10.0
        assert env == (world, rank, rank)


def test_single_process_needs_no_process_group():
    assert bench.max_over_ranks(3.25, torch.device("cpu")) == 3.25


def test_layer_work_counts_only_algorithmic_flops():
    s = CONFIGS["mixtral"]
    w = bench.layer_work(s, None, kept_total=2 * s.T, dropped_tokens=0)
    # three matrices of d x d_ff per kept assignment, 2 FLOP per multiply-add
    assert w["expert_ffn"]["flops"] == 2.0 * 3 * (2 * s.T) * s.d * s.d_ff
    assert w["dispatch"]["bytes"] == s.T * s.d * 2 + 2 * s.T * s.d * 2 + s.T * s.k * 9
    # the fused alternative moves a row table instead
    assert w["dispatch_rows"]["bytes"] == bench.perm_rows(s) * 4 + s.T * s.k * 9 + 2 * s.T * 4
    assert bench.perm_rows(s) == (2 * s.T + 127 * s.E + 127) // 128 * 128
    ds = CONFIGS["deepseekmoe"]
    wd = bench.layer_work(ds, None, kept_total=ds.T * ds.k, dropped_tokens=0)
    shared = 2.0 * 3 * ds.n_shared * ds.T * ds.d * ds.d_ff_shared
    assert wd["expert_ffn"]["flops"] == 2.0 * 3 * ds.T * ds.k * ds.d * ds.d_ff + shared
    assert wd["route"]["bytes"] == ds.T * ds.d * 2 + ds.d * ds.E * 4 + ds.T * ds.k * 8 + \
        math.ceil(ds.T / 32) * (ds.E + 1) * 4


def test_clock_summary_flags_throttle_reasons():
    c = bench.ClockSampler(0)
    c.lines = ["0, 1900, 1965, 900.0, 0x1, Not Active, Not Active, Not Active, Active",
               "0, 1800, 1965, 990.0, 0x1, Not Active, Active, Not Active, Active",
               "garbage"]
    s = c.summary()
    assert s["sm_mhz"] == 1850.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"] and s["samples"] == 2


def test_peaks_fall_back_when_the_file_is_missing(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    peaks, src = bench.load_peaks()
    assert src == "fallback" and peaks["hbm_gbs"] == 6650.0


def test_layer_summary_rates_and_roofline():
    peaks = dict(bench.FALLBACK_PEAKS)
    s = CONFIGS["deepseek_v3"]
    kept = s.T * s.k
    stage_ms = {"route": 0.1, "capacity": 0.01, "dispatch": 0.1, "expert_ffn": 4.0,
                "combine": 0.1, "losses": 0.01}
    ms = sum(stage_ms.values())
    out = bench.summarize_layer(s, ms, stage_ms, kept, 0, steps=100, peaks=peaks)
    w = bench.layer_work(s, None, kept, 0)
    ffn = out["expert_ffn"]
    assert ffn["TFLOP/s"] == round(w["expert_ffn"]["flops"] / 4e-3 / 1e12, 1)
    # 22.6 GB of expert weights: the layer is bound by its bytes, not its FLOPs
    assert out["layer_roofline"]["bound"] == "hbm" and ffn["bound"] == "hbm"
    assert 0 < out["layer_roofline"]["frac"] <= 1
    assert out["stages"]["dispatch"]["GB/s"] == round(w["dispatch"]["bytes"] / 1e-4 / 1e9, 1)
    assert bench.summarize_layer(CONFIGS["mixtral"], 4.3, {**stage_ms, "expert_ffn": 4.0}, 16384,
                                 0, 200, peaks)["layer_roofline"]["bound"] == "tensor"


def test_launch_count_follows_the_forward():
    # router 1 (bf16, <= 16 experts) or 3, capacity 2, dispatch 1, two GEMMs,
    # combine 1 unless top-1 without shared experts
    assert bench.kernels_per_step(CONFIGS["mixtral"]) == 1 + 2 + 1 + 2 + 1
    assert bench.kernels_per_step(CONFIGS["switch"]) == 1 + 2 + 1 + 2
    assert bench.kernels_per_step(CONFIGS["deepseekmoe"]) == 3 + 2 + 1 + 2 + 1
    assert bench.kernels_per_step(CONFIGS["deepseek_v3"]) == 3 + 2 + 1 + 2 + 1
