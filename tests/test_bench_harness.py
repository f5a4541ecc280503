"""CPU checks of bench.py's host logic: the max-over-ranks reduction on a
2-rank gloo group (the replicas path runs one independent layer per GPU and
only this reduction crosses ranks), clock-sample parsing, and the
algorithmic work the roofline divides by."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from expert_layer_dual_b200.configs import CONFIGS


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    bench.init_dist(world, "gloo")
    try:
        got = bench.max_over_ranks(10.0 + 5 * rank, "cpu")
        bench.barrier()
        out[rank] = got
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_with_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    mp.start_processes(_rank_main, args=(2, _free_port(), out), nprocs=2, start_method="spawn",
                       join=True)
    assert dict(out) == {0: 15.0, 1: 15.0}


def test_max_over_ranks_without_a_group_is_identity():
    assert bench.max_over_ranks(3.5, "cpu") == 3.5


def test_clock_samples_parse_median_under_load_and_reasons():
    lines = [
        "0, 1965, 1965, 150.0, 0x0, Not Active, Not Active, Not Active, Not Active",
        "0, 1800, 1965, 900.0, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1700, 1965, 950.0, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1750, 1965, 920.0, 0x4, Not Active, Not Active, Not Active, Active",
        "garbage",
    ]
    c = bench.parse_clock_samples(lines)
    assert c["sm_mhz"] == 1750 and c["sm_max_mhz"] == 1965 and c["reasons"] == ["sw_power_cap"]
    assert bench.parse_clock_samples([])["sm_mhz"] is None


def test_algorithmic_work_of_the_gemms():
    cfg = CONFIGS["decode"]
    f, b = bench.gateup_algorithmic(cfg, cfg.T, n_active=200)
    R = 64 * 8 + 64
    assert f == 2.0 * R * 4096 * 2 * 1536
    # 200 routed experts + the shared one, each 2I x d bf16, plus x in and h out
    assert b == 201 * 2 * 1536 * 4096 * 2 + 64 * 4096 * 2 + R * 1536 * 2
    f8, b8 = bench.gateup_algorithmic(CONFIGS["fp8"], 4096, n_active=256)
    assert b8 == 257 * 2 * 2048 * 6144 + 4096 * 6144 + (4096 * 9) * 2048
    # MXFP8 adds one scale byte per 32 elements of weights, x and h
    fm, bm = bench.gateup_algorithmic(CONFIGS["mxfp8"], 4096, n_active=256)
    assert fm == f8 and bm == b8 + (257 * 2 * 2048 * 6144 + 4096 * 6144 + (4096 * 9) * 2048) // 32
    fd, bd = bench.down_algorithmic(cfg, cfg.T, n_active=200)
    assert fd == 2.0 * R * 1536 * 4096
    assert CONFIGS["prefill"].flops() == pytest.approx(2.82e12, rel=0.01)


def test_peak_regime_follows_the_clock_under_load():
    capped = {"sm_mhz": 1342.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    flagged_full_clock = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    assert bench.power_capped(capped, 50.0)
    assert not bench.power_capped(flagged_full_clock, 800.0)
    # without clock samples, the length of the timed region decides
    assert not bench.power_capped({"sm_mhz": None, "sm_max_mhz": None, "reasons": []}, 50.0)
    assert bench.power_capped({"sm_mhz": None, "sm_max_mhz": None, "reasons": []}, 800.0)
    hbm, burst, _ = bench.load_peaks(False)
    _, sustained, _ = bench.load_peaks(True)
    assert sustained <= burst and hbm > 0


def test_gateup_kernel_follows_the_library_dispatch():
    from expert_layer_dual_b200.configs import CONFIGS
    names = {n: bench.gateup_kernel(CONFIGS[n], CONFIGS[n].T, 148) for n in CONFIGS}
    assert names["decode"] == names["tiny"] == "k_gateup_bf16"
    assert names["prefill"] == names["skew"] == "k_gateup_bf16_2sm"
    assert names["fp8"] == "k_gateup_fp8" and names["mxfp8"] == "k_gateup_mx"
    assert names["fp8t"] == "k_gateup_f8t"
    assert set(names.values()) <= set(bench.KERNEL_SOURCES)


def test_launch_count_follows_the_library_dispatch():
    from expert_layer_dual_b200.configs import CONFIGS
    n = {k: bench.kernels_per_step(c, c.T) for k, c in CONFIGS.items()}
    # decode splits the router's K: router, top-k, the one-block permute (<= 1024
    # assignments), gate-up, down, combine
    assert n["decode"] == 6
    assert bench.router_ksplit(64, 4096, 256) == 8 and bench.router_ksplit(8192, 4096, 256) == 1
    # one CTA per router tile and E <= 64: the top-k runs inside the router kernel
    assert n["tiny"] == 5
    # 256 experts: router, top-k, the permute in three kernels (count, scan, scatter), the
    # copy of x into the permuted row order for the CTA-pair gate-up
    assert n["prefill"] == n["skew"] == 9
    # + the activation quantiser
    assert n["fp8"] == n["mxfp8"] == n["fp8t"] == 9
