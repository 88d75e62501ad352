"""Host-side logic of bench.py (no GPU): the clock record it attaches to its line."""
import os
import sys
import threading

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import bench  # noqa: E402


def _sampler_with(samples, source="nvml"):
    c = bench.ClockSampler(0)
    c.source = source
    c._t = threading.Thread(target=lambda: None)
    c._t.start()
    c.samples = list(samples)
    return c


def test_clock_record_median_max_and_reasons():
    rec = _sampler_with([(1965.0, 1965.0, []), (1800.0, 1965.0, ["sw_power_cap"]),
                         (1900.0, 1965.0, [])]).stop()
    assert rec["sm_mhz"] == 1900.0 and rec["sm_max_mhz"] == 1965.0
    assert rec["reasons"] == ["sw_power_cap"] and rec["samples"] == 3


def test_clock_record_without_samples():
    rec = _sampler_with([]).stop()
    assert rec["sm_mhz"] is None and rec["samples"] == 0


def test_clock_reason_bits_are_the_nvml_ones():
    # clocks-event reason masks of NVML: power cap, hw slowdown, sw / hw thermal slowdown
    assert dict(bench.ClockSampler.REASONS) == {"sw_power_cap": 0x4, "hw_slowdown": 0x8,
                                                "sw_thermal_slowdown": 0x20,
                                                "hw_thermal_slowdown": 0x40}


# ---------------------------------------------------------------------------
# N > 1: each rank times its own layer; the job's time is the slowest rank's and
# its value counts every rank's work.  Two gloo ranks on the CPU.
# ---------------------------------------------------------------------------
def _two_rank_worker(rank, port, out_dir):
    import datetime

    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=2,
                            timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = 10.0 + 3.0 * rank           # rank 1 is the slower one
        ms = bench.max_over_ranks(local_ms, 2, "cpu")
        value = bench.weak_value(2, 1e12, ms)
        with open(os.path.join(out_dir, f"r{rank}.txt"), "w") as f:
            f.write(f"{ms} {value}")
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time_and_count_all_work(tmp_path):
    import socket

    import torch.multiprocessing as mp
    with socket.socket() as s_:
        s_.bind(("127.0.0.1", 0))
        port = s_.getsockname()[1]
    mp.start_processes(_two_rank_worker, args=(port, str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    for r in range(2):
        ms, value = map(float, open(tmp_path / f"r{r}.txt").read().split())
        assert ms == 13.0
        assert abs(value - 2 * 1e12 / 13e-3 / 1e12) < 1e-9


def test_one_rank_needs_no_process_group():
    assert bench.max_over_ranks(7.5, 1, "cpu") == 7.5
    assert bench.weak_value(1, 2e12, 4.0) == 2e12 / 4e-3 / 1e12


# ---------------------------------------------------------------------------
# N > 1 with --shard kv-heads: one layer's KV heads split over the ranks (the path's
# units are independent, so nothing is exchanged); the job's value counts one layer's
# FLOP over the slowest rank's time.  Two gloo ranks on the CPU.
# ---------------------------------------------------------------------------
def _shard_worker(rank, port, out_dir):
    import datetime

    import torch
    import torch.distributed as dist

    import workloads as W
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=2,
                            timeout=datetime.timedelta(seconds=60))
    try:
        wl = W.small_workload("gqa-32k", 256, 8, 4, head_dim=32, page_size=32, q_block=64,
                              shuffle_pages=True)
        x = W.make_inputs(wl, seed=0)        # every rank draws the same layer
        h0, h1 = bench.kv_head_shard(rank, 2, wl.num_kv_heads)
        xs = bench.shard_inputs(x, wl.num_q_heads, wl.num_kv_heads, h0, h1)
        ranges = [None, None]
        dist.all_gather_object(ranges, (h0, h1))
        parts = {k: [torch.empty_like(xs[k]) for _ in range(2)] for k in ("q", "k_pool", "v_pool")}
        for k in parts:
            dist.all_gather(parts[k], xs[k])
        whole = all(torch.equal(torch.cat(parts["q"], 1), x["q"]) for _ in [0]) and \
            torch.equal(torch.cat(parts["k_pool"], 1), x["k_pool"]) and \
            torch.equal(torch.cat(parts["v_pool"], 1), x["v_pool"]) and \
            torch.equal(xs["page_table"], x["page_table"])
        local_ms = 10.0 + 3.0 * rank
        ms = bench.max_over_ranks(local_ms, 2, "cpu")
        value = bench.strong_value(wl.dense_flops(), ms)
        with open(os.path.join(out_dir, f"s{rank}.txt"), "w") as f:
            f.write(f"{ranges} {int(whole)} {ms} {value} {wl.dense_flops()}")
    finally:
        dist.destroy_process_group()


def test_two_ranks_split_one_layer_by_kv_heads(tmp_path):
    import ast
    import socket

    import torch.multiprocessing as mp
    with socket.socket() as s_:
        s_.bind(("127.0.0.1", 0))
        port = s_.getsockname()[1]
    mp.start_processes(_shard_worker, args=(port, str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    for r in range(2):
        txt = open(tmp_path / f"s{r}.txt").read()
        ranges = ast.literal_eval(txt[:txt.index("]") + 1])
        whole, ms, value, flop = txt[txt.index("]") + 2:].split()
        heads = [h for a, b in ranges for h in range(a, b)]
        assert sorted(heads) == list(range(4)) and len(heads) == 4  # every KV head once
        assert int(whole) == 1              # the shards put together are the layer
        assert float(ms) == 13.0
        # strong scaling: one layer's FLOP over the slowest rank's time, not two layers'
        assert abs(float(value) - float(flop) / 13e-3 / 1e12) < 1e-9


def test_kv_head_shard_edges():
    assert bench.kv_head_shard(0, 1, 8) == (0, 8)
    assert [bench.kv_head_shard(r, 8, 8) for r in range(8)] == [(r, r + 1) for r in range(8)]
    import pytest
    with pytest.raises(ValueError):
        bench.kv_head_shard(0, 3, 8)


def test_kap_pool_bytes_closed_form():
    # 128K layer, 32 / 8 heads: Q 1.074 GB + K 0.268 GB read, pooled vectors written as
    # two fp32 terms: 8 * 128 * (32 * 4096 + 8 * 8192) bytes
    b = bench.kap_pool_bytes(1, 32, 8, 131072, 128, 32, 16)
    assert b == 2 * 131072 * 128 * 40 + 8 * 128 * (32 * 4096 + 8 * 8192)
