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
