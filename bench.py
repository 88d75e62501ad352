#!/usr/bin/env python
"""Benchmark: CoSA causal prefill attention (KAP select + OSK attention) on the
128K long-context GQA layer (B1, 32 q-heads / 8 KV heads, N=131072, D=128,
64-token pages through a shuffled page table, q-block 128), synthetic seeded
inputs resident in HBM.

One step = one pass of the whole sparse path over one layer: cosa_kap_select
(pool, score, MaxPool, MaxNorm, HRM, select, order) then cosa_osk_attention.
Metric: effective TFLOP/s = dense-equivalent causal FLOP 4*B*H_q*D*N(N+1)/2
divided by the step time (plus the step time in ms).  The own dense kernel is
timed beside it on the same inputs.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl cosa|reference]

Multi-GPU (torchrun): every rank runs its own independent layer (weak
scaling; the path needs no data exchange), timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "128K causal prefill attention ms & effective TFLOP/s; % of bf16 tensor peak"
WORKLOAD = "gqa-128k"


# DRAM traffic (read + write) of one OSK launch at gqa-128k, from one ncu capture
# (profiles/osk_attention_gqa-128k_traffic.md).  It describes the kernel source the
# capture ran, identified by the hash below; any other source reports null.
OSK_TRAFFIC = {"workload": "gqa-128k", "bytes": 2695605504, "source_sha256_16": "37ec78a68845158c"}


def _osk_traffic(workload: str):
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(os.path.dirname(os.path.abspath(__file__)), "block_sparse_long_kap_b200",
                        "csrc")
    for f in ("attn_tc.cuh", "tc_ptx.cuh", "common.cuh"):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    if workload != OSK_TRAFFIC["workload"] or h.hexdigest()[:16] != OSK_TRAFFIC["source_sha256_16"]:
        return None
    return OSK_TRAFFIC["bytes"]


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p, "measured"
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "sm_max_mhz": 1965.0}, "fallback"


class ClockSampler:
    """SM clocks and clock-event (throttle) reasons of this process's GPU, sampled every
    10 ms during the timed region through NVML (read-only queries), nvidia-smi if NVML
    cannot be used."""
    REASONS = (("hw_slowdown", 0x8), ("sw_thermal_slowdown", 0x20), ("hw_thermal_slowdown", 0x40),
               ("sw_power_cap", 0x4))
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, torch_device: int):
        self.dev = torch_device
        self.samples = []       # (sm MHz, max MHz, reason names)
        self.proc = None
        self.lines = []
        self._stop = threading.Event()
        self._t = None
        self.source = None

    def _nvml_handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        props = torch.cuda.get_device_properties(self.dev)
        try:
            return pynvml, pynvml.nvmlDeviceGetHandleByUUID("GPU-" + str(props.uuid))
        except Exception:
            bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus)

    def start(self):
        try:
            nv, h = self._nvml_handle()
            mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)

            def poll():
                while not self._stop.is_set():
                    try:
                        sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                        bits = nv.nvmlDeviceGetCurrentClocksThrottleReasons(h)
                        self.samples.append((float(sm), float(mx),
                                             [n for n, b in self.REASONS if bits & b]))
                    except Exception:
                        pass
                    self._stop.wait(0.01)
            self._t = threading.Thread(target=poll, daemon=True)
            self._t.start()
            self.source = "nvml"
            return
        except Exception:
            pass
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
            self.source = "nvidia-smi"
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.source == "nvml":
            self._stop.set()
            self._t.join(timeout=1)
        elif self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
            for ln in self.lines:
                parts = [p.strip() for p in ln.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm, mx = float(parts[1]), float(parts[2])
                except ValueError:
                    continue
                self.samples.append((sm, mx, [n for n, v in zip(names, parts[5:9])
                                              if v.lower().startswith("active")]))
        else:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["clock query unavailable"],
                    "samples": 0}
        sm = [x[0] for x in self.samples]
        reasons = sorted({r for x in self.samples for r in x[2]})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": self.samples[-1][1] if self.samples else None,
                "reasons": reasons, "samples": len(sm), "source": self.source}


def max_over_ranks(v: float, world: int, device) -> float:
    """The largest of the ranks' values (every rank gets it); each rank times its
    own shard, and the job takes as long as the slowest."""
    if world <= 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_value(world: int, flop_per_rank: float, ms: float) -> float:
    """Whole-job TFLOP/s when every rank runs its own layer (weak scaling): all
    ranks' work over the slowest rank's time."""
    return world * flop_per_rank / (ms * 1e-3) / 1e12


def _cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def oracle_sample(wl, x_host, budget, eps, q_heads=(0,), qblocks=None, time_budget_s=20.0):
    """Time the CPU oracle (KAP + OSK) on a bounded sample of the workload:
    the given q-heads x evenly spaced q-blocks, added until time_budget_s.
    Returns (seconds, dense-equivalent FLOP of the sampled rows, description)."""
    import numpy as np
    import oracle as O
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        threads = 1
    nQB = wl.num_q_blocks
    if qblocks is None:
        qblocks = [int(v) for v in np.linspace(nQB - 1, 0, 16)]
    scale = 1.0 / math.sqrt(wl.head_dim)
    G = wl.num_q_heads // wl.num_kv_heads
    pt = x_host["page_table"].numpy()
    t0 = time.perf_counter()
    flops = 0.0
    done = []
    cache = {}
    for h in q_heads:
        hk = h // G
        if hk not in cache:
            kp = x_host["k_pool"][:, hk].float().numpy().astype(np.float64)[:, None]
            vp = x_host["v_pool"][:, hk].float().numpy().astype(np.float64)[:, None]
            k_log = O.gather_logical(kp, pt, 0, 0)
            v_log = O.gather_logical(vp, pt, 0, 0)
            khat = O.kap_pool_keys(k_log, wl.page_size, 16)
            cache[hk] = (k_log, v_log, khat)
        k_log, v_log, khat = cache[hk]
        q_bh = x_host["q"][0, h].float().numpy().astype(np.float64)
        for qb in qblocks:
            order, _, _, _ = O.kap_select_block(q_bh, None, qb, q_block=wl.q_block,
                                                page_size=wl.page_size, q_sub=wl.q_block // 4,
                                                k_sub=16, scale=scale, budget=budget,
                                                sink_pages=1, khat=khat)
            rows = slice(qb * wl.q_block, (qb + 1) * wl.q_block)
            O.osk_block(q_bh[rows], k_log, v_log, qb, wl.q_block, wl.page_size, order, eps, scale)
            r0 = qb * wl.q_block
            n_keys = sum(r0 + i + 1 for i in range(wl.q_block))
            flops += 4.0 * wl.head_dim * n_keys
            done.append((h, qb))
            if time.perf_counter() - t0 > time_budget_s:
                break
    secs = time.perf_counter() - t0
    desc = (f"{len(done)} (q-head, q-block) tiles of {wl.name} (q-heads {sorted(set(h for h, _ in done))}, "
            f"q-blocks evenly spaced from the last); KAP + OSK per tile, pooled keys of the "
            f"KV head included; dense-equivalent FLOP of the sampled rows / wall time")
    return secs, flops, desc, threads


def run_reference(args):
    """The reference arm: the CPU oracle as it stands, on the host cores."""
    import torch
    import workloads as W
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    wl = W.WORKLOADS[args.workload]
    x = W.make_inputs(wl, seed=0, device="cpu")
    budget, eps = args.budget, args.eps
    cores = _cpu_cores()
    per_step = max(2.0, min(20.0, 150.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_sample(wl, x, budget, eps, qblocks=[wl.num_q_blocks - 1], time_budget_s=per_step)
    tot_s = tot_f = 0.0
    desc = threads = None
    for _ in range(args.steps):
        s, f, desc, threads = oracle_sample(wl, x, budget, eps, time_budget_s=per_step)
        tot_s += s
        tot_f += f
    value = tot_f / tot_s / 1e12
    full_ms = wl.dense_flops() / (value * 1e12) * 1e3
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": full_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": _config(wl, budget, eps),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads or cores,
                         "kind": "oracle", "sample": desc + " (ms_per_step extrapolated to the full layer)"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def _config(wl, budget, eps):
    return {"workload": wl.name, "batch": wl.batch, "num_q_heads": wl.num_q_heads,
            "num_kv_heads": wl.num_kv_heads, "seq_len": wl.seq_len, "head_dim": wl.head_dim,
            "page_size": wl.page_size, "q_block": wl.q_block, "page_table": "shuffled",
            "budget": budget, "eps": eps, "q_sub": wl.q_block // 4, "k_sub": 16, "sink_pages": 1,
            "l2": "inputs larger than L2 (Q 1 GiB + K/V 0.5 GiB read per step)",
            "parallelism": "independent layer per GPU"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="cosa", choices=["cosa", "reference"])
    ap.add_argument("--workload", default=WORKLOAD)
    ap.add_argument("--budget", type=float, default=0.2)
    ap.add_argument("--eps", type=float, default=1e-4)
    ap.add_argument("--no-extras", action="store_true", help="skip dense/sweep/e2e/cpu legs")
    ap.add_argument("--dense-only", action="store_true",
                    help="time only the dense kernel on the workload (for profiling it)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)

    import numpy as np
    import torch
    import torch.distributed as dist

    import block_sparse_long_kap_b200 as C
    import workloads as W

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    wl = W.WORKLOADS[args.workload]
    x = W.make_inputs(wl, seed=rank, device=str(dev))
    shape = C.Shape(wl.batch, wl.num_q_heads, wl.num_kv_heads, wl.seq_len, wl.head_dim,
                    wl.page_size, wl.q_block)
    kap = C.KapParams(budget=args.budget, q_sub=wl.q_block // 4, k_sub=16, sink_pages=1)
    osk = C.OskParams(eps=args.eps)
    B, Hq, N, D = wl.batch, wl.num_q_heads, wl.seq_len, wl.head_dim
    kc = C.cosa_kap_kcap(shape, kap)
    order = torch.empty(B, Hq, shape.num_q_blocks, kc, dtype=torch.int32, device=dev)
    count = torch.empty(B, Hq, shape.num_q_blocks, dtype=torch.int32, device=dev)
    ws = torch.empty(C.cosa_kap_workspace_size(shape, kap), dtype=torch.uint8, device=dev)
    out = torch.empty(B, Hq, N, D, dtype=torch.bfloat16, device=dev)
    computed = torch.empty(B, Hq, shape.num_q_blocks, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        C.cosa_kap_select(shape, kap, x["q"], x["k_pool"], x["page_table"], order, count, ws,
                          stream=stream)
        if ev is not None:
            ev[1].record(stream)
        C.cosa_osk_attention(shape, osk, x["q"], x["k_pool"], x["v_pool"], x["page_table"], order,
                             count, out, computed=computed, stream=stream)
        if ev is not None:
            ev[2].record(stream)

    def barrier():
        if world > 1:
            dist.barrier()


    if args.dense_only:
        dense_flop = 4.0 * B * Hq * D * N * (N + 1) / 2
        for _ in range(args.warmup):
            C.cosa_dense_attention(shape, x["q"], x["k_pool"], x["v_pool"], x["page_table"], out,
                                   stream=stream)
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            C.cosa_dense_attention(shape, x["q"], x["k_pool"], x["v_pool"], x["page_table"], out,
                                   stream=stream)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        assert C.cosa_get_status(stream) == 0
        ms = e0.elapsed_time(e1) / max(args.steps, 1)
        if rank == 0:
            print(json.dumps({"kernel": "dense_attention", "workload": args.workload, "ms": ms,
                              "tflops": dense_flop / (ms * 1e-3) / 1e12, "steps": args.steps,
                              "warmup": args.warmup}), flush=True)
        if world > 1:
            dist.destroy_process_group()
        return 0

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    assert C.cosa_get_status(stream) == 0

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    clocks = ClockSampler(torch.cuda.current_device())
    barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    clk = clocks.stop()
    total_ms = max_over_ranks(t_start.elapsed_time(t_end), world, dev)
    kap_ms = [e[0].elapsed_time(e[1]) for e in evs]
    osk_ms = [e[1].elapsed_time(e[2]) for e in evs]
    assert C.cosa_get_status(stream) == 0

    ms_per_step = total_ms / args.steps
    dense_flop = wl.dense_flops()
    value = weak_value(world, dense_flop, ms_per_step)

    # algorithmic work of the dominant kernel (OSK) for the roofline
    cnt = count.to(torch.int64)
    steps_visited = int(cnt.sum().item())
    steps_computed = int(computed.to(torch.int64).sum().item())
    tile = 2.0 * wl.q_block * wl.page_size * wl.head_dim
    osk_flop = tile * (steps_visited + steps_computed)
    osk_avg_ms = statistics.mean(osk_ms)
    peaks, peak_src = _peaks()
    burst = float(peaks.get("bf16_tflops", 1590.0))
    sustained = float(peaks.get("bf16_tflops_sustained", burst))
    # the burst figure unless the clocks seen in the timed region sat well below max
    # (the sustained figure is a seconds-long GEMM under the power cap, at ~1.35 GHz)
    throttled = (clk.get("sm_mhz") is not None and clk.get("sm_max_mhz")
                 and clk["sm_mhz"] < 0.9 * clk["sm_max_mhz"])
    peak_tflops = sustained if throttled else burst
    peak_kind = "sustained (SM clock under 90 % of max in the timed region)" if throttled else \
        "burst (SM clock at max in the timed region)"
    achieved = osk_flop / (osk_avg_ms * 1e-3) / 1e12
    n_b_total = sum(((qb + 1) * wl.q_block + wl.page_size - 1) // wl.page_size
                    for qb in range(shape.num_q_blocks)) * B * Hq

    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": _config(wl, args.budget, args.eps),
        "gpu_launches": 4 * args.steps,
        "clocks": clk,
        "roofline": {"kernel": "osk_attention", "bound": "tensor", "achieved": achieved,
                     "peak": peak_tflops, "unit": "TFLOP/s", "frac": achieved / peak_tflops,
                     "peak_source": f"{peak_src} bf16 {peak_kind}",
                     "frac_vs_burst": achieved / burst, "frac_vs_sustained": achieved / sustained,
                     "traffic": _osk_traffic(args.workload),
                     "traffic_unit": "bytes per launch (DRAM read + write, ncu)",
                     "work": "visited FLOP = 2*Bq*P*D*(visited pages + computed pages) per launch"},
        "breakdown_ms": {"kap_select": statistics.mean(kap_ms), "osk_attention": osk_avg_ms},
        "budgets": {"kap_kept_frac": steps_visited / n_b_total,
                    "osk_computed_frac": steps_computed / n_b_total},
    }
    # ---- end to end through the C-ABI with host buffers (every rank, every N) ---
    def e2e_leg():
        # through the library's host-buffer entry point: every step copies its inputs in
        # from page-locked host memory and its output back, one KV head at a time, the
        # copies overlapping the kernels
        qh = x["q"].cpu().pin_memory()
        kh = x["k_pool"].cpu().pin_memory()
        vh = x["v_pool"].cpu().pin_memory()
        pth = x["page_table"].cpu().pin_memory()
        outh = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        wsh = torch.empty(C.cosa_attention_host_workspace_size(shape, kap), dtype=torch.uint8,
                          device=dev)
        e2e_steps = max(1, min(args.steps, 3))

        def e2e_step():
            C.cosa_attention_host(shape, kap, osk, qh, kh, vh, pth, outh, wsh, stream=stream)

        e2e_step()
        torch.cuda.synchronize(dev)
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, world, dev)
        h2d = sum(t.numel() * t.element_size() for t in (qh, kh, vh, pth))
        d2h = outh.numel() * outh.element_size()
        return {"value": weak_value(world, dense_flop, e2e_ms), "unit": "TFLOP/s",
                "ms_per_step": e2e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}

    if world > 1:
        line["e2e"] = e2e_leg()
    if args.no_extras or world > 1:
        if rank == 0:
            print(json.dumps(line), flush=True)
        if world > 1:
            dist.destroy_process_group()
        return 0

    # ---- own dense kernel on the same inputs -------------------------------
    dense_out = torch.empty_like(out)
    for _ in range(2):
        C.cosa_dense_attention(shape, x["q"], x["k_pool"], x["v_pool"], x["page_table"], dense_out,
                               stream=stream)
    torch.cuda.synchronize(dev)
    d_ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    d_ev[0].record(stream)
    for _ in range(3):
        C.cosa_dense_attention(shape, x["q"], x["k_pool"], x["v_pool"], x["page_table"], dense_out,
                               stream=stream)
    d_ev[1].record(stream)
    torch.cuda.synchronize(dev)
    dense_ms = d_ev[0].elapsed_time(d_ev[1]) / 3
    dense_tf = dense_flop / (dense_ms * 1e-3) / 1e12
    line["dense"] = {"ms": dense_ms, "tflops": dense_tf, "frac_vs_burst": dense_tf / burst,
                     "frac_vs_sustained": dense_tf / sustained,
                     "speedup_sparse_vs_dense": dense_ms / ms_per_step}

    # ---- eps sweep at this budget (OSK only, KAP list reused) --------------
    sweep = []
    for eps in wl.eps_list:
        o2 = C.OskParams(eps=eps)
        C.cosa_osk_attention(shape, o2, x["q"], x["k_pool"], x["v_pool"], x["page_table"], order,
                             count, out, computed=computed, stream=stream)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(3):
            C.cosa_osk_attention(shape, o2, x["q"], x["k_pool"], x["v_pool"], x["page_table"],
                                 order, count, out, computed=computed, stream=stream)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ms = e0.elapsed_time(e1) / 3
        comp = int(computed.to(torch.int64).sum().item())
        fl = tile * (steps_visited + comp)
        sweep.append({"eps": eps, "osk_ms": ms, "kap_plus_osk_ms": ms + statistics.mean(kap_ms),
                      "computed_frac": comp / n_b_total, "visited_tflops": fl / (ms * 1e-3) / 1e12,
                      "speedup_vs_dense": dense_ms / (ms + statistics.mean(kap_ms))})
    line["eps_sweep"] = sweep

    # ---- group-shared selection: one list per KV head and q-block (KAP group +
    # OSK over head pairs), same budget and eps; quality against the dense output
    Hk = wl.num_kv_heads
    og = torch.empty(B, Hk, shape.num_q_blocks, kc, dtype=torch.int32, device=dev)
    cg = torch.empty(B, Hk, shape.num_q_blocks, dtype=torch.int32, device=dev)
    outg = torch.empty_like(out)
    compg = torch.empty_like(computed)

    def gstep(ev=None):
        if ev is not None:
            ev[0].record(stream)
        C.cosa_kap_select_group(shape, kap, x["q"], x["k_pool"], x["page_table"], og, cg, ws,
                                stream=stream)
        if ev is not None:
            ev[1].record(stream)
        C.cosa_osk_attention_group(shape, osk, x["q"], x["k_pool"], x["v_pool"], x["page_table"],
                                   og, cg, outg, computed=compg, stream=stream)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(args.warmup):
        gstep()
    torch.cuda.synchronize(dev)
    gevs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    for i in range(args.steps):
        gstep(gevs[i])
    torch.cuda.synchronize(dev)
    assert C.cosa_get_status(stream) == 0
    g_kap = statistics.mean(e[0].elapsed_time(e[1]) for e in gevs)
    g_osk = statistics.mean(e[1].elapsed_time(e[2]) for e in gevs)
    g_ms = g_kap + g_osk
    # the per-head output at this eps, for the same quality measure
    C.cosa_osk_attention(shape, osk, x["q"], x["k_pool"], x["v_pool"], x["page_table"], order,
                         count, out, computed=computed, stream=stream)
    torch.cuda.synchronize(dev)
    dref = dense_out.float()

    def rel_l2(a):
        return float((a.float() - dref).norm() / dref.norm())

    G_ = Hq // Hk
    vis_g = G_ * int(cg.to(torch.int64).sum().item())
    comp_g = int(compg.to(torch.int64).sum().item())
    vis_tf = tile * (vis_g + comp_g) / (g_osk * 1e-3) / 1e12
    line["group_shared"] = {
        "kap_ms": g_kap, "osk_ms": g_osk, "ms": g_ms, "tflops": dense_flop / (g_ms * 1e-3) / 1e12,
        "speedup_vs_dense": dense_ms / g_ms, "speedup_vs_per_head": ms_per_step / g_ms,
        "visited_tflops": vis_tf, "visited_frac_vs_burst": vis_tf / burst,
        "kap_kept_frac": vis_g / n_b_total, "osk_computed_frac": comp_g / n_b_total,
        "rel_l2_vs_dense": rel_l2(outg), "per_head_rel_l2_vs_dense": rel_l2(out)}

    # ---- early break (max_run: not part of the pages' method): OSK only, the lists
    # reused; output against the pages' rule at this eps (in `out`) and against dense
    def early_break_leg():
        bout = torch.empty_like(out)
        bcomp = torch.empty_like(computed)
        pref = out.float()
        k_ms = statistics.mean(kap_ms)
        res = []
        for r in (16, 8):
            o3 = C.OskParams(eps=args.eps, max_run=r)

            def run():
                C.cosa_osk_attention(shape, o3, x["q"], x["k_pool"], x["v_pool"], x["page_table"],
                                     order, count, bout, computed=bcomp, stream=stream)

            run()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(3):
                run()
            e1.record(stream)
            torch.cuda.synchronize(dev)
            if C.cosa_get_status(stream) != 0:
                raise RuntimeError("in-kernel error status")
            ms = e0.elapsed_time(e1) / 3
            comp = int(bcomp.to(torch.int64).sum().item())
            res.append({"max_run": r, "eps": args.eps, "osk_ms": ms, "kap_plus_osk_ms": ms + k_ms,
                        "tflops": dense_flop / ((ms + k_ms) * 1e-3) / 1e12,
                        "speedup_vs_dense": dense_ms / (ms + k_ms),
                        "computed_frac": comp / n_b_total,
                        "rel_l2_vs_pages_rule": float((bout.float() - pref).norm() / pref.norm()),
                        "rel_l2_vs_dense": rel_l2(bout)})
        return res

    try:
        line["early_break"] = early_break_leg()
    except Exception as exc:  # an extra leg: report the failure, keep the line
        line["early_break"] = {"error": repr(exc)}

    line["e2e"] = e2e_leg()

    # ---- CPU oracle on a bounded sample of the same workload ----------------
    xh = {"q": x["q"][:, :1].cpu(), "k_pool": x["k_pool"][:, :1].cpu(),
          "v_pool": x["v_pool"][:, :1].cpu(), "page_table": x["page_table"].cpu()}
    secs, fl, desc, threads = oracle_sample(wl, xh, args.budget, args.eps, time_budget_s=15.0)
    line["cpu_baseline"] = {"value": fl / secs / 1e12, "unit": "TFLOP/s", "cores": threads,
                            "host_cores": _cpu_cores(), "kind": "oracle", "sample": desc,
                            "extrapolated_full_layer_s": dense_flop / (fl / secs)}
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
