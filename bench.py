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


# DRAM traffic (read + write) of one launch at gqa-128k, from the ncu traffic captures
# of these kernels.  Each figure describes the kernel source the capture ran,
# identified by a hash of the files below; any other source reports null.
TRAFFIC = {
    "osk": {"workload": "gqa-128k", "bytes": 1652753920 + 1035382784,
            "source_sha256_16": "58ec01c35dcc6e5a",
            "files": ("attn_tc.cuh", "tc_ptx.cuh", "common.cuh")},
    "kap_pool": {"workload": "gqa-128k", "bytes": 1342215168 + 184500224,
                 "source_sha256_16": "db13d4d202b518c7",
                 "files": ("kap.cuh", "common.cuh")},
}


def source_hash(files) -> str:
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(os.path.dirname(os.path.abspath(__file__)), "block_sparse_long_kap_b200",
                        "csrc")
    for f in files:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def _traffic(kernel: str, workload: str):
    t = TRAFFIC[kernel]
    if t["bytes"] is None or workload != t["workload"] or \
            source_hash(t["files"]) != t["source_sha256_16"]:
        return None
    return t["bytes"]


def _osk_traffic(workload: str):
    return _traffic("osk", workload)


def _pool_traffic(workload: str):
    return _traffic("kap_pool", workload)


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
            import torch
            # by UUID: under CUDA_VISIBLE_DEVICES the torch ordinal can name another GPU
            gid = "GPU-" + str(torch.cuda.get_device_properties(self.dev).uuid)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={gid}", f"--query-gpu={self.FIELDS}",
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
        "ms_per_step": full_ms, "higher_is_better": True,
        "scaling": "strong" if args.shard == "kv-heads" else "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": _config(wl, budget, eps, args.shard, args.gpus),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads or cores,
                         "kind": "oracle", "sample": desc + " (ms_per_step extrapolated to the full layer)"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def kv_head_shard(rank: int, world: int, num_kv_heads: int):
    """KV heads [h0, h1) of this rank when one layer's KV heads are split evenly over
    the ranks.  Heads are independent in both stages (per-head pooling, scoring,
    lists and attention), so each rank runs its heads' Q and KV pages alone and the
    outputs stay head-sharded, as in tensor-parallel attention: no data exchange."""
    if world < 1 or num_kv_heads % world:
        raise ValueError(f"{num_kv_heads} KV heads do not split evenly over {world} ranks")
    n = num_kv_heads // world
    return rank * n, (rank + 1) * n


def shard_inputs(x: dict, num_q_heads: int, num_kv_heads: int, h0: int, h1: int) -> dict:
    """The inputs of KV heads [h0, h1): their G query heads of Q and their column of
    the K and V page pools (contiguous copies); the page table is shared."""
    G = num_q_heads // num_kv_heads
    return {"q": x["q"][:, h0 * G:h1 * G].contiguous(),
            "k_pool": x["k_pool"][:, h0:h1].contiguous(),
            "v_pool": x["v_pool"][:, h0:h1].contiguous(),
            "page_table": x["page_table"]}


def strong_value(flop_job: float, ms: float) -> float:
    """Whole-job TFLOP/s when the ranks split one job: its FLOP over the slowest
    rank's time."""
    return flop_job / (ms * 1e-3) / 1e12


def kap_pool_bytes(batch, num_q_heads, num_kv_heads, seq_len, head_dim, q_sub, k_sub) -> float:
    """Algorithmic DRAM bytes of one KAP pooling launch: Q and K read once (bf16), the
    pooled vectors written once as two fp32 TF32 terms."""
    read = 2.0 * batch * seq_len * head_dim * (num_q_heads + num_kv_heads)
    write = 2 * 4.0 * head_dim * batch * (num_q_heads * seq_len / q_sub + num_kv_heads * seq_len / k_sub)
    return read + write


def _config(wl, budget, eps, shard, world):
    par = ("kv-head shards: one layer's KV heads split evenly over the GPUs, outputs "
           "head-sharded, no data exchange" if shard == "kv-heads"
           else "independent layer per GPU")
    return {"workload": wl.name, "batch": wl.batch, "num_q_heads": wl.num_q_heads,
            "num_kv_heads": wl.num_kv_heads, "seq_len": wl.seq_len, "head_dim": wl.head_dim,
            "page_size": wl.page_size, "q_block": wl.q_block,
            "page_table": "shuffled" if wl.shuffle_pages else "identity",
            "budget": budget, "eps": eps, "q_sub": wl.q_block // 4, "k_sub": 16, "sink_pages": 1,
            "l2": "inputs larger than L2 (Q 1 GiB + K/V 0.5 GiB read per step)",
            "parallelism": f"{par} ({world} GPU{'s' if world > 1 else ''})"}


def _timed(fn, reps, stream, warm=1):
    """Mean CUDA-event time (ms) of fn() over reps calls on stream, after warm calls."""
    import torch
    for _ in range(warm):
        fn()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        fn()
    e1.record(stream)
    e1.synchronize()
    return e0.elapsed_time(e1) / reps


# Per-budget sweep (the speedup over the own dense kernel at each budget, and the ordered
# against the page-order visit): workload -> (budgets, eps values, visit orders)
SWEEP = (
    ("wide-head-128k", (0.05, 0.10, 0.15, 0.20, 0.25, 0.30, 0.40, 0.50), (1e-4, 0.0), (False,)),
    ("narrow-kv-64k", (0.05, 0.10, 0.20), (1e-4,), (False, True)),
    ("gqa-32k", (0.10, 0.25, 0.50), (1e-4, 0.0), (False,)),
)


def budget_sweep(C, W, dev, stream, burst, reps=3):
    """KAP + OSK at every budget / eps / visit order of SWEEP on each workload's seeded
    inputs, against the own dense kernel on the same inputs: ms, speedup, the pages kept
    and computed as fractions of the causal pages, visited TFLOP/s and the output's
    relative L2 distance from the dense output."""
    import torch
    res = {}
    for name, budgets, eps_list, modes in SWEEP:
        wl = W.WORKLOADS[name]
        x = W.make_inputs(wl, seed=0, device=str(dev))
        B, Hq, N, D = wl.batch, wl.num_q_heads, wl.seq_len, wl.head_dim
        shape = C.Shape(B, Hq, wl.num_kv_heads, N, D, wl.page_size, wl.q_block)
        dense_out = torch.empty(B, Hq, N, D, dtype=torch.bfloat16, device=dev)
        dense_ms = _timed(lambda: C.cosa_dense_attention(shape, x["q"], x["k_pool"], x["v_pool"],
                                                         x["page_table"], dense_out,
                                                         stream=stream), reps, stream)
        dref = dense_out.float()
        dnorm = float(dref.norm())
        out = torch.empty_like(dense_out)
        comp = torch.empty(B, Hq, shape.num_q_blocks, dtype=torch.int32, device=dev)
        n_b_total = sum(((qb + 1) * wl.q_block + wl.page_size - 1) // wl.page_size
                        for qb in range(shape.num_q_blocks)) * B * Hq
        tile = 2.0 * wl.q_block * wl.page_size * D
        pts = []
        for asc in modes:
            for budget in budgets:
                kap = C.KapParams(budget=budget, q_sub=wl.q_block // 4, k_sub=16, sink_pages=1,
                                  ascending=asc)
                kc = C.cosa_kap_kcap(shape, kap)
                order = torch.empty(B, Hq, shape.num_q_blocks, kc, dtype=torch.int32, device=dev)
                count = torch.empty(B, Hq, shape.num_q_blocks, dtype=torch.int32, device=dev)
                ws = torch.empty(C.cosa_kap_workspace_size(shape, kap), dtype=torch.uint8,
                                 device=dev)
                kap_ms = _timed(lambda: C.cosa_kap_select(shape, kap, x["q"], x["k_pool"],
                                                          x["page_table"], order, count, ws,
                                                          stream=stream), reps, stream)
                listed = int(count.to(torch.int64).sum().item())
                for eps in eps_list:
                    osk = C.OskParams(eps=eps)
                    osk_ms = _timed(lambda: C.cosa_osk_attention(
                        shape, osk, x["q"], x["k_pool"], x["v_pool"], x["page_table"], order,
                        count, out, computed=comp, stream=stream), reps, stream)
                    if C.cosa_get_status(stream) != 0:
                        raise RuntimeError(f"in-kernel error status in the sweep ({name})")
                    cmp_ = int(comp.to(torch.int64).sum().item())
                    vis_tf = tile * (listed + cmp_) / (osk_ms * 1e-3) / 1e12
                    pts.append({
                        "budget": budget, "eps": eps, "visit": "page order" if asc else "ordered",
                        "kap_ms": kap_ms, "osk_ms": osk_ms, "ms": kap_ms + osk_ms,
                        "speedup_vs_dense": dense_ms / (kap_ms + osk_ms),
                        "kept_frac": listed / n_b_total, "computed_frac": cmp_ / n_b_total,
                        "visited_tflops": vis_tf, "visited_frac_vs_burst": vis_tf / burst,
                        "effective_tflops": wl.dense_flops() / ((kap_ms + osk_ms) * 1e-3) / 1e12,
                        "rel_l2_vs_dense": float((out.float() - dref).norm()) / dnorm})
                del order, count, ws
        res[name] = {"dense_ms": dense_ms,
                     "dense_tflops": wl.dense_flops() / (dense_ms * 1e-3) / 1e12,
                     "points": pts}
        del x, dense_out, out, dref
        torch.cuda.empty_cache()
    return res


def decode_leg(C, torch, x, shape, wl, order, count, dev, stream, eps_run, hbm, reps=20):
    """Decode (the pages' future work): the last token of every head with the list KAP
    wrote for its q-block, against the same kernel visiting every page."""
    B, Hq, N, D = shape.batch, shape.num_q_heads, shape.seq_len, shape.head_dim
    t = N - 1
    P_ = wl.page_size
    qdec = x["q"][:, :, t].contiguous()
    pos = torch.full((B,), t, dtype=torch.int32, device=dev)
    o_dec, c_dec = order[:, :, -1].contiguous(), count[:, :, -1].contiguous()
    n_all = t // P_ + 1
    o_full = torch.full((B, Hq, wl.num_pages), -1, dtype=torch.int32, device=dev)
    o_full[:, :, :n_all] = torch.arange(n_all, dtype=torch.int32, device=dev)
    c_full = torch.full((B, Hq), n_all, dtype=torch.int32, device=dev)
    outd = torch.empty(B, Hq, D, dtype=torch.bfloat16, device=dev)
    compd = torch.empty(B, Hq, dtype=torch.int32, device=dev)
    wsd = torch.empty(C.cosa_osk_decode_workspace_size(shape, wl.num_pages), dtype=torch.uint8,
                      device=dev)
    page_bytes = P_ * D * 2
    res = []
    for label, o, c, eps in (("KAP list", o_dec, c_dec, eps_run), ("KAP list", o_dec, c_dec, 0.0),
                             ("every page", o_full, c_full, 0.0)):
        od = C.OskParams(eps=eps)
        ms = _timed(lambda: C.cosa_osk_decode(shape, od, qdec, x["k_pool"], x["v_pool"],
                                              x["page_table"], pos, o, c, outd, wsd,
                                              computed=compd, stream=stream), reps, stream, warm=3)
        if C.cosa_get_status(stream) != 0:
            raise RuntimeError("in-kernel error status in decode")
        listed = int(c.to(torch.int64).sum().item())
        kept = int(compd.to(torch.int64).sum().item())
        byts = (listed + kept) * page_bytes  # K of every listed page, V of every kept one
        res.append({"list": label, "eps": eps, "us": ms * 1e3, "listed_pages": listed,
                    "computed_pages": kept, "bytes": byts,
                    "gbs": byts / (ms * 1e-3) / 1e9, "frac_vs_hbm": byts / (ms * 1e-3) / 1e9 / hbm})
    for r in res:
        r["speedup_vs_every_page"] = res[-1]["us"] / r["us"]
    return {"position": t, "heads": B * Hq, "points": res,
            "note": "bytes: K of the listed pages + V of the kept pages, read by each head "
                    "(the G heads of a KV head share pages through L2)"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="cosa", choices=["cosa", "reference"])
    ap.add_argument("--workload", default=WORKLOAD)
    ap.add_argument("--budget", type=float, default=0.2)
    ap.add_argument("--eps", type=float, default=1e-4)
    ap.add_argument("--shard", default="kv-heads", choices=["kv-heads", "replica"],
                    help="N > 1: split one layer's KV heads over the GPUs (strong scaling), "
                         "or run an independent layer on each (weak scaling)")
    ap.add_argument("--kv-heads", type=int, default=0,
                    help="run only the first K KV heads of the layer (a smaller case of the "
                         "same layer, for profiling; one GPU)")
    ap.add_argument("--no-extras", action="store_true", help="skip dense/sweep/e2e/cpu legs")
    ap.add_argument("--no-sweep", action="store_true",
                    help="skip the per-budget sweep leg (the same fixed layers whatever --workload)")
    ap.add_argument("--sweep-only", action="store_true",
                    help="run only the per-budget sweep and print it")
    ap.add_argument("--decode-only", action="store_true",
                    help="time only the decode leg on the workload (for profiling it)")
    ap.add_argument("--dense-only", action="store_true",
                    help="time only the dense kernel on the workload (for profiling it)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)

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
    stream = torch.cuda.current_stream(dev)
    peaks, peak_src = _peaks()
    burst = float(peaks.get("bf16_tflops", 1590.0))
    sustained = float(peaks.get("bf16_tflops_sustained", burst))
    hbm = float(peaks.get("hbm_gbs", 6650.0))

    if args.sweep_only:
        sw = budget_sweep(C, W, dev, stream, burst)
        if rank == 0:
            print(json.dumps({"budget_sweep": sw}), flush=True)
        if world > 1:
            dist.destroy_process_group()
        return 0

    wl = W.WORKLOADS[args.workload]
    B, N, D = wl.batch, wl.seq_len, wl.head_dim
    G = wl.num_q_heads // wl.num_kv_heads
    if args.kv_heads > 0:
        if world > 1 or args.kv_heads > wl.num_kv_heads:
            raise SystemExit("--kv-heads: one GPU, at most the layer's KV heads")
        h0, h1 = 0, args.kv_heads
        x = shard_inputs(W.make_inputs(wl, seed=0, device=str(dev)), wl.num_q_heads,
                         wl.num_kv_heads, h0, h1)
        torch.cuda.empty_cache()
    elif args.shard == "kv-heads":
        # every rank draws the same layer and keeps its KV heads' share
        h0, h1 = kv_head_shard(rank, world, wl.num_kv_heads)
        x = shard_inputs(W.make_inputs(wl, seed=0, device=str(dev)), wl.num_q_heads,
                         wl.num_kv_heads, h0, h1)
        torch.cuda.empty_cache()
    else:
        h0, h1 = 0, wl.num_kv_heads
        x = W.make_inputs(wl, seed=rank, device=str(dev))
    Hk = h1 - h0
    Hq = Hk * G
    shape = C.Shape(B, Hq, Hk, N, D, wl.page_size, wl.q_block,
                    pages_per_seq=x["page_table"].shape[1], num_phys_pages=x["k_pool"].shape[0])
    kap = C.KapParams(budget=args.budget, q_sub=wl.q_block // 4, k_sub=16, sink_pages=1)
    osk = C.OskParams(eps=args.eps)
    kc = C.cosa_kap_kcap(shape, kap)
    order = torch.empty(B, Hq, shape.num_q_blocks, kc, dtype=torch.int32, device=dev)
    count = torch.empty(B, Hq, shape.num_q_blocks, dtype=torch.int32, device=dev)
    ws = torch.empty(C.cosa_kap_workspace_size(shape, kap), dtype=torch.uint8, device=dev)
    out = torch.empty(B, Hq, N, D, dtype=torch.bfloat16, device=dev)
    computed = torch.empty(B, Hq, shape.num_q_blocks, dtype=torch.int32, device=dev)
    dense_flop = wl.dense_flops()  # of one whole layer
    if args.kv_heads > 0:
        dense_flop *= Hk / wl.num_kv_heads

    def job_value(ms):
        if args.shard == "kv-heads":
            return strong_value(dense_flop, ms)
        return weak_value(world, dense_flop, ms)

    def step(ev=None):
        # cosa_kap_pool + cosa_kap_rank is cosa_kap_select, with an event between the two
        if ev is not None:
            ev[0].record(stream)
        C.cosa_kap_pool(shape, kap, x["q"], x["k_pool"], x["page_table"], ws, stream=stream)
        if ev is not None:
            ev[1].record(stream)
        C.cosa_kap_rank(shape, kap, order, count, ws, stream=stream)
        if ev is not None:
            ev[2].record(stream)
        C.cosa_osk_attention(shape, osk, x["q"], x["k_pool"], x["v_pool"], x["page_table"], order,
                             count, out, computed=computed, stream=stream)
        if ev is not None:
            ev[3].record(stream)

    def barrier():
        if world > 1:
            dist.barrier()

    if args.dense_only:
        ms = _timed(lambda: C.cosa_dense_attention(shape, x["q"], x["k_pool"], x["v_pool"],
                                                   x["page_table"], out, stream=stream),
                    args.steps, stream, warm=args.warmup)
        assert C.cosa_get_status(stream) == 0
        if rank == 0:
            print(json.dumps({"kernel": "dense_attention", "workload": args.workload, "ms": ms,
                              "tflops": dense_flop * Hq / wl.num_q_heads / (ms * 1e-3) / 1e12,
                              "steps": args.steps, "warmup": args.warmup}), flush=True)
        if world > 1:
            dist.destroy_process_group()
        return 0

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    assert C.cosa_get_status(stream) == 0
    if args.decode_only:
        res = decode_leg(C, torch, x, shape, wl, order, count, dev, stream, args.eps, hbm,
                         reps=args.steps)
        if rank == 0:
            print(json.dumps({"decode": res, "workload": args.workload}), flush=True)
        if world > 1:
            dist.destroy_process_group()
        return 0

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
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
    pool_ms = [e[0].elapsed_time(e[1]) for e in evs]
    kap_ms = [e[0].elapsed_time(e[2]) for e in evs]
    osk_ms = [e[2].elapsed_time(e[3]) for e in evs]
    assert C.cosa_get_status(stream) == 0

    ms_per_step = total_ms / args.steps
    value = job_value(ms_per_step)

    # algorithmic work of the dominant kernel (OSK) for the roofline
    steps_visited = int(count.to(torch.int64).sum().item())
    steps_computed = int(computed.to(torch.int64).sum().item())
    tile = 2.0 * wl.q_block * wl.page_size * wl.head_dim
    osk_flop = tile * (steps_visited + steps_computed)
    osk_avg_ms = statistics.mean(osk_ms)
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
    pool_bytes = kap_pool_bytes(B, Hq, Hk, N, D, wl.q_block // 4, 16)
    pool_avg_ms = statistics.mean(pool_ms)
    pool_gbs = pool_bytes / (pool_avg_ms * 1e-3) / 1e9

    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "strong" if args.shard == "kv-heads" else "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": _config(wl, args.budget, args.eps, args.shard, world),
        "gpu_launches": 4 * args.steps,  # pool, score, order, OSK per step
        "clocks": clk,
        "roofline": {"kernel": "osk_attention", "bound": "tensor", "achieved": achieved,
                     "peak": peak_tflops, "unit": "TFLOP/s", "frac": achieved / peak_tflops,
                     "peak_source": f"{peak_src} bf16 {peak_kind}",
                     "frac_vs_burst": achieved / burst, "frac_vs_sustained": achieved / sustained,
                     "traffic": _osk_traffic(args.workload) if Hq == wl.num_q_heads else None,
                     "traffic_unit": "bytes per launch (DRAM read + write, ncu)",
                     "work": "visited FLOP = 2*Bq*P*D*(visited pages + computed pages) per launch",
                     "others": [{
                         "kernel": "kap_pool_kernel", "bound": "hbm", "achieved": pool_gbs,
                         "peak": hbm, "unit": "GB/s", "frac": pool_gbs / hbm,
                         "peak_source": f"{peak_src} HBM copy bandwidth",
                         "traffic": _pool_traffic(args.workload) if Hq == wl.num_q_heads else None,
                         "traffic_unit": "bytes per launch (DRAM read + write, ncu)",
                         "work": "Q and K read once (bf16) + pooled vectors written once "
                                 f"(2 fp32 terms): {pool_bytes:.4g} B per launch",
                         "ms": pool_avg_ms}]},
        "breakdown_ms": {"kap_select": statistics.mean(kap_ms), "kap_pool": pool_avg_ms,
                         "kap_rank": statistics.mean(kap_ms) - pool_avg_ms,
                         "osk_attention": osk_avg_ms},
        "budgets": {"kap_kept_frac": steps_visited / n_b_total,
                    "osk_computed_frac": steps_computed / n_b_total},
    }
    if world > 1:
        line["shard"] = {"rank0_kv_heads": [h0, h1], "kv_heads_per_rank": Hk}
    if args.kv_heads > 0:
        line["config"]["kv_heads_run"] = [h0, h1]

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
        return {"value": job_value(e2e_ms), "unit": "TFLOP/s",
                "ms_per_step": e2e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "entry_point": "cosa_attention_host"}

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
    dense_ms = _timed(lambda: C.cosa_dense_attention(shape, x["q"], x["k_pool"], x["v_pool"],
                                                     x["page_table"], dense_out, stream=stream),
                      3, stream, warm=2)
    dense_tf = dense_flop / (dense_ms * 1e-3) / 1e12
    line["dense"] = {"ms": dense_ms, "tflops": dense_tf, "frac_vs_burst": dense_tf / burst,
                     "frac_vs_sustained": dense_tf / sustained,
                     "speedup_sparse_vs_dense": dense_ms / ms_per_step}
    k_mean = statistics.mean(kap_ms)

    # ---- eps sweep at this budget (OSK only, KAP list reused) --------------
    sweep = []
    for eps in wl.eps_list:
        o2 = C.OskParams(eps=eps)
        ms = _timed(lambda: C.cosa_osk_attention(shape, o2, x["q"], x["k_pool"], x["v_pool"],
                                                 x["page_table"], order, count, out,
                                                 computed=computed, stream=stream), 3, stream)
        comp = int(computed.to(torch.int64).sum().item())
        fl = tile * (steps_visited + comp)
        sweep.append({"eps": eps, "osk_ms": ms, "kap_plus_osk_ms": ms + k_mean,
                      "computed_frac": comp / n_b_total, "visited_tflops": fl / (ms * 1e-3) / 1e12,
                      "visited_frac_vs_burst": fl / (ms * 1e-3) / 1e12 / burst,
                      "speedup_vs_dense": dense_ms / (ms + k_mean)})
    line["eps_sweep"] = sweep

    # ---- group-shared selection: one list per KV head and q-block (KAP group +
    # OSK over head pairs), same budget and eps; quality against the dense output
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

    vis_g = G * int(cg.to(torch.int64).sum().item())
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
        res = []
        for r in (16, 8):
            o3 = C.OskParams(eps=args.eps, max_run=r)
            ms = _timed(lambda: C.cosa_osk_attention(shape, o3, x["q"], x["k_pool"], x["v_pool"],
                                                     x["page_table"], order, count, bout,
                                                     computed=bcomp, stream=stream), 3, stream)
            if C.cosa_get_status(stream) != 0:
                raise RuntimeError("in-kernel error status")
            comp = int(bcomp.to(torch.int64).sum().item())
            res.append({"max_run": r, "eps": args.eps, "osk_ms": ms, "kap_plus_osk_ms": ms + k_mean,
                        "tflops": dense_flop / ((ms + k_mean) * 1e-3) / 1e12,
                        "speedup_vs_dense": dense_ms / (ms + k_mean),
                        "computed_frac": comp / n_b_total,
                        "rel_l2_vs_pages_rule": float((bout.float() - pref).norm() / pref.norm()),
                        "rel_l2_vs_dense": rel_l2(bout)})
        return res

    try:
        line["early_break"] = early_break_leg()
    except Exception as exc:  # an extra leg: report the failure, keep the line
        line["early_break"] = {"error": repr(exc)}

    # ---- proxy-bound pre-skip (not part of the pages' method): KAP, the pre-skip
    # filter, then the pages' rule on the survivors; output against the pages' rule on
    # the full lists (in `out`) and against dense
    def preskip_leg():
        po, pc = torch.empty_like(order), torch.empty_like(count)
        pout, pcomp = torch.empty_like(out), torch.empty_like(computed)
        pref = out.float()
        res = []
        for eps_pre, margin in ((1e-4, 0.0), (1e-4, 2.0), (1e-4, 4.0), (1e-3, 4.0), (1e-2, 0.0)):
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]

            def run(rec):
                if rec:
                    ev[0].record(stream)
                C.cosa_kap_select(shape, kap, x["q"], x["k_pool"], x["page_table"], po, pc, ws,
                                  stream=stream)
                if rec:
                    ev[1].record(stream)
                C.cosa_kap_preskip(shape, kap, eps_pre, margin, po, pc, ws, stream=stream)
                if rec:
                    ev[2].record(stream)
                C.cosa_osk_attention(shape, osk, x["q"], x["k_pool"], x["v_pool"], x["page_table"],
                                     po, pc, pout, computed=pcomp, stream=stream)
                if rec:
                    ev[3].record(stream)

            run(False)
            tms = [0.0, 0.0, 0.0]
            for _ in range(3):
                run(True)
                ev[3].synchronize()
                for i in range(3):
                    tms[i] += ev[i].elapsed_time(ev[i + 1]) / 3
            if C.cosa_get_status(stream) != 0:
                raise RuntimeError("in-kernel error status")
            vis = int(pc.to(torch.int64).sum().item())
            comp = int(pcomp.to(torch.int64).sum().item())
            fl = tile * (vis + comp)
            tot = sum(tms)
            res.append({"eps_pre": eps_pre, "margin": margin, "eps": args.eps,
                        "kap_ms": tms[0], "preskip_ms": tms[1], "osk_ms": tms[2], "ms": tot,
                        "tflops": dense_flop / (tot * 1e-3) / 1e12,
                        "speedup_vs_dense": dense_ms / tot,
                        "visited_frac": vis / n_b_total, "computed_frac": comp / n_b_total,
                        "visited_tflops": fl / (tms[2] * 1e-3) / 1e12,
                        "rel_l2_vs_pages_rule": float((pout.float() - pref).norm() / pref.norm()),
                        "rel_l2_vs_dense": rel_l2(pout)})
        return res

    try:
        line["preskip"] = preskip_leg()
    except Exception as exc:  # an extra leg: report the failure, keep the line
        line["preskip"] = {"error": repr(exc)}

    try:
        line["decode"] = decode_leg(C, torch, x, shape, wl, order, count, dev, stream, args.eps,
                                    hbm)
    except Exception as exc:  # an extra leg: report the failure, keep the line
        line["decode"] = {"error": repr(exc)}

    # ---- KAP pooling fused into the prefill's write of Q / K / V: the plain write then
    # cosa_kap_select, against the fused write then cosa_kap_rank (same lists)
    def fused_write_leg():
        P_ = wl.page_size
        pt = x["page_table"].long()
        tok = lambda pool: torch.stack([pool[pt[b_]].permute(0, 2, 1, 3).reshape(N, Hk, D)
                                        for b_ in range(B)]).contiguous()
        q_tok, k_tok, v_tok = x["q"].permute(0, 2, 1, 3).contiguous(), tok(x["k_pool"]), tok(x["v_pool"])
        q2, kp2, vp2 = torch.empty_like(x["q"]), torch.empty_like(x["k_pool"]), torch.empty_like(x["v_pool"])
        ws2 = torch.empty_like(ws)
        o2, c2 = torch.empty_like(order), torch.empty_like(count)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]

        def run(fused):
            ev[0].record(stream)
            C.cosa_prefill_write(shape, kap, q_tok, k_tok, v_tok, x["page_table"], q2, kp2, vp2,
                                 workspace=ws2 if fused else None, stream=stream)
            ev[1].record(stream)
            if fused:
                C.cosa_kap_rank(shape, kap, o2, c2, ws2, stream=stream)
            else:
                C.cosa_kap_select(shape, kap, q2, kp2, x["page_table"], o2, c2, ws2, stream=stream)
            ev[2].record(stream)
            C.cosa_osk_attention(shape, osk, q2, kp2, vp2, x["page_table"], o2, c2, out,
                                 stream=stream)
            ev[3].record(stream)
            ev[3].synchronize()
            return [ev[i].elapsed_time(ev[i + 1]) for i in range(3)]

        res = {}
        for fused in (False, True):
            run(fused)
            t = [0.0, 0.0, 0.0]
            for _ in range(3):
                t = [a + b_ / 3 for a, b_ in zip(t, run(fused))]
            res["fused" if fused else "plain"] = {"write_ms": t[0], "stage1_ms": t[1],
                                                  "osk_ms": t[2], "ms": sum(t)}
        if C.cosa_get_status(stream) != 0:
            raise RuntimeError("in-kernel error status")
        rw = 2.0 * 2 * B * N * D * (Hq + 2 * Hk)  # Q, K, V read once and written once (bf16)
        pooled = 2 * 4.0 * D * B * (Hq * N / (wl.q_block // 4) + Hk * N / 16)
        fw = res["fused"]["write_ms"]
        res["fused_write_roofline"] = {"bound": "hbm", "bytes": rw + pooled,
                                       "achieved": (rw + pooled) / (fw * 1e-3) / 1e9, "peak": hbm,
                                       "unit": "GB/s", "frac": (rw + pooled) / (fw * 1e-3) / 1e9 / hbm}
        res["saved_ms"] = res["plain"]["ms"] - res["fused"]["ms"]
        return res

    try:
        line["fused_write"] = fused_write_leg()
    except Exception as exc:  # an extra leg: report the failure, keep the line
        line["fused_write"] = {"error": repr(exc)}

    line["e2e"] = e2e_leg()
    del dense_out, dref, outg
    torch.cuda.empty_cache()

    # ---- speedup per budget on the other long-context layers ----------------
    if not args.no_sweep:
        try:
            line["budget_sweep"] = budget_sweep(C, W, dev, stream, burst)
        except Exception as exc:  # an extra leg: report the failure, keep the line
            line["budget_sweep"] = {"error": repr(exc)}

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
