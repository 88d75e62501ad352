"""Seeded synthetic inputs for causal prefill attention over a paged KV cache.

This module only draws random numbers and lays them out; it holds none of the
attention or proxy arithmetic.  Both the CPU oracle (through the tests) and the
GPU path consume what it produces, so it imports neither of them.

The recipes stand in for the long-context prompts the CoSA pages evaluate on
(RULER and LongBench-v2 on Qwen3-8B / Llama-3.1-8B-Instruct, gist.science/pt
"4. Resultados Experimentais"), which are not available here.  Shapes follow
the GQA attention layers of those backbones at 2K-128K context.

Recipe (per sequence b and KV head h_kv; G = H_q / H_kv query heads per group):
  * base: Q, K, V ~ N(0, 1) per element;
  * drift (locality): w_0 = 0, w_t = w_{t-1} + sigma * z_t with z_t ~ N(0, I_D);
    w_t is added to K[b, h_kv, t] and to Q[b, h, t] for every q-head h of the group;
  * planted salient pages: a set of pages is drawn without replacement; a unit
    Gaussian direction u is drawn; keys of those pages get += mag * u and the
    chosen queries (the last 256, or all) of every q-head of the group get += u;
  * sink: the first `sink_keys` keys get += sink_mag * mu, mu = unit vector of
    the mean of the group's queries over all positions;
  * everything is rounded to bf16 (an fp32 copy is kept when asked);
  * K and V are scattered into page pools [num_phys_pages][H_kv][P][D] through a
    page table [B][pages_per_seq] (identity, or a seeded shuffle).
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import torch

__all__ = ["Workload", "WORKLOADS", "make_inputs", "make_score_inputs", "small_workload"]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    num_q_heads: int
    num_kv_heads: int
    seq_len: int
    head_dim: int
    page_size: int
    q_block: int
    drift_sigma: float = 0.0
    sink_keys: int = 0
    sink_mag: float = 3.0
    planted_count: int = 0          # pages per (b, h_kv); overrides planted_frac when > 0
    planted_frac: float = 0.0
    planted_mag: float = 4.0
    planted_queries: str = "all"    # "all" or "last256"
    shuffle_pages: bool = False
    keep_fp32: bool = False
    budgets: tuple = (0.25,)
    eps_list: tuple = (1e-4,)

    @property
    def num_pages(self) -> int:
        return self.seq_len // self.page_size

    @property
    def num_q_blocks(self) -> int:
        return self.seq_len // self.q_block

    def dense_flops(self) -> float:
        """Dense-equivalent causal FLOP: 4 * B * H_q * D * N (N + 1) / 2."""
        n = self.seq_len
        return 4.0 * self.batch * self.num_q_heads * self.head_dim * n * (n + 1) / 2.0

    def n_planted(self) -> int:
        if self.planted_count > 0:
            return self.planted_count
        if self.planted_frac <= 0:
            return 0
        return max(1, int(round(self.planted_frac * self.num_pages)))


WORKLOADS = {
    # 2K tiny causal prefill, 3 planted pages seen by the last 256 queries.
    "tiny-2k": Workload("tiny-2k", 1, 2, 2, 2048, 64, 64, 64,
                        planted_count=3, planted_mag=4.0, planted_queries="last256",
                        keep_fp32=True, budgets=(0.25,), eps_list=(1e-4,)),
    # Llama-3-8B-shaped GQA layer at 32K.
    "gqa-32k": Workload("gqa-32k", 1, 32, 8, 32768, 128, 64, 128,
                        drift_sigma=0.02, sink_keys=64, planted_frac=0.01, planted_mag=4.0,
                        budgets=(0.10, 0.25, 0.50), eps_list=(1e-4, 0.0)),
    # Long-context GQA layer at 128K with a shuffled page table.
    "gqa-128k": Workload("gqa-128k", 1, 32, 8, 131072, 128, 64, 128,
                         drift_sigma=0.02, sink_keys=64, planted_frac=0.005, planted_mag=4.0,
                         shuffle_pages=True, budgets=(0.20,), eps_list=(0.0, 1e-5, 1e-4, 1e-3)),
    # Narrow-KV GQA layer (G = 7) at 64K, batch 2.
    "narrow-kv-64k": Workload("narrow-kv-64k", 2, 28, 4, 65536, 128, 64, 128,
                              drift_sigma=0.05, sink_keys=16, planted_frac=0.02, planted_mag=6.0,
                              budgets=(0.05, 0.10, 0.20), eps_list=(1e-4,)),
    # Wide-head GQA layer (G = 8) at 128K with 128-token pages.
    "wide-head-128k": Workload("wide-head-128k", 1, 64, 8, 131072, 128, 128, 128,
                               drift_sigma=0.02, sink_keys=64, planted_frac=0.005, planted_mag=4.0,
                               shuffle_pages=True,
                               budgets=(0.05, 0.10, 0.15, 0.20, 0.25, 0.30, 0.40, 0.50),
                               eps_list=(1e-4, 0.0)),
}


def small_workload(base: str, seq_len: int, num_q_heads: Optional[int] = None,
                   num_kv_heads: Optional[int] = None, batch: Optional[int] = None,
                   **overrides) -> Workload:
    """A shrunken copy of a named workload (same generator, fewer tokens/heads)."""
    wl = WORKLOADS[base]
    kw = dict(seq_len=seq_len, name=f"{base}@{seq_len}")
    if num_q_heads is not None:
        kw["num_q_heads"] = num_q_heads
    if num_kv_heads is not None:
        kw["num_kv_heads"] = num_kv_heads
    if batch is not None:
        kw["batch"] = batch
    kw.update(overrides)
    return dataclasses.replace(wl, **kw)


def _unit(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm()


@torch.no_grad()
def make_inputs(wl: Workload, seed: int = 0, device: str = "cpu",
                keep_logical: bool = False) -> dict:
    """Draw one seeded problem.

    Returns a dict with
      q          bf16 [B][H_q][N][D]
      k_pool     bf16 [B * nP][H_kv][P][D]   (physical pages)
      v_pool     bf16 [B * nP][H_kv][P][D]
      page_table int32 [B][nP]  (logical page -> physical page)
      planted    int64 [B][H_kv][n_planted]  (logical page ids, sorted)
    and, when wl.keep_fp32, q_f32 / k_f32 / v_f32 (logical, [B][H][N][D]);
    when keep_logical, k_log / v_log bf16 [B][H_kv][N][D].
    The same seed gives the same values on the same device type.
    """
    B, Hq, Hk, N, D, P = (wl.batch, wl.num_q_heads, wl.num_kv_heads, wl.seq_len,
                          wl.head_dim, wl.page_size)
    if Hq % Hk:
        raise ValueError("num_q_heads must be a multiple of num_kv_heads")
    if N % P or N % wl.q_block:
        raise ValueError("seq_len must be a multiple of page_size and q_block")
    G = Hq // Hk
    nP = N // P
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    # host generator for the small integer draws (page choices, shuffles)
    gh = torch.Generator(device="cpu")
    gh.manual_seed(seed + 0x5EED)

    q = torch.randn(B, Hq, N, D, generator=g, device=device, dtype=torch.float32)
    k = torch.randn(B, Hk, N, D, generator=g, device=device, dtype=torch.float32)
    v = torch.randn(B, Hk, N, D, generator=g, device=device, dtype=torch.float32)

    if wl.drift_sigma > 0:
        for b in range(B):
            for h in range(Hk):
                steps = torch.randn(N, D, generator=g, device=device, dtype=torch.float32)
                steps.mul_(wl.drift_sigma)
                steps[0].zero_()
                w = torch.cumsum(steps, dim=0)
                k[b, h].add_(w)
                q[b, h * G:(h + 1) * G].add_(w.unsqueeze(0))
                del steps, w

    n_pl = wl.n_planted()
    planted = torch.zeros(B, Hk, n_pl, dtype=torch.int64)
    if n_pl > 0:
        if wl.planted_queries == "last256":
            last_tok = N - 256
            hi = last_tok // P          # pages overlapping the last 256 tokens are excluded
            cand = torch.arange(1, max(1, hi))
            q_rows = slice(max(0, N - 256), N)
        else:
            cand = torch.arange(1, max(1, nP - 1))  # neither page 0 nor the last page
            q_rows = slice(0, N)
        if cand.numel() < n_pl:
            raise ValueError("not enough candidate pages to plant")
        for b in range(B):
            for h in range(Hk):
                pick = cand[torch.randperm(cand.numel(), generator=gh)[:n_pl]]
                pick, _ = torch.sort(pick)
                planted[b, h] = pick
                u = _unit(torch.randn(D, generator=g, device=device, dtype=torch.float32))
                tok = (pick.to(device).unsqueeze(1) * P + torch.arange(P, device=device)).reshape(-1)
                k[b, h, tok] += wl.planted_mag * u
                q[b, h * G:(h + 1) * G, q_rows] += u

    if wl.sink_keys > 0:
        for b in range(B):
            for h in range(Hk):
                mu = _unit(q[b, h * G:(h + 1) * G].mean(dim=(0, 1)))
                k[b, h, :wl.sink_keys] += wl.sink_mag * mu

    if wl.shuffle_pages:
        perm = torch.randperm(B * nP, generator=gh)
    else:
        perm = torch.arange(B * nP)
    page_table = perm.view(B, nP).to(torch.int32)

    out = {"planted": planted, "page_table": page_table.to(device)}
    if wl.keep_fp32:
        out["q_f32"], out["k_f32"], out["v_f32"] = q.clone(), k.clone(), v.clone()
    qb16 = q.to(torch.bfloat16)
    del q
    kb16 = k.to(torch.bfloat16)
    vb16 = v.to(torch.bfloat16)
    del k, v
    out["q"] = qb16
    out["k_pool"] = _to_pool(kb16, page_table.to(device), P)
    out["v_pool"] = _to_pool(vb16, page_table.to(device), P)
    if keep_logical:
        out["k_log"], out["v_log"] = kb16, vb16
    return out


def _to_pool(x: torch.Tensor, page_table: torch.Tensor, P: int) -> torch.Tensor:
    """Scatter logical [B][H][N][D] into physical pages [B*nP][H][P][D]."""
    B, H, N, D = x.shape
    nP = N // P
    pool = torch.empty(B * nP, H, P, D, dtype=x.dtype, device=x.device)
    src = x.view(B, H, nP, P, D).permute(0, 2, 1, 3, 4).reshape(B * nP, H, P, D)
    pool[page_table.reshape(-1).long()] = src
    return pool


@torch.no_grad()
def make_score_inputs(batch: int, num_q_heads: int, seq_len: int, page_size: int,
                      q_block: int, seed: int = 0, tie_frac: float = 0.1,
                      hrm_frac: float = 0.02) -> dict:
    """Random proxy scores S in (0, 1] (fp32) and HRM flags (u8), laid out
    [B][H_q][nQB][nP], with a fraction of exactly repeated values so that the
    page-index tie-break is exercised.  Every entry of the rectangle is
    drawn; consumers read only a q-block's causal pages."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    nP = seq_len // page_size
    nQB = seq_len // q_block
    s = torch.rand(batch, num_q_heads, nQB, nP, generator=g, dtype=torch.float32)
    s = 1.0 - s                              # (0, 1]
    # plant exact ties: copy a value from a random other column
    tie = torch.rand(s.shape, generator=g) < tie_frac
    src = torch.randint(0, nP, s.shape, generator=g)
    s = torch.where(tie, torch.gather(s, 3, src), s)
    hrm = (torch.rand(s.shape, generator=g) < hrm_frac).to(torch.uint8)
    return {"scores": s.contiguous(), "hrm": hrm.contiguous()}
