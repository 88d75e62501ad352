"""Shared helpers for the GPU parity tests: run the C-ABI path on seeded inputs,
run the oracle on the same inputs, and compare.  Tolerances are stated here
once and derived in the comments."""
from __future__ import annotations

import math

import numpy as np
import torch

import block_sparse_long_kap_b200 as C
import oracle as O
import workloads as W

# Output tolerance for bf16 attention with fp32 accumulation (the bar the
# method is held to): max-abs 2e-2 and mean-abs 2e-3 against the float64 oracle.
OUT_MAX_ABS = 2e-2
OUT_MEAN_ABS = 2e-3
# LSE: fp32 logits from bf16 products; error grows with the logit magnitude.
LSE_REL = 2e-5
LSE_ABS = 2e-3
# Skip decisions: the kernel decides in fp32 (log2 domain), the oracle in
# float64 (natural log).  A tile whose float64 margin |max_i d_i - ln eps| is
# below this many nats may legitimately go either way.
SKIP_MARGIN = 1e-3


def shape_of(wl: W.Workload, x: dict) -> C.Shape:
    return C.Shape(wl.batch, wl.num_q_heads, wl.num_kv_heads, wl.seq_len, wl.head_dim,
                   wl.page_size, wl.q_block, pages_per_seq=x["page_table"].shape[1],
                   num_phys_pages=x["k_pool"].shape[0])


def to_dev(x: dict, device="cuda") -> dict:
    return {k: (v.to(device) if torch.is_tensor(v) and k in ("q", "k_pool", "v_pool", "page_table")
                else v) for k, v in x.items()}


def np64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def gpu_kap(shape: C.Shape, kap: C.KapParams, xd: dict, export=True):
    B, Hq = shape.batch, shape.num_q_heads
    kc = C.cosa_kap_kcap(shape, kap)
    dev = xd["q"].device
    order = torch.full((B, Hq, shape.num_q_blocks, kc), -7, dtype=torch.int32, device=dev)
    count = torch.full((B, Hq, shape.num_q_blocks), -7, dtype=torch.int32, device=dev)
    ws = torch.empty(C.cosa_kap_workspace_size(shape, kap), dtype=torch.uint8, device=dev)
    scores = hrm = None
    if export:
        scores = torch.full((B, Hq, shape.num_q_blocks, shape.num_pages), float("nan"),
                            dtype=torch.float32, device=dev)
        hrm = torch.full((B, Hq, shape.num_q_blocks, shape.num_pages), 7, dtype=torch.uint8,
                         device=dev)
    C.cosa_kap_select(shape, kap, xd["q"], xd["k_pool"], xd["page_table"], order, count, ws,
                      scores=scores, hrm=hrm)
    torch.cuda.synchronize()
    assert C.cosa_get_status() == 0
    return order, count, scores, hrm


def gpu_osk(shape: C.Shape, eps: float, xd: dict, order: torch.Tensor, count: torch.Tensor,
            max_run: int = 0):
    B, Hq, N, D = shape.batch, shape.num_q_heads, shape.seq_len, shape.head_dim
    dev = xd["q"].device
    out = torch.full((B, Hq, N, D), float("nan"), dtype=torch.bfloat16, device=dev)
    lse = torch.full((B, Hq, N), float("nan"), dtype=torch.float32, device=dev)
    computed = torch.full((B, Hq, shape.num_q_blocks), -7, dtype=torch.int32, device=dev)
    skip = torch.full(tuple(order.shape), 7, dtype=torch.uint8, device=dev)
    C.cosa_osk_attention(shape, C.OskParams(eps, max_run), xd["q"], xd["k_pool"], xd["v_pool"],
                         xd["page_table"], order, count, out, lse=lse, computed=computed,
                         skip_log=skip)
    torch.cuda.synchronize()
    assert C.cosa_get_status() == 0
    return out, lse, computed, skip


def gpu_dense(shape: C.Shape, xd: dict):
    B, Hq, N, D = shape.batch, shape.num_q_heads, shape.seq_len, shape.head_dim
    dev = xd["q"].device
    out = torch.full((B, Hq, N, D), float("nan"), dtype=torch.bfloat16, device=dev)
    lse = torch.full((B, Hq, N), float("nan"), dtype=torch.float32, device=dev)
    C.cosa_dense_attention(shape, xd["q"], xd["k_pool"], xd["v_pool"], xd["page_table"], out,
                           lse=lse)
    torch.cuda.synchronize()
    assert C.cosa_get_status() == 0
    return out, lse


def assert_out_close(got: np.ndarray, want: np.ndarray, what: str, rows_mask=None):
    """Element-wise bf16-output check: max-abs <= 2e-2 and mean-abs <= 2e-3."""
    err = np.abs(got - want)
    if rows_mask is not None:
        err = err[rows_mask]
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    mx, mean = float(err.max()) if err.size else 0.0, float(err.mean()) if err.size else 0.0
    assert mx <= OUT_MAX_ABS, f"{what}: max-abs {mx:.3e} > {OUT_MAX_ABS}"
    assert mean <= OUT_MEAN_ABS, f"{what}: mean-abs {mean:.3e} > {OUT_MEAN_ABS}"
    return mx, mean


def assert_lse_close(got: np.ndarray, want: np.ndarray, what: str, rows_mask=None):
    d = np.abs(got - want)
    tol = LSE_ABS + LSE_REL * np.abs(want)
    if rows_mask is not None:
        d, tol = d[rows_mask], tol[rows_mask]
    bad = d > tol
    assert not bad.any(), f"{what}: lse off by up to {float(d.max()):.3e}"


def score_tolerance(qhat_bound: float) -> float:
    """|S_gpu - S_oracle| bound.  S = mean_r exp(a - m_r) has |dS| <= 2 max|da|.
    The kernel's a is an fp32 dot product of length D of fp32 pooled vectors
    scaled by 1/sqrt(D): |da| <= gamma_D * scale * sum_d |q_d k_d| + pooling
    rounding, with gamma_D = D u / (1 - D u), u = 2^-24.  qhat_bound is
    max over (rep, sub-key) of scale * sum_d |q_d k_d|; the factor 2 covers the
    pooled-vector rounding."""
    gamma = 128 * 2.0 ** -24 / (1 - 128 * 2.0 ** -24)
    return 1e-5 + 2 * 2 * gamma * qhat_bound


def check_order_valid(order_g, count_g, S_ref, hrm_g, qb, Bq, P, sink, budget, delta, ascending):
    """The GPU list for one q-block is a correct KAP list for scores within
    +-delta of the oracle's: right size, forced pages kept, every kept
    non-forced page at least as good (up to delta) as every dropped one, and
    listed by (HRM, score) descending up to delta (or by page id)."""
    n_b = O.causal_pages(qb, Bq, P)
    k_b = O.budget_count(qb, Bq, P, sink, budget)
    assert count_g == k_b
    lst = [int(p) for p in order_g[:count_g]]
    assert len(set(lst)) == k_b and all(0 <= p < n_b for p in lst)
    assert all(p == -1 for p in order_g[count_g:])
    forced = set(O.forced_pages(qb, Bq, P, sink))
    assert forced <= set(lst)
    kept = [p for p in lst if p not in forced]
    dropped = [p for p in range(n_b) if p not in set(lst)]

    def val(p):
        return (int(hrm_g[p]), float(S_ref[p]))
    if kept and dropped:
        worst_kept = min(kept, key=val)
        best_drop = max(dropped, key=val)
        wk, bd = val(worst_kept), val(best_drop)
        assert wk[0] > bd[0] or (wk[0] == bd[0] and wk[1] >= bd[1] - delta), \
            f"qb {qb}: kept {worst_kept} {wk} worse than dropped {best_drop} {bd}"
    if ascending:
        assert lst == sorted(lst)
    else:
        for a, b in zip(lst, lst[1:]):
            va, vb = val(a), val(b)
            assert va[0] > vb[0] or (va[0] == vb[0] and va[1] >= vb[1] - delta), \
                f"qb {qb}: {a} {va} listed before {b} {vb}"


def check_osk_tiles(skip, computed, out, lse, ref, count, tiles, q_block, page_size, eps, vmax,
                    what):
    """Compare one OSK launch with the oracle on the given (b, h, qb) tiles.

    skip / computed / out / lse are the kernel's (numpy; the skip log was
    pre-filled with 7 so that writes past count show), ref the oracle's
    osk_attention on the same lists.  Skip decisions are bit-exact outside the
    float64 margin SKIP_MARGIN; a tile with a decision inside it is held to the
    skip error bound instead of the element-wise bar.  Returns the number of
    steps checked and of steps inside the margin."""
    rows_ok = np.zeros(out.shape[:3], dtype=bool)
    n_amb = n_steps = 0
    for (b, h, qb) in tiles:
        idx = (b, h, qb)
        n = int(count[idx])
        n_steps += n
        gs, rs, mg = skip[idx][:n], ref["skip"][idx][:n], ref["margin"][idx][:n]
        assert np.all(skip[idx][n:] == 7), f"{what}: skip log written past count at {idx}"
        assert computed[idx] == n - int(gs.sum()), f"{what}: computed != unskipped at {idx}"
        amb = np.abs(mg) <= SKIP_MARGIN
        n_amb += int(amb.sum())
        dis = gs != rs
        assert not np.any(dis & ~amb), f"{what}: skip decision differs outside the margin at {idx}"
        rows = slice(qb * q_block, (qb + 1) * q_block)
        if dis.any():
            bound = 2 * int(dis.sum()) * page_size * eps * vmax
            assert np.abs(out[b, h, rows] - ref["out"][b, h, rows]).max() <= bound + OUT_MAX_ABS
        else:
            assert computed[idx] == ref["computed"][idx], f"{what}: computed differs at {idx}"
            rows_ok[b, h, rows] = True
    assert n_amb <= max(2, n_steps // 1000), f"{what}: {n_amb} of {n_steps} steps in the margin"
    assert rows_ok.any(), f"{what}: no tile compared element-wise"
    assert_out_close(out, ref["out"], what, rows_mask=rows_ok)
    assert_lse_close(lse, ref["lse"], what, rows_mask=rows_ok)
    return n_steps, n_amb
