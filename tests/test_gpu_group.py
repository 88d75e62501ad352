"""GPU parity of the group-shared path (one ordered list per KV head and
q-block): cosa_kap_select_group against the oracle's kap_select_group.  The
list is compared bit-exactly with the oracle's selection and ordering run on the
GPU's own exported group scores and flags, and checked valid under the oracle's
float64 scores; the scores are compared within the derived bound."""
import math

import numpy as np
import pytest
import torch

import block_sparse_long_kap_b200 as C
import oracle as O
import workloads as W
from helpers import check_order_valid, np64, score_tolerance, shape_of, to_dev

pytestmark = pytest.mark.gpu

GROUP_CASES = {
    "tiny-2k-g2": (W.small_workload("tiny-2k", 2048, 4, 2), 0.25),
    "gqa-4k": (W.small_workload("gqa-32k", 4096, 8, 2, shuffle_pages=True), 0.25),
    "narrow-kv-4k-g7": (W.small_workload("narrow-kv-64k", 4096, 14, 2), 0.1),
    "wide-head-4k-p128": (W.small_workload("wide-head-128k", 4096, 16, 2), 0.15),
    "gqa-2k-bq64": (W.small_workload("gqa-32k", 2048, 4, 1, q_block=64), 0.3),
}


def gpu_kap_group(shape, kap, xd):
    B, Hk = shape.batch, shape.num_kv_heads
    kc = C.cosa_kap_kcap(shape, kap)
    dev = xd["q"].device
    order = torch.full((B, Hk, shape.num_q_blocks, kc), -7, dtype=torch.int32, device=dev)
    count = torch.full((B, Hk, shape.num_q_blocks), -7, dtype=torch.int32, device=dev)
    ws = torch.empty(C.cosa_kap_workspace_size(shape, kap), dtype=torch.uint8, device=dev)
    scores = torch.full((B, Hk, shape.num_q_blocks, shape.num_pages), float("nan"),
                        dtype=torch.float32, device=dev)
    hrm = torch.full((B, Hk, shape.num_q_blocks, shape.num_pages), 7, dtype=torch.uint8,
                     device=dev)
    C.cosa_kap_select_group(shape, kap, xd["q"], xd["k_pool"], xd["page_table"], order, count, ws,
                            scores=scores, hrm=hrm)
    torch.cuda.synchronize()
    assert C.cosa_get_status() == 0
    return order, count, scores, hrm


@pytest.mark.parametrize("case", sorted(GROUP_CASES))
def test_kap_select_group_parity(case):
    wl, budget = GROUP_CASES[case]
    x = W.make_inputs(wl, seed=2)
    xd = to_dev(x)
    shape = shape_of(wl, x)
    kap = C.KapParams(budget=budget, q_sub=wl.q_block // 4, k_sub=16, sink_pages=1)
    order, count, scores, hrm = gpu_kap_group(shape, kap, xd)
    o, c, S_g, h_g = (order.cpu().numpy(), count.cpu().numpy(), scores.cpu().numpy(),
                      hrm.cpu().numpy())
    q, kp, pt = np64(x["q"]), np64(x["k_pool"]), x["page_table"].cpu().numpy()
    scale = 1 / math.sqrt(wl.head_dim)
    ref = O.kap_select_group(q, kp, pt, num_kv_heads=wl.num_kv_heads, page_size=wl.page_size,
                             q_block=wl.q_block, q_sub=wl.q_block // 4, k_sub=16, scale=scale,
                             budget=budget, sink_pages=1)
    G = wl.num_q_heads // wl.num_kv_heads
    bound = 0.0
    for b in range(wl.batch):
        for hk in range(wl.num_kv_heads):
            kh = O.kap_pool_keys(O.gather_logical(kp, pt, b, hk), wl.page_size, 16)
            for h in range(hk * G, (hk + 1) * G):
                qh = O.kap_pool_queries(q[b, h], wl.q_block, wl.q_block // 4)
                bound = max(bound, scale * float(np.abs(qh).max(axis=(0, 1)) @ np.abs(kh).max(axis=(0, 1))))
    tol = score_tolerance(bound)
    np.testing.assert_array_equal(c, ref["count"])
    n_hrm_diff = n_rows = 0
    for b in range(wl.batch):
        for hk in range(wl.num_kv_heads):
            for qb in range(wl.num_q_blocks):
                n_rows += 1
                n_b = O.causal_pages(qb, wl.q_block, wl.page_size)
                dS = np.abs(S_g[b, hk, qb, :n_b] - ref["S"][b, hk, qb, :n_b])
                assert dS.max() <= tol, f"S off by {dS.max():.2e} > {tol:.2e} at {(b, hk, qb)}"
                assert np.all(S_g[b, hk, qb, n_b:] == 0) and np.all(h_g[b, hk, qb, n_b:] == 0)
                n_hrm_diff += not np.array_equal(h_g[b, hk, qb, :n_b], ref["hrm"][b, hk, qb, :n_b])
                # bit-exact: the oracle's selection + order on the GPU's own fp32 scores/flags
                want = O.kap_order_from_scores(S_g[b, hk, qb, :n_b], h_g[b, hk, qb, :n_b], qb,
                                               wl.q_block, wl.page_size, budget, 1)
                assert o[b, hk, qb, :c[b, hk, qb]].tolist() == want.tolist(), (b, hk, qb)
                assert np.all(o[b, hk, qb, c[b, hk, qb]:] == -1)
                check_order_valid(o[b, hk, qb], int(c[b, hk, qb]), ref["S"][b, hk, qb],
                                  h_g[b, hk, qb], qb, wl.q_block, wl.page_size, 1, budget, 2 * tol,
                                  False)
    # HRM may differ only where some head's two best pages tie within rounding (rare)
    assert n_hrm_diff <= max(1, n_rows // 100)


def test_kap_select_group_with_one_head_per_group_equals_per_head():
    wl = W.small_workload("gqa-32k", 2048, 4, 4, shuffle_pages=True)
    x = W.make_inputs(wl, seed=3)
    xd = to_dev(x)
    shape = shape_of(wl, x)
    kap = C.KapParams(budget=0.25, q_sub=wl.q_block // 4, k_sub=16, sink_pages=1)
    og, cg, sg, hg = gpu_kap_group(shape, kap, xd)
    from helpers import gpu_kap
    oh, ch, sh, hh = gpu_kap(shape, kap, xd)
    assert torch.equal(og, oh) and torch.equal(cg, ch) and torch.equal(sg, sh) and torch.equal(hg, hh)


# ---------------------------------------------------------------------------
# OSK over group-shared lists: every head on its KV head's list, against the
# oracle's per-head OSK given those lists
# ---------------------------------------------------------------------------
GROUP_OSK_CASES = {
    "tiny-2k-g2": (W.small_workload("tiny-2k", 2048, 4, 2), 0.25, (1e-4, 0.0)),
    "gqa-4k": (W.small_workload("gqa-32k", 4096, 8, 2, shuffle_pages=True), 0.25, (1e-4, 1e-3, 0.0)),
    "narrow-kv-4k-g7": (W.small_workload("narrow-kv-64k", 4096, 7, 1, batch=2), 0.2, (1e-4,)),
    "wide-head-4k-p128": (W.small_workload("wide-head-128k", 4096, 8, 1), 0.3, (1e-4, 0.0)),
    "gqa-2k-bq64": (W.small_workload("gqa-32k", 2048, 4, 1, q_block=64), 0.5, (1e-3,)),
}


def gpu_osk_group(shape, eps, xd, order, count):
    B, Hq, N, D = shape.batch, shape.num_q_heads, shape.seq_len, shape.head_dim
    dev = xd["q"].device
    out = torch.full((B, Hq, N, D), float("nan"), dtype=torch.bfloat16, device=dev)
    lse = torch.full((B, Hq, N), float("nan"), dtype=torch.float32, device=dev)
    computed = torch.full((B, Hq, shape.num_q_blocks), -7, dtype=torch.int32, device=dev)
    skip = torch.full((B, Hq, shape.num_q_blocks, order.shape[-1]), 7, dtype=torch.uint8,
                      device=dev)
    C.cosa_osk_attention_group(shape, C.OskParams(eps), xd["q"], xd["k_pool"], xd["v_pool"],
                               xd["page_table"], order, count, out, lse=lse, computed=computed,
                               skip_log=skip)
    torch.cuda.synchronize()
    assert C.cosa_get_status() == 0
    return out, lse, computed, skip


@pytest.mark.parametrize("case,eps", [(c, e) for c in sorted(GROUP_OSK_CASES)
                                      for e in GROUP_OSK_CASES[c][2]])
def test_osk_group_parity(case, eps):
    from helpers import SKIP_MARGIN, assert_lse_close, assert_out_close
    wl, budget, _ = GROUP_OSK_CASES[case]
    x = W.make_inputs(wl, seed=4)
    xd = to_dev(x)
    shape = shape_of(wl, x)
    q, kp, vp, pt = np64(x["q"]), np64(x["k_pool"]), np64(x["v_pool"]), x["page_table"].cpu().numpy()
    scale = 1 / math.sqrt(wl.head_dim)
    sel = O.kap_select_group(q, kp, pt, num_kv_heads=wl.num_kv_heads, page_size=wl.page_size,
                             q_block=wl.q_block, q_sub=wl.q_block // 4, k_sub=16, scale=scale,
                             budget=budget, sink_pages=1)
    out, lse, computed, skip = gpu_osk_group(shape, eps, xd, torch.from_numpy(sel["order"]).cuda(),
                                             torch.from_numpy(sel["count"]).cuda())
    out, lse, computed, skip = np64(out), lse.cpu().numpy(), computed.cpu().numpy(), skip.cpu().numpy()
    o_h, c_h = O.expand_group_order(sel["order"], sel["count"], wl.num_q_heads)
    ref = O.osk_attention(q, kp, vp, pt, o_h, c_h, num_kv_heads=wl.num_kv_heads,
                          page_size=wl.page_size, q_block=wl.q_block, eps=eps, scale=scale)
    vmax = float(np.abs(vp).max())
    rows_ok = np.ones(out.shape[:3], dtype=bool)
    n_amb = n_steps = 0
    for idx in np.ndindex(*c_h.shape):
        b, h, qb = idx
        n = int(c_h[idx])
        n_steps += n
        gs, rs, mg = skip[idx][:n], ref["skip"][idx][:n], ref["margin"][idx][:n]
        assert np.all(skip[idx][n:] == 7), "skip log written past count"
        assert computed[idx] == n - int(gs.sum())
        amb = np.abs(mg) <= SKIP_MARGIN
        n_amb += int(amb.sum())
        dis = gs != rs
        assert not np.any(dis & ~amb), f"skip decision differs outside the margin at {idx}"
        if dis.any():
            rows = slice(qb * wl.q_block, (qb + 1) * wl.q_block)
            rows_ok[b, h, rows] = False
            bound = 2 * int(dis.sum()) * wl.page_size * eps * vmax
            assert np.abs(out[b, h, rows] - ref["out"][b, h, rows]).max() <= bound + 2e-2
        else:
            assert computed[idx] == ref["computed"][idx]
    assert n_amb <= max(2, n_steps // 1000), f"{n_amb} of {n_steps} steps within the skip margin"
    assert_out_close(out, ref["out"], f"osk group {case} eps={eps}", rows_mask=rows_ok)
    assert_lse_close(lse, ref["lse"], f"osk group {case} eps={eps}", rows_mask=rows_ok)


def test_osk_group_equals_per_head_kernel_on_expanded_lists():
    """The pair kernel's decisions are those of the per-head kernel given each
    head its KV head's list (same fp32 logits and the same vote arithmetic)."""
    wl = W.small_workload("gqa-32k", 4096, 8, 2, shuffle_pages=True)
    x = W.make_inputs(wl, seed=9)
    xd = to_dev(x)
    shape = shape_of(wl, x)
    kap = C.KapParams(budget=0.25, q_sub=wl.q_block // 4, k_sub=16, sink_pages=1)
    og, cg, _, _ = gpu_kap_group(shape, kap, xd)
    G = wl.num_q_heads // wl.num_kv_heads
    hk = torch.arange(wl.num_q_heads, device="cuda") // G
    from helpers import gpu_osk
    for eps in (1e-4, 0.0):
        o1, l1, c1, s1 = gpu_osk_group(shape, eps, xd, og, cg)
        o2, l2, c2, s2 = gpu_osk(shape, eps, xd, og[:, hk].contiguous(), cg[:, hk].contiguous())
        assert torch.equal(c1, c2) and torch.equal(s1, s2)
        d = (o1.float() - o2.float()).abs().max().item()
        assert d <= 2 ** -7 * max(1.0, o2.float().abs().max().item())
