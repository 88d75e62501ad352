"""GPU parity at the sizes the benchmark runs, and on inputs that reach the
kernels' rarely taken paths.

At 128K tokens (64-token pages, 128-row q-blocks) a q-block has up to 2048
causal pages: the KAP order kernel then handles several keys per thread, runs
its radix passes and bitonic stages over more than one block of threads, and
sorts up to 2048 kept keys; the OSK kernel's kept-page queue (64 entries)
wraps several times on a 410-page list.  One or two query heads per case keep
the oracle's share to seconds while every kernel still sees the work of one
(head, q-block) of the 32-head layer.  Large planted logits (a jump of tens of
nats) move the OSK kernels' exponent base, which ordinary inputs never do.

Methodology as in test_gpu_parity: lists bit-exact against the oracle's
selection and ordering run on the GPU's own fp32 scores (gist.science/pt §2.2
"Ordenação por Grupo de Flags"), skip decisions bit-exact outside a float64
margin, outputs within max-abs 2e-2 / mean-abs 2e-3 of the float64 oracle
(gist.science/pt §2.3)."""
import math

import numpy as np
import pytest
import torch

import block_sparse_long_kap_b200 as C
import oracle as O
import workloads as W
from helpers import (assert_lse_close, assert_out_close, check_osk_tiles, gpu_dense, gpu_kap,
                     gpu_osk, np64, score_tolerance, shape_of, SKIP_MARGIN)

pytestmark = pytest.mark.gpu

N128K = 131072
# tiles the oracle checks on a 128K sequence: the four longest lists, then spread ones
QB_SAMPLE = [1023, 1022, 1021, 1020, 800, 512, 256, 64]


def _host(x):
    return dict(q=np64(x["q"]), k_pool=np64(x["k_pool"]), v_pool=np64(x["v_pool"]),
                page_table=x["page_table"].cpu().numpy())


# ---------------------------------------------------------------------------
# KAP order kernel on caller-given scores at n_b up to 2048
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("budget", [0.2, 1.0])
def test_kap_order_bit_exact_128k(budget):
    si = W.make_score_inputs(1, 1, N128K, 64, 128, seed=77, tie_frac=0.1, hrm_frac=0.02)
    shape = C.Shape(1, 1, 1, N128K, 128, 64, 128)
    kap = C.KapParams(budget=budget, sink_pages=1)
    kc = C.cosa_kap_kcap(shape, kap)
    order = torch.full((1, 1, 1024, kc), -7, dtype=torch.int32, device="cuda")
    count = torch.full((1, 1, 1024), -7, dtype=torch.int32, device="cuda")
    C.cosa_kap_order(shape, kap, si["scores"].cuda(), si["hrm"].cuda(), order, count)
    torch.cuda.synchronize()
    assert C.cosa_get_status() == 0
    want_o, want_c = O.kap_order(si["scores"].numpy(), si["hrm"].numpy(), page_size=64,
                                 q_block=128, budget=budget, sink_pages=1)
    np.testing.assert_array_equal(count.cpu().numpy(), want_c)
    np.testing.assert_array_equal(order.cpu().numpy(), want_o)
    assert int(want_c.max()) == (2048 if budget == 1.0 else 410)


# ---------------------------------------------------------------------------
# fused KAP (pool, tensor-core scores, MaxNorm/HRM, select, order) at 128K:
# the list equals the oracle's selection + order on the GPU's exported scores
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("budget", [0.2, 1.0])
def test_kap_select_128k_order_equals_oracle_order_of_gpu_scores(budget):
    wl = W.small_workload("gqa-128k", N128K, 2, 1)
    x = W.make_inputs(wl, seed=31, device="cuda")
    shape = shape_of(wl, x)
    kap = C.KapParams(budget=budget, q_sub=32, k_sub=16, sink_pages=1)
    order, count, scores, hrm = gpu_kap(shape, kap, x)
    o, c = order.cpu().numpy(), count.cpu().numpy()
    S_g, h_g = scores.cpu().numpy(), hrm.cpu().numpy()
    # parity mode (i): bit-exact on identical fp32 scores and flags, every q-block
    want_o, want_c = O.kap_order(S_g, h_g, page_size=64, q_block=128, budget=budget,
                                 sink_pages=1)
    np.testing.assert_array_equal(c, want_c)
    np.testing.assert_array_equal(o, want_o)
    # the exported scores themselves against the float64 oracle on sampled q-blocks
    xh = _host(x)
    scale = 1 / math.sqrt(128)
    k_log = O.gather_logical(xh["k_pool"], xh["page_table"], 0, 0)
    khat = O.kap_pool_keys(k_log, 64, 16)
    n_hrm_diff = 0
    for h in range(2):
        qhat_all = O.kap_pool_queries(xh["q"][0, h], 128, 32)
        bound = scale * float(np.abs(qhat_all).max(axis=(0, 1)) @ np.abs(khat).max(axis=(0, 1)))
        tol = score_tolerance(bound)
        for qb in QB_SAMPLE:
            _, S, hr, a = O.kap_select_block(xh["q"][0, h], None, qb, q_block=128, page_size=64,
                                             q_sub=32, k_sub=16, scale=scale, budget=budget,
                                             sink_pages=1, khat=khat)
            n_b = O.causal_pages(qb, 128, 64)
            dS = np.abs(S_g[0, h, qb, :n_b] - S)
            assert dS.max() <= tol, f"S off by {dS.max():.2e} > {tol:.2e} at h {h} qb {qb}"
            if not np.array_equal(h_g[0, h, qb, :n_b], hr):
                n_hrm_diff += 1
                top2 = np.sort(a, axis=1)[:, -2:]
                assert np.min(top2[:, 1] - top2[:, 0]) <= 2 * tol
    assert n_hrm_diff <= 1


def test_kap_select_group_128k_order_equals_oracle_order_of_gpu_scores():
    wl = W.small_workload("gqa-128k", N128K, 2, 1)
    x = W.make_inputs(wl, seed=32, device="cuda")
    shape = shape_of(wl, x)
    kap = C.KapParams(budget=0.2, q_sub=32, k_sub=16, sink_pages=1)
    kc = C.cosa_kap_kcap(shape, kap)
    order = torch.full((1, 1, 1024, kc), -7, dtype=torch.int32, device="cuda")
    count = torch.full((1, 1, 1024), -7, dtype=torch.int32, device="cuda")
    scores = torch.full((1, 1, 1024, 2048), float("nan"), device="cuda")
    hrm = torch.full((1, 1, 1024, 2048), 7, dtype=torch.uint8, device="cuda")
    ws = torch.empty(C.cosa_kap_workspace_size(shape, kap), dtype=torch.uint8, device="cuda")
    C.cosa_kap_select_group(shape, kap, x["q"], x["k_pool"], x["page_table"], order, count, ws,
                            scores=scores, hrm=hrm)
    torch.cuda.synchronize()
    assert C.cosa_get_status() == 0
    want_o, want_c = O.kap_order(scores.cpu().numpy(), hrm.cpu().numpy(), page_size=64,
                                 q_block=128, budget=0.2, sink_pages=1)
    np.testing.assert_array_equal(count.cpu().numpy(), want_c)
    np.testing.assert_array_equal(order.cpu().numpy(), want_o)


# ---------------------------------------------------------------------------
# OSK on 128K lists from the GPU's own KAP: the kept-page queue wraps
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("eps", [0.0, 1e-4])
def test_osk_128k_long_lists(eps):
    wl = W.small_workload("gqa-128k", N128K, 1, 1)
    x = W.make_inputs(wl, seed=33, device="cuda")
    shape = shape_of(wl, x)
    kap = C.KapParams(budget=0.2, q_sub=32, k_sub=16, sink_pages=1)
    order, count, _, _ = gpu_kap(shape, kap, x, export=False)
    out, lse, computed, skip = gpu_osk(shape, eps, x, order, count)
    o, c = order.cpu().numpy(), count.cpu().numpy()
    assert int(c[0, 0, 1023]) == 410
    if eps == 0.0:  # every listed page computed: 410 kept pages through a 64-entry queue
        np.testing.assert_array_equal(computed.cpu().numpy(), c)
    xh = _host(x)
    ref = O.osk_attention(xh["q"], xh["k_pool"], xh["v_pool"], xh["page_table"], o, c,
                          num_kv_heads=1, page_size=64, q_block=128, eps=eps,
                          scale=1 / math.sqrt(128), heads=[(0, 0)], qblocks=QB_SAMPLE)
    check_osk_tiles(skip.cpu().numpy(), computed.cpu().numpy(), np64(out), lse.cpu().numpy(), ref,
                    c, [(0, 0, qb) for qb in QB_SAMPLE], 128, 64, eps,
                    float(np.abs(xh["v_pool"]).max()), f"osk 128k eps={eps}")


@pytest.mark.parametrize("eps", [0.0, 1e-4])
def test_osk_group_128k_long_lists(eps):
    wl = W.small_workload("gqa-128k", N128K, 2, 1)
    x = W.make_inputs(wl, seed=34, device="cuda")
    shape = shape_of(wl, x)
    kap = C.KapParams(budget=0.2, q_sub=32, k_sub=16, sink_pages=1)
    kc = C.cosa_kap_kcap(shape, kap)
    og = torch.full((1, 1, 1024, kc), -7, dtype=torch.int32, device="cuda")
    cg = torch.full((1, 1, 1024), -7, dtype=torch.int32, device="cuda")
    ws = torch.empty(C.cosa_kap_workspace_size(shape, kap), dtype=torch.uint8, device="cuda")
    C.cosa_kap_select_group(shape, kap, x["q"], x["k_pool"], x["page_table"], og, cg, ws)
    out = torch.full((1, 2, N128K, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((1, 2, N128K), float("nan"), device="cuda")
    computed = torch.full((1, 2, 1024), -7, dtype=torch.int32, device="cuda")
    skip = torch.full((1, 2, 1024, kc), 7, dtype=torch.uint8, device="cuda")
    C.cosa_osk_attention_group(shape, C.OskParams(eps), x["q"], x["k_pool"], x["v_pool"],
                               x["page_table"], og, cg, out, lse=lse, computed=computed,
                               skip_log=skip)
    torch.cuda.synchronize()
    assert C.cosa_get_status() == 0
    o_h, c_h = O.expand_group_order(og.cpu().numpy(), cg.cpu().numpy(), 2)
    xh = _host(x)
    ref = O.osk_attention(xh["q"], xh["k_pool"], xh["v_pool"], xh["page_table"], o_h, c_h,
                          num_kv_heads=1, page_size=64, q_block=128, eps=eps,
                          scale=1 / math.sqrt(128), qblocks=QB_SAMPLE)
    check_osk_tiles(skip.cpu().numpy(), computed.cpu().numpy(), np64(out), lse.cpu().numpy(), ref,
                    c_h, [(0, h, qb) for h in range(2) for qb in QB_SAMPLE], 128, 64, eps,
                    float(np.abs(xh["v_pool"]).max()), f"osk group 128k eps={eps}")


# ---------------------------------------------------------------------------
# exponent-base moves: planted pages whose logits jump by tens of nats
# ---------------------------------------------------------------------------
# (page, key magnitude): listed in page order, page 21 lifts the running max of the rows
# that see it by about 3 * 400 / sqrt(128) = 106 nats (153 in the kernels' log2 units,
# far past their 2^32 rescale slack) as the second page of its 128-key group, page 40
# by about as much again as the first page of its group
RESCALE_PAGES = ((21, 400.0), (40, 800.0))


def _rescale_inputs(num_q_heads):
    wl = W.small_workload("gqa-32k", 4096, num_q_heads, 1, drift_sigma=0.0, sink_keys=0,
                          planted_frac=0.0)
    x = W.make_inputs(wl, seed=41)
    g = torch.Generator().manual_seed(42)
    u = torch.randn(128, generator=g)
    u /= u.norm()
    q, kp = x["q"].float(), x["k_pool"].float()
    for page, mag in RESCALE_PAGES:
        kp[int(x["page_table"][0, page]), 0] += mag * u
    q[:, :, RESCALE_PAGES[0][0] * 64:] += 3.0 * u
    x["q"], x["k_pool"] = q.to(torch.bfloat16), kp.to(torch.bfloat16)
    return wl, x


def _ascending_lists(rows, nqb, kc):
    o = np.full((1, rows, nqb, kc), -1, dtype=np.int32)
    c = np.zeros((1, rows, nqb), dtype=np.int32)
    for r in range(rows):
        for qb in range(nqb):
            n = O.causal_pages(qb, 128, 64)
            o[0, r, qb, :n] = np.arange(n)
            c[0, r, qb] = n
    return o, c


@pytest.mark.parametrize("kernel", ["per-head", "group"])
@pytest.mark.parametrize("eps", [0.0, 1e-4])
def test_osk_exponent_base_moves_on_large_logits(kernel, eps):
    wl, x = _rescale_inputs(2)
    xd = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in x.items()}
    shape = shape_of(wl, x)
    nqb, kc = wl.num_q_blocks, O.causal_pages(wl.num_q_blocks - 1, 128, 64)
    xh = _host(x)
    # the planted logits really jump past the kernels' slack of 2^32 (in exp2 units)
    k_log = O.gather_logical(xh["k_pool"], xh["page_table"], 0, 0)
    s = xh["q"][0, 0, 40 * 64 + 63] @ k_log[:41 * 64].T / math.sqrt(128)
    assert (s[40 * 64:].max() - s[21 * 64:22 * 64].max()) / math.log(2) > 32
    assert (s[21 * 64:22 * 64].max() - s[:21 * 64].max()) / math.log(2) > 32
    if kernel == "per-head":
        o, c = _ascending_lists(2, nqb, kc)
        out, lse, computed, skip = gpu_osk(shape, eps, xd, torch.from_numpy(o).cuda(),
                                           torch.from_numpy(c).cuda())
    else:
        og, cg = _ascending_lists(1, nqb, kc)
        out = torch.full((1, 2, 4096, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
        lse = torch.full((1, 2, 4096), float("nan"), device="cuda")
        computed = torch.full((1, 2, nqb), -7, dtype=torch.int32, device="cuda")
        skip = torch.full((1, 2, nqb, kc), 7, dtype=torch.uint8, device="cuda")
        C.cosa_osk_attention_group(shape, C.OskParams(eps), xd["q"], xd["k_pool"], xd["v_pool"],
                                   xd["page_table"], torch.from_numpy(og).cuda(),
                                   torch.from_numpy(cg).cuda(), out, lse=lse, computed=computed,
                                   skip_log=skip)
        torch.cuda.synchronize()
        assert C.cosa_get_status() == 0
        o, c = O.expand_group_order(og, cg, 2)
    ref = O.osk_attention(xh["q"], xh["k_pool"], xh["v_pool"], xh["page_table"], o, c,
                          num_kv_heads=1, page_size=64, q_block=128, eps=eps,
                          scale=1 / math.sqrt(128))
    tiles = [(0, h, qb) for h in range(2) for qb in range(nqb)]
    check_osk_tiles(skip.cpu().numpy(), computed.cpu().numpy(), np64(out), lse.cpu().numpy(), ref,
                    c, tiles, 128, 64, eps, float(np.abs(xh["v_pool"]).max()),
                    f"osk {kernel} rescale eps={eps}")


def test_dense_on_large_logits():
    wl, x = _rescale_inputs(2)
    xd = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in x.items()}
    out, lse = gpu_dense(shape_of(wl, x), xd)
    xh = _host(x)
    ref = O.dense_attention(xh["q"], xh["k_pool"], xh["v_pool"], xh["page_table"],
                            num_kv_heads=1, scale=1 / math.sqrt(128))
    assert_out_close(np64(out), ref["out"], "dense rescale")
    assert_lse_close(lse.cpu().numpy(), ref["lse"], "dense rescale")


# ---------------------------------------------------------------------------
# early break deep in long lists (many ring wraps before the break)
# ---------------------------------------------------------------------------
def test_osk_early_break_long_lists():
    """16K tokens, budget 0.5 (lists of up to 128 pages), r = 8: tiles break after
    visiting 40-70 pages, i.e. past many rotations of the K ring and S buffers.
    Skip logs, computed counts, outputs and LSE against osk_block_rules(max_run=8);
    a decision within rounding of the threshold is taken as the kernel took it and
    the oracle run on from there."""
    r = 8
    wl = W.small_workload("gqa-32k", 16384, 1, 1)
    x = W.make_inputs(wl, seed=5)
    xd = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in x.items()}
    shape = shape_of(wl, x)
    xh = _host(x)
    scale = 1 / math.sqrt(128)
    sel = O.kap_select(xh["q"], xh["k_pool"], xh["page_table"], num_kv_heads=1, page_size=64,
                       q_block=128, q_sub=32, k_sub=16, scale=scale, budget=0.5, sink_pages=1)
    out, lse, computed, skip = gpu_osk(shape, 1e-4, xd, torch.from_numpy(sel["order"]).cuda(),
                                       torch.from_numpy(sel["count"]).cuda(), max_run=r)
    out, lse = np64(out), lse.cpu().numpy()
    computed, skip = computed.cpu().numpy(), skip.cpu().numpy()
    k_log = O.gather_logical(xh["k_pool"], xh["page_table"], 0, 0)
    v_log = O.gather_logical(xh["v_pool"], xh["page_table"], 0, 0)
    deep = n_forced = 0
    qbs = list(range(wl.num_q_blocks - 16, wl.num_q_blocks)) + [20, 50, 80]
    rows_all = np.zeros(out.shape[:3], dtype=bool)
    want_out = np.zeros_like(out)
    want_lse = np.full_like(lse, -np.inf)
    for qb in qbs:
        n = int(sel["count"][0, 0, qb])
        lst = sel["order"][0, 0, qb, :n]
        rows = slice(qb * 128, (qb + 1) * 128)
        gs = skip[0, 0, qb, :n]
        assert np.all(skip[0, 0, qb, n:] == 7)
        force = {}
        for _ in range(n + 1):
            ref = O.osk_block_rules(xh["q"][0, 0, rows], k_log, v_log, qb, 128, 64, lst, 1e-4,
                                    scale, force=force, max_run=r)
            dis = np.nonzero(gs != ref["skip"])[0]
            if len(dis) == 0:
                break
            j = int(dis[0])
            assert abs(ref["margin"][j]) <= SKIP_MARGIN, f"decision differs outside the margin, qb {qb}"
            force[j] = bool(gs[j])
        assert np.array_equal(gs, ref["skip"])
        assert computed[0, 0, qb] == ref["computed"]
        want_out[0, 0, rows] = ref["out"]
        want_lse[0, 0, rows] = ref["lse"]
        rows_all[0, 0, rows] = True
        # broke after more than two rotations of the S buffers (2 * 3 groups of 2 pages)
        deep += int(12 < ref["visited"] < n)
        n_forced += len(force)
    assert n_forced <= 2
    assert deep >= len(qbs) // 2, f"only {deep} tiles broke deep in their list"
    assert_out_close(out, want_out, "osk break 16k r=8", rows_mask=rows_all)
    assert_lse_close(lse, want_lse, "osk break 16k r=8", rows_mask=rows_all)
