"""GPU parity: the C-ABI CUDA path against the CPU oracle on the same seeded
inputs.  Indices (order, count) are compared bit-exactly where the inputs to
the decision are identical (cosa_kap_order on given fp32 scores); where the
GPU computes the scores itself, scores are compared within a derived bound and
the lists are checked to be valid under the oracle's scores.  Attention
outputs are compared element by element (max-abs 2e-2, mean-abs 2e-3)."""
import math

import numpy as np
import pytest
import torch

import block_sparse_long_kap_b200 as C
import oracle as O
import workloads as W
from helpers import (SKIP_MARGIN, assert_lse_close, assert_out_close, check_order_valid,
                     check_osk_tiles, gpu_dense, gpu_kap, gpu_osk, np64, score_tolerance,
                     shape_of, to_dev)

pytestmark = pytest.mark.gpu


def _oracle_args(wl, x):
    return dict(q=np64(x["q"]), k_pool=np64(x["k_pool"]), v_pool=np64(x["v_pool"]),
                page_table=x["page_table"].cpu().numpy())


# ---------------------------------------------------------------------------
# selection + ordering: bit-exact on identical fp32 scores
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("B,Hq,N,P,Bq,budget,sink,asc", [
    (1, 4, 8192, 64, 128, 0.2, 1, 0),
    (2, 3, 4096, 64, 64, 0.1, 1, 0),
    (1, 2, 8192, 128, 128, 0.37, 2, 0),
    (1, 2, 4096, 128, 64, 0.05, 0, 0),
    (1, 2, 4096, 64, 128, 0.25, 1, 1),
    (1, 2, 2048, 64, 128, 1.0, 1, 0),
    (1, 2, 2048, 64, 128, 0.0, 3, 0),
    (1, 1, 128, 64, 128, 0.5, 1, 0),
    (1, 1, 64, 64, 64, 0.5, 1, 0),
])
def test_kap_order_bit_exact(B, Hq, N, P, Bq, budget, sink, asc):
    si = W.make_score_inputs(B, Hq, N, P, Bq, seed=N + Hq)
    shape = C.Shape(B, Hq, 1, N, 128, P, Bq)
    kap = C.KapParams(budget=budget, sink_pages=sink, ascending=bool(asc))
    kc = C.cosa_kap_kcap(shape, kap)
    order = torch.full((B, Hq, N // Bq, kc), -7, dtype=torch.int32, device="cuda")
    count = torch.full((B, Hq, N // Bq), -7, dtype=torch.int32, device="cuda")
    C.cosa_kap_order(shape, kap, si["scores"].cuda(), si["hrm"].cuda(), order, count)
    torch.cuda.synchronize()
    want_o, want_c = O.kap_order(si["scores"].numpy(), si["hrm"].numpy(), page_size=P, q_block=Bq,
                                 budget=budget, sink_pages=sink, ascending=bool(asc))
    np.testing.assert_array_equal(count.cpu().numpy(), want_c)
    np.testing.assert_array_equal(order.cpu().numpy(), want_o)


# ---------------------------------------------------------------------------
# full KAP on generated inputs
# ---------------------------------------------------------------------------
KAP_CASES = {
    "tiny-2k": (W.WORKLOADS["tiny-2k"], 0.25),
    "gqa-4k-shuffled": (W.small_workload("gqa-32k", 4096, 8, 2, shuffle_pages=True), 0.25),
    "narrow-kv-4k-g7": (W.small_workload("narrow-kv-64k", 4096, 14, 2), 0.1),
    "wide-head-4k-p128": (W.small_workload("wide-head-128k", 4096, 16, 2), 0.15),
    "gqa-2k-bq64": (W.small_workload("gqa-32k", 2048, 4, 1, q_block=64), 0.3),
}


@pytest.mark.parametrize("case", sorted(KAP_CASES))
def test_kap_select_parity(case):
    wl, budget = KAP_CASES[case]
    x = W.make_inputs(wl, seed=1)
    xd = to_dev(x)
    shape = shape_of(wl, x)
    kap = C.KapParams(budget=budget, q_sub=wl.q_block // 4, k_sub=16, sink_pages=1)
    order, count, scores, hrm = gpu_kap(shape, kap, xd)
    o, c, S_g, h_g = (order.cpu().numpy(), count.cpu().numpy(), scores.cpu().numpy(),
                      hrm.cpu().numpy())
    oa = _oracle_args(wl, x)
    scale = 1 / math.sqrt(wl.head_dim)
    ref = O.kap_select(oa["q"], oa["k_pool"], oa["page_table"], num_kv_heads=wl.num_kv_heads,
                       page_size=wl.page_size, q_block=wl.q_block, q_sub=wl.q_block // 4,
                       k_sub=16, scale=scale, budget=budget, sink_pages=1)
    # score bound from the pooled magnitudes (see helpers.score_tolerance)
    G = wl.num_q_heads // wl.num_kv_heads
    bound = 0.0
    for b in range(wl.batch):
        for hk in range(wl.num_kv_heads):
            kh = O.kap_pool_keys(O.gather_logical(oa["k_pool"], oa["page_table"], b, hk),
                                 wl.page_size, 16)
            for h in range(hk * G, (hk + 1) * G):
                qh = O.kap_pool_queries(oa["q"][b, h], wl.q_block, wl.q_block // 4)
                bound = max(bound, scale * float(np.abs(qh).max(axis=(0, 1)) @ np.abs(kh).max(axis=(0, 1))))
    tol = score_tolerance(bound)
    np.testing.assert_array_equal(c, ref["count"])
    nP, nQB = wl.num_pages, wl.num_q_blocks
    n_hrm_diff = 0
    for b in range(wl.batch):
        for h in range(wl.num_q_heads):
            for qb in range(nQB):
                n_b = O.causal_pages(qb, wl.q_block, wl.page_size)
                dS = np.abs(S_g[b, h, qb, :n_b] - ref["S"][b, h, qb, :n_b])
                assert dS.max() <= tol, f"S off by {dS.max():.2e} > {tol:.2e} at {(b, h, qb)}"
                assert np.all(S_g[b, h, qb, n_b:] == 0) and np.all(h_g[b, h, qb, n_b:] == 0)
                if not np.array_equal(h_g[b, h, qb, :n_b], ref["hrm"][b, h, qb, :n_b]):
                    # allowed only where a representative's two best pages tie within rounding
                    n_hrm_diff += 1
                    _, _, _, a = O.kap_select_block(
                        oa["q"][b, h], O.gather_logical(oa["k_pool"], oa["page_table"], b,
                                                        h // G), qb, q_block=wl.q_block,
                        page_size=wl.page_size, q_sub=wl.q_block // 4, k_sub=16, scale=scale,
                        budget=budget, sink_pages=1)
                    top2 = np.sort(a, axis=1)[:, -2:]
                    assert np.min(top2[:, 1] - top2[:, 0]) <= 2 * tol
                check_order_valid(o[b, h, qb], int(c[b, h, qb]), ref["S"][b, h, qb],
                                  h_g[b, h, qb], qb, wl.q_block, wl.page_size, 1, budget, 2 * tol,
                                  False)
    assert n_hrm_diff <= max(1, wl.batch * wl.num_q_heads * nQB // 100)
    # bit-exact: the oracle's selection and order run on the GPU's own fp32 scores and
    # flags give the GPU's list (the fused order kernel ranks by exactly those values)
    want_o, want_c = O.kap_order(S_g, h_g, page_size=wl.page_size, q_block=wl.q_block,
                                 budget=budget, sink_pages=1)
    np.testing.assert_array_equal(c, want_c)
    np.testing.assert_array_equal(o, want_o)


def test_kap_planted_pages_first_on_gpu():
    wl = W.WORKLOADS["tiny-2k"]
    x = W.make_inputs(wl, seed=0)
    shape = shape_of(wl, x)
    kap = C.KapParams(budget=0.25, q_sub=16, k_sub=16, sink_pages=1)
    order, count, _, _ = gpu_kap(shape, kap, to_dev(x), export=False)
    o = order.cpu().numpy()
    for h in range(2):
        planted = set(x["planted"][0, h].tolist())
        for qb in range(wl.num_q_blocks - 4, wl.num_q_blocks):
            assert set(o[0, h, qb, :3].tolist()) == planted


def test_kap_unordered_mode_lists_same_set_ascending():
    wl = W.small_workload("gqa-32k", 4096, 4, 1)
    x = W.make_inputs(wl, seed=2)
    xd = to_dev(x)
    shape = shape_of(wl, x)
    o1, c1, _, _ = gpu_kap(shape, C.KapParams(budget=0.2, q_sub=32), xd, export=False)
    o2, c2, _, _ = gpu_kap(shape, C.KapParams(budget=0.2, q_sub=32, ascending=True), xd,
                           export=False)
    assert torch.equal(c1, c2)
    a, b = o1.cpu().numpy(), o2.cpu().numpy()
    for idx in np.ndindex(*c1.shape):
        n = int(c1[idx])
        assert sorted(a[idx][:n].tolist()) == b[idx][:n].tolist()


# ---------------------------------------------------------------------------
# OSK on the oracle's lists
# ---------------------------------------------------------------------------
OSK_CASES = {
    "tiny-2k": (W.WORKLOADS["tiny-2k"], 0.25, (1e-4, 0.0)),
    "gqa-4k": (W.small_workload("gqa-32k", 4096, 8, 2, shuffle_pages=True), 0.25, (1e-4, 1e-3, 0.0)),
    "narrow-kv-4k-g7": (W.small_workload("narrow-kv-64k", 4096, 7, 1, batch=2), 0.2, (1e-4,)),
    "wide-head-4k-p128": (W.small_workload("wide-head-128k", 4096, 8, 1), 0.3, (1e-4, 1e-5)),
    "gqa-2k-bq64": (W.small_workload("gqa-32k", 2048, 4, 1, q_block=64), 0.5, (1e-3,)),
}


def _osk_case(case, eps):
    wl, budget, _ = OSK_CASES[case]
    x = W.make_inputs(wl, seed=4)
    xd = to_dev(x)
    shape = shape_of(wl, x)
    oa = _oracle_args(wl, x)
    scale = 1 / math.sqrt(wl.head_dim)
    sel = O.kap_select(oa["q"], oa["k_pool"], oa["page_table"], num_kv_heads=wl.num_kv_heads,
                       page_size=wl.page_size, q_block=wl.q_block, q_sub=wl.q_block // 4,
                       k_sub=16, scale=scale, budget=budget, sink_pages=1)
    order = torch.from_numpy(sel["order"]).cuda()
    count = torch.from_numpy(sel["count"]).cuda()
    out, lse, computed, skip = gpu_osk(shape, eps, xd, order, count)
    ref = O.osk_attention(oa["q"], oa["k_pool"], oa["v_pool"], oa["page_table"], sel["order"],
                          sel["count"], num_kv_heads=wl.num_kv_heads, page_size=wl.page_size,
                          q_block=wl.q_block, eps=eps, scale=scale)
    return wl, x, sel, ref, np64(out), lse.cpu().numpy(), computed.cpu().numpy(), skip.cpu().numpy()


@pytest.mark.parametrize("case,eps", [(c, e) for c in sorted(OSK_CASES) for e in OSK_CASES[c][2]])
def test_osk_parity(case, eps):
    wl, x, sel, ref, out, lse, computed, skip = _osk_case(case, eps)
    cnt = sel["count"]
    vmax = float(np.abs(np64(x["v_pool"])).max())
    rows_ok = np.ones(out.shape[:3], dtype=bool)
    n_amb = n_dis = n_steps = 0
    for idx in np.ndindex(*cnt.shape):
        b, h, qb = idx
        n = int(cnt[idx])
        n_steps += n
        gs, rs, mg = skip[idx][:n], ref["skip"][idx][:n], ref["margin"][idx][:n]
        assert np.all(skip[idx][n:] == 7), "skip log written past count"
        assert computed[idx] == n - int(gs.sum())
        amb = np.abs(mg) <= SKIP_MARGIN
        n_amb += int(amb.sum())
        dis = gs != rs
        assert not np.any(dis & ~amb), f"skip decision differs outside the margin at {idx}"
        if dis.any():
            n_dis += int(dis.sum())
            rows = slice(qb * wl.q_block, (qb + 1) * wl.q_block)
            rows_ok[b, h, rows] = False
            # the alternative decision moves the output by at most the skip error bound
            bound = 2 * int(dis.sum()) * wl.page_size * eps * vmax
            assert np.abs(out[b, h, rows] - ref["out"][b, h, rows]).max() <= bound + 2e-2
        else:
            assert computed[idx] == ref["computed"][idx]
    assert n_amb <= max(2, n_steps // 1000), f"{n_amb} of {n_steps} steps within the skip margin"
    assert_out_close(out, ref["out"], f"osk {case} eps={eps}", rows_mask=rows_ok)
    assert_lse_close(lse, ref["lse"], f"osk {case} eps={eps}", rows_mask=rows_ok)
    if eps > 0 and case != "tiny-2k":
        assert skip.sum() > 0 or wl.drift_sigma == 0


def test_osk_full_budget_no_skip_equals_dense_and_is_order_invariant():
    wl = W.small_workload("gqa-32k", 4096, 4, 1, shuffle_pages=True)
    x = W.make_inputs(wl, seed=6)
    xd = to_dev(x)
    shape = shape_of(wl, x)
    order, count, _, _ = gpu_kap(shape, C.KapParams(budget=1.0, q_sub=32), xd, export=False)
    assert torch.all(count == torch.tensor([O.causal_pages(qb, 128, 64) for qb in range(32)],
                                           dtype=torch.int32, device="cuda"))
    out1, lse1, comp1, _ = gpu_osk(shape, 0.0, xd, order, count)
    assert torch.equal(comp1, count)
    # a seeded random permutation of every list (host-side)
    g = np.random.default_rng(7)
    o = order.cpu().numpy().copy()
    for idx in np.ndindex(*count.shape):
        n = int(count[idx])
        o[idx][:n] = g.permutation(o[idx][:n])
    out2, lse2, _, _ = gpu_osk(shape, 0.0, xd, torch.from_numpy(o).cuda(), count)
    oa = _oracle_args(wl, x)
    dense = O.dense_attention(oa["q"], oa["k_pool"], oa["v_pool"], oa["page_table"],
                              num_kv_heads=1, scale=1 / math.sqrt(128))
    assert_out_close(np64(out1), dense["out"], "osk beta=1 vs dense")
    assert_out_close(np64(out2), dense["out"], "osk permuted vs dense")
    assert_lse_close(lse1.cpu().numpy(), dense["lse"], "lse beta=1")
    # order invariance on the GPU itself: fp32 reassociation only
    d = (np64(out1) - np64(out2))
    assert np.abs(d).max() <= 2 ** -7 * max(1.0, float(np.abs(np64(out1)).max()))


def test_osk_never_reads_unlisted_pages():
    """Lists are built host-side from a seeded generator: the forced pages plus
    random odd pages.  The even pages 2..18 are then filled with NaN, as are
    physical pages no page-table entry names.  A q-block from 10 on lists none
    of them (its own pages are 2qb, 2qb+1 >= 20), so its output must not change
    by a single bit; earlier q-blocks own a poisoned page and are not checked."""
    wl = W.small_workload("gqa-32k", 4096, 4, 1, shuffle_pages=True)
    x = W.make_inputs(wl, seed=8)
    xd = to_dev(x)
    B, nP, nQB, Hq = 1, wl.num_pages, wl.num_q_blocks, 4
    extra = 5
    nanpad = lambda t: torch.cat([t, torch.full((extra,) + tuple(t.shape[1:]), float("nan"),
                                                dtype=t.dtype, device=t.device)])
    kp, vp = nanpad(xd["k_pool"]), nanpad(xd["v_pool"])
    pt = torch.full((B, nP + 3), -1, dtype=torch.int32, device="cuda")   # stride > nP
    pt[:, :nP] = xd["page_table"]
    shape = C.Shape(1, 4, 1, 4096, 128, 64, 128, pages_per_seq=nP + 3,
                    num_phys_pages=B * nP + extra)
    g = np.random.default_rng(8)
    kc = O.causal_pages(nQB - 1, 128, 64)
    o = np.full((B, Hq, nQB, kc), -1, dtype=np.int32)
    c = np.zeros((B, Hq, nQB), dtype=np.int32)
    for h in range(Hq):
        for qb in range(nQB):
            n_b = O.causal_pages(qb, 128, 64)
            forced = O.forced_pages(qb, 128, 64, 1)
            odds = [p for p in range(1, n_b, 2) if p not in forced]
            pick = [int(p) for p in g.permutation(odds)[:len(odds) // 2]]
            lst = [int(p) for p in g.permutation(forced + pick)]
            o[0, h, qb, :len(lst)] = lst
            c[0, h, qb] = len(lst)
    order, count = torch.from_numpy(o).cuda(), torch.from_numpy(c).cuda()
    xd2 = dict(xd, k_pool=kp, v_pool=vp, page_table=pt)
    out_a, lse_a, _, _ = gpu_osk(shape, 1e-4, xd2, order, count)
    poisoned = list(range(2, 20, 2))
    phys = pt[0, torch.tensor(poisoned, device="cuda")].long()
    kp2, vp2 = kp.clone(), vp.clone()
    kp2[phys] = float("nan")
    vp2[phys] = float("nan")
    out_b, lse_b, _, _ = gpu_osk(shape, 1e-4, dict(xd2, k_pool=kp2, v_pool=vp2), order, count)
    r0 = 10 * 128
    assert torch.isfinite(out_a.float()).all()
    assert torch.equal(out_a[:, :, r0:], out_b[:, :, r0:])
    assert torch.equal(lse_a[:, :, r0:], lse_b[:, :, r0:])
    assert not torch.isfinite(out_b[:, :, :r0].float()).all()   # the poison is really read there
    # and the OSK result on these lists matches the oracle on them
    oa = _oracle_args(wl, x)
    ref = O.osk_attention(oa["q"], oa["k_pool"], oa["v_pool"], oa["page_table"], o, c,
                          num_kv_heads=1, page_size=64, q_block=128, eps=1e-4,
                          scale=1 / math.sqrt(128))
    # every tile whose decisions are clear of the threshold's rounding is compared
    # element-wise (check_osk_tiles), the others against the skip error bound
    tiles = [(0, h, qb) for h in range(Hq) for qb in range(nQB)]
    skip_a = torch.full((B, Hq, nQB, kc), 7, dtype=torch.uint8, device="cuda")
    comp_a = torch.full((B, Hq, nQB), -7, dtype=torch.int32, device="cuda")
    out_c = torch.empty_like(out_a)
    lse_c = torch.empty_like(lse_a)
    C.cosa_osk_attention(shape, C.OskParams(1e-4), xd2["q"], kp, vp, pt, order, count, out_c,
                         lse=lse_c, computed=comp_a, skip_log=skip_a)
    torch.cuda.synchronize()
    assert C.cosa_get_status() == 0
    assert torch.equal(out_c, out_a)
    check_osk_tiles(skip_a.cpu().numpy(), comp_a.cpu().numpy(), np64(out_a), lse_a.cpu().numpy(),
                    ref, c, tiles, 128, 64, 1e-4, float(np.abs(oa["v_pool"]).max()),
                    "osk on host-built lists")


def test_osk_infinite_eps_with_page0_first():
    wl = W.small_workload("gqa-32k", 2048, 2, 1)
    x = W.make_inputs(wl, seed=9)
    xd = to_dev(x)
    shape = shape_of(wl, x)
    nQB = wl.num_q_blocks
    kc = O.causal_pages(nQB - 1, 128, 64)
    o = np.full((1, 2, nQB, kc), -1, dtype=np.int32)
    c = np.zeros((1, 2, nQB), dtype=np.int32)
    for h in range(2):
        for qb in range(nQB):
            n = O.causal_pages(qb, 128, 64)
            o[0, h, qb, :n] = np.arange(n)
            c[0, h, qb] = n
    out, _, computed, _ = gpu_osk(shape, math.inf, xd, torch.from_numpy(o).cuda(),
                                  torch.from_numpy(c).cuda())
    oa = _oracle_args(wl, x)
    ref = O.osk_attention(oa["q"], oa["k_pool"], oa["v_pool"], oa["page_table"], o, c,
                          num_kv_heads=1, page_size=64, q_block=128, eps=math.inf,
                          scale=1 / math.sqrt(128))
    np.testing.assert_array_equal(computed.cpu().numpy(), ref["computed"])
    assert_out_close(np64(out), ref["out"], "eps=inf")


# ---------------------------------------------------------------------------
# dense
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("case", ["tiny-2k", "gqa-4k", "wide-head-4k-p128", "gqa-2k-bq64",
                                  "single-qblock", "single-page", "ragged-320", "ragged-448"])
def test_dense_parity(case):
    # the dense kernel takes query rows in pairs of 128-row tiles: N = 64 and 320 end
    # on a 64-row first tile, 448 on a 64-row second tile with a 64-key diagonal block
    extra = {"single-qblock": W.small_workload("gqa-32k", 128, 2, 1, planted_frac=0.0),
             "single-page": W.small_workload("gqa-32k", 64, 2, 1, q_block=64, planted_frac=0.0),
             "ragged-320": W.small_workload("gqa-32k", 320, 4, 2, q_block=64, planted_frac=0.0),
             "ragged-448": W.small_workload("gqa-32k", 448, 3, 1, q_block=64, planted_frac=0.0)}
    wl = extra[case] if case in extra else OSK_CASES[case][0]
    x = W.make_inputs(wl, seed=10)
    xd = to_dev(x)
    shape = shape_of(wl, x)
    out, lse = gpu_dense(shape, xd)
    oa = _oracle_args(wl, x)
    ref = O.dense_attention(oa["q"], oa["k_pool"], oa["v_pool"], oa["page_table"],
                            num_kv_heads=wl.num_kv_heads, scale=1 / math.sqrt(wl.head_dim))
    assert_out_close(np64(out), ref["out"], f"dense {case}")
    assert_lse_close(lse.cpu().numpy(), ref["lse"], f"dense {case}")


def test_status_word_clear_after_runs():
    assert C.cosa_get_status() == 0


# ---------------------------------------------------------------------------
# early break (max_run): not part of the pages' method; parity with the oracle's
# osk_block_rules(max_run=r)
# ---------------------------------------------------------------------------
BREAK_CASES = {  # workload, budget, eps, max_run values (eps large enough that tiles break)
    "gqa-4k": (W.small_workload("gqa-32k", 4096, 8, 2, shuffle_pages=True), 0.25, 0.5, (2, 3)),
    "narrow-kv-4k-g7": (W.small_workload("narrow-kv-64k", 4096, 7, 1, batch=2), 0.2, 1e-4, (2, 3)),
    "wide-head-4k-p128": (W.small_workload("wide-head-128k", 4096, 8, 1), 0.3, 0.5, (2, 3)),
}


@pytest.mark.parametrize("case,r", [(c, r) for c in sorted(BREAK_CASES) for r in BREAK_CASES[c][3]])
def test_osk_early_break_parity(case, r):
    """The skip log equals the oracle's decisions page for page: where a decision lies
    within rounding of the threshold, the oracle takes the kernel's decision there and
    runs on (the break point moves with it); the first difference always precedes any
    break, so its margin is defined.  Outputs and LSE then match the oracle run that
    takes the same decisions, and some tiles do break."""
    wl, budget, eps, _ = BREAK_CASES[case]
    x = W.make_inputs(wl, seed=4)
    xd = to_dev(x)
    shape = shape_of(wl, x)
    oa = _oracle_args(wl, x)
    scale = 1 / math.sqrt(wl.head_dim)
    sel = O.kap_select(oa["q"], oa["k_pool"], oa["page_table"], num_kv_heads=wl.num_kv_heads,
                       page_size=wl.page_size, q_block=wl.q_block, q_sub=wl.q_block // 4,
                       k_sub=16, scale=scale, budget=budget, sink_pages=1)
    order = torch.from_numpy(sel["order"]).cuda()
    count = torch.from_numpy(sel["count"]).cuda()
    out, lse, computed, skip = gpu_osk(shape, eps, xd, order, count, max_run=r)
    out, lse = np64(out), lse.cpu().numpy()
    computed, skip = computed.cpu().numpy(), skip.cpu().numpy()
    want_out = np.zeros_like(out)
    want_lse = np.full_like(lse, -np.inf)
    G = wl.num_q_heads // wl.num_kv_heads
    N, Bq, P = wl.seq_len, wl.q_block, wl.page_size
    logical = {}
    n_breaks = n_forced = 0
    for idx in np.ndindex(*sel["count"].shape):
        b, h, qb = idx
        n = int(sel["count"][idx])
        lst = sel["order"][idx][:n]
        if (b, h // G) not in logical:
            logical[(b, h // G)] = (O.gather_logical(oa["k_pool"], oa["page_table"], b, h // G, N),
                                    O.gather_logical(oa["v_pool"], oa["page_table"], b, h // G, N))
        k_log, v_log = logical[(b, h // G)]
        rows = slice(qb * Bq, (qb + 1) * Bq)
        gs = skip[idx][:n]
        assert np.all(skip[idx][n:] == 7), "skip log written past count"
        force = {}
        for _ in range(n + 1):
            ref = O.osk_block_rules(oa["q"][b, h, rows], k_log, v_log, qb, Bq, P, lst, eps, scale,
                                    force=force, max_run=r)
            dis = np.nonzero(gs != ref["skip"])[0]
            if len(dis) == 0:
                break
            j = int(dis[0])
            assert abs(ref["margin"][j]) <= SKIP_MARGIN, f"decision differs outside the margin at {idx}"
            force[j] = bool(gs[j])
        assert np.array_equal(gs, ref["skip"])
        assert computed[idx] == ref["computed"]
        want_out[b, h, rows] = ref["out"]
        want_lse[b, h, rows] = ref["lse"]
        n_breaks += int(ref["visited"] < n)
        n_forced += len(force)
    n_tiles = int(np.prod(sel["count"].shape))
    assert n_forced <= max(2, n_tiles // 100), f"{n_forced} decisions within the skip margin"
    assert_out_close(out, want_out, f"osk break {case} r={r}")
    assert_lse_close(lse, want_lse, f"osk break {case} r={r}")
    assert n_breaks > 0, "no tile broke early: the case does not exercise the break"


def test_kap_pool_then_rank_equals_kap_select():
    """The two stage entry points on one workspace are cosa_kap_select, bit for bit."""
    wl = W.small_workload("narrow-kv-64k", 4096, 14, 2, batch=2)
    x = W.make_inputs(wl, seed=12)
    xd = to_dev(x)
    shape = shape_of(wl, x)
    kap = C.KapParams(budget=0.2, q_sub=32, k_sub=16, sink_pages=1)
    o1, c1, s1, h1 = gpu_kap(shape, kap, xd)
    o2, c2, s2, h2 = (torch.full_like(o1, -7), torch.full_like(c1, -7), torch.full_like(s1, -1),
                      torch.full_like(h1, 9))
    ws = torch.empty(C.cosa_kap_workspace_size(shape, kap), dtype=torch.uint8, device="cuda")
    C.cosa_kap_pool(shape, kap, xd["q"], xd["k_pool"], xd["page_table"], ws)
    C.cosa_kap_rank(shape, kap, o2, c2, ws, scores=s2, hrm=h2)
    torch.cuda.synchronize()
    assert C.cosa_get_status() == 0
    assert torch.equal(o1, o2) and torch.equal(c1, c2)
    assert torch.equal(s1, s2) and torch.equal(h1, h2)
