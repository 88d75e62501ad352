"""GPU parity of the proxy-bound pre-skip (cosa_kap_preskip; a variant the pages do
not give) against the oracle's kap_preskip on the same ordered lists.

The kernel decides in fp32 on its own page maxima a[r][p] (tensor-core scores),
the oracle in float64 on its own: decisions are compared bit for bit wherever the
oracle's tested quantity lies farther than twice the derived score bound from the
threshold, and the compacted list must be the GPU's original list with exactly the
logged positions removed.  Then the pages' rule (cosa_osk_attention) runs on the
survivors and is compared with the oracle on the same survivors."""
import math

import numpy as np
import pytest
import torch

import block_sparse_long_kap_b200 as C
import oracle as O
import workloads as W
from helpers import check_osk_tiles, gpu_osk, np64, score_tolerance, shape_of, to_dev

pytestmark = pytest.mark.gpu


def _gpu_lists(wl, x, budget):
    xd = to_dev(x) if not x["q"].is_cuda else x
    shape = shape_of(wl, xd)
    kap = C.KapParams(budget=budget, q_sub=wl.q_block // 4, k_sub=16, sink_pages=1)
    kc = C.cosa_kap_kcap(shape, kap)
    B, Hq, nQB = wl.batch, wl.num_q_heads, wl.num_q_blocks
    order = torch.full((B, Hq, nQB, kc), -7, dtype=torch.int32, device="cuda")
    count = torch.full((B, Hq, nQB), -7, dtype=torch.int32, device="cuda")
    ws = torch.empty(C.cosa_kap_workspace_size(shape, kap), dtype=torch.uint8, device="cuda")
    C.cosa_kap_select(shape, kap, xd["q"], xd["k_pool"], xd["page_table"], order, count, ws)
    return xd, shape, kap, order, count, ws


def _oracle_a(wl, xh, tiles):
    """The oracle's page maxima a [R][n_b] of the given tiles, and the score bound."""
    G = wl.num_q_heads // wl.num_kv_heads
    scale = 1 / math.sqrt(wl.head_dim)
    out, khats, bound = {}, {}, 0.0
    for (b, h, qb) in tiles:
        hk = h // G
        if (b, hk) not in khats:
            khats[(b, hk)] = O.kap_pool_keys(O.gather_logical(xh["k_pool"], xh["page_table"], b, hk),
                                             wl.page_size, 16)
        khat = khats[(b, hk)]
        qh = O.kap_pool_queries(xh["q"][b, h], wl.q_block, wl.q_block // 4)
        bound = max(bound, scale * float(np.abs(qh).max(axis=(0, 1)) @ np.abs(khat).max(axis=(0, 1))))
        *_, a = O.kap_select_block(xh["q"][b, h], None, qb, q_block=wl.q_block,
                                   page_size=wl.page_size, q_sub=wl.q_block // 4, k_sub=16,
                                   scale=scale, budget=1.0, sink_pages=1, khat=khat)
        out[(b, h, qb)] = a
    return out, score_tolerance(bound)


def _check_filter(o0, c0, o1, c1, log, ref, tiles, tol):
    n_amb = n_pre = 0
    for idx in tiles:
        n = int(c0[idx])
        gs = log[idx][:n]
        assert np.all(log[idx][n:] == 7), f"pre-skip log written past count at {idx}"
        rs, mg = ref["skipped"][idx][:n], ref["margin"][idx][:n]
        amb = np.abs(np.nan_to_num(mg, nan=np.inf)) <= 2 * tol
        n_amb += int(amb.sum())
        dis = (gs != rs) & ~amb
        assert not dis.any(), f"pre-skip decision differs outside the rounding band at {idx}"
        assert gs[0] == 0, "the first listed page is never pre-skipped"
        survivors = o0[idx][:n][gs == 0]
        assert int(c1[idx]) == len(survivors)
        assert o1[idx][:len(survivors)].tolist() == survivors.tolist()
        assert np.all(o1[idx][len(survivors):] == -1)
        n_pre += int(gs.sum())
    return n_amb, n_pre


@pytest.mark.parametrize("eps,margin", [(1e-2, 0.0), (1e-3, 0.0), (1e-2, 1.0)])
def test_preskip_parity_and_osk_on_survivors(eps, margin):
    wl = W.small_workload("gqa-32k", 4096, 8, 2, shuffle_pages=True)
    x = W.make_inputs(wl, seed=61)
    xd, shape, kap, order, count, ws = _gpu_lists(wl, x, 0.5)
    o0, c0 = order.cpu().numpy(), count.cpu().numpy()
    log = torch.full(tuple(order.shape), 7, dtype=torch.uint8, device="cuda")
    C.cosa_kap_preskip(shape, kap, eps, margin, order, count, ws, skip_log=log)
    torch.cuda.synchronize()
    assert C.cosa_get_status() == 0
    o1, c1, lg = order.cpu().numpy(), count.cpu().numpy(), log.cpu().numpy()
    xh = dict(q=np64(x["q"]), k_pool=np64(x["k_pool"]), v_pool=np64(x["v_pool"]),
              page_table=x["page_table"].cpu().numpy())
    tiles = [(0, h, qb) for h in range(wl.num_q_heads) for qb in range(wl.num_q_blocks)]
    a, tol = _oracle_a(wl, xh, tiles)
    ref = O.kap_preskip_lists(o0, c0, lambda b, h, qb: a[(b, h, qb)], eps, margin, tiles=tiles)
    n_amb, n_pre = _check_filter(o0, c0, o1, c1, lg, ref, tiles, tol)
    assert n_pre > 0, "the case removes no page"
    assert n_amb <= max(4, int(c0.sum()) // 500)
    # the pages' rule on the survivors
    out, lse, computed, skip = gpu_osk(shape, 1e-4, xd, order, count)
    oref = O.osk_attention(xh["q"], xh["k_pool"], xh["v_pool"], xh["page_table"], o1, c1,
                           num_kv_heads=wl.num_kv_heads, page_size=64, q_block=128, eps=1e-4,
                           scale=1 / math.sqrt(128))
    check_osk_tiles(skip.cpu().numpy(), computed.cpu().numpy(), np64(out), lse.cpu().numpy(), oref,
                    c1, tiles, 128, 64, 1e-4, float(np.abs(xh["v_pool"]).max()),
                    f"osk after pre-skip eps={eps} margin={margin}")


def test_preskip_off_leaves_the_lists():
    wl = W.small_workload("narrow-kv-64k", 4096, 7, 1, batch=2)
    x = W.make_inputs(wl, seed=62)
    xd, shape, kap, order, count, ws = _gpu_lists(wl, x, 0.2)
    o0, c0 = order.clone(), count.clone()
    log = torch.full(tuple(order.shape), 7, dtype=torch.uint8, device="cuda")
    C.cosa_kap_preskip(shape, kap, 0.0, 0.0, order, count, ws, skip_log=log)
    torch.cuda.synchronize()
    assert C.cosa_get_status() == 0
    assert torch.equal(order, o0) and torch.equal(count, c0)
    for idx in np.ndindex(*c0.shape):
        n = int(c0[idx])
        assert int(log[idx][:n].sum()) == 0 and bool(torch.all(log[idx][n:] == 7))


def test_preskip_128k_long_lists():
    wl = W.small_workload("gqa-128k", 131072, 1, 1)
    x = W.make_inputs(wl, seed=63, device="cuda")
    xd, shape, kap, order, count, ws = _gpu_lists(wl, x, 0.2)
    o0, c0 = order.cpu().numpy(), count.cpu().numpy()
    log = torch.full(tuple(order.shape), 7, dtype=torch.uint8, device="cuda")
    C.cosa_kap_preskip(shape, kap, 1e-3, 0.0, order, count, ws, skip_log=log)
    torch.cuda.synchronize()
    assert C.cosa_get_status() == 0
    o1, c1, lg = order.cpu().numpy(), count.cpu().numpy(), log.cpu().numpy()
    xh = dict(q=np64(x["q"]), k_pool=np64(x["k_pool"]), page_table=x["page_table"].cpu().numpy())
    tiles = [(0, 0, qb) for qb in (1023, 1022, 1021, 1020, 800, 512, 256, 64)]
    a, tol = _oracle_a(wl, xh, tiles)
    ref = O.kap_preskip_lists(o0, c0, lambda b, h, qb: a[(b, h, qb)], 1e-3, 0.0, tiles=tiles)
    n_amb, n_pre = _check_filter(o0, c0, o1, c1, lg, ref, tiles, tol)
    # positions within twice the score bound of the threshold may go either way
    assert n_pre > 0 and n_amb <= max(4, sum(int(c0[t]) for t in tiles) // 500)
    # every other tile: the compaction matches its own log
    for qb in range(1024):
        n = int(c0[0, 0, qb])
        keep = o0[0, 0, qb, :n][lg[0, 0, qb, :n] == 0]
        assert int(c1[0, 0, qb]) == len(keep) and o1[0, 0, qb, :len(keep)].tolist() == keep.tolist()


def test_preskip_invalid_list_is_reported_and_left():
    wl = W.small_workload("gqa-32k", 2048, 2, 1)
    x = W.make_inputs(wl, seed=64)
    xd, shape, kap, order, count, ws = _gpu_lists(wl, x, 0.5)
    assert int(count[0, 0, 5]) >= 2
    order[0, 0, 5, 1] = 40  # q-block 5 sees pages 0..11 only
    o0, c0 = order.clone(), count.clone()
    C.cosa_kap_preskip(shape, kap, 1e-2, 0.0, order, count, ws)
    torch.cuda.synchronize()
    assert C.cosa_get_status() == 1  # COSA_ERR_INVALID_ARG
    assert torch.equal(order[0, 0, 5], o0[0, 0, 5]) and count[0, 0, 5] == c0[0, 0, 5]
    # the other lists were filtered: each is a subsequence of its input that keeps its
    # first page
    for (b, h, qb) in [(0, 0, 4), (0, 1, 10), (0, 1, 15)]:
        n0, n = int(c0[b, h, qb]), int(count[b, h, qb])
        src, got = o0[b, h, qb, :n0].tolist(), order[b, h, qb, :n].tolist()
        assert got[0] == src[0] and 1 <= n <= n0
        it = iter(src)
        assert all(pg in it for pg in got)
