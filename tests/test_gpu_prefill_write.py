"""The prefill's write of Q / K / V with KAP's downsampling fused in
(cosa_prefill_write): the written head-major Q and paged K / V equal the inputs bit
for bit, and Stage 1 finished from the fused pooling (cosa_kap_rank) equals
cosa_kap_select on the written tensors bit for bit: lists, counts, scores and HRM
flags (gist.science/pt §2.2: the same downsampling, only read once)."""
import pytest
import torch

import block_sparse_long_kap_b200 as C
import workloads as W
from helpers import gpu_kap, shape_of

pytestmark = pytest.mark.gpu

CASES = {
    "gqa-4k-shuffled": W.small_workload("gqa-32k", 4096, 8, 2, shuffle_pages=True),
    "narrow-kv-4k-g7-b2": W.small_workload("narrow-kv-64k", 4096, 14, 2, batch=2, shuffle_pages=True),
    "wide-head-4k-p128": W.small_workload("wide-head-128k", 4096, 16, 2),
    "tiny-2k-d64": W.WORKLOADS["tiny-2k"],
}


@pytest.mark.parametrize("case", sorted(CASES))
def test_fused_write_and_pooling(case):
    wl = CASES[case]
    x = W.make_inputs(wl, seed=81, device="cuda", keep_logical=True)
    shape = shape_of(wl, x)
    kap = C.KapParams(budget=0.25, q_sub=wl.q_block // 4, k_sub=16, sink_pages=1)
    q_tok = x["q"].permute(0, 2, 1, 3).contiguous()
    k_tok = x["k_log"].permute(0, 2, 1, 3).contiguous()
    v_tok = x["v_log"].permute(0, 2, 1, 3).contiguous()
    for pooled in (True, False):
        q = torch.full_like(x["q"], float("nan"))
        kp = torch.full_like(x["k_pool"], float("nan"))
        vp = torch.full_like(x["v_pool"], float("nan"))
        ws = torch.empty(C.cosa_kap_workspace_size(shape, kap), dtype=torch.uint8, device="cuda")
        C.cosa_prefill_write(shape, kap, q_tok, k_tok, v_tok, x["page_table"], q, kp, vp,
                             workspace=ws if pooled else None)
        torch.cuda.synchronize()
        assert C.cosa_get_status() == 0
        assert torch.equal(q, x["q"]) and torch.equal(kp, x["k_pool"]) and torch.equal(vp, x["v_pool"])
        if not pooled:
            continue
        kc = C.cosa_kap_kcap(shape, kap)
        B, Hq, nQB, nP = wl.batch, wl.num_q_heads, wl.num_q_blocks, wl.num_pages
        o2 = torch.full((B, Hq, nQB, kc), -7, dtype=torch.int32, device="cuda")
        c2 = torch.full((B, Hq, nQB), -7, dtype=torch.int32, device="cuda")
        s2 = torch.full((B, Hq, nQB, nP), -1.0, device="cuda")
        h2 = torch.full((B, Hq, nQB, nP), 9, dtype=torch.uint8, device="cuda")
        C.cosa_kap_rank(shape, kap, o2, c2, ws, scores=s2, hrm=h2)
        torch.cuda.synchronize()
        assert C.cosa_get_status() == 0
        o1, c1, s1, h1 = gpu_kap(shape, kap, dict(x, q=q, k_pool=kp))
        assert torch.equal(o1, o2) and torch.equal(c1, c2)
        assert torch.equal(s1, s2) and torch.equal(h1, h2)


def test_fused_write_padded_page_table_and_spare_pages():
    """A page-table row longer than the sequence's pages and a pool with spare physical
    pages: the named pages are written, the spare ones left untouched."""
    wl = W.small_workload("gqa-32k", 2048, 4, 2, shuffle_pages=True)
    x = W.make_inputs(wl, seed=82, device="cuda", keep_logical=True)
    nP, extra = wl.num_pages, 3
    pt = torch.full((1, nP + 5), -1, dtype=torch.int32, device="cuda")
    pt[:, :nP] = x["page_table"] + extra  # physical pages extra .. extra + nP - 1
    shape = C.Shape(1, 4, 2, 2048, 128, 64, 128, pages_per_seq=nP + 5, num_phys_pages=nP + extra)
    kap = C.KapParams(budget=0.25, q_sub=32, k_sub=16, sink_pages=1)
    q_tok = x["q"].permute(0, 2, 1, 3).contiguous()
    k_tok = x["k_log"].permute(0, 2, 1, 3).contiguous()
    v_tok = x["v_log"].permute(0, 2, 1, 3).contiguous()
    q = torch.full_like(x["q"], float("nan"))
    kp = torch.full((nP + extra, 2, 64, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    vp = torch.full_like(kp, 7.0)
    ws = torch.empty(C.cosa_kap_workspace_size(shape, kap), dtype=torch.uint8, device="cuda")
    C.cosa_prefill_write(shape, kap, q_tok, k_tok, v_tok, pt, q, kp, vp, workspace=ws)
    torch.cuda.synchronize()
    assert C.cosa_get_status() == 0
    assert torch.equal(q, x["q"])
    assert torch.equal(kp[extra:], x["k_pool"]) and torch.equal(vp[extra:], x["v_pool"])
    assert bool(torch.all(kp[:extra] == 7.0)) and bool(torch.all(vp[:extra] == 7.0))


def test_fused_write_page_outside_the_pool_is_reported_not_written():
    """A page-table entry outside [0, num_phys_pages): reported in the status word,
    that page written nowhere, every other page and Q written exactly, and the pooled
    key vectors (taken from the token-major input) unchanged, so Stage 1 from the
    workspace equals cosa_kap_select on the intended tensors."""
    wl = W.small_workload("gqa-32k", 2048, 4, 2, shuffle_pages=True)
    x = W.make_inputs(wl, seed=83, device="cuda", keep_logical=True)
    shape = shape_of(wl, x)
    kap = C.KapParams(budget=0.25, q_sub=32, k_sub=16, sink_pages=1)
    bad_page = 9
    pt = x["page_table"].clone()
    lost = int(pt[0, bad_page])
    pt[0, bad_page] = wl.num_pages  # one past the pool
    q_tok = x["q"].permute(0, 2, 1, 3).contiguous()
    k_tok = x["k_log"].permute(0, 2, 1, 3).contiguous()
    v_tok = x["v_log"].permute(0, 2, 1, 3).contiguous()
    q = torch.full_like(x["q"], float("nan"))
    kp = torch.full_like(x["k_pool"], 3.0)
    vp = torch.full_like(x["v_pool"], 3.0)
    ws = torch.empty(C.cosa_kap_workspace_size(shape, kap), dtype=torch.uint8, device="cuda")
    C.cosa_prefill_write(shape, kap, q_tok, k_tok, v_tok, pt, q, kp, vp, workspace=ws)
    torch.cuda.synchronize()
    assert C.cosa_get_status() == 1  # COSA_ERR_INVALID_ARG
    keep = [p for p in range(wl.num_pages) if p != lost]
    assert torch.equal(q, x["q"])
    assert torch.equal(kp[keep], x["k_pool"][keep]) and torch.equal(vp[keep], x["v_pool"][keep])
    assert bool(torch.all(kp[lost] == 3.0)) and bool(torch.all(vp[lost] == 3.0))
    kc = C.cosa_kap_kcap(shape, kap)
    o2 = torch.full((1, 4, wl.num_q_blocks, kc), -7, dtype=torch.int32, device="cuda")
    c2 = torch.full((1, 4, wl.num_q_blocks), -7, dtype=torch.int32, device="cuda")
    C.cosa_kap_rank(shape, kap, o2, c2, ws)
    torch.cuda.synchronize()
    assert C.cosa_get_status() == 0
    o1, c1, _, _ = gpu_kap(shape, kap, x, export=False)
    assert torch.equal(o1, o2) and torch.equal(c1, c2)


def test_kap_pooling_page_outside_the_pool_is_reported_not_read():
    """cosa_kap_select with a page-table entry outside the pool: reported, the page
    not read (its pooled keys zero), every list still a valid list of causal pages."""
    wl = W.small_workload("gqa-32k", 2048, 4, 2)
    x = W.make_inputs(wl, seed=84, device="cuda")
    shape = shape_of(wl, x)
    kap = C.KapParams(budget=0.25, q_sub=32, k_sub=16, sink_pages=1)
    pt = x["page_table"].clone()
    pt[0, 20] = -3
    kc = C.cosa_kap_kcap(shape, kap)
    order = torch.full((1, 4, wl.num_q_blocks, kc), -7, dtype=torch.int32, device="cuda")
    count = torch.full((1, 4, wl.num_q_blocks), -7, dtype=torch.int32, device="cuda")
    ws = torch.empty(C.cosa_kap_workspace_size(shape, kap), dtype=torch.uint8, device="cuda")
    C.cosa_kap_select(shape, kap, x["q"], x["k_pool"], pt, order, count, ws)
    torch.cuda.synchronize()
    assert C.cosa_get_status() == 1
    for qb in range(wl.num_q_blocks):
        n_b = (qb + 1) * wl.q_block // wl.page_size
        for h in range(4):
            n = int(count[0, h, qb])
            lst = order[0, h, qb, :n].tolist()
            assert 1 <= n <= n_b and len(set(lst)) == n and all(0 <= p < n_b for p in lst)
