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
