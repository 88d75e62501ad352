"""GPU parity of single-query decode (cosa_osk_decode) against the oracle's
osk_decode on the same lists: skip decisions bit-exact outside a float64 margin,
outputs within max-abs 2e-2 / mean-abs 2e-3, LSE and computed counts (the pages'
in-kernel rule, gist.science/pt §2.3, as a q-block of one row)."""
import math

import numpy as np
import pytest
import torch

import block_sparse_long_kap_b200 as C
import oracle as O
import workloads as W
from helpers import (SKIP_MARGIN, assert_lse_close, assert_out_close, gpu_kap, np64, shape_of,
                     to_dev)

pytestmark = pytest.mark.gpu


def _decode(shape, eps, xd, q, pos, order, count):
    B, Hq, D = shape.batch, shape.num_q_heads, shape.head_dim
    kc = order.shape[-1]
    out = torch.full((B, Hq, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((B, Hq), float("nan"), device="cuda")
    comp = torch.full((B, Hq), -7, dtype=torch.int32, device="cuda")
    skip = torch.full((B, Hq, kc), 7, dtype=torch.uint8, device="cuda")
    ws = torch.empty(C.cosa_osk_decode_workspace_size(shape, kc), dtype=torch.uint8, device="cuda")
    C.cosa_osk_decode(shape, C.OskParams(eps), q, xd["k_pool"], xd["v_pool"], xd["page_table"], pos,
                      order, count, out, ws, lse=lse, computed=comp, skip_log=skip)
    torch.cuda.synchronize()
    assert C.cosa_get_status() == 0
    return np64(out), lse.cpu().numpy(), comp.cpu().numpy(), skip.cpu().numpy()


def _check(got, ref, count, eps, vmax, what):
    out, lse, comp, skip = got
    rows_ok = np.zeros(count.shape, dtype=bool)
    n_amb = n_steps = 0
    for idx in np.ndindex(*count.shape):
        n = int(count[idx])
        n_steps += n
        gs, rs, mg = skip[idx][:n], ref["skip"][idx][:n], ref["margin"][idx][:n]
        assert np.all(skip[idx][n:] == 7), f"{what}: skip log written past count at {idx}"
        assert comp[idx] == n - int(gs.sum())
        amb = np.abs(mg) <= SKIP_MARGIN
        n_amb += int(amb.sum())
        dis = gs != rs
        assert not np.any(dis & ~amb), f"{what}: decision differs outside the margin at {idx}"
        if dis.any():
            bound = 2 * int(dis.sum()) * 64 * eps * vmax
            assert np.abs(out[idx] - ref["out"][idx]).max() <= bound + 2e-2
        else:
            assert comp[idx] == ref["computed"][idx]
            rows_ok[idx] = True
    assert n_amb <= max(2, n_steps // 1000)
    assert_out_close(out, ref["out"], what, rows_mask=rows_ok)
    assert_lse_close(lse, ref["lse"], what, rows_mask=rows_ok)


CASES = {  # workload, decode positions (one per sequence)
    "gqa-4k-shuffled": (W.small_workload("gqa-32k", 4096, 8, 2, shuffle_pages=True), (4095,)),
    "narrow-kv-4k-g7-b2": (W.small_workload("narrow-kv-64k", 4096, 7, 1, batch=2), (4000, 1234)),
    "wide-head-4k-p128": (W.small_workload("wide-head-128k", 4096, 8, 1), (3071,)),
    "tiny-2k-d64": (W.WORKLOADS["tiny-2k"], (2047,)),
}


@pytest.mark.parametrize("case", sorted(CASES))
@pytest.mark.parametrize("eps", [0.0, 1e-4, 1e-2])
def test_decode_parity_on_random_lists(case, eps):
    wl, positions = CASES[case]
    x = W.make_inputs(wl, seed=71)
    xd = to_dev(x)
    shape = shape_of(wl, x)
    B, Hq, P = wl.batch, wl.num_q_heads, wl.page_size
    rng = np.random.default_rng(71)
    kc = wl.num_pages
    order = np.full((B, Hq, kc), -1, dtype=np.int32)
    count = np.zeros((B, Hq), dtype=np.int32)
    for b in range(B):
        n_all = positions[b] // P + 1
        for h in range(Hq):
            n = int(rng.integers(1, n_all + 1))
            order[b, h, :n] = rng.permutation(n_all)[:n]
            count[b, h] = n
    qdec = x["q"][torch.arange(B), :, torch.tensor(positions)].contiguous()  # [B][H_q][D]: row t
    pos = torch.tensor(positions, dtype=torch.int32)
    got = _decode(shape, eps, xd, qdec.cuda(), pos.cuda(), torch.from_numpy(order).cuda(),
                  torch.from_numpy(count).cuda())
    ref = O.osk_decode(np64(qdec), np64(x["k_pool"]), np64(x["v_pool"]), x["page_table"].numpy(),
                       positions, order, count, num_kv_heads=wl.num_kv_heads, page_size=P, eps=eps,
                       scale=1 / math.sqrt(wl.head_dim))
    _check(got, ref, count, eps, float(np.abs(np64(x["v_pool"])).max()), f"decode {case} eps={eps}")


@pytest.mark.parametrize("eps", [0.0, 1e-4])
def test_decode_128k_with_kap_lists(eps):
    """The last token of a 128K sequence decodes with the list KAP wrote for its
    q-block (410 pages at budget 0.2); 4 query heads on one KV head."""
    wl = W.small_workload("gqa-128k", 131072, 4, 1)
    x = W.make_inputs(wl, seed=72, device="cuda")
    shape = shape_of(wl, x)
    order, count, _, _ = gpu_kap(shape, C.KapParams(budget=0.2, q_sub=32, k_sub=16, sink_pages=1), x,
                                 export=False)
    t = 131071
    o_dec = order[:, :, -1].contiguous()
    c_dec = count[:, :, -1].contiguous()
    qdec = x["q"][:, :, t].contiguous()
    pos = torch.tensor([t], dtype=torch.int32, device="cuda")
    got = _decode(shape, eps, x, qdec, pos, o_dec, c_dec)
    ref = O.osk_decode(np64(qdec), np64(x["k_pool"]), np64(x["v_pool"]),
                       x["page_table"].cpu().numpy(), [t], o_dec.cpu().numpy(), c_dec.cpu().numpy(),
                       num_kv_heads=1, page_size=64, eps=eps, scale=1 / math.sqrt(128))
    assert int(c_dec.min()) == 410
    _check(got, ref, c_dec.cpu().numpy(), eps, float(np.abs(np64(x["v_pool"])).max()),
           f"decode 128k eps={eps}")


def test_decode_every_page_equals_dense_row():
    wl = W.small_workload("gqa-32k", 4096, 4, 2, shuffle_pages=True)
    x = W.make_inputs(wl, seed=73)
    xd = to_dev(x)
    shape = shape_of(wl, x)
    t = 3000
    n = t // 64 + 1
    order = torch.full((1, 4, 64), -1, dtype=torch.int32)
    order[:, :, :n] = torch.arange(n, dtype=torch.int32)
    count = torch.full((1, 4), n, dtype=torch.int32)
    qdec = x["q"][:, :, t].contiguous()
    got = _decode(shape, 0.0, xd, qdec.cuda(), torch.tensor([t], dtype=torch.int32).cuda(),
                  order.cuda(), count.cuda())
    dense = O.dense_attention(np64(x["q"]), np64(x["k_pool"]), np64(x["v_pool"]),
                              x["page_table"].numpy(), num_kv_heads=2, scale=1 / math.sqrt(128),
                              rows=np.array([t]))
    assert_out_close(got[0], dense["out"][:, :, t], "decode every page")
    assert_lse_close(got[1], dense["lse"][:, :, t], "decode every page lse")
    np.testing.assert_array_equal(got[2], count.numpy())


def test_decode_list_entry_past_the_query_is_reported_not_read():
    wl = W.small_workload("gqa-32k", 4096, 2, 1)
    x = W.make_inputs(wl, seed=74)
    xd = to_dev(x)
    shape = shape_of(wl, x)
    t = 1000  # its page is 15; page 40 lies past it
    order = torch.tensor([[[0, 15, 40, 3] + [-1] * 60, [15, 0] + [-1] * 62]], dtype=torch.int32)
    count = torch.tensor([[4, 2]], dtype=torch.int32)
    out = torch.zeros(1, 2, 128, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(C.cosa_osk_decode_workspace_size(shape, 64), dtype=torch.uint8, device="cuda")
    C.cosa_osk_decode(shape, C.OskParams(0.0), x["q"][:, :, t].contiguous().cuda(), xd["k_pool"],
                      xd["v_pool"], xd["page_table"], torch.tensor([t], dtype=torch.int32).cuda(),
                      order.cuda(), count.cuda(), out, ws)
    torch.cuda.synchronize()
    assert C.cosa_get_status() == 1  # COSA_ERR_INVALID_ARG, read and cleared
    assert C.cosa_get_status() == 0
    assert torch.isfinite(out.float()).all()
    with pytest.raises(C.CosaError):  # eps > 1 is outside the decode rule's range
        C.cosa_osk_decode(shape, C.OskParams(2.0), x["q"][:, :, t].contiguous().cuda(), xd["k_pool"],
                          xd["v_pool"], xd["page_table"], torch.tensor([t], dtype=torch.int32).cuda(),
                          order.cuda(), count.cuda(), out, ws)


def test_decode_empty_list_and_position_out_of_range():
    """A head with an empty list gets a zero output, LSE -inf and 0 computed; a
    sequence whose position lies outside the cache is reported (status word) and its
    heads get the same empty result, while the other sequence decodes normally."""
    wl = W.small_workload("narrow-kv-64k", 4096, 7, 1, batch=2)
    x = W.make_inputs(wl, seed=75)
    xd = to_dev(x)
    shape = shape_of(wl, x)
    B, Hq, P = 2, 7, 64
    positions = [3000, 5000]  # the second lies past the 4096-token cache
    order = torch.full((B, Hq, 64), -1, dtype=torch.int32)
    count = torch.zeros((B, Hq), dtype=torch.int32)
    n = positions[0] // P + 1
    order[0, :, :n] = torch.arange(n, dtype=torch.int32)
    count[0, :] = n
    count[0, 3] = 0  # an empty list
    order[1, :, :5] = torch.arange(5, dtype=torch.int32)
    count[1, :] = 5
    qdec = torch.stack([x["q"][0, :, positions[0]], x["q"][1, :, 100]]).contiguous()
    out = torch.full((B, Hq, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((B, Hq), float("nan"), device="cuda")
    comp = torch.full((B, Hq), -7, dtype=torch.int32, device="cuda")
    ws = torch.empty(C.cosa_osk_decode_workspace_size(shape, 64), dtype=torch.uint8, device="cuda")
    C.cosa_osk_decode(shape, C.OskParams(1e-4), qdec.cuda(), xd["k_pool"], xd["v_pool"],
                      xd["page_table"], torch.tensor(positions, dtype=torch.int32).cuda(),
                      order.cuda(), count.cuda(), out, ws, lse=lse, computed=comp)
    torch.cuda.synchronize()
    assert C.cosa_get_status() == 1  # the position out of range, reported
    o, l, c = out.float().cpu(), lse.cpu(), comp.cpu()
    for b, h in [(0, 3)] + [(1, h) for h in range(Hq)]:
        assert torch.all(o[b, h] == 0) and l[b, h] == -math.inf and c[b, h] == 0
    ref = O.osk_decode(np64(qdec[:1]), np64(x["k_pool"]), np64(x["v_pool"]),
                       x["page_table"][:1].numpy(), positions[:1], order[:1].numpy(),
                       count[:1].numpy(), num_kv_heads=1, page_size=P, eps=1e-4,
                       scale=1 / math.sqrt(128))
    heads = [h for h in range(Hq) if h != 3]
    assert_out_close(o[0, heads].double().numpy(), ref["out"][0, heads], "decode batch row 0")


def test_decode_page_outside_the_pool_is_reported_not_read():
    """A list entry whose page-table entry lies outside the pool is reported and
    treated as an invalid entry: the result equals the oracle's on the list without
    it (a local max of -inf moves no running max and the entry is skipped)."""
    wl = W.small_workload("gqa-32k", 4096, 4, 2, shuffle_pages=True)
    x = W.make_inputs(wl, seed=76)
    xd = to_dev(x)
    shape = shape_of(wl, x)
    t, bad_page, eps = 3500, 17, 1e-4
    pt = xd["page_table"].clone()
    pt[0, bad_page] = wl.num_pages + 5
    n_all = t // 64 + 1
    rng = np.random.default_rng(76)
    order = np.full((1, 4, 64), -1, dtype=np.int32)
    count = np.zeros((1, 4), dtype=np.int32)
    for h in range(4):
        lst = [p for p in rng.permutation(n_all) if p != bad_page][:30]
        lst.insert(3 + h, bad_page)  # never first
        order[0, h, :len(lst)] = lst
        count[0, h] = len(lst)
    qdec = x["q"][:, :, t].contiguous()
    out = torch.full((1, 4, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((1, 4), float("nan"), device="cuda")
    comp = torch.full((1, 4), -7, dtype=torch.int32, device="cuda")
    skip = torch.full((1, 4, 64), 7, dtype=torch.uint8, device="cuda")
    ws = torch.empty(C.cosa_osk_decode_workspace_size(shape, 64), dtype=torch.uint8, device="cuda")
    C.cosa_osk_decode(shape, C.OskParams(eps), qdec.cuda(), xd["k_pool"], xd["v_pool"], pt,
                      torch.tensor([t], dtype=torch.int32).cuda(), torch.from_numpy(order).cuda(),
                      torch.from_numpy(count).cuda(), out, ws, lse=lse, computed=comp,
                      skip_log=skip)
    torch.cuda.synchronize()
    assert C.cosa_get_status() == 1
    sk = skip.cpu().numpy()
    order2 = np.full_like(order, -1)
    count2 = count - 1
    for h in range(4):
        assert sk[0, h, 3 + h] == 1  # the entry is skipped
        order2[0, h, :count2[0, h]] = [p for p in order[0, h, :count[0, h]] if p != bad_page]
    ref = O.osk_decode(np64(qdec), np64(x["k_pool"]), np64(x["v_pool"]), x["page_table"].numpy(),
                       [t], order2, count2, num_kv_heads=2, page_size=64, eps=eps,
                       scale=1 / math.sqrt(128))
    for h in range(4):
        n = int(count[0, h])
        mine = np.delete(sk[0, h, :n], 3 + h)
        amb = np.abs(ref["margin"][0, h, :n - 1]) <= SKIP_MARGIN
        assert np.all((mine == ref["skip"][0, h, :n - 1]) | amb)
    assert_out_close(np64(out), ref["out"], "decode without the bad page")
    assert_lse_close(lse.cpu().numpy(), ref["lse"], "decode without the bad page")
