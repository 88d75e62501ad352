"""Failure detection without a GPU fault: one of the attention kernel's bounded
waits is made to run out on purpose (the K tile copies of one listed group are
never issued, and the wait limit is cut to 20 ms through the test hook
cosa_debug_osk_wait_fault).  The launch must end by itself with
COSA_ERR_TIMEOUT in the status word, after draining the copies and MMAs it did
issue and freeing its tensor memory; the next normal call on the same device
must run clean and match the oracle.  Nothing here traps, hangs or reads out
of bounds: every wait in the kernel is bounded, and the withheld copies are
simply never issued."""
import math
import time

import numpy as np
import pytest
import torch

import block_sparse_long_kap_b200 as C
import oracle as O
import workloads as W
from helpers import check_osk_tiles, gpu_osk, np64, shape_of, to_dev

pytestmark = pytest.mark.gpu

COSA_ERR_TIMEOUT = 4


def _case():
    wl = W.small_workload("gqa-32k", 4096, 4, 1, shuffle_pages=True)
    x = W.make_inputs(wl, seed=51)
    xh = dict(q=np64(x["q"]), k_pool=np64(x["k_pool"]), v_pool=np64(x["v_pool"]),
              page_table=x["page_table"].cpu().numpy())
    sel = O.kap_select(xh["q"], xh["k_pool"], xh["page_table"], num_kv_heads=1, page_size=64,
                       q_block=128, q_sub=32, k_sub=16, scale=1 / math.sqrt(128), budget=0.5,
                       sink_pages=1)
    return wl, x, xh, sel


@pytest.mark.parametrize("withhold", [0, 5])
def test_osk_wait_runs_out_is_reported_and_the_next_call_is_clean(withhold):
    wl, x, xh, sel = _case()
    xd = to_dev(x)
    shape = shape_of(wl, x)
    order = torch.from_numpy(sel["order"]).cuda()
    count = torch.from_numpy(sel["count"]).cuda()
    # lists of the last q-blocks reach group 5 (32 pages at budget 0.5)
    assert int(sel["count"].max()) > 2 * 5 + 1
    assert C.cosa_get_status() == 0
    out = torch.zeros(wl.batch, wl.num_q_heads, wl.seq_len, 128, dtype=torch.bfloat16,
                      device="cuda")
    C.cosa_debug_osk_wait_fault(withhold, 20_000_000)
    t0 = time.perf_counter()
    C.cosa_osk_attention(shape, C.OskParams(1e-4), xd["q"], xd["k_pool"], xd["v_pool"],
                         xd["page_table"], order, count, out)
    torch.cuda.synchronize()  # the launch ends by itself
    secs = time.perf_counter() - t0
    assert C.cosa_get_status() == COSA_ERR_TIMEOUT
    assert C.cosa_get_status() == 0  # read and cleared
    assert secs < 10.0
    # the hook was one-shot: the next call runs normally and matches the oracle
    out, lse, computed, skip = gpu_osk(shape, 1e-4, xd, order, count)
    ref = O.osk_attention(xh["q"], xh["k_pool"], xh["v_pool"], xh["page_table"], sel["order"],
                          sel["count"], num_kv_heads=1, page_size=64, q_block=128, eps=1e-4,
                          scale=1 / math.sqrt(128))
    tiles = [(0, h, qb) for h in range(wl.num_q_heads) for qb in range(wl.num_q_blocks)]
    check_osk_tiles(skip.cpu().numpy(), computed.cpu().numpy(), np64(out), lse.cpu().numpy(), ref,
                    sel["count"], tiles, 128, 64, 1e-4, float(np.abs(xh["v_pool"]).max()),
                    "osk after a timed-out launch")


def test_short_wait_limit_alone_changes_nothing():
    """With no copy withheld, a 20 ms wait limit is far above any wait of a healthy
    launch: the call is clean and bit-identical to one with the default limit."""
    wl, x, xh, sel = _case()
    xd = to_dev(x)
    shape = shape_of(wl, x)
    order = torch.from_numpy(sel["order"]).cuda()
    count = torch.from_numpy(sel["count"]).cuda()
    C.cosa_debug_osk_wait_fault(-1, 20_000_000)
    a = gpu_osk(shape, 1e-4, xd, order, count)
    b = gpu_osk(shape, 1e-4, xd, order, count)
    for u, v in zip(a, b):
        assert torch.equal(u, v)


def test_fault_hook_argument_checks():
    with pytest.raises(RuntimeError):
        C.cosa_debug_osk_wait_fault(-2, 0)
    # consumed by a call whose arguments fail: the hook does not leak to a later call
    wl, x, _, sel = _case()
    shape = shape_of(wl, x)
    C.cosa_debug_osk_wait_fault(0, 1000)
    xd = to_dev(x)
    out = torch.empty(wl.batch, wl.num_q_heads, wl.seq_len, 128, dtype=torch.bfloat16,
                      device="cuda")
    with pytest.raises(RuntimeError):  # the hook needs max_run = 0
        C.cosa_osk_attention(shape, C.OskParams(1e-4, 4), xd["q"], xd["k_pool"], xd["v_pool"],
                             xd["page_table"], torch.from_numpy(sel["order"]).cuda(),
                             torch.from_numpy(sel["count"]).cuda(), out)
    gpu_osk(shape, 1e-4, xd, torch.from_numpy(sel["order"]).cuda(),
            torch.from_numpy(sel["count"]).cuda())  # asserts a clean status
