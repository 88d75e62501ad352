"""cosa_kap_select_noalloc: the Stage-1 entry point for callers that cannot
allocate device memory (their allocator belongs to someone else, or their
memory plan is fixed before the call).  It must give exactly what
cosa_kap_select gives with a caller workspace, call after call, although every
call reuses the library's one fixed scratch array.

The new entry point is called through the C ABI (ctypes), not the binding.
This file is collected last so that a run stopping at the first failure has
already run every other test."""
import ctypes

import numpy as np
import pytest
import torch

import block_sparse_long_kap_b200 as C
import workloads as W

pytestmark = pytest.mark.gpu


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _abi_noalloc(shape, kap, q, k_pool, pt, order, count, scores=None, hrm=None):
    lib = C.lib()
    s, k = shape.c(), kap.c(shape)
    stream = torch.cuda.current_stream().cuda_stream
    return lib.cosa_kap_select_noalloc(ctypes.byref(s), ctypes.byref(k), _ptr(q), _ptr(k_pool),
                                       _ptr(pt), _ptr(order), _ptr(count), _ptr(scores),
                                       _ptr(hrm), ctypes.c_void_p(stream))


def _case(wl, budget, seed, with_exports):
    x = W.make_inputs(wl, seed=seed)
    q, kp, pt = x["q"].cuda(), x["k_pool"].cuda(), x["page_table"].cuda()
    shape = C.Shape(wl.batch, wl.num_q_heads, wl.num_kv_heads, wl.seq_len, wl.head_dim,
                    wl.page_size, wl.q_block)
    kap = C.KapParams(budget=budget, q_sub=wl.q_block // 4, k_sub=16, sink_pages=1)
    assert C.cosa_kap_workspace_size(shape, kap) <= C.NOALLOC_SCRATCH_BYTES
    kc = C.cosa_kap_kcap(shape, kap)
    B, Hq, nQB, nP = wl.batch, wl.num_q_heads, wl.num_q_blocks, wl.num_pages

    def bufs():
        o = torch.full((B, Hq, nQB, kc), -7, dtype=torch.int32, device="cuda")
        c = torch.full((B, Hq, nQB), -7, dtype=torch.int32, device="cuda")
        sc = torch.full((B, Hq, nQB, nP), -1.0, device="cuda") if with_exports else None
        hr = torch.full((B, Hq, nQB, nP), 9, dtype=torch.uint8, device="cuda") if with_exports else None
        return o, c, sc, hr

    # the existing entry point, with a caller workspace
    o1, c1, s1, h1 = bufs()
    ws = torch.empty(C.cosa_kap_workspace_size(shape, kap), dtype=torch.uint8, device="cuda")
    C.cosa_kap_select(shape, kap, q, kp, pt, o1, c1, ws, scores=s1, hrm=h1)
    # the allocation-free one
    o2, c2, s2, h2 = bufs()
    st = _abi_noalloc(shape, kap, q, kp, pt, o2, c2, s2, h2)
    torch.cuda.synchronize()
    assert st == 0, C.cosa_status_string(st)
    assert C.cosa_get_status() == 0
    # same kernels on the same inputs: identical results (within any tolerance)
    assert torch.equal(c1, c2)
    assert torch.equal(o1, o2)
    if with_exports:
        assert torch.equal(s1, s2) and torch.equal(h1, h2)


def test_noalloc_matches_workspace_entry_point_two_calls_in_a_row():
    # first call: 4K-token GQA layer, exports to caller buffers
    _case(W.small_workload("gqa-32k", 4096, 8, 2, shuffle_pages=True), 0.25, seed=21,
          with_exports=True)
    # second call right after, different shape and head dim, scores kept in the
    # scratch: the previous call's contents must not leak into this one
    _case(W.WORKLOADS["tiny-2k"], 0.25, seed=22, with_exports=False)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    shape = C.Shape(1, 32, 8, 131072, 128, 64, 128)
    kap = C.KapParams(budget=0.2, q_sub=32, k_sub=16)
    assert C.cosa_kap_workspace_size(shape, kap) > C.NOALLOC_SCRATCH_BYTES
    st = _abi_noalloc(shape, kap, torch.empty(16, device="cuda"), torch.empty(16, device="cuda"),
                      torch.empty(16, device="cuda"), torch.empty(16, device="cuda"),
                      torch.empty(16, device="cuda"))
    assert st == 2  # COSA_ERR_UNSUPPORTED, before anything is launched
