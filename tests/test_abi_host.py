"""Host-side checks of the C-ABI library (no GPU): it loads, exports every
symbol include/cosa.h declares, and validates arguments on the host before any
CUDA call."""
import ctypes
import math
import os
import re

import pytest

import block_sparse_long_kap_b200 as C
import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    text = open(os.path.join(ROOT, "include", "cosa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(cosa_[a-z_0-9]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(C.library_path)
    declared = _declared_symbols()
    assert declared, "no declarations parsed"
    for name in declared:
        assert hasattr(lib, name), f"{name} declared in cosa.h but not exported"
    assert set(declared) == set(C.EXPORTED_SYMBOLS)


def test_status_strings_and_version():
    for code in range(6):
        assert C.cosa_status_string(code)
    assert C.cosa_status_string(99) == "unknown status"
    assert C.cosa_version() > 0


@pytest.mark.parametrize("N,P,Bq,budget,sink", [
    (131072, 64, 128, 0.2, 1), (32768, 64, 128, 0.1, 1), (65536, 64, 128, 0.05, 1),
    (131072, 128, 128, 0.15, 1), (2048, 64, 64, 0.25, 1), (4096, 128, 64, 0.5, 2),
    (1024, 64, 128, 0.0, 0), (1024, 64, 128, 1.0, 1)])
def test_kcap_matches_oracle(N, P, Bq, budget, sink):
    s = C.Shape(1, 4, 2, N, 128, P, Bq)
    k = C.KapParams(budget=budget, sink_pages=sink)
    assert C.cosa_kap_kcap(s, k) == O.k_cap(N, Bq, P, sink, budget)


def test_workspace_size_covers_pooled_vectors_and_page_maxima():
    s = C.Shape(1, 32, 8, 131072, 128, 64, 128)
    k = C.KapParams(0.2, q_sub=32, k_sub=16)
    rows = 32 * 1024 * 4                       # representatives
    keys = 8 * 2048 * 4                        # sub-keys
    tri = sum(O.causal_pages(qb, 128, 64) for qb in range(1024))
    need = 2 * rows * 128 * 4 + 2 * keys * 128 * 4 + 8 * 16 * tri * 4 + rows * 8
    got = C.cosa_kap_workspace_size(s, k)
    assert need <= got <= need + 8 * 256


def _status(fn):
    try:
        fn()
    except C.CosaError as e:
        return e.status
    return 0


@pytest.mark.parametrize("bad,code", [
    (dict(head_dim=96), 2), (dict(page_size=32), 2), (dict(q_block=256), 2),
    (dict(seq_len=1000), 1), (dict(num_kv_heads=3), 1), (dict(batch=0), 1),
    (dict(softmax_scale=-1.0), 1), (dict(pages_per_seq=3), 1)])
def test_invalid_shapes_rejected_on_host(bad, code):
    kw = dict(batch=1, num_q_heads=4, num_kv_heads=2, seq_len=1024, head_dim=128, page_size=64,
              q_block=128)
    kw.update(bad)
    s = C.Shape(**kw)
    if "softmax_scale" in bad:
        s.softmax_scale = bad["softmax_scale"]
    assert _status(lambda: C.cosa_kap_kcap(s, C.KapParams())) == code


@pytest.mark.parametrize("bad,code", [
    (dict(budget=1.5), 1), (dict(budget=-0.1), 1), (dict(budget=float("nan")), 1),
    (dict(q_sub=48), 1), (dict(k_sub=5), 1), (dict(q_sub=8), 2), (dict(k_sub=4), 2),
    (dict(sink_pages=-1), 1)])
def test_invalid_kap_params_rejected_on_host(bad, code):
    s = C.Shape(1, 4, 2, 1024, 128, 64, 128)
    assert _status(lambda: C.cosa_kap_kcap(s, C.KapParams(**bad))) == code


def test_null_pointers_and_bad_eps_rejected_before_launch():
    lib = C.lib()
    s = C.Shape(1, 4, 2, 1024, 128, 64, 128).c()
    k = C.KapParams().c(C.Shape(1, 4, 2, 1024, 128, 64, 128))
    o = C._Osk(1e-4)
    # null q
    assert lib.cosa_osk_attention(ctypes.byref(s), ctypes.byref(o), None, 16, 16, 16, 16, 16, 4,
                                  16, None, None, None, None) == 1
    # negative / NaN eps
    for eps in (-1.0, float("nan")):
        ob = C._Osk(eps)
        assert lib.cosa_osk_attention(ctypes.byref(s), ctypes.byref(ob), 16, 16, 16, 16, 16, 16, 4,
                                      16, None, None, None, None) == 1
    # k_cap out of range
    assert lib.cosa_osk_attention(ctypes.byref(s), ctypes.byref(o), 16, 16, 16, 16, 16, 16, 0,
                                  16, None, None, None, None) == 1
    # misaligned tensor pointer
    assert lib.cosa_dense_attention(ctypes.byref(s), 18, 16, 16, 16, 16, None, None) == 1
    # workspace missing / too small / misaligned
    assert lib.cosa_kap_select(ctypes.byref(s), ctypes.byref(k), 16, 16, 16, 16, 16, None, None,
                               None, 0, None) == 5
    assert lib.cosa_kap_select(ctypes.byref(s), ctypes.byref(k), 16, 16, 16, 16, 16, None, None,
                               256, 100, None) == 5
    assert lib.cosa_kap_select(ctypes.byref(s), ctypes.byref(k), 16, 16, 16, 16, 16, None, None,
                               16, 1 << 40, None) == 5
    # null shape
    assert lib.cosa_dense_attention(None, 16, 16, 16, 16, 16, None, None) == 1


def test_group_entry_points_reject_bad_arguments_before_launch():
    lib = C.lib()
    shp = C.Shape(1, 4, 2, 1024, 128, 64, 128)
    s = shp.c()
    k = C.KapParams().c(shp)
    o = C._Osk(1e-4)
    # null q / negative eps / k_cap out of range / misaligned output
    assert lib.cosa_osk_attention_group(ctypes.byref(s), ctypes.byref(o), None, 16, 16, 16, 16, 16,
                                        4, 16, None, None, None, None) == 1
    ob = C._Osk(-1.0)
    assert lib.cosa_osk_attention_group(ctypes.byref(s), ctypes.byref(ob), 16, 16, 16, 16, 16, 16,
                                        4, 16, None, None, None, None) == 1
    assert lib.cosa_osk_attention_group(ctypes.byref(s), ctypes.byref(o), 16, 16, 16, 16, 16, 16,
                                        0, 16, None, None, None, None) == 1
    assert lib.cosa_osk_attention_group(ctypes.byref(s), ctypes.byref(o), 16, 16, 16, 16, 16, 16,
                                        4, 24, None, None, None, None) == 1
    # workspace missing / too small; ascending lists unsupported in group mode
    assert lib.cosa_kap_select_group(ctypes.byref(s), ctypes.byref(k), 16, 16, 16, 16, 16, None,
                                     None, None, 0, None) == 5
    assert lib.cosa_kap_select_group(ctypes.byref(s), ctypes.byref(k), 16, 16, 16, 16, 16, None,
                                     None, 256, 100, None) == 5
    ka = C.KapParams(ascending=True).c(shp)
    assert lib.cosa_kap_select_group(ctypes.byref(s), ctypes.byref(ka), 16, 16, 16, 16, 16, None,
                                     None, 256, 1 << 40, None) == 2


def test_host_pipeline_workspace_and_argument_checks():
    """cosa_attention_host: the workspace holds two sets of one KV head's K and V pool
    columns, three slots of one query head's Q and O (over the batch), and one query
    head's lists and KAP workspace; bad arguments return before anything is queued
    (no CUDA call is made on these paths)."""
    lib = C.lib()
    shp = C.Shape(2, 8, 2, 2048, 128, 64, 128)
    kap = C.KapParams(budget=0.25, q_sub=32, k_sub=16)
    ws = C.cosa_attention_host_workspace_size(shp, kap)
    sub = C.Shape(2, 1, 1, 2048, 128, 64, 128, num_phys_pages=shp.c().num_phys_pages)
    q_head = 2 * 1 * 2048 * 128 * 2
    kv_head = shp.c().num_phys_pages * 64 * 128 * 2
    need = 2 * 2 * kv_head + 3 * 2 * q_head + C.cosa_kap_workspace_size(sub, kap)
    assert need <= ws <= need + 64 * 1024 + 2 * 2 * 1024 * C.cosa_kap_kcap(sub, kap) * 4
    s, k, o = shp.c(), kap.c(shp), C._Osk(1e-4)
    # null host buffer, negative eps, missing / small / misaligned workspace
    assert lib.cosa_attention_host(ctypes.byref(s), ctypes.byref(k), ctypes.byref(o), None, 16, 16,
                                   16, 16, 256, ws, None) == 1
    ob = C._Osk(-1.0)
    assert lib.cosa_attention_host(ctypes.byref(s), ctypes.byref(k), ctypes.byref(ob), 16, 16, 16,
                                   16, 16, 256, ws, None) == 1
    assert lib.cosa_attention_host(ctypes.byref(s), ctypes.byref(k), ctypes.byref(o), 16, 16, 16,
                                   16, 16, None, 0, None) == 5
    assert lib.cosa_attention_host(ctypes.byref(s), ctypes.byref(k), ctypes.byref(o), 16, 16, 16,
                                   16, 16, 256, ws - 1, None) == 5
    assert lib.cosa_attention_host(ctypes.byref(s), ctypes.byref(k), ctypes.byref(o), 16, 16, 16,
                                   16, 16, 128, ws, None) == 5
    # invalid shape (H_q not a multiple of H_kv) and null size pointer
    bad = C.Shape(1, 6, 4, 1024, 128, 64, 128).c()
    assert lib.cosa_attention_host_workspace_size(ctypes.byref(bad), ctypes.byref(k),
                                                  ctypes.byref(ctypes.c_size_t(0))) == 1
    assert lib.cosa_attention_host_workspace_size(ctypes.byref(s), ctypes.byref(k), None) == 1
    # the binding refuses device-resident host arguments before calling in
    with pytest.raises((TypeError, ValueError)):
        C.cosa_attention_host(shp, kap, C.OskParams(1e-4), None, None, None, None, None, None)


def test_early_break_argument_checks():
    """max_run < 0 is an argument error; the group-shared kernel has no early break."""
    lib = C.lib()
    shp = C.Shape(1, 4, 2, 1024, 128, 64, 128)
    s = shp.c()
    neg = C._Osk(1e-4, -1)
    assert lib.cosa_osk_attention(ctypes.byref(s), ctypes.byref(neg), 16, 16, 16, 16, 16, 16, 4,
                                  16, None, None, None, None) == 1
    brk = C._Osk(1e-4, 4)
    assert lib.cosa_osk_attention_group(ctypes.byref(s), ctypes.byref(brk), 16, 16, 16, 16, 16,
                                        16, 4, 16, None, None, None, None) == 2
    assert C.OskParams(1e-3, 8).c().max_run == 8 and C.OskParams().c().max_run == 0


def test_wait_fault_hook_argument_checks_on_host():
    """The test hook (cosa_debug_osk_wait_fault) only records a one-shot setting:
    no CUDA call, so it is checked here; a group below -1 is rejected."""
    lib = C.lib()
    assert lib.cosa_debug_osk_wait_fault(-2, 0) == 1
    assert lib.cosa_debug_osk_wait_fault(-1, 0) == 0
    # consumed by the next OSK call even when that call fails its own checks
    assert lib.cosa_osk_attention(None, None, None, None, None, None, None, None, 0, None, None,
                                  None, None, None) == 1


def test_prefill_write_argument_checks_on_host():
    lib = C.lib()
    s = C.Shape(1, 4, 2, 256, 128, 64, 128).c()
    k = C.KapParams(budget=0.2, q_sub=32, k_sub=16).c(C.Shape(1, 4, 2, 256, 128, 64, 128))
    # a missing buffer, then a misaligned one, both before anything is launched
    assert lib.cosa_prefill_write(ctypes.byref(s), ctypes.byref(k), None, 16, 16, 16, 16, 16, 16,
                                  None, 0, None) == 1
    assert lib.cosa_prefill_write(ctypes.byref(s), ctypes.byref(k), 8, 16, 16, 16, 16, 16, 16,
                                  None, 0, None) == 1
    # a workspace smaller than cosa_kap_workspace_size
    assert lib.cosa_prefill_write(ctypes.byref(s), ctypes.byref(k), 16, 16, 16, 16, 16, 16, 16,
                                  256, 16, None) == 5


def test_host_pipeline_checks_its_host_page_table():
    """cosa_attention_host reads its page table on the host: an entry outside
    [0, num_phys_pages) returns COSA_ERR_INVALID_ARG before any CUDA call."""
    import numpy as np
    lib = C.lib()
    shp = C.Shape(2, 4, 2, 1024, 128, 64, 128)
    kap = C.KapParams(budget=0.25, q_sub=32, k_sub=16)
    ws = C.cosa_attention_host_workspace_size(shp, kap)
    s, k, o = shp.c(), kap.c(shp), C._Osk(1e-4)
    for bad in (-1, s.num_phys_pages):
        pt = np.arange(2 * 16, dtype=np.int32).reshape(2, 16)
        pt[1, 9] = bad
        assert lib.cosa_attention_host(ctypes.byref(s), ctypes.byref(k), ctypes.byref(o), 16, 16,
                                       16, pt.ctypes.data, 16, 256, ws, None) == 1
    # padded rows (stride 20 for 16 pages): the bad entry sits where only the
    # row stride, not the page count, reaches it
    s2 = C.Shape(2, 4, 2, 1024, 128, 64, 128, pages_per_seq=20).c()
    pt = np.zeros((2, 20), dtype=np.int32)
    pt[:, :16] = np.arange(32, dtype=np.int32).reshape(2, 16)
    pt[1, 14] = 99
    assert lib.cosa_attention_host(ctypes.byref(s2), ctypes.byref(k), ctypes.byref(o), 16, 16, 16,
                                   pt.ctypes.data, 16, 256, 1 << 40, None) == 1
