"""The host-buffer entry point cosa_attention_host (copies in, KAP + OSK per KV
head, copies out, overlapped on streams) gives exactly the output of the
whole-layer device calls on the same inputs: heads are independent in both
stages, so running them one KV head at a time changes no arithmetic.  The cases
cover batch > 1 (strided copies of Q and O), four KV heads (each device buffer
set reused), D = 64, P = 128 and a repeated call on the same workspace."""
import pytest
import torch

import block_sparse_long_kap_b200 as C
import workloads as W
from helpers import shape_of, to_dev

pytestmark = pytest.mark.gpu

HOST_CASES = {
    "gqa-4k-b2-kv4": W.small_workload("gqa-32k", 4096, 16, 4, batch=2, shuffle_pages=True),
    "narrow-kv-4k-g7": W.small_workload("narrow-kv-64k", 4096, 14, 2),
    "wide-head-4k-p128": W.small_workload("wide-head-128k", 4096, 16, 2),
    "tiny-2k-d64": W.WORKLOADS["tiny-2k"],
}


def _device_path(shape, kap, osk, xd):
    B, Hq = shape.batch, shape.num_q_heads
    kc = C.cosa_kap_kcap(shape, kap)
    order = torch.empty((B, Hq, shape.num_q_blocks, kc), dtype=torch.int32, device="cuda")
    count = torch.empty((B, Hq, shape.num_q_blocks), dtype=torch.int32, device="cuda")
    ws = torch.empty(C.cosa_kap_workspace_size(shape, kap), dtype=torch.uint8, device="cuda")
    C.cosa_kap_select(shape, kap, xd["q"], xd["k_pool"], xd["page_table"], order, count, ws)
    out = torch.empty_like(xd["q"])
    C.cosa_osk_attention(shape, osk, xd["q"], xd["k_pool"], xd["v_pool"], xd["page_table"],
                         order, count, out)
    torch.cuda.synchronize()
    assert C.cosa_get_status() == 0
    return out.cpu()


@pytest.mark.parametrize("case", sorted(HOST_CASES))
def test_host_path_equals_device_path(case):
    wl = HOST_CASES[case]
    x = W.make_inputs(wl, seed=5)
    shape = shape_of(wl, x)
    kap = C.KapParams(budget=0.25, q_sub=wl.q_block // 4, k_sub=16)
    osk = C.OskParams(1e-4)
    ref = _device_path(shape, kap, osk, to_dev(x))

    pin = lambda t: t.detach().cpu().contiguous().pin_memory()
    qh, kh, vh, pth = pin(x["q"]), pin(x["k_pool"]), pin(x["v_pool"]), pin(x["page_table"])
    ws = torch.empty(C.cosa_attention_host_workspace_size(shape, kap), dtype=torch.uint8,
                     device="cuda")
    for _ in range(2):  # the second call reuses the workspace and the pinned buffers
        out = torch.full(tuple(ref.shape), 7.0, dtype=torch.bfloat16).pin_memory()
        C.cosa_attention_host(shape, kap, osk, qh, kh, vh, pth, out, ws)
        torch.cuda.synchronize()
        assert C.cosa_get_status() == 0
        assert torch.equal(out, ref), f"{case}: host path differs from the device path"
