"""Python binding of libcosa.so: CoSA block-sparse causal prefill attention
(Kernel-Aware Proxy + Ordered-Skipping Kernel) on B200 (sm_100a).

Argument marshalling only: every step of the method runs in the library's CUDA
kernels.  Functions carry the C names (include/cosa.h) and take torch tensors
for device memory; the current torch CUDA stream is used unless one is given.
There is no CPU fallback: if the library cannot be loaded, calls raise.
"""
from __future__ import annotations

import ctypes
import dataclasses
import math
import os
from typing import Optional

__all__ = [
    "CosaError", "Shape", "KapParams", "OskParams", "lib", "library_path",
    "cosa_status_string", "cosa_version", "cosa_kap_kcap", "cosa_kap_workspace_size",
    "cosa_kap_select", "cosa_kap_select_noalloc", "cosa_kap_order", "cosa_osk_attention",
    "cosa_dense_attention", "cosa_get_status", "EXPORTED_SYMBOLS", "NOALLOC_SCRATCH_BYTES",
    "cosa_kap_select_group", "cosa_osk_attention_group", "cosa_attention_host_workspace_size",
    "cosa_attention_host", "cosa_debug_osk_wait_fault", "cosa_kap_pool", "cosa_kap_rank",
    "cosa_kap_preskip", "cosa_osk_decode", "cosa_osk_decode_workspace_size",
    "cosa_prefill_write",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "libcosa.so")

EXPORTED_SYMBOLS = (
    "cosa_status_string", "cosa_version", "cosa_kap_kcap", "cosa_kap_workspace_size",
    "cosa_kap_select", "cosa_kap_select_noalloc", "cosa_kap_order", "cosa_osk_attention",
    "cosa_dense_attention", "cosa_get_status", "cosa_kap_select_group", "cosa_osk_attention_group",
    "cosa_attention_host_workspace_size", "cosa_attention_host", "cosa_debug_osk_wait_fault",
    "cosa_kap_pool", "cosa_kap_rank", "cosa_kap_preskip", "cosa_osk_decode",
    "cosa_osk_decode_workspace_size", "cosa_prefill_write",
)

# Largest workspace the allocation-free Stage-1 entry point accepts (cosa.h).
NOALLOC_SCRATCH_BYTES = 128 << 20

STATUS_NAMES = {0: "COSA_OK", 1: "COSA_ERR_INVALID_ARG", 2: "COSA_ERR_UNSUPPORTED",
                3: "COSA_ERR_CUDA", 4: "COSA_ERR_TIMEOUT", 5: "COSA_ERR_WORKSPACE"}


class CosaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = STATUS_NAMES.get(status, str(status))
        try:
            msg += ": " + lib().cosa_status_string(status).decode()
        except Exception:
            pass
        super().__init__(f"{where}: {msg}")


class _Shape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("num_q_heads", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("seq_len", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("page_size", ctypes.c_int32),
                ("q_block", ctypes.c_int32), ("pages_per_seq", ctypes.c_int32),
                ("num_phys_pages", ctypes.c_int32), ("softmax_scale", ctypes.c_float)]


class _Kap(ctypes.Structure):
    _fields_ = [("budget", ctypes.c_float), ("q_sub", ctypes.c_int32), ("k_sub", ctypes.c_int32),
                ("sink_pages", ctypes.c_int32), ("ascending", ctypes.c_int32)]


class _Osk(ctypes.Structure):
    _fields_ = [("eps", ctypes.c_float), ("max_run", ctypes.c_int32)]


@dataclasses.dataclass
class Shape:
    batch: int
    num_q_heads: int
    num_kv_heads: int
    seq_len: int
    head_dim: int
    page_size: int
    q_block: int
    pages_per_seq: int = 0      # 0 -> seq_len // page_size
    num_phys_pages: int = 0     # 0 -> batch * pages_per_seq
    softmax_scale: float = 0.0  # 0 -> 1/sqrt(head_dim)

    def c(self) -> _Shape:
        pps = self.pages_per_seq or self.seq_len // self.page_size
        nphys = self.num_phys_pages or self.batch * pps
        scale = self.softmax_scale or 1.0 / math.sqrt(self.head_dim)
        return _Shape(self.batch, self.num_q_heads, self.num_kv_heads, self.seq_len, self.head_dim,
                      self.page_size, self.q_block, pps, nphys, scale)

    @property
    def num_pages(self) -> int:
        return self.seq_len // self.page_size

    @property
    def num_q_blocks(self) -> int:
        return self.seq_len // self.q_block


@dataclasses.dataclass
class KapParams:
    budget: float = 0.2
    q_sub: int = 0         # 0 -> q_block // 4
    k_sub: int = 16
    sink_pages: int = 1
    ascending: bool = False

    def c(self, shape: Shape) -> _Kap:
        q_sub = self.q_sub or shape.q_block // 4
        return _Kap(self.budget, q_sub, self.k_sub, self.sink_pages, int(bool(self.ascending)))


@dataclasses.dataclass
class OskParams:
    eps: float = 1e-4
    max_run: int = 0        # > 0: early break after this many consecutive skipped pages

    def c(self) -> _Osk:
        return _Osk(self.eps, self.max_run)


_lib = None


def lib():
    """Load libcosa.so (once).  Raises if it is missing: there is no fallback."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(library_path):
        raise RuntimeError(f"libcosa.so not built ({library_path}); run "
                           "python -m block_sparse_long_kap_b200.build")
    L = ctypes.CDLL(library_path)
    P = ctypes.POINTER
    vp, sz, i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32
    L.cosa_status_string.argtypes = [ctypes.c_int]
    L.cosa_status_string.restype = ctypes.c_char_p
    L.cosa_version.argtypes = []
    L.cosa_version.restype = i32
    L.cosa_kap_kcap.argtypes = [P(_Shape), P(_Kap), P(i32)]
    L.cosa_kap_workspace_size.argtypes = [P(_Shape), P(_Kap), P(sz)]
    L.cosa_kap_select.argtypes = [P(_Shape), P(_Kap), vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.cosa_kap_select_noalloc.argtypes = [P(_Shape), P(_Kap), vp, vp, vp, vp, vp, vp, vp, vp]
    L.cosa_kap_select_group.argtypes = [P(_Shape), P(_Kap), vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.cosa_kap_order.argtypes = [P(_Shape), P(_Kap), vp, vp, vp, vp, vp]
    L.cosa_osk_attention.argtypes = [P(_Shape), P(_Osk), vp, vp, vp, vp, vp, vp, i32, vp, vp, vp,
                                     vp, vp]
    L.cosa_dense_attention.argtypes = [P(_Shape), vp, vp, vp, vp, vp, vp, vp]
    L.cosa_osk_attention_group.argtypes = [P(_Shape), P(_Osk), vp, vp, vp, vp, vp, vp, i32, vp, vp,
                                           vp, vp, vp]
    L.cosa_get_status.argtypes = [vp]
    L.cosa_attention_host_workspace_size.argtypes = [P(_Shape), P(_Kap), P(sz)]
    L.cosa_attention_host.argtypes = [P(_Shape), P(_Kap), P(_Osk), vp, vp, vp, vp, vp, vp, sz, vp]
    L.cosa_debug_osk_wait_fault.argtypes = [i32, ctypes.c_uint64]
    L.cosa_kap_pool.argtypes = [P(_Shape), P(_Kap), vp, vp, vp, vp, sz, vp]
    L.cosa_kap_rank.argtypes = [P(_Shape), P(_Kap), vp, vp, vp, vp, vp, sz, vp]
    L.cosa_osk_decode_workspace_size.argtypes = [P(_Shape), i32, P(sz)]
    L.cosa_osk_decode.argtypes = [P(_Shape), P(_Osk), vp, vp, vp, vp, vp, vp, vp, i32, vp, vp, vp,
                                  vp, vp, sz, vp]
    L.cosa_prefill_write.argtypes = [P(_Shape), P(_Kap), vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.cosa_kap_preskip.argtypes = [P(_Shape), P(_Kap), ctypes.c_float, ctypes.c_float, vp, vp, vp,
                                   vp, sz, vp]
    for name in EXPORTED_SYMBOLS:
        if name not in ("cosa_status_string", "cosa_version"):
            getattr(L, name).restype = ctypes.c_int
    _lib = L
    return L


def _check(status: int, where: str) -> None:
    if status != 0:
        raise CosaError(status, where)


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _expect(t, name, dtype, shape, device=None):
    import torch
    if t is None:
        raise ValueError(f"{name} is required")
    if t.dtype != dtype:
        raise TypeError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")


def cosa_status_string(status: int) -> str:
    return lib().cosa_status_string(status).decode()


def cosa_version() -> int:
    return lib().cosa_version()


def cosa_kap_kcap(shape: Shape, kap: KapParams) -> int:
    out = ctypes.c_int32(0)
    s, k = shape.c(), kap.c(shape)
    _check(lib().cosa_kap_kcap(ctypes.byref(s), ctypes.byref(k), ctypes.byref(out)), "cosa_kap_kcap")
    return out.value


def cosa_kap_workspace_size(shape: Shape, kap: KapParams) -> int:
    out = ctypes.c_size_t(0)
    s, k = shape.c(), kap.c(shape)
    _check(lib().cosa_kap_workspace_size(ctypes.byref(s), ctypes.byref(k), ctypes.byref(out)),
           "cosa_kap_workspace_size")
    return out.value


def _kv_shape(shape: Shape):
    s = shape.c()
    return (s.num_phys_pages, shape.num_kv_heads, shape.page_size, shape.head_dim)


def cosa_kap_select(shape: Shape, kap: KapParams, q, k_pool, page_table, order, count,
                    workspace, scores=None, hrm=None, stream=None) -> None:
    """Stage 1: write the ordered page lists (order, count) for every q-block."""
    import torch
    s, k = shape.c(), kap.c(shape)
    B, Hq, N, D = shape.batch, shape.num_q_heads, shape.seq_len, shape.head_dim
    kc = cosa_kap_kcap(shape, kap)
    _expect(q, "q", torch.bfloat16, (B, Hq, N, D))
    _expect(k_pool, "k_pool", torch.bfloat16, _kv_shape(shape))
    _expect(page_table, "page_table", torch.int32, (B, s.pages_per_seq))
    _expect(order, "order", torch.int32, (B, Hq, shape.num_q_blocks, kc))
    _expect(count, "count", torch.int32, (B, Hq, shape.num_q_blocks))
    if scores is not None:
        _expect(scores, "scores", torch.float32, (B, Hq, shape.num_q_blocks, shape.num_pages))
    if hrm is not None:
        _expect(hrm, "hrm", torch.uint8, (B, Hq, shape.num_q_blocks, shape.num_pages))
    if workspace is None or not workspace.is_cuda:
        raise ValueError("workspace must be a CUDA tensor")
    nbytes = workspace.numel() * workspace.element_size()
    _check(lib().cosa_kap_select(ctypes.byref(s), ctypes.byref(k), _ptr(q), _ptr(k_pool),
                                 _ptr(page_table), _ptr(order), _ptr(count), _ptr(scores),
                                 _ptr(hrm), _ptr(workspace), nbytes, _stream(stream)),
           "cosa_kap_select")


def cosa_kap_pool(shape: Shape, kap: KapParams, q, k_pool, page_table, workspace,
                  stream=None) -> None:
    """Stage 1, downsampling alone: pooled queries and keys into the workspace."""
    import torch
    s, k = shape.c(), kap.c(shape)
    B, Hq, N, D = shape.batch, shape.num_q_heads, shape.seq_len, shape.head_dim
    _expect(q, "q", torch.bfloat16, (B, Hq, N, D))
    _expect(k_pool, "k_pool", torch.bfloat16, _kv_shape(shape))
    _expect(page_table, "page_table", torch.int32, (B, s.pages_per_seq))
    if workspace is None or not workspace.is_cuda:
        raise ValueError("workspace must be a CUDA tensor")
    nbytes = workspace.numel() * workspace.element_size()
    _check(lib().cosa_kap_pool(ctypes.byref(s), ctypes.byref(k), _ptr(q), _ptr(k_pool),
                               _ptr(page_table), _ptr(workspace), nbytes, _stream(stream)),
           "cosa_kap_pool")


def cosa_kap_rank(shape: Shape, kap: KapParams, order, count, workspace, scores=None, hrm=None,
                  stream=None) -> None:
    """Stage 1 after cosa_kap_pool on the same workspace: scores, MaxPool, MaxNorm,
    HRM, selection and ordering (order, count, optional scores / hrm)."""
    import torch
    s, k = shape.c(), kap.c(shape)
    B, Hq = shape.batch, shape.num_q_heads
    kc = cosa_kap_kcap(shape, kap)
    _expect(order, "order", torch.int32, (B, Hq, shape.num_q_blocks, kc))
    _expect(count, "count", torch.int32, (B, Hq, shape.num_q_blocks))
    if scores is not None:
        _expect(scores, "scores", torch.float32, (B, Hq, shape.num_q_blocks, shape.num_pages))
    if hrm is not None:
        _expect(hrm, "hrm", torch.uint8, (B, Hq, shape.num_q_blocks, shape.num_pages))
    if workspace is None or not workspace.is_cuda:
        raise ValueError("workspace must be a CUDA tensor")
    nbytes = workspace.numel() * workspace.element_size()
    _check(lib().cosa_kap_rank(ctypes.byref(s), ctypes.byref(k), _ptr(order), _ptr(count),
                               _ptr(scores), _ptr(hrm), _ptr(workspace), nbytes, _stream(stream)),
           "cosa_kap_rank")


def cosa_prefill_write(shape: Shape, kap: KapParams, q_tok, k_tok, v_tok, page_table, q, k_pool,
                       v_pool, workspace=None, stream=None) -> None:
    """Write token-major Q / K / V ([B][N][H][D]) as head-major q and the paged k_pool /
    v_pool, pooling Q and K into the KAP workspace in the same pass (workspace None: the
    plain write).  cosa_kap_rank on that workspace then finishes Stage 1."""
    import torch
    s, k = shape.c(), kap.c(shape)
    B, Hq, Hk, N, D = shape.batch, shape.num_q_heads, shape.num_kv_heads, shape.seq_len, shape.head_dim
    _expect(q_tok, "q_tok", torch.bfloat16, (B, N, Hq, D))
    _expect(k_tok, "k_tok", torch.bfloat16, (B, N, Hk, D))
    _expect(v_tok, "v_tok", torch.bfloat16, (B, N, Hk, D))
    _expect(page_table, "page_table", torch.int32, (B, s.pages_per_seq))
    _expect(q, "q", torch.bfloat16, (B, Hq, N, D))
    _expect(k_pool, "k_pool", torch.bfloat16, _kv_shape(shape))
    _expect(v_pool, "v_pool", torch.bfloat16, _kv_shape(shape))
    nbytes = 0
    if workspace is not None:
        if not workspace.is_cuda:
            raise ValueError("workspace must be a CUDA tensor")
        nbytes = workspace.numel() * workspace.element_size()
    _check(lib().cosa_prefill_write(ctypes.byref(s), ctypes.byref(k), _ptr(q_tok), _ptr(k_tok),
                                    _ptr(v_tok), _ptr(page_table), _ptr(q), _ptr(k_pool),
                                    _ptr(v_pool), _ptr(workspace), nbytes, _stream(stream)),
           "cosa_prefill_write")


def cosa_kap_preskip(shape: Shape, kap: KapParams, eps: float, margin: float, order, count,
                     workspace, skip_log=None, stream=None) -> None:
    """Proxy-bound pre-skip (not the pages' rule): filter the lists cosa_kap_select just
    wrote with this workspace, in place; skip_log gets 1 at the removed positions."""
    import torch
    s, k = shape.c(), kap.c(shape)
    B, Hq = shape.batch, shape.num_q_heads
    kc = cosa_kap_kcap(shape, kap)
    _expect(order, "order", torch.int32, (B, Hq, shape.num_q_blocks, kc))
    _expect(count, "count", torch.int32, (B, Hq, shape.num_q_blocks))
    if skip_log is not None:
        _expect(skip_log, "skip_log", torch.uint8, (B, Hq, shape.num_q_blocks, kc))
    if workspace is None or not workspace.is_cuda:
        raise ValueError("workspace must be a CUDA tensor")
    nbytes = workspace.numel() * workspace.element_size()
    _check(lib().cosa_kap_preskip(ctypes.byref(s), ctypes.byref(k), float(eps), float(margin),
                                  _ptr(order), _ptr(count), _ptr(skip_log), _ptr(workspace),
                                  nbytes, _stream(stream)), "cosa_kap_preskip")


def cosa_kap_select_group(shape: Shape, kap: KapParams, q, k_pool, page_table, order, count,
                          workspace, scores=None, hrm=None, stream=None) -> None:
    """Stage 1 with one list per KV head (group-shared selection): order
    [B][H_kv][nQB][k_cap], count [B][H_kv][nQB]; scores / hrm, when given,
    [B][H_kv][nQB][nP]."""
    import torch
    s, k = shape.c(), kap.c(shape)
    B, Hq, Hk, N, D = shape.batch, shape.num_q_heads, shape.num_kv_heads, shape.seq_len, shape.head_dim
    kc = cosa_kap_kcap(shape, kap)
    _expect(q, "q", torch.bfloat16, (B, Hq, N, D))
    _expect(k_pool, "k_pool", torch.bfloat16, _kv_shape(shape))
    _expect(page_table, "page_table", torch.int32, (B, s.pages_per_seq))
    _expect(order, "order", torch.int32, (B, Hk, shape.num_q_blocks, kc))
    _expect(count, "count", torch.int32, (B, Hk, shape.num_q_blocks))
    if scores is not None:
        _expect(scores, "scores", torch.float32, (B, Hk, shape.num_q_blocks, shape.num_pages))
    if hrm is not None:
        _expect(hrm, "hrm", torch.uint8, (B, Hk, shape.num_q_blocks, shape.num_pages))
    if workspace is None or not workspace.is_cuda:
        raise ValueError("workspace must be a CUDA tensor")
    nbytes = workspace.numel() * workspace.element_size()
    _check(lib().cosa_kap_select_group(ctypes.byref(s), ctypes.byref(k), _ptr(q), _ptr(k_pool),
                                       _ptr(page_table), _ptr(order), _ptr(count), _ptr(scores),
                                       _ptr(hrm), _ptr(workspace), nbytes, _stream(stream)),
           "cosa_kap_select_group")


def cosa_kap_select_noalloc(shape: Shape, kap: KapParams, q, k_pool, page_table, order, count,
                            scores=None, hrm=None, stream=None) -> None:
    """Stage 1 without a caller workspace: for callers that cannot allocate
    device memory.  The library's fixed scratch array is used instead; shapes
    whose workspace exceeds NOALLOC_SCRATCH_BYTES are rejected.  Calls that
    overlap on the GPU share that array and race."""
    import torch
    s, k = shape.c(), kap.c(shape)
    B, Hq, N, D = shape.batch, shape.num_q_heads, shape.seq_len, shape.head_dim
    kc = cosa_kap_kcap(shape, kap)
    _expect(q, "q", torch.bfloat16, (B, Hq, N, D))
    _expect(k_pool, "k_pool", torch.bfloat16, _kv_shape(shape))
    _expect(page_table, "page_table", torch.int32, (B, s.pages_per_seq))
    _expect(order, "order", torch.int32, (B, Hq, shape.num_q_blocks, kc))
    _expect(count, "count", torch.int32, (B, Hq, shape.num_q_blocks))
    if scores is not None:
        _expect(scores, "scores", torch.float32, (B, Hq, shape.num_q_blocks, shape.num_pages))
    if hrm is not None:
        _expect(hrm, "hrm", torch.uint8, (B, Hq, shape.num_q_blocks, shape.num_pages))
    _check(lib().cosa_kap_select_noalloc(ctypes.byref(s), ctypes.byref(k), _ptr(q), _ptr(k_pool),
                                         _ptr(page_table), _ptr(order), _ptr(count), _ptr(scores),
                                         _ptr(hrm), _stream(stream)), "cosa_kap_select_noalloc")


def cosa_kap_order(shape: Shape, kap: KapParams, scores, hrm, order, count, stream=None) -> None:
    """Stage 1, selection + ordering only, from given fp32 scores and u8 HRM flags."""
    import torch
    s, k = shape.c(), kap.c(shape)
    B, Hq = shape.batch, shape.num_q_heads
    kc = cosa_kap_kcap(shape, kap)
    _expect(scores, "scores", torch.float32, (B, Hq, shape.num_q_blocks, shape.num_pages))
    _expect(hrm, "hrm", torch.uint8, (B, Hq, shape.num_q_blocks, shape.num_pages))
    _expect(order, "order", torch.int32, (B, Hq, shape.num_q_blocks, kc))
    _expect(count, "count", torch.int32, (B, Hq, shape.num_q_blocks))
    _check(lib().cosa_kap_order(ctypes.byref(s), ctypes.byref(k), _ptr(scores), _ptr(hrm),
                                _ptr(order), _ptr(count), _stream(stream)), "cosa_kap_order")


def cosa_osk_attention(shape: Shape, osk: OskParams, q, k_pool, v_pool, page_table, order, count,
                       out, lse=None, computed=None, skip_log=None, stream=None) -> None:
    """Stage 2: ordered-skipping attention over the listed pages."""
    import torch
    s, o = shape.c(), osk.c()
    B, Hq, N, D = shape.batch, shape.num_q_heads, shape.seq_len, shape.head_dim
    if order is None or order.dim() != 4:
        raise ValueError("order must be int32 [B][H_q][nQB][k_cap]")
    kc = int(order.shape[-1])
    _expect(q, "q", torch.bfloat16, (B, Hq, N, D))
    _expect(k_pool, "k_pool", torch.bfloat16, _kv_shape(shape))
    _expect(v_pool, "v_pool", torch.bfloat16, _kv_shape(shape))
    _expect(page_table, "page_table", torch.int32, (B, s.pages_per_seq))
    _expect(order, "order", torch.int32, (B, Hq, shape.num_q_blocks, kc))
    _expect(count, "count", torch.int32, (B, Hq, shape.num_q_blocks))
    _expect(out, "out", torch.bfloat16, (B, Hq, N, D))
    if lse is not None:
        _expect(lse, "lse", torch.float32, (B, Hq, N))
    if computed is not None:
        _expect(computed, "computed", torch.int32, (B, Hq, shape.num_q_blocks))
    if skip_log is not None:
        _expect(skip_log, "skip_log", torch.uint8, (B, Hq, shape.num_q_blocks, kc))
    _check(lib().cosa_osk_attention(ctypes.byref(s), ctypes.byref(o), _ptr(q), _ptr(k_pool),
                                    _ptr(v_pool), _ptr(page_table), _ptr(order), _ptr(count), kc,
                                    _ptr(out), _ptr(lse), _ptr(computed), _ptr(skip_log),
                                    _stream(stream)), "cosa_osk_attention")


def cosa_osk_attention_group(shape: Shape, osk: OskParams, q, k_pool, v_pool, page_table, order,
                             count, out, lse=None, computed=None, skip_log=None,
                             stream=None) -> None:
    """Stage 2 over group-shared lists: order [B][H_kv][nQB][k_cap], count
    [B][H_kv][nQB]; every query head runs its own skip rule on its KV head's list."""
    import torch
    s, o = shape.c(), osk.c()
    B, Hq, Hk, N, D = shape.batch, shape.num_q_heads, shape.num_kv_heads, shape.seq_len, shape.head_dim
    if order is None or order.dim() != 4:
        raise ValueError("order must be int32 [B][H_kv][nQB][k_cap]")
    kc = int(order.shape[-1])
    _expect(q, "q", torch.bfloat16, (B, Hq, N, D))
    _expect(k_pool, "k_pool", torch.bfloat16, _kv_shape(shape))
    _expect(v_pool, "v_pool", torch.bfloat16, _kv_shape(shape))
    _expect(page_table, "page_table", torch.int32, (B, s.pages_per_seq))
    _expect(order, "order", torch.int32, (B, Hk, shape.num_q_blocks, kc))
    _expect(count, "count", torch.int32, (B, Hk, shape.num_q_blocks))
    _expect(out, "out", torch.bfloat16, (B, Hq, N, D))
    if lse is not None:
        _expect(lse, "lse", torch.float32, (B, Hq, N))
    if computed is not None:
        _expect(computed, "computed", torch.int32, (B, Hq, shape.num_q_blocks))
    if skip_log is not None:
        _expect(skip_log, "skip_log", torch.uint8, (B, Hq, shape.num_q_blocks, kc))
    _check(lib().cosa_osk_attention_group(ctypes.byref(s), ctypes.byref(o), _ptr(q), _ptr(k_pool),
                                          _ptr(v_pool), _ptr(page_table), _ptr(order), _ptr(count),
                                          kc, _ptr(out), _ptr(lse), _ptr(computed), _ptr(skip_log),
                                          _stream(stream)), "cosa_osk_attention_group")


def cosa_osk_decode_workspace_size(shape: Shape, k_cap: int) -> int:
    s = shape.c()
    n = ctypes.c_size_t(0)
    _check(lib().cosa_osk_decode_workspace_size(ctypes.byref(s), int(k_cap), ctypes.byref(n)),
           "cosa_osk_decode_workspace_size")
    return n.value


def cosa_osk_decode(shape: Shape, osk: OskParams, q, k_pool, v_pool, page_table, positions, order,
                    count, out, workspace, lse=None, computed=None, skip_log=None,
                    stream=None) -> None:
    """Decode: the query of each sequence and head (q [B][H_q][D], at positions [B])
    visits its ordered page list (order [B][H_q][k_cap], count [B][H_q]) under the
    in-kernel skip rule; out [B][H_q][D]."""
    import torch
    s, o = shape.c(), osk.c()
    B, Hq, D = shape.batch, shape.num_q_heads, shape.head_dim
    kc = order.shape[-1]
    _expect(q, "q", torch.bfloat16, (B, Hq, D))
    _expect(k_pool, "k_pool", torch.bfloat16, _kv_shape(shape))
    _expect(v_pool, "v_pool", torch.bfloat16, _kv_shape(shape))
    _expect(page_table, "page_table", torch.int32, (B, s.pages_per_seq))
    _expect(positions, "positions", torch.int32, (B,))
    _expect(order, "order", torch.int32, (B, Hq, kc))
    _expect(count, "count", torch.int32, (B, Hq))
    _expect(out, "out", torch.bfloat16, (B, Hq, D))
    if lse is not None:
        _expect(lse, "lse", torch.float32, (B, Hq))
    if computed is not None:
        _expect(computed, "computed", torch.int32, (B, Hq))
    if skip_log is not None:
        _expect(skip_log, "skip_log", torch.uint8, (B, Hq, kc))
    if workspace is None or not workspace.is_cuda:
        raise ValueError("workspace must be a CUDA tensor")
    nbytes = workspace.numel() * workspace.element_size()
    _check(lib().cosa_osk_decode(ctypes.byref(s), ctypes.byref(o), _ptr(q), _ptr(k_pool),
                                 _ptr(v_pool), _ptr(page_table), _ptr(positions), _ptr(order),
                                 _ptr(count), kc, _ptr(out), _ptr(lse), _ptr(computed),
                                 _ptr(skip_log), _ptr(workspace), nbytes, _stream(stream)),
           "cosa_osk_decode")


def cosa_dense_attention(shape: Shape, q, k_pool, v_pool, page_table, out, lse=None,
                         stream=None) -> None:
    """Dense causal attention over the same paged cache (comparison point)."""
    import torch
    s = shape.c()
    B, Hq, N, D = shape.batch, shape.num_q_heads, shape.seq_len, shape.head_dim
    _expect(q, "q", torch.bfloat16, (B, Hq, N, D))
    _expect(k_pool, "k_pool", torch.bfloat16, _kv_shape(shape))
    _expect(v_pool, "v_pool", torch.bfloat16, _kv_shape(shape))
    _expect(page_table, "page_table", torch.int32, (B, s.pages_per_seq))
    _expect(out, "out", torch.bfloat16, (B, Hq, N, D))
    if lse is not None:
        _expect(lse, "lse", torch.float32, (B, Hq, N))
    _check(lib().cosa_dense_attention(ctypes.byref(s), _ptr(q), _ptr(k_pool), _ptr(v_pool),
                                      _ptr(page_table), _ptr(out), _ptr(lse), _stream(stream)),
           "cosa_dense_attention")


def cosa_attention_host_workspace_size(shape: Shape, kap: KapParams) -> int:
    out = ctypes.c_size_t(0)
    s, k = shape.c(), kap.c(shape)
    _check(lib().cosa_attention_host_workspace_size(ctypes.byref(s), ctypes.byref(k),
                                                    ctypes.byref(out)),
           "cosa_attention_host_workspace_size")
    return out.value


def _expect_host(t, name, dtype, shape):
    if t is None:
        raise ValueError(f"{name} is required")
    if t.dtype != dtype:
        raise TypeError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.is_cuda:
        raise ValueError(f"{name} must be a host (CPU) tensor, page-locked for overlap")


def cosa_attention_host(shape: Shape, kap: KapParams, osk: OskParams, q, k_pool, v_pool,
                        page_table, out, workspace, stream=None) -> None:
    """Both stages from host tensors, pipelined per KV head (copies overlap the kernels)."""
    import torch
    s, k, o = shape.c(), kap.c(shape), osk.c()
    B, Hq, N, D = shape.batch, shape.num_q_heads, shape.seq_len, shape.head_dim
    _expect_host(q, "q", torch.bfloat16, (B, Hq, N, D))
    _expect_host(k_pool, "k_pool", torch.bfloat16, _kv_shape(shape))
    _expect_host(v_pool, "v_pool", torch.bfloat16, _kv_shape(shape))
    _expect_host(page_table, "page_table", torch.int32, (B, s.pages_per_seq))
    _expect_host(out, "out", torch.bfloat16, (B, Hq, N, D))
    if workspace is None or workspace.dtype != torch.uint8 or not workspace.is_cuda:
        raise ValueError("workspace must be a CUDA uint8 tensor")
    _check(lib().cosa_attention_host(ctypes.byref(s), ctypes.byref(k), ctypes.byref(o), _ptr(q),
                                     _ptr(k_pool), _ptr(v_pool), _ptr(page_table), _ptr(out),
                                     _ptr(workspace), workspace.numel(), _stream(stream)),
           "cosa_attention_host")


def cosa_debug_osk_wait_fault(withhold_k_group: int, wait_limit_ns: int = 0) -> None:
    """Test hook: the next cosa_osk_attention call from this thread runs with its waits
    limited to wait_limit_ns and the K copies of listed group withhold_k_group never
    issued (-1: none), so that a wait runs out on purpose (see cosa.h)."""
    _check(lib().cosa_debug_osk_wait_fault(int(withhold_k_group), int(wait_limit_ns)),
           "cosa_debug_osk_wait_fault")


def cosa_get_status(stream=None) -> int:
    """Read and clear the device status word (0 = ok); synchronises the stream."""
    return lib().cosa_get_status(_stream(stream))
