"""Plain, slow CPU oracle for CoSA: Kernel-Aware Proxy (KAP) + Ordered-Skipping
Kernel (OSK) causal prefill attention over a paged KV cache.

TEST INFRASTRUCTURE.  Only tests, the smoke check and the benchmark's
CPU-baseline leg may import this module; the product path never does.  It
shares no code with the CUDA library: it reads the same seeded inputs and
nothing else.

Sources (the only description of the method; no code was published with it):
  [ABS]   "CoSA: Accelerating Long-Context Inference via Proxy-Kernel
          Co-Designed Sparse Attention", abstract (as printed on
          insight.artgrammer.co.kr/papers/23508 and fugumt.com).
  [TS]    the same paper's technical summary on gist.science/pt/paper/2607.25291:
          §2.1 "Princípios de Design Central", §2.2 "Estágio 1: KAP"
          ("Ranking de Blocos", "Geração de Flag HRM", "Ordenação por Grupo de
          Flags"), §2.3 "Estágio 2: OSK" ("Saltado pela Máscara", "Saltado no
          Kernel", "Computado").
Where the pages leave a step open, the reading taken is stated at the step.

All arithmetic is float64 on the (bf16-rounded) input values, except where a
floating-point value decides an integer result: the page ranking key packs the
score as float32 bits, the kernel's precision, on both sides.

Notation: B batch, H_q / H_kv heads, G = H_q / H_kv, N tokens, D head dim,
P page size, Bq q-block, nP = N / P pages, nQB = N / Bq q-blocks,
R = Bq / q_sub query representatives per q-block, T = P / k_sub sub-keys per page.

Pins (tests/test_oracle_pins.py) tie every function here to something other
than itself: brute force, closed forms, library routines, invariants.  The
absolute *quality* of the proxy's selection has no worked values on the pages;
it is reported (softmax-mass recall), not pinned.
"""
from __future__ import annotations

import math
from typing import Optional, Sequence

import numpy as np

__all__ = [
    "causal_pages", "forced_pages", "budget_count", "k_cap",
    "gather_logical", "kap_pool_queries", "kap_pool_keys", "kap_block_scores",
    "kap_maxnorm_hrm", "rank_key", "kap_order_from_scores", "kap_select_block",
    "kap_select", "kap_order", "osk_block", "osk_block_rules", "osk_attention", "dense_rows",
    "dense_attention", "kap_group_scores", "kap_select_group", "expand_group_order",
    "kap_preskip", "kap_preskip_lists", "osk_decode",
]

NEG_INF = -math.inf


# ----------------------------------------------------------------------------
# page arithmetic
# ----------------------------------------------------------------------------
def causal_pages(qb: int, q_block: int, page_size: int) -> int:
    """n_b: pages holding at least one key a row of q-block qb may see under
    the causal mask (query i sees keys 0..i).  Last row is (qb+1)*Bq - 1."""
    return ((qb + 1) * q_block + page_size - 1) // page_size


def forced_pages(qb: int, q_block: int, page_size: int, sink_pages: int) -> list:
    """Pages always kept (reading: the sink page(s) and the "local" pages,
    i.e. the pages overlapping the q-block's own token range).  The pages fix
    neither; this is the plainest sink + local-window choice."""
    n_b = causal_pages(qb, q_block, page_size)
    first_diag = (qb * q_block) // page_size
    forced = set(range(min(sink_pages, n_b)))
    forced.update(range(first_diag, n_b))
    return sorted(forced)


def budget_count(qb: int, q_block: int, page_size: int, sink_pages: int,
                 budget: float) -> int:
    """k_b: pages KAP keeps for q-block qb under a "moderate budget" [ABS],
    [TS §2.2].  Reading: budget = fraction of the block's causal pages,
    rounded up, never below the forced set, never above n_b.  The product
    beta * n_b is the float32 product (round to nearest) of the float32 budget
    the C interface carries and n_b, so that a 10% budget of 10 pages is
    exactly one page; its ceiling then decides the integer on both sides."""
    n_b = causal_pages(qb, q_block, page_size)
    n_f = len(forced_pages(qb, q_block, page_size, sink_pages))
    prod = np.float32(budget) * np.float32(n_b)
    want = int(math.ceil(float(prod)))
    return min(n_b, max(n_f, want))


def k_cap(seq_len: int, q_block: int, page_size: int, sink_pages: int, budget: float) -> int:
    """Row length of the ordered page list: the largest k_b over q-blocks."""
    return max(budget_count(qb, q_block, page_size, sink_pages, budget)
               for qb in range(seq_len // q_block))


def gather_logical(pool: np.ndarray, page_table: np.ndarray, b: int, h_kv: int,
                   n_tokens: Optional[int] = None) -> np.ndarray:
    """Logical keys (or values) of sequence b, KV head h_kv, through the page
    table: token t lives at pool[page_table[b, t // P], h_kv, t % P]
    ("KV page remapping", [TS §2.3] "Saltado pela Máscara")."""
    P, D = pool.shape[2], pool.shape[3]
    pt = np.asarray(page_table[b], dtype=np.int64)
    if n_tokens is not None:
        pt = pt[: n_tokens // P]
    return np.asarray(pool[pt, h_kv], dtype=np.float64).reshape(-1, D)


# ----------------------------------------------------------------------------
# Stage 1: Kernel-Aware Proxy  ([TS §2.2])
# ----------------------------------------------------------------------------
def kap_pool_queries(q_bh: np.ndarray, q_block: int, q_sub: int) -> np.ndarray:
    """Query downsampling ("downsampling de queries", [TS §2.2] "Ranking de
    Blocos").  Reading: mean over each run of q_sub consecutive rows, so a
    q-block of Bq rows has R = Bq / q_sub representatives.
    q_bh [N][D] -> [nQB][R][D]."""
    N, D = q_bh.shape
    R = q_block // q_sub
    x = np.asarray(q_bh, dtype=np.float64).reshape(N // q_block, R, q_sub, D)
    return x.sum(axis=2) / q_sub


def kap_pool_keys(k_log: np.ndarray, page_size: int, k_sub: int) -> np.ndarray:
    """Key downsampling ([TS §2.2] "Ranking de Blocos").  Reading: mean over
    each run of k_sub consecutive keys of a page, T = P / k_sub sub-keys per
    page.  k_log [N][D] -> [nP][T][D]."""
    N, D = k_log.shape
    T = page_size // k_sub
    x = np.asarray(k_log, dtype=np.float64).reshape(N // page_size, T, k_sub, D)
    return x.sum(axis=2) / k_sub


def kap_block_scores(qhat_qb: np.ndarray, khat: np.ndarray, qb: int, q_block: int,
                     q_sub: int, page_size: int, k_sub: int, scale: float) -> np.ndarray:
    """Approximate scores then MaxPool over the keys of each page ([TS §2.2]
    "computa scores aproximados e aplica MaxPool sobre as chaves").

    a[r, p] = max over visible sub-keys t of scale * <qhat_r, khat_{p,t}>,
    -inf when rep r sees no sub-key of page p.  Reading for causality: sub-key
    t of page p is visible to rep r iff its first token p*P + t*k_sub is at or
    before the rep's last row qb*Bq + (r+1)*q_sub - 1.  Only the n_b causal
    pages are scored.  Returns a [R][n_b]."""
    R = qhat_qb.shape[0]
    T = khat.shape[1]
    n_b = causal_pages(qb, q_block, page_size)
    raw = np.einsum("rd,ptd->rpt", np.asarray(qhat_qb, np.float64),
                    np.asarray(khat[:n_b], np.float64)) * scale
    first_tok = (np.arange(n_b)[:, None] * page_size + np.arange(T)[None, :] * k_sub)
    last_row = qb * q_block + (np.arange(R) + 1) * q_sub - 1
    visible = first_tok[None, :, :] <= last_row[:, None, None]
    raw = np.where(visible, raw, NEG_INF)
    return raw.max(axis=2)


def kap_maxnorm_hrm(a: np.ndarray):
    """MaxNorm and Have-RowMax flags ([TS §2.2] "MaxNorm ... contribuições de
    ranking relativo", "Geração de Flag HRM").

    Reading of MaxNorm: normalise each representative row by its row max in
    the logit domain, exp(a - rowmax) in [0, 1], then average over the R rows:
        m_r  = max_p a[r, p]
        S[p] = (1/R) * sum_r exp(a[r, p] - m_r)
    HRM: page p is flagged when it holds the row max of some representative
    row r; if several pages tie for m_r, the lowest page index holds it.
    Returns (S float64 [n_b], hrm uint8 [n_b])."""
    R, n_b = a.shape
    m = a.max(axis=1)
    with np.errstate(invalid="ignore"):
        e = np.exp(a - m[:, None])          # exp(-inf) = 0
    S = e.sum(axis=0) / R
    hrm = np.zeros(n_b, dtype=np.uint8)
    for r in range(R):
        hrm[int(np.argmax(a[r]))] = 1       # argmax returns the first maximum
    return S, hrm


def rank_key(s32: float, hrm: int, page: int) -> int:
    """Ranking key of a page ([TS §2.2] "Ordenação por Grupo de Flags": HRM
    pages first, the rest by descending estimated score).  Reading for the
    order inside each flag group and for ties: score descending, then the
    lower page index first.  Packed as one unsigned 64-bit integer:
        hrm << 63 | float32_bits(S) << 31 | (2^31 - 1 - page)
    (S >= 0, so its float32 bit pattern orders like its value)."""
    bits = int(np.array([s32], dtype=np.float32).view(np.uint32)[0])
    return (int(hrm) << 63) | (bits << 31) | ((1 << 31) - 1 - int(page))


def kap_order_from_scores(S: Sequence[float], hrm: Sequence[int], qb: int, q_block: int,
                          page_size: int, budget: float, sink_pages: int,
                          ascending: bool = False) -> np.ndarray:
    """Budgeted selection and the computation-order mask M_KAP for one
    q-block ([ABS] "selects blocks under a moderate budget and produces an
    ordered mask"; [TS §2.1] "Máscara de Computação-Ordem"; [TS §2.2]).

    S (rounded to float32 here: the precision the kernel decides in) and hrm
    cover the block's n_b causal pages.  The forced pages are kept; the
    remaining k_b - |forced| slots go to the non-forced pages with the largest
    keys; the kept set is then listed by key, largest first.  With
    ascending=True the kept set is listed by page index instead (a
    binary-mask proxy's visit order, the comparison the pages argue against).
    Returns int32 [k_b] logical page ids."""
    n_b = causal_pages(qb, q_block, page_size)
    forced = forced_pages(qb, q_block, page_size, sink_pages)
    k_b = budget_count(qb, q_block, page_size, sink_pages, budget)
    s32 = np.asarray(S[:n_b], dtype=np.float64).astype(np.float32)
    keys = {p: rank_key(float(s32[p]), int(hrm[p]), p) for p in range(n_b)}
    fset = set(forced)
    rest = sorted((p for p in range(n_b) if p not in fset), key=lambda p: keys[p], reverse=True)
    kept = list(forced) + rest[: k_b - len(forced)]
    if ascending:
        kept.sort()
    else:
        kept.sort(key=lambda p: keys[p], reverse=True)
    return np.asarray(kept, dtype=np.int32)


def kap_select_block(q_bh: np.ndarray, k_log: np.ndarray, qb: int, *, q_block: int,
                     page_size: int, q_sub: int, k_sub: int, scale: float,
                     budget: float, sink_pages: int, ascending: bool = False,
                     khat: Optional[np.ndarray] = None):
    """All KAP steps for one (b, h_q, q-block): pool, score, MaxPool, MaxNorm,
    HRM, select, order.  Returns (order int32 [k_b], S float64 [n_b],
    hrm uint8 [n_b], a float64 [R][n_b])."""
    rows = slice(qb * q_block, (qb + 1) * q_block)
    qhat = kap_pool_queries(q_bh[rows], q_block, q_sub)[0]
    if khat is None:
        khat = kap_pool_keys(k_log, page_size, k_sub)
    a = kap_block_scores(qhat, khat, qb, q_block, q_sub, page_size, k_sub, scale)
    S, hrm = kap_maxnorm_hrm(a)
    order = kap_order_from_scores(S, hrm, qb, q_block, page_size, budget, sink_pages, ascending)
    return order, S, hrm, a


def kap_select(q: np.ndarray, k_pool: np.ndarray, page_table: np.ndarray, *,
               num_kv_heads: int, page_size: int, q_block: int, q_sub: int,
               k_sub: int, scale: float, budget: float, sink_pages: int,
               ascending: bool = False, heads: Optional[Sequence] = None,
               qblocks: Optional[Sequence[int]] = None):
    """KAP over a whole problem (or a subset of (b, h_q) heads / q-blocks).

    q [B][H_q][N][D]; k_pool [phys][H_kv][P][D]; page_table [B][nP].
    Returns dict with order int32 [B][H_q][nQB][k_cap] (-1 padded), count
    int32 [B][H_q][nQB], S float64 [B][H_q][nQB][nP] and hrm uint8 (zero past
    n_b).  Entries for heads / q-blocks not requested stay -1 / 0."""
    B, Hq, N, D = q.shape
    G = Hq // num_kv_heads
    nP, nQB = N // page_size, N // q_block
    kc = k_cap(N, q_block, page_size, sink_pages, budget)
    order = np.full((B, Hq, nQB, kc), -1, dtype=np.int32)
    count = np.zeros((B, Hq, nQB), dtype=np.int32)
    S_all = np.zeros((B, Hq, nQB, nP), dtype=np.float64)
    hrm_all = np.zeros((B, Hq, nQB, nP), dtype=np.uint8)
    if heads is None:
        heads = [(b, h) for b in range(B) for h in range(Hq)]
    if qblocks is None:
        qblocks = range(nQB)
    khat_cache = {}
    for (b, h) in heads:
        hk = h // G
        if (b, hk) not in khat_cache:
            k_log = gather_logical(k_pool, page_table, b, hk, N)
            khat_cache[(b, hk)] = kap_pool_keys(k_log, page_size, k_sub)
        khat = khat_cache[(b, hk)]
        q_bh = np.asarray(q[b, h], dtype=np.float64)
        for qb in qblocks:
            o, S, hr, _ = kap_select_block(q_bh, None, qb, q_block=q_block, page_size=page_size,
                                           q_sub=q_sub, k_sub=k_sub, scale=scale, budget=budget,
                                           sink_pages=sink_pages, ascending=ascending, khat=khat)
            order[b, h, qb, :len(o)] = o
            count[b, h, qb] = len(o)
            S_all[b, h, qb, :len(S)] = S
            hrm_all[b, h, qb, :len(hr)] = hr
    return {"order": order, "count": count, "S": S_all, "hrm": hrm_all, "k_cap": kc}


def kap_order(scores: np.ndarray, hrm: np.ndarray, *, page_size: int, q_block: int,
              budget: float, sink_pages: int, ascending: bool = False):
    """Selection and ordering alone, from given float32 scores and HRM flags
    laid out [B][H_q][nQB][nP] (entries past n_b ignored)."""
    B, Hq, nQB, nP = scores.shape
    N = nQB * q_block
    kc = k_cap(N, q_block, page_size, sink_pages, budget)
    order = np.full((B, Hq, nQB, kc), -1, dtype=np.int32)
    count = np.zeros((B, Hq, nQB), dtype=np.int32)
    for b in range(B):
        for h in range(Hq):
            for qb in range(nQB):
                o = kap_order_from_scores(scores[b, h, qb], hrm[b, h, qb], qb, q_block,
                                          page_size, budget, sink_pages, ascending)
                order[b, h, qb, :len(o)] = o
                count[b, h, qb] = len(o)
    return order, count


# ----------------------------------------------------------------------------
# Group-shared selection: one ordered list per (b, h_kv, q-block) for the G
# query heads that read the same KV head.  The pages do not describe it; the
# readings are:
#   S_group[p]   = max over the G heads of that head's MaxNorm score S_h[p]
#                  (a page one head ranks highly stays high for the group),
#   HRM_group[p] = 1 when the page holds a row max of any head's rows,
# then the same forced pages, budget, key and order as per-head selection
# ([TS §2.2]).  Every head of the group then runs the per-head OSK skip rule
# on the shared list (osk_block, unchanged).
# ----------------------------------------------------------------------------
def kap_group_scores(S_heads: np.ndarray, hrm_heads: np.ndarray):
    """Aggregate per-head MaxNorm scores [G][n_b] and HRM flags [G][n_b] of one
    (b, h_kv, q-block) into the group's (S float64 [n_b], hrm uint8 [n_b])."""
    S = np.max(np.asarray(S_heads, dtype=np.float64), axis=0)
    hrm = (np.asarray(hrm_heads) != 0).any(axis=0).astype(np.uint8)
    return S, hrm


def kap_select_group(q: np.ndarray, k_pool: np.ndarray, page_table: np.ndarray, *,
                     num_kv_heads: int, page_size: int, q_block: int, q_sub: int,
                     k_sub: int, scale: float, budget: float, sink_pages: int,
                     groups: Optional[Sequence] = None,
                     qblocks: Optional[Sequence[int]] = None):
    """Group-shared KAP over a whole problem (or a subset of (b, h_kv) groups /
    q-blocks).  Each head's S and HRM come from the per-head steps
    (kap_select_block); kap_group_scores aggregates them; kap_order_from_scores
    selects and orders.  Returns dict with order int32 [B][H_kv][nQB][k_cap]
    (-1 padded), count int32 [B][H_kv][nQB], S float64 and hrm uint8
    [B][H_kv][nQB][nP] (zero past n_b)."""
    B, Hq, N, D = q.shape
    G = Hq // num_kv_heads
    nP, nQB = N // page_size, N // q_block
    kc = k_cap(N, q_block, page_size, sink_pages, budget)
    order = np.full((B, num_kv_heads, nQB, kc), -1, dtype=np.int32)
    count = np.zeros((B, num_kv_heads, nQB), dtype=np.int32)
    S_all = np.zeros((B, num_kv_heads, nQB, nP), dtype=np.float64)
    hrm_all = np.zeros((B, num_kv_heads, nQB, nP), dtype=np.uint8)
    if groups is None:
        groups = [(b, hk) for b in range(B) for hk in range(num_kv_heads)]
    if qblocks is None:
        qblocks = range(nQB)
    for (b, hk) in groups:
        k_log = gather_logical(k_pool, page_table, b, hk, N)
        khat = kap_pool_keys(k_log, page_size, k_sub)
        q_heads = [np.asarray(q[b, hk * G + g], dtype=np.float64) for g in range(G)]
        for qb in qblocks:
            Sh, Hh = [], []
            for g in range(G):
                _, S_g, h_g, _ = kap_select_block(q_heads[g], None, qb, q_block=q_block,
                                                  page_size=page_size, q_sub=q_sub, k_sub=k_sub,
                                                  scale=scale, budget=budget,
                                                  sink_pages=sink_pages, khat=khat)
                Sh.append(S_g)
                Hh.append(h_g)
            S, hr = kap_group_scores(np.stack(Sh), np.stack(Hh))
            o = kap_order_from_scores(S, hr, qb, q_block, page_size, budget, sink_pages)
            order[b, hk, qb, :len(o)] = o
            count[b, hk, qb] = len(o)
            S_all[b, hk, qb, :len(S)] = S
            hrm_all[b, hk, qb, :len(hr)] = hr
    return {"order": order, "count": count, "S": S_all, "hrm": hrm_all, "k_cap": kc}


def expand_group_order(order_g: np.ndarray, count_g: np.ndarray, num_q_heads: int):
    """Per-head lists [B][H_q][nQB][k_cap] from group lists [B][H_kv][nQB][k_cap]:
    head h reads the list of its KV head h // G (for osk_attention)."""
    B, Hkv = count_g.shape[:2]
    G = num_q_heads // Hkv
    hk = np.arange(num_q_heads) // G
    return order_g[:, hk], count_g[:, hk]


# ----------------------------------------------------------------------------
# Proxy-bound pre-skip: a variant the pages do not give (off unless asked).
# The pages' in-kernel rule ([TS §2.3] "Saltado no Kernel") compares a page's
# exact local max with the exact running max, so every listed page still costs
# its K load and QK^T.  This variant applies the same kind of test one stage
# earlier, on the proxy's page maxima a[r][p] (kap_block_scores) and the proxy's
# own running max along the ordered list, and removes the pages it rejects from
# the list, so the kernel never visits them.  Reading (a proxy-estimated logit
# compared with a running max, in its plainest form): along the list
# L = (p_0, p_1, ...),
#   ahat_r(j) = max over positions j' < j of a[r][p_j'];
#   representative r keeps position j iff a[r][p_j] > -inf and (ahat_r(j) = -inf
#     or a[r][p_j] + margin - ahat_r(j) >= ln(eps));
#   position j >= 1 is pre-skipped iff no representative keeps it; position 0
#   is always kept; eps = 0 pre-skips nothing.
# The surviving pages keep their order and go to the kernel's own rule.  The
# margin (>= 0, in nats) is slack for the proxy's error: pooled scores are
# estimates of a page's logits, not bounds on them, so the quality of the
# pages this removes is measured against the full rule, not guaranteed.
# ----------------------------------------------------------------------------
def kap_preskip(order: Sequence[int], a: np.ndarray, eps: float, margin: float):
    """Pre-skip along one q-block's ordered list.  order: logical page ids;
    a [R][n_b]: the block's proxy page maxima.  Returns (kept int32 list,
    skipped uint8 [len(order)], margin float64 [len(order)] = max over the
    representatives that see the page of (a + margin - ahat) minus ln(eps),
    +inf where a representative that sees the page has ahat = -inf, NaN at
    position 0)."""
    a = np.asarray(a, dtype=np.float64)
    R = a.shape[0]
    n = len(order)
    log_eps = math.log(eps) if eps > 0 else NEG_INF
    ahat = np.full(R, NEG_INF)
    skipped = np.zeros(n, dtype=np.uint8)
    tested = np.full(n, np.nan)
    kept = []
    for j, p in enumerate(order):
        col = a[:, int(p)]
        if j > 0:
            best = NEG_INF
            for r in range(R):
                if col[r] == NEG_INF:
                    continue                    # this representative sees no key of p
                if ahat[r] == NEG_INF:
                    best = math.inf             # its first visible page: kept
                else:
                    best = max(best, col[r] + margin - ahat[r])
            tested[j] = best - log_eps if log_eps > NEG_INF else math.inf
            if log_eps > NEG_INF and best < log_eps:
                skipped[j] = 1
        if not skipped[j]:
            kept.append(int(p))
        ahat = np.maximum(ahat, col)
    return np.asarray(kept, dtype=np.int32), skipped, tested


def kap_preskip_lists(order: np.ndarray, count: np.ndarray, a_of, eps: float, margin: float,
                      tiles: Optional[Sequence] = None):
    """kap_preskip over whole lists [B][H][nQB][k_cap] / counts [B][H][nQB].
    a_of(b, h, qb) gives that block's a [R][n_b].  Returns dict with order
    (survivors first, -1 padded), count, skipped uint8 [B][H][nQB][k_cap] (at the
    original list positions) and margin float64 (same layout, NaN past count).
    Tiles not requested keep their list (skipped 0, margin NaN)."""
    B, H, nQB, kc = order.shape
    out_o = order.copy()
    out_c = count.copy()
    skipped = np.zeros(order.shape, dtype=np.uint8)
    tested = np.full(order.shape, np.nan)
    if tiles is None:
        tiles = [(b, h, qb) for b in range(B) for h in range(H) for qb in range(nQB)]
    for (b, h, qb) in tiles:
        n = int(count[b, h, qb])
        kept, sk, mg = kap_preskip(order[b, h, qb, :n], a_of(b, h, qb), eps, margin)
        out_o[b, h, qb, :] = -1
        out_o[b, h, qb, :len(kept)] = kept
        out_c[b, h, qb] = len(kept)
        skipped[b, h, qb, :n] = sk
        tested[b, h, qb, :n] = mg
    return {"order": out_o, "count": out_c, "skipped": skipped, "margin": tested}


# ----------------------------------------------------------------------------
# Stage 2: Ordered-Skipping Kernel  ([TS §2.1], [TS §2.3])
# ----------------------------------------------------------------------------
def osk_block_rules(q_rows: np.ndarray, k_log: np.ndarray, v_log: np.ndarray, qb: int,
                    q_block: int, page_size: int, order: Sequence[int], eps: float,
                    scale: float, force: Optional[dict] = None, rule: str = "max",
                    max_run: Optional[int] = None) -> dict:
    """Ordered-skipping online-softmax attention for one q-block, under the
    pages' skip rule (rule="max") or one of two variants the pages do not give
    (rule="sum", max_run): see the end of this docstring.

    Pages are visited in the order given ([ABS] "the order in which KV pages
    are visited in the kernel inner loop"); online-softmax accumulation is
    order-independent ([TS §2.1] "Invariância de Ordem").  Unlisted pages are
    never touched ([TS §2.3] "Saltado pela Máscara").  For each listed page:
      s_ic   = scale * <q_i, k_c> for keys c of the page, -inf where c > i;
      m_loc_i = max_c s_ic;
      d_i    = m_loc_i - m_i (the "local max minus running max" of [TS §2.3]
               "Saltado no Kernel"); +inf when m_i = -inf; rows with
               m_loc_i = -inf take no part.
      Reading of the rule: the page is skipped iff it is not the first visited
      page and max_i d_i < ln(eps) (eps = 0 never skips).  One decision per
      q-block tile: a single row with a large d_i keeps the page (the "bucket
      effect" the pages name).  A skipped page leaves m, l and o unchanged.
      Otherwise ("Computado"):
        m'_i = max(m_i, m_loc_i); l_i = l_i e^{m_i - m'_i} + sum_c e^{s_ic - m'_i};
        o_i = o_i e^{m_i - m'_i} + sum_c e^{s_ic - m'_i} v_c; m_i = m'_i.
    Output o_i / l_i and lse_i = m_i + ln l_i (rows that saw no key: 0, -inf).

    force: optional {step j: bool skipped} overriding the rule at listed steps
    (used by tests to evaluate the alternative at steps whose decision lies
    within rounding of the threshold).

    Variants (not on the pages; stated here as they are computed):
      rule="sum": a row's test also weighs the page against the mass the row
        already holds: the page is skipped iff max_i (d_i + ln P - ln l_i) <
        ln(eps), l_i the running sum relative to the running max m_i.  Each of
        the page's at most P visible keys has weight <= e^{d_i} relative to m_i,
        so a skipped page would have added less than eps * l_i to row i's sum.
      max_run=r: after r consecutive skipped pages the rest of the list is
        skipped without being visited (no QK^T, no K load).
    Returns dict: out [Bq][D], lse [Bq], computed (pages with P V), visited
    (pages whose QK^T was evaluated), skip uint8 [len(order)], margin float64
    [len(order)] = the tested maximum minus ln(eps) (NaN past a break)."""
    Bq, D = q_rows.shape
    rows = qb * q_block + np.arange(Bq)
    qf = np.asarray(q_rows, dtype=np.float64)
    m = np.full(Bq, NEG_INF)
    l = np.zeros(Bq)
    o = np.zeros((Bq, D))
    log_eps = math.log(eps) if eps > 0 else NEG_INF
    n = len(order)
    skip_log = np.zeros(n, dtype=np.uint8)
    margin = np.full(n, np.nan)
    computed = 0
    visited = 0
    run = 0
    for j, p in enumerate(order):
        if max_run is not None and run >= max_run:
            skip_log[j:] = 1
            break
        visited += 1
        keys = int(p) * page_size + np.arange(page_size)
        s = (qf @ k_log[keys].T) * scale
        s = np.where(keys[None, :] > rows[:, None], NEG_INF, s)
        m_loc = s.max(axis=1)
        live = m_loc > NEG_INF
        d = np.full(Bq, NEG_INF)
        first_seen = live & (m == NEG_INF)
        d[first_seen] = math.inf
        both = live & (m > NEG_INF)
        d[both] = m_loc[both] - m[both]
        if rule == "sum":
            d[both] += math.log(page_size) - np.log(l[both])
        elif rule != "max":
            raise ValueError(f"unknown skip rule {rule!r}")
        dmax = d.max() if live.any() else NEG_INF
        if log_eps == NEG_INF or log_eps == math.inf:
            margin[j] = math.inf if log_eps == NEG_INF else NEG_INF
        else:
            margin[j] = dmax - log_eps
        skip = (j >= 1) and live.any() and (dmax < log_eps)
        if force is not None and j in force:
            skip = bool(force[j])
        skip_log[j] = 1 if skip else 0
        if skip:
            run += 1
            continue
        run = 0
        computed += 1
        m_new = np.maximum(m, m_loc)
        upd = m_new > NEG_INF
        alpha = np.ones(Bq)
        alpha[upd] = np.exp(m[upd] - m_new[upd])      # exp(-inf) = 0 for first contact
        pexp = np.zeros_like(s)
        pexp[upd] = np.exp(s[upd] - m_new[upd, None])
        l = l * alpha + pexp.sum(axis=1)
        o = o * alpha[:, None] + pexp @ v_log[keys]
        m = m_new
    out = np.zeros((Bq, D))
    lse = np.full(Bq, NEG_INF)
    seen = l > 0
    out[seen] = o[seen] / l[seen, None]
    lse[seen] = m[seen] + np.log(l[seen])
    return {"out": out, "lse": lse, "computed": computed, "visited": visited,
            "skip": skip_log, "margin": margin}


def osk_block(q_rows: np.ndarray, k_log: np.ndarray, v_log: np.ndarray, qb: int,
              q_block: int, page_size: int, order: Sequence[int], eps: float,
              scale: float, force: Optional[dict] = None):
    """The pages' rule for one q-block (osk_block_rules with rule="max", no
    break).  Returns (out [Bq][D], lse [Bq], computed int, skip_log uint8
    [len(order)], margin float64 [len(order)] = max_i d_i - ln(eps))."""
    r = osk_block_rules(q_rows, k_log, v_log, qb, q_block, page_size, order, eps, scale,
                        force=force)
    return r["out"], r["lse"], r["computed"], r["skip"], r["margin"]


def osk_attention(q: np.ndarray, k_pool: np.ndarray, v_pool: np.ndarray,
                  page_table: np.ndarray, order: np.ndarray, count: np.ndarray, *,
                  num_kv_heads: int, page_size: int, q_block: int, eps: float,
                  scale: float, heads: Optional[Sequence] = None,
                  qblocks: Optional[Sequence[int]] = None, rule: str = "max",
                  max_run: Optional[int] = None):
    """OSK over a whole problem (or a subset).  order [B][H_q][nQB][k_cap],
    count [B][H_q][nQB]; rule / max_run select a skip-rule variant
    (osk_block_rules).  Returns dict with out float64 [B][H_q][N][D],
    lse [B][H_q][N], computed and visited int32 [B][H_q][nQB], skip uint8
    [B][H_q][nQB][k_cap], margin float64 [B][H_q][nQB][k_cap]."""
    B, Hq, N, D = q.shape
    G = Hq // num_kv_heads
    nQB = N // q_block
    kc = order.shape[-1]
    out = np.zeros((B, Hq, N, D))
    lse = np.full((B, Hq, N), NEG_INF)
    computed = np.zeros((B, Hq, nQB), dtype=np.int32)
    visited = np.zeros((B, Hq, nQB), dtype=np.int32)
    skip = np.zeros((B, Hq, nQB, kc), dtype=np.uint8)
    margin = np.full((B, Hq, nQB, kc), np.nan)
    if heads is None:
        heads = [(b, h) for b in range(B) for h in range(Hq)]
    if qblocks is None:
        qblocks = range(nQB)
    cache = {}
    for (b, h) in heads:
        hk = h // G
        if (b, hk) not in cache:
            cache[(b, hk)] = (gather_logical(k_pool, page_table, b, hk, N),
                              gather_logical(v_pool, page_table, b, hk, N))
        k_log, v_log = cache[(b, hk)]
        for qb in qblocks:
            rows = slice(qb * q_block, (qb + 1) * q_block)
            c = int(count[b, h, qb])
            r = osk_block_rules(q[b, h, rows], k_log, v_log, qb, q_block, page_size,
                                order[b, h, qb, :c], eps, scale, rule=rule, max_run=max_run)
            out[b, h, rows] = r["out"]
            lse[b, h, rows] = r["lse"]
            computed[b, h, qb] = r["computed"]
            visited[b, h, qb] = r["visited"]
            skip[b, h, qb, :c] = r["skip"]
            margin[b, h, qb, :c] = r["margin"]
    return {"out": out, "lse": lse, "computed": computed, "visited": visited, "skip": skip,
            "margin": margin}


# ----------------------------------------------------------------------------
# Decode: one new query per sequence and head, after the prefill.  The pages
# leave decoding as future work ([TS] closing section); the reading here is the
# plainest continuation of the prefill method: the query at position t sees keys
# 0..t of the paged cache and visits an ordered page list (for instance the list
# KAP produced for the q-block holding t) under the same in-kernel rule, as a
# q-block of one row (osk_block_rules with q_block = 1 and qb = t).
# ----------------------------------------------------------------------------
def osk_decode(q: np.ndarray, k_pool: np.ndarray, v_pool: np.ndarray, page_table: np.ndarray,
               positions: Sequence[int], order: np.ndarray, count: np.ndarray, *,
               num_kv_heads: int, page_size: int, eps: float, scale: float,
               heads: Optional[Sequence] = None):
    """Single-query ordered-skipping attention.  q [B][H_q][D] (the new query of
    each sequence and head), positions [B] (its position t: it sees keys 0..t),
    order [B][H_q][k_cap] (logical pages, each <= t // P), count [B][H_q].
    Returns dict with out float64 [B][H_q][D], lse [B][H_q], computed int32
    [B][H_q], skip uint8 [B][H_q][k_cap], margin float64 [B][H_q][k_cap]."""
    B, Hq, D = q.shape
    G = Hq // num_kv_heads
    kc = order.shape[-1]
    out = np.zeros((B, Hq, D))
    lse = np.full((B, Hq), NEG_INF)
    computed = np.zeros((B, Hq), dtype=np.int32)
    skip = np.zeros((B, Hq, kc), dtype=np.uint8)
    margin = np.full((B, Hq, kc), np.nan)
    if heads is None:
        heads = [(b, h) for b in range(B) for h in range(Hq)]
    cache = {}
    for (b, h) in heads:
        t = int(positions[b])
        hk = h // G
        if (b, hk) not in cache:
            n_tok = (t // page_size + 1) * page_size
            cache[(b, hk)] = (gather_logical(k_pool, page_table, b, hk, n_tok),
                              gather_logical(v_pool, page_table, b, hk, n_tok))
        k_log, v_log = cache[(b, hk)]
        c = int(count[b, h])
        r = osk_block_rules(np.asarray(q[b, h], dtype=np.float64)[None, :], k_log, v_log, t, 1,
                            page_size, order[b, h, :c], eps, scale)
        out[b, h] = r["out"][0]
        lse[b, h] = r["lse"][0]
        computed[b, h] = r["computed"]
        skip[b, h, :c] = r["skip"]
        margin[b, h, :c] = r["margin"]
    return {"out": out, "lse": lse, "computed": computed, "skip": skip, "margin": margin}


# ----------------------------------------------------------------------------
# dense causal attention: the plain definition
# ----------------------------------------------------------------------------
def dense_rows(q_rows: np.ndarray, k_log: np.ndarray, v_log: np.ndarray,
               row_ids: np.ndarray, scale: float):
    """softmax_c(scale * <q_i, k_c>, c <= i) @ V for the given query rows,
    brute force over the full logit row.  Returns (out [n][D], lse [n])."""
    qf = np.asarray(q_rows, dtype=np.float64)
    row_ids = np.asarray(row_ids)
    hi = int(row_ids.max()) + 1
    s = (qf @ k_log[:hi].T) * scale
    s = np.where(np.arange(hi)[None, :] > row_ids[:, None], NEG_INF, s)
    m = s.max(axis=1)
    e = np.exp(s - m[:, None])
    l = e.sum(axis=1)
    out = (e @ v_log[:hi]) / l[:, None]
    return out, m + np.log(l)


def dense_attention(q: np.ndarray, k_pool: np.ndarray, v_pool: np.ndarray,
                    page_table: np.ndarray, *, num_kv_heads: int, scale: float,
                    heads: Optional[Sequence] = None, rows: Optional[np.ndarray] = None,
                    chunk: int = 512):
    """Dense causal attention over the paged cache.  Returns dict with out
    float64 [B][H_q][N][D] and lse [B][H_q][N] (rows not requested are 0)."""
    B, Hq, N, D = q.shape
    G = Hq // num_kv_heads
    out = np.zeros((B, Hq, N, D))
    lse = np.full((B, Hq, N), NEG_INF)
    if heads is None:
        heads = [(b, h) for b in range(B) for h in range(Hq)]
    if rows is None:
        rows = np.arange(N)
    rows = np.asarray(rows)
    cache = {}
    for (b, h) in heads:
        hk = h // G
        if (b, hk) not in cache:
            cache[(b, hk)] = (gather_logical(k_pool, page_table, b, hk, N),
                              gather_logical(v_pool, page_table, b, hk, N))
        k_log, v_log = cache[(b, hk)]
        for i in range(0, len(rows), chunk):
            r = rows[i:i + chunk]
            o, ls = dense_rows(q[b, h, r], k_log, v_log, r, scale)
            out[b, h, r] = o
            lse[b, h, r] = ls
    return {"out": out, "lse": lse}
