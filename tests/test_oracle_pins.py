"""Pins for the CPU oracle: each test ties an oracle function to something other
than itself (brute force, a closed form, a library routine, an invariant the
method fixes, or the method's own error bound), chosen so that a dropped term,
a wrong sign, a wrong index or a transposed operand fails at least one of them.
No GPU is needed."""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle as O
import workloads as W


# --------------------------------------------------------------------------
# page arithmetic
# --------------------------------------------------------------------------
def test_causal_pages_brute_force():
    for Bq, P in [(64, 64), (128, 64), (128, 128), (64, 128), (16, 16), (32, 16)]:
        N = 8 * max(Bq, P)
        for qb in range(N // Bq):
            rows = range(qb * Bq, (qb + 1) * Bq)
            # pages with at least one key c <= i for some row i of the block
            seen = {c // P for i in rows for c in range(0, i + 1)}
            assert O.causal_pages(qb, Bq, P) == len(seen) == max(seen) + 1


def test_forced_pages_are_sink_and_own_range():
    for Bq, P, sink in [(128, 64, 1), (64, 64, 1), (64, 128, 2), (128, 64, 0)]:
        for qb in range(12):
            own = {t // P for t in range(qb * Bq, (qb + 1) * Bq)}
            want = sorted(own | set(range(min(sink, O.causal_pages(qb, Bq, P)))))
            assert O.forced_pages(qb, Bq, P, sink) == want


def test_budget_count_closed_forms():
    # qb=5, Bq=128, P=64: n_b = 12, forced = {0, 10, 11}
    assert O.causal_pages(5, 128, 64) == 12
    assert O.budget_count(5, 128, 64, 1, 1.0) == 12
    assert O.budget_count(5, 128, 64, 1, 0.0) == 3
    assert O.budget_count(5, 128, 64, 1, 0.25) == 3        # 0.25 * 12 = 3 exactly
    assert O.budget_count(5, 128, 64, 1, 0.26) == 4        # 3.12 -> 4
    assert O.budget_count(5, 128, 64, 1, 0.5) == 6
    # 10% of 10 pages is one page (float32 product), not two
    # qb=4, Bq=128, P=64 -> n_b = 10, forced {0, 8, 9} -> max(3, 1) = 3
    assert O.budget_count(4, 128, 64, 0, 0.1) == 2         # forced {8, 9}
    n_b = O.causal_pages(1023, 128, 64)
    assert n_b == 2048
    assert O.budget_count(1023, 128, 64, 1, 0.2) == 410   # ceil(409.6)
    assert O.k_cap(131072, 128, 64, 1, 0.2) == 410


# --------------------------------------------------------------------------
# page-table gather: against the generator's own logical copy
# --------------------------------------------------------------------------
def test_gather_logical_matches_generator_scatter():
    wl = W.small_workload("gqa-128k", 2048, num_q_heads=4, num_kv_heads=2, batch=2)
    x = W.make_inputs(wl, seed=3, keep_logical=True)
    assert wl.shuffle_pages
    pt = x["page_table"].numpy()
    assert not np.array_equal(pt.reshape(-1), np.arange(pt.size))  # really shuffled
    for b in range(2):
        for h in range(2):
            got = O.gather_logical(x["k_pool"].float().numpy(), pt, b, h)
            want = x["k_log"][b, h].float().numpy()
            np.testing.assert_array_equal(got, want)


# --------------------------------------------------------------------------
# KAP pooling: against torch's avg_pool1d (library routine)
# --------------------------------------------------------------------------
def test_pooling_matches_avg_pool1d():
    rng = np.random.default_rng(0)
    N, D = 512, 16
    x = rng.standard_normal((N, D))
    for Bq, q_sub in [(64, 16), (128, 32), (128, 128)]:
        got = O.kap_pool_queries(x, Bq, q_sub).reshape(-1, D)
        want = torch.nn.functional.avg_pool1d(torch.from_numpy(x.T[None]), q_sub).numpy()[0].T
        np.testing.assert_allclose(got, want, rtol=1e-14, atol=1e-14)
    for P, k_sub in [(64, 16), (128, 16), (64, 64)]:
        got = O.kap_pool_keys(x, P, k_sub).reshape(-1, D)
        want = torch.nn.functional.avg_pool1d(torch.from_numpy(x.T[None]), k_sub).numpy()[0].T
        np.testing.assert_allclose(got, want, rtol=1e-14, atol=1e-14)


# --------------------------------------------------------------------------
# KAP scores + MaxPool: brute force at token level
# --------------------------------------------------------------------------
def test_block_scores_brute_force():
    rng = np.random.default_rng(1)
    N, D, Bq, P, q_sub, k_sub = 96, 3, 32, 16, 8, 4
    scale = 0.7
    qf = rng.standard_normal((N, D))
    kf = rng.standard_normal((N, D))
    qhat = O.kap_pool_queries(qf, Bq, q_sub)
    khat = O.kap_pool_keys(kf, P, k_sub)
    for qb in range(N // Bq):
        a = O.kap_block_scores(qhat[qb], khat, qb, Bq, q_sub, P, k_sub, scale)
        R = Bq // q_sub
        for r in range(R):
            rep_rows = list(range(qb * Bq + r * q_sub, qb * Bq + (r + 1) * q_sub))
            rep = [sum(qf[i][d] for i in rep_rows) / q_sub for d in range(D)]
            n_b = O.causal_pages(qb, Bq, P)
            for p in range(n_b):
                best = -math.inf
                for t in range(P // k_sub):
                    toks = list(range(p * P + t * k_sub, p * P + (t + 1) * k_sub))
                    # visible iff some row of the rep may see some key of the sub-key
                    if not any(c <= i for i in rep_rows for c in toks):
                        continue
                    sk = [sum(kf[c][d] for c in toks) / k_sub for d in range(D)]
                    best = max(best, scale * sum(rep[d] * sk[d] for d in range(D)))
                if best == -math.inf:
                    assert a[r, p] == -math.inf
                else:
                    assert abs(a[r, p] - best) < 1e-12


def test_kap_hand_worked_example():
    """N=4, D=1, P=2, Bq=2, q_sub=k_sub=1, scale=1, q=[1,2,3,4], k=[1,0,2,-1].
    q-block 1 holds rows 2 and 3 (the two representatives).
      rep row 2: page 0 -> max(3*1, 3*0) = 3; page 1 -> key 2 only (key 3 is
                 in the future) -> 3*2 = 6.
      rep row 3: page 0 -> max(4, 0) = 4; page 1 -> max(8, -4) = 8.
    a = [[3, 6], [4, 8]], row maxima 6 and 8, so
    S = [(e^-3 + e^-4)/2, 1], HRM = [0, 1]; both pages are forced (sink and
    own range); page 1 (HRM) is visited first."""
    q = np.array([[1.0], [2.0], [3.0], [4.0]])
    k = np.array([[1.0], [0.0], [2.0], [-1.0]])
    order, S, hrm, a = O.kap_select_block(q, k, 1, q_block=2, page_size=2, q_sub=1,
                                          k_sub=1, scale=1.0, budget=0.0, sink_pages=1)
    np.testing.assert_allclose(a, [[3, 6], [4, 8]], rtol=0, atol=1e-15)
    np.testing.assert_allclose(S, [(math.exp(-3) + math.exp(-4)) / 2, 1.0], rtol=1e-15)
    assert list(hrm) == [0, 1]
    assert list(order) == [1, 0]


# --------------------------------------------------------------------------
# MaxNorm + HRM: closed forms and invariants
# --------------------------------------------------------------------------
def test_maxnorm_closed_forms():
    S, hrm = O.kap_maxnorm_hrm(np.array([[0.0, math.log(0.5), -math.inf]]))
    np.testing.assert_allclose(S, [1.0, 0.5, 0.0], rtol=1e-15)
    assert list(hrm) == [1, 0, 0]
    # mean (not sum) over representatives
    S, hrm = O.kap_maxnorm_hrm(np.array([[0.0, -math.log(2)], [-math.log(2), 0.0]]))
    np.testing.assert_allclose(S, [0.75, 0.75], rtol=1e-15)
    assert list(hrm) == [1, 1]
    # ties: the lowest page index holds the row max
    S, hrm = O.kap_maxnorm_hrm(np.array([[1.0, 2.0, 2.0, 0.5]]))
    assert list(hrm) == [0, 1, 0, 0]
    np.testing.assert_allclose(S, [math.exp(-1), 1, 1, math.exp(-1.5)], rtol=1e-15)


def test_maxnorm_invariants():
    rng = np.random.default_rng(2)
    for _ in range(50):
        R, n = rng.integers(1, 6), rng.integers(1, 40)
        a = rng.standard_normal((R, n)) * 3
        S, hrm = O.kap_maxnorm_hrm(a)
        assert np.all(S > 0) and np.all(S <= 1 + 1e-15)
        # per-row shift invariance
        S2, hrm2 = O.kap_maxnorm_hrm(a + rng.standard_normal((R, 1)) * 10)
        np.testing.assert_allclose(S, S2, rtol=1e-12)
        assert np.array_equal(hrm, hrm2)
        # HRM pages carry at least 1/R of the mass; S = 1 iff all rows peak there
        assert np.all(S[hrm == 1] >= 1.0 / R - 1e-15)
        assert 1 <= hrm.sum() <= R
        am = a.argmax(axis=1)
        for p in range(n):
            assert (abs(S[p] - 1) < 1e-15) == bool(np.all(am == p))


# --------------------------------------------------------------------------
# ranking key, budgeted selection, ordering: brute force
# --------------------------------------------------------------------------
def test_rank_key_orders_like_tuples():
    rng = np.random.default_rng(3)
    vals = rng.random(200).astype(np.float32)
    vals[::7] = vals[3]                       # ties in score
    vals[::11] = 0.0
    hr = (rng.random(200) < 0.2).astype(int)
    pages = rng.permutation(200)
    items = list(zip(hr, vals, pages))
    by_key = sorted(items, key=lambda t: O.rank_key(float(t[1]), t[0], t[2]), reverse=True)
    by_tuple = sorted(items, key=lambda t: (t[0], float(t[1]), -t[2]), reverse=True)
    assert [t[2] for t in by_key] == [t[2] for t in by_tuple]


def test_selection_is_best_subset_brute_force():
    rng = np.random.default_rng(4)
    Bq, P, sink = 16, 8, 1
    for trial in range(60):
        qb = int(rng.integers(0, 6))
        n_b = O.causal_pages(qb, Bq, P)
        S = rng.random(n_b).astype(np.float32)
        if trial % 3 == 0:
            S[rng.integers(0, n_b, 3)] = S[0]            # exact ties
        hrm = (rng.random(n_b) < 0.25).astype(np.uint8)
        budget = float(rng.choice([0.0, 0.3, 0.5, 0.75, 1.0]))
        order = O.kap_order_from_scores(S, hrm, qb, Bq, P, budget, sink)
        forced = set(O.forced_pages(qb, Bq, P, sink))
        k_b = O.budget_count(qb, Bq, P, sink, budget)
        assert len(order) == k_b == len(set(order.tolist()))

        def tup(p):
            return (int(hrm[p]), float(S[p]), -p)
        # exhaustive: among all k_b-subsets containing the forced set, the one
        # whose non-forced members, sorted descending, are lexicographically largest
        free = [p for p in range(n_b) if p not in forced]
        best = None
        for combo in itertools.combinations(free, k_b - len(forced)):
            cand = sorted((tup(p) for p in combo), reverse=True)
            if best is None or cand > best[0]:
                best = (cand, set(combo) | forced)
        assert set(order.tolist()) == best[1]
        # listed by (hrm, S, lower index) descending: HRM pages first
        assert [tup(p) for p in order] == sorted((tup(p) for p in order), reverse=True)
        seen_non_hrm = False
        for p in order:
            if hrm[p] == 0:
                seen_non_hrm = True
            else:
                assert not seen_non_hrm
        asc = O.kap_order_from_scores(S, hrm, qb, Bq, P, budget, sink, ascending=True)
        assert list(asc) == sorted(order.tolist())


def test_planted_pages_come_first_tiny_2k():
    """On the tiny 2K workload, every q-block among the last 256 queries lists
    the 3 planted pages first ([TS §2.2]: ordering puts the blocks holding the
    row maxima first)."""
    wl = W.WORKLOADS["tiny-2k"]
    x = W.make_inputs(wl, seed=0)
    r = O.kap_select(x["q"].float().numpy(), x["k_pool"].float().numpy(), x["page_table"].numpy(),
                     num_kv_heads=2, page_size=64, q_block=64, q_sub=16, k_sub=16,
                     scale=1 / math.sqrt(64), budget=0.25, sink_pages=1)
    nQB = wl.seq_len // wl.q_block
    for h in range(2):
        planted = set(x["planted"][0, h].tolist())
        for qb in range(nQB - 256 // wl.q_block, nQB):
            assert set(r["order"][0, h, qb, :3].tolist()) == planted
            assert r["count"][0, h, qb] == O.budget_count(qb, 64, 64, 1, 0.25)


# --------------------------------------------------------------------------
# dense attention: against torch's scaled_dot_product_attention in float64
# --------------------------------------------------------------------------
def test_dense_matches_torch_sdpa():
    wl = W.small_workload("gqa-32k", 512, num_q_heads=4, num_kv_heads=2, head_dim=32, page_size=32,
                          q_block=64, shuffle_pages=True)
    x = W.make_inputs(wl, seed=5, keep_logical=True)
    scale = 1 / math.sqrt(32)
    r = O.dense_attention(x["q"].float().numpy(), x["k_pool"].float().numpy(),
                          x["v_pool"].float().numpy(), x["page_table"].numpy(),
                          num_kv_heads=2, scale=scale, chunk=100)
    q = x["q"].double()
    k = x["k_log"].double().repeat_interleave(2, dim=1)
    v = x["v_log"].double().repeat_interleave(2, dim=1)
    want = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True, scale=scale)
    np.testing.assert_allclose(r["out"], want.numpy(), rtol=0, atol=1e-12)
    s = torch.einsum("bhid,bhjd->bhij", q, k) * scale
    s = s.masked_fill(torch.ones(512, 512, dtype=torch.bool).triu(1), -math.inf)
    np.testing.assert_allclose(r["lse"], torch.logsumexp(s, -1).numpy(), rtol=0, atol=1e-11)


# --------------------------------------------------------------------------
# OSK: closed forms, invariance, brute-force skip decisions, error bound
# --------------------------------------------------------------------------
def _tiny_problem(seed=6, N=256, D=8, P=16, Bq=16, drift=0.0):
    wl = W.Workload("t", 1, 1, 1, N, D, P, Bq, drift_sigma=drift, planted_count=2,
                    planted_mag=3.0)
    x = W.make_inputs(wl, seed=seed, keep_logical=True)
    k = x["k_log"][0, 0].double().numpy()
    v = x["v_log"][0, 0].double().numpy()
    q = x["q"][0, 0].double().numpy()
    return q, k, v


def test_osk_full_budget_no_skip_equals_dense():
    q, k, v = _tiny_problem()
    N, P, Bq, scale = 256, 16, 16, 1 / math.sqrt(8)
    for qb in range(N // Bq):
        rows = np.arange(qb * Bq, (qb + 1) * Bq)
        n_b = O.causal_pages(qb, Bq, P)
        order = np.random.default_rng(qb).permutation(n_b)
        out, lse, comp, sk, _ = O.osk_block(q[rows], k, v, qb, Bq, P, order, 0.0, scale)
        want, wlse = O.dense_rows(q[rows], k, v, rows, scale)
        np.testing.assert_allclose(out, want, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse, wlse, rtol=0, atol=1e-12)
        assert comp == n_b and sk.sum() == 0


def test_osk_attention_whole_problem_gqa_equals_sdpa():
    """osk_attention over a whole GQA problem (4 query heads on 2 KV heads, batch 2,
    shuffled page table, 32-token pages, 64-row q-blocks) with every causal page
    listed in a random order and eps = 0 is exact causal attention in which query
    head h reads KV head h // 2 (torch SDPA on repeat-interleaved K and V).  A wrong
    head map (h % H_kv), a wrong page-table gather or a q-block row offset fails it."""
    wl = W.small_workload("gqa-32k", 512, num_q_heads=4, num_kv_heads=2, batch=2, head_dim=32,
                          page_size=32, q_block=64, shuffle_pages=True)
    x = W.make_inputs(wl, seed=15, keep_logical=True)
    scale = 1 / math.sqrt(32)
    nQB, kc = 512 // 64, 512 // 32
    g = np.random.default_rng(15)
    order = np.full((2, 4, nQB, kc), -1, dtype=np.int32)
    count = np.zeros((2, 4, nQB), dtype=np.int32)
    for b in range(2):
        for h in range(4):
            for qb in range(nQB):
                n = O.causal_pages(qb, 64, 32)
                order[b, h, qb, :n] = g.permutation(n)
                count[b, h, qb] = n
    r = O.osk_attention(x["q"].double().numpy(), x["k_pool"].double().numpy(),
                        x["v_pool"].double().numpy(), x["page_table"].numpy(), order, count,
                        num_kv_heads=2, page_size=32, q_block=64, eps=0.0, scale=scale)
    q = x["q"].double()
    k = x["k_log"].double().repeat_interleave(2, dim=1)
    v = x["v_log"].double().repeat_interleave(2, dim=1)
    want = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True, scale=scale)
    np.testing.assert_allclose(r["out"], want.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_array_equal(r["computed"], count)
    s = torch.einsum("bhid,bhjd->bhij", q, k) * scale
    s = s.masked_fill(torch.ones(512, 512, dtype=torch.bool).triu(1), -math.inf)
    np.testing.assert_allclose(r["lse"], torch.logsumexp(s, -1).numpy(), rtol=0, atol=1e-11)


def test_osk_order_invariance_every_permutation():
    q, k, v = _tiny_problem(seed=7)
    P, Bq, scale = 16, 16, 1 / math.sqrt(8)
    qb = 4                                    # n_b = 5 pages: all 120 orders
    rows = slice(qb * Bq, (qb + 1) * Bq)
    ref = None
    for perm in itertools.permutations(range(5)):
        out, lse, comp, _, _ = O.osk_block(q[rows], k, v, qb, Bq, P, perm, 0.0, scale)
        if ref is None:
            ref = (out, lse)
        np.testing.assert_allclose(out, ref[0], rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse, ref[1], rtol=0, atol=1e-13)


def test_osk_skip_decisions_from_full_logit_matrix():
    """For eps < 1 a skipped page lies wholly below the running max, so the
    running max before step j equals the max over ALL earlier listed pages.
    Recompute every decision from the full N x N logit matrix."""
    q, k, v = _tiny_problem(seed=8, drift=0.3)
    N, P, Bq, scale = 256, 16, 16, 1 / math.sqrt(8)
    L = (q @ k.T) * scale
    L[np.triu(np.ones((N, N), dtype=bool), 1)] = -np.inf
    rng = np.random.default_rng(9)
    n_skips = 0
    for eps in [1e-1, 1e-2, 1e-4]:
        for qb in range(N // Bq):
            n_b = O.causal_pages(qb, Bq, P)
            order = rng.permutation(n_b)
            rows = np.arange(qb * Bq, (qb + 1) * Bq)
            _, _, comp, sk, _ = O.osk_block(q[rows], k, v, qb, Bq, P, order, eps, scale)
            for j, p in enumerate(order):
                blk = L[rows][:, p * P:(p + 1) * P]
                loc = blk.max(axis=1)
                if j == 0:
                    assert sk[j] == 0
                    continue
                prev = np.concatenate([np.arange(pp * P, (pp + 1) * P) for pp in order[:j]])
                run = L[rows][:, prev].max(axis=1)
                live = loc > -np.inf
                with np.errstate(invalid="ignore"):
                    d = np.where(run == -np.inf, np.inf, loc - run)
                want = bool(d[live].max() < math.log(eps))
                assert bool(sk[j]) == want
            assert comp == len(order) - sk.sum()
            n_skips += int(sk.sum())
    assert n_skips > 0                          # the rule actually fired


def test_osk_skip_error_bound():
    """Each skipped page holds less than P * eps of softmax mass relative to the
    row max, so |out - out_noskip| <= 2 * n_skipped * P * eps * max|v|."""
    q, k, v = _tiny_problem(seed=10, drift=0.2)
    N, P, Bq, scale = 256, 16, 16, 1 / math.sqrt(8)
    vmax = np.abs(v).max()
    total_skipped = 0
    for eps in [1e-1, 1e-2, 1e-3]:
        for qb in range(N // Bq):
            rows = np.arange(qb * Bq, (qb + 1) * Bq)
            order = np.arange(O.causal_pages(qb, Bq, P))[::-1]
            out, _, _, sk, _ = O.osk_block(q[rows], k, v, qb, Bq, P, order, eps, scale)
            ref, _ = O.dense_rows(q[rows], k, v, rows, scale)
            bound = 2 * sk.sum() * P * eps * vmax
            assert np.abs(out - ref).max() <= bound + 1e-12
            total_skipped += int(sk.sum())
    assert total_skipped > 0


def test_osk_infinite_eps_keeps_first_page_only():
    """eps = inf with page 0 listed first: every later page is skipped, so each
    row attends to keys 0..min(P-1, i) only (a textbook masked softmax)."""
    q, k, v = _tiny_problem(seed=11)
    N, P, Bq, scale = 256, 16, 16, 1 / math.sqrt(8)
    mask = torch.zeros(N, N, dtype=torch.bool)
    for i in range(N):
        mask[i, :min(P, i + 1)] = True
    want = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None], torch.from_numpy(k)[None], torch.from_numpy(v)[None],
        attn_mask=mask, scale=scale)[0].numpy()
    for qb in range(1, N // Bq):
        rows = np.arange(qb * Bq, (qb + 1) * Bq)
        order = [0] + list(range(1, O.causal_pages(qb, Bq, P)))
        out, _, comp, _, _ = O.osk_block(q[rows], k, v, qb, Bq, P, order, math.inf, scale)
        assert comp == 1
        np.testing.assert_allclose(out, want[rows], rtol=0, atol=1e-12)


def test_osk_sink_plus_local_budget_is_local_sink_mask():
    """Budget 0: only the sink page and the q-block's own pages are kept; with
    eps = 0 the result is attention under a sink + local-window mask."""
    q, k, v = _tiny_problem(seed=12)
    N, P, Bq, scale = 256, 16, 32, 1 / math.sqrt(8)
    for qb in range(N // Bq):
        rows = np.arange(qb * Bq, (qb + 1) * Bq)
        order = O.kap_order_from_scores(np.ones(64, np.float32), np.zeros(64, np.uint8),
                                        qb, Bq, P, 0.0, 1)
        out, _, _, _, _ = O.osk_block(q[rows], k, v, qb, Bq, P, order, 0.0, scale)
        mask = torch.zeros(Bq, N, dtype=torch.bool)
        for a, i in enumerate(rows):
            for c in range(i + 1):
                if c < P or c >= qb * Bq:
                    mask[a, c] = True
        want = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q[rows])[None], torch.from_numpy(k)[None], torch.from_numpy(v)[None],
            attn_mask=mask[None], scale=scale)[0].numpy()
        np.testing.assert_allclose(out, want, rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# group-shared selection: reductions and invariances
# --------------------------------------------------------------------------
def _group_problem(G=3, seed=11, N=256, D=16, P=16, Bq=32):
    wl = W.small_workload("gqa-32k", N, num_q_heads=2 * G, num_kv_heads=2, head_dim=D, page_size=P,
                          q_block=Bq, planted_frac=0.05, shuffle_pages=True)
    x = W.make_inputs(wl, seed=seed)
    return wl, x["q"].float().numpy(), x["k_pool"].float().numpy(), x["page_table"].numpy()


def _kw(wl):
    return dict(num_kv_heads=wl.num_kv_heads, page_size=wl.page_size, q_block=wl.q_block,
                q_sub=wl.q_block // 4, k_sub=wl.page_size // 2, scale=1 / math.sqrt(wl.head_dim),
                budget=0.3, sink_pages=1)


def test_group_selection_with_one_head_per_group_is_per_head_selection():
    wl = W.small_workload("gqa-32k", 256, num_q_heads=2, num_kv_heads=2, head_dim=16, page_size=16,
                          q_block=32, planted_frac=0.05)
    x = W.make_inputs(wl, seed=3)
    args = (x["q"].float().numpy(), x["k_pool"].float().numpy(), x["page_table"].numpy())
    g = O.kap_select_group(*args, **_kw(wl))
    h = O.kap_select(*args, **_kw(wl))
    assert np.array_equal(g["order"], h["order"]) and np.array_equal(g["count"], h["count"])
    np.testing.assert_array_equal(g["S"], h["S"])


def test_group_selection_does_not_depend_on_head_order():
    wl, q, kp, pt = _group_problem()
    base = O.kap_select_group(q, kp, pt, **_kw(wl))
    G = 3
    perm = np.concatenate([hk * G + np.random.default_rng(hk).permutation(G) for hk in range(2)])
    other = O.kap_select_group(q[:, perm], kp, pt, **_kw(wl))
    assert np.array_equal(base["order"], other["order"])


def test_group_selection_of_identical_heads_is_each_heads_selection():
    wl, q, kp, pt = _group_problem()
    G = 3
    q2 = q.copy()
    for hk in range(2):
        q2[:, hk * G + 1: hk * G + G] = q2[:, hk * G: hk * G + 1]
    g = O.kap_select_group(q2, kp, pt, **_kw(wl))
    h = O.kap_select(q2, kp, pt, **_kw(wl))
    for hq in range(2 * G):
        assert np.array_equal(g["order"][:, hq // G], h["order"][:, hq])


def test_group_aggregate_with_a_dominant_head_follows_it():
    """If one head's scores and HRM flags dominate the others' page by page, the
    group list is that head's list (selection and order only depend on the key)."""
    rng = np.random.default_rng(9)
    Bq, P, sink = 16, 8, 1
    for trial in range(40):
        qb = int(rng.integers(1, 6))
        n_b = O.causal_pages(qb, Bq, P)
        G = int(rng.integers(2, 5))
        S0 = rng.random(n_b)
        h0 = (rng.random(n_b) < 0.3).astype(np.uint8)
        Sh = [S0] + [S0 * rng.random(n_b) for _ in range(G - 1)]
        Hh = [h0] + [h0 * (rng.random(n_b) < 0.5) for _ in range(G - 1)]
        S, hr = O.kap_group_scores(np.stack(Sh), np.stack(Hh))
        budget = float(rng.choice([0.25, 0.5, 1.0]))
        got = O.kap_order_from_scores(S, hr, qb, Bq, P, budget, sink)
        want = O.kap_order_from_scores(S0, h0, qb, Bq, P, budget, sink)
        assert got.tolist() == want.tolist()


def test_group_selection_is_best_subset_brute_force():
    """Exhaustive check on tiny blocks: the group list is the best k_b-subset
    (forced pages included) under (any head flags it, largest head score, lower
    page) compared lexicographically, listed in that order."""
    rng = np.random.default_rng(12)
    Bq, P, sink = 16, 8, 1
    for trial in range(40):
        qb = int(rng.integers(0, 6))
        n_b = O.causal_pages(qb, Bq, P)
        G = int(rng.integers(1, 4))
        Sh = rng.random((G, n_b)).astype(np.float32).astype(np.float64)
        Hh = (rng.random((G, n_b)) < 0.2).astype(np.uint8)
        S, hr = O.kap_group_scores(Sh, Hh)
        budget = float(rng.choice([0.3, 0.5, 0.75]))
        order = O.kap_order_from_scores(S, hr, qb, Bq, P, budget, sink)
        forced = set(O.forced_pages(qb, Bq, P, sink))
        k_b = O.budget_count(qb, Bq, P, sink, budget)

        def tup(p):
            return (int(any(Hh[g, p] for g in range(G))), max(float(Sh[g, p]) for g in range(G)), -p)
        free = [p for p in range(n_b) if p not in forced]
        best = None
        for combo in itertools.combinations(free, k_b - len(forced)):
            cand = sorted((tup(p) for p in combo), reverse=True)
            if best is None or cand > best[0]:
                best = (cand, set(combo) | forced)
        assert set(order.tolist()) == best[1]
        assert [tup(p) for p in order] == sorted((tup(p) for p in order), reverse=True)


def test_group_planted_pages_come_first():
    """Two query heads share a KV head whose planted pages every query of the
    last 256 rows is drawn towards: the group list opens with them."""
    wl = W.small_workload("tiny-2k", 2048, num_q_heads=4, num_kv_heads=2)
    x = W.make_inputs(wl, seed=0)
    r = O.kap_select_group(x["q"].float().numpy(), x["k_pool"].float().numpy(),
                           x["page_table"].numpy(), num_kv_heads=2, page_size=64, q_block=64,
                           q_sub=16, k_sub=16, scale=1 / math.sqrt(64), budget=0.25, sink_pages=1)
    nQB = wl.seq_len // wl.q_block
    for hk in range(2):
        planted = set(x["planted"][0, hk].tolist())
        for qb in range(nQB - 256 // wl.q_block, nQB):
            assert set(r["order"][0, hk, qb, :3].tolist()) == planted


def test_expand_group_order_maps_heads_to_their_kv_head():
    og = np.arange(2 * 3 * 4 * 5, dtype=np.int32).reshape(2, 3, 4, 5)
    cg = np.arange(2 * 3 * 4, dtype=np.int32).reshape(2, 3, 4)
    o, c = O.expand_group_order(og, cg, 6)
    for h in range(6):
        assert np.array_equal(o[:, h], og[:, h // 2]) and np.array_equal(c[:, h], cg[:, h // 2])


# ---------------------------------------------------------------------------
# skip-rule variants (not on the pages): the sum-aware test and the early break
# ---------------------------------------------------------------------------
def test_sum_rule_skipped_pages_hold_less_than_eps_of_the_row_mass():
    """Under rule="sum" a skipped page would have added less than eps times the
    row's mass so far.  Recompute that mass from the full logit matrix over the
    pages computed before the skip (not online), and the page's own mass."""
    q, k, v = _tiny_problem(seed=12, drift=0.3)
    N, P, Bq, scale = 256, 16, 16, 1 / math.sqrt(8)
    L = (q @ k.T) * scale
    L[np.triu(np.ones((N, N), dtype=bool), 1)] = -np.inf
    rng = np.random.default_rng(13)
    n_skips = 0
    for eps in [0.3, 1e-1, 1e-2]:
        for qb in range(N // Bq):
            n_b = O.causal_pages(qb, Bq, P)
            order = rng.permutation(n_b)
            rows = np.arange(qb * Bq, (qb + 1) * Bq)
            r = O.osk_block_rules(q[rows], k, v, qb, Bq, P, order, eps, scale, rule="sum")
            sk = r["skip"]
            assert sk[0] == 0 and r["computed"] == len(order) - sk.sum()
            for j in np.nonzero(sk)[0]:
                done = [order[t] for t in range(j) if sk[t] == 0]
                cols = np.concatenate([np.arange(pp * P, (pp + 1) * P) for pp in done])
                M = L[rows][:, cols].max(axis=1)
                page = L[rows][:, order[j] * P:(order[j] + 1) * P]
                sees = (page > -np.inf).any(axis=1)
                assert np.all(M[sees] > -np.inf)          # no row meets its first key here
                S = np.exp(L[rows][:, cols] - M[:, None]).sum(axis=1)
                Wp = np.exp(page - M[:, None]).sum(axis=1)
                assert np.all(Wp[sees] < eps * S[sees] * (1 + 1e-12))
            n_skips += int(sk.sum())
    assert n_skips > 0


def test_sum_rule_extremes_match_the_pages_rule():
    """eps = 0 skips nothing and eps = inf keeps only the first page and pages
    where some row meets its first key, under both rules."""
    q, k, v = _tiny_problem(seed=14, drift=0.2)
    N, P, Bq, scale = 256, 16, 16, 1 / math.sqrt(8)
    rng = np.random.default_rng(15)
    for qb in range(N // Bq):
        rows = np.arange(qb * Bq, (qb + 1) * Bq)
        order = rng.permutation(O.causal_pages(qb, Bq, P))
        for eps in (0.0, math.inf):
            a = O.osk_block_rules(q[rows], k, v, qb, Bq, P, order, eps, scale, rule="sum")
            b = O.osk_block_rules(q[rows], k, v, qb, Bq, P, order, eps, scale, rule="max")
            assert np.array_equal(a["skip"], b["skip"])
            np.testing.assert_array_equal(a["out"], b["out"])
    with pytest.raises(ValueError):
        O.osk_block_rules(q[:Bq], k, v, 0, Bq, P, [0], 1e-3, scale, rule="mean")


def test_early_break_is_the_pages_rule_cut_after_r_skips():
    """A skipped page changes no state, so with max_run = r the decisions equal
    the pages' rule up to its first run of r consecutive skips and every later
    page is skipped unvisited; the output equals the pages' rule with those
    later pages forced skipped (osk_block's force path)."""
    q, k, v = _tiny_problem(seed=16, drift=0.3)
    N, P, Bq, scale = 256, 16, 16, 1 / math.sqrt(8)
    rng = np.random.default_rng(17)
    cuts = 0
    for eps in [1e-1, 1e-2]:
        for qb in range(N // Bq):
            rows = np.arange(qb * Bq, (qb + 1) * Bq)
            order = rng.permutation(O.causal_pages(qb, Bq, P))
            base = O.osk_block_rules(q[rows], k, v, qb, Bq, P, order, eps, scale)
            for r in (1, 2, 3):
                got = O.osk_block_rules(q[rows], k, v, qb, Bq, P, order, eps, scale, max_run=r)
                sk = base["skip"]
                t = next((i for i in range(r - 1, len(order)) if sk[i - r + 1:i + 1].all()),
                         None)
                want = sk.copy()
                if t is not None:
                    want[t + 1:] = 1
                    cuts += int(t + 1 < len(order))
                assert np.array_equal(got["skip"], want)
                assert got["visited"] == (len(order) if t is None else min(t + 1, len(order)))
                forced = {j: True for j in range(t + 1, len(order))} if t is not None else None
                out, lse, comp, _, _ = O.osk_block(q[rows], k, v, qb, Bq, P, order, eps, scale,
                                                   force=forced)
                np.testing.assert_array_equal(got["out"], out)
                assert got["computed"] == comp
    assert cuts > 0
