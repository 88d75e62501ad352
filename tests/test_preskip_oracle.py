"""Pins for the oracle's proxy-bound pre-skip (kap_preskip), a variant the
pages do not give: it removes listed pages on the proxy's own scores before the
kernel runs.  Pinned against the pages' in-kernel rule ([TS §2.3] "Saltado no
Kernel"), which is itself pinned against the full logit matrix
(test_oracle_pins): with one-row representatives and one-key sub-keys the proxy
is exact, and a skipped page cannot raise the running max, so the proxy's
running max over every earlier listed page is the kernel's running max; the
pre-skip at margin 0 must then take exactly the kernel rule's decisions."""
import math

import numpy as np
import pytest

import oracle as O
import workloads as W


def _problem(seed, N=512, D=16, P=16, Bq=32, drift=0.05):
    wl = W.Workload("t", 1, 1, 1, N, D, P, Bq, drift_sigma=drift, planted_count=3,
                    planted_mag=4.0, sink_keys=8)
    x = W.make_inputs(wl, seed=seed, keep_logical=True)
    q = x["q"][0, 0].double().numpy()
    k = x["k_log"][0, 0].double().numpy()
    v = x["v_log"][0, 0].double().numpy()
    return q, k, v


@pytest.mark.parametrize("seed,eps", [(1, 0.1), (2, 0.2), (3, 0.3), (4, 0.5)])
def test_exact_proxy_preskip_takes_the_kernel_rules_decisions(seed, eps):
    q, k, v = _problem(seed)
    N, P, Bq, scale = 512, 16, 32, 1 / math.sqrt(16)
    khat = O.kap_pool_keys(k, P, 1)                      # one key per sub-key: exact keys
    rng = np.random.default_rng(seed)
    n_checked = n_skipped = 0
    for qb in range(N // Bq):
        rows = slice(qb * Bq, (qb + 1) * Bq)
        qhat = O.kap_pool_queries(q[rows], Bq, 1)[0]      # one row per representative
        a = O.kap_block_scores(qhat, khat, qb, Bq, 1, P, 1, scale)
        n_b = O.causal_pages(qb, Bq, P)
        for order in (O.kap_order_from_scores(*O.kap_maxnorm_hrm(a), qb, Bq, P, 1.0, 1),
                      rng.permutation(n_b)):
            _, sk, _ = O.kap_preskip(order, a, eps, 0.0)
            _, _, _, ref_skip, ref_margin = O.osk_block(q[rows], k, v, qb, Bq, P, order, eps, scale)
            clear = np.abs(ref_margin) > 1e-9
            assert np.array_equal(sk[clear], ref_skip[clear]), (qb, order)
            n_checked += int(clear.sum())
            n_skipped += int(sk.sum())
    assert n_skipped > 0 and n_checked > 0


def test_preskip_off_cases_keep_the_list():
    q, k, _ = _problem(5)
    khat = O.kap_pool_keys(k, 16, 4)
    for qb in (3, 9, 15):
        qhat = O.kap_pool_queries(q[qb * 32:(qb + 1) * 32], 32, 8)[0]
        a = O.kap_block_scores(qhat, khat, qb, 32, 8, 16, 4, 0.25)
        order = np.arange(O.causal_pages(qb, 32, 16))[::-1]
        for eps, margin in ((0.0, 0.0), (1e-2, 1e9)):       # eps 0, or an unbounded margin
            kept, sk, _ = O.kap_preskip(order, a, eps, margin)
            assert kept.tolist() == order.tolist() and sk.sum() == 0


def test_preskip_is_monotone_in_margin_and_eps_and_never_drops_the_first_page():
    q, k, _ = _problem(6)
    khat = O.kap_pool_keys(k, 16, 4)
    rng = np.random.default_rng(6)
    for qb in range(4, 16):
        qhat = O.kap_pool_queries(q[qb * 32:(qb + 1) * 32], 32, 8)[0]
        a = O.kap_block_scores(qhat, khat, qb, 32, 8, 16, 4, 0.25)
        order = rng.permutation(O.causal_pages(qb, 32, 16))
        prev = None
        for margin in (0.0, 0.5, 1.0, 2.0, 4.0):
            _, sk, _ = O.kap_preskip(order, a, 1e-2, margin)
            assert sk[0] == 0
            if prev is not None:
                assert np.all(sk <= prev)                  # a larger margin removes a subset
            prev = sk
        prev = None
        for eps in (0.3, 1e-1, 1e-2, 1e-3, 0.0):
            _, sk, _ = O.kap_preskip(order, a, eps, 0.5)
            if prev is not None:
                assert np.all(sk <= prev)                  # a smaller eps removes a subset
            prev = sk


def test_preskip_lists_wrapper_compacts_in_order():
    order = np.array([[[[5, 2, 7, 0, -1], [1, 0, -1, -1, -1]]]], dtype=np.int32)
    count = np.array([[[4, 2]]], dtype=np.int32)
    # page 7 and page 0 fall far below page 5's proxy maximum for both representatives
    a = {0: np.array([[-1.0, 0.0, 2.5, 0.0, 0.0, 3.0, 0.0, -9.0],
                      [-2.0, 0.0, 2.0, 0.0, 0.0, 3.0, 0.0, -9.0]]),
         1: np.array([[1.0, 1.0], [1.0, 1.0]])}
    r = O.kap_preskip_lists(order, count, lambda b, h, qb: a[qb], 0.1, 0.0)
    # position 1 (page 2): 2.5 - 3 = -0.5 >= ln 0.1 kept; page 7: -12 < ln 0.1 skipped;
    # page 0: -4, -5 < ln 0.1 skipped
    assert r["order"][0, 0, 0].tolist() == [5, 2, -1, -1, -1] and r["count"][0, 0, 0] == 2
    assert r["skipped"][0, 0, 0].tolist() == [0, 0, 1, 1, 0]
    assert r["order"][0, 0, 1].tolist() == [1, 0, -1, -1, -1] and r["count"][0, 0, 1] == 2
