"""Skip-rule variants compared on the oracle (CPU): the pages' rule (page max
against the running max), a sum-aware rule (the page's largest possible mass
against the mass the row already holds) and an early break after r consecutive
skipped pages.  Measured: pages whose QK^T is evaluated (visited), pages with
P V (computed), and the output error against dense attention and against the
listed pages with nothing skipped, on small synthetic layers with the shapes of
the benchmark workloads (8K tokens, budget 0.25) and on the last q-blocks of a
32K layer (lists of about 80 pages, budget 0.2).  The table prints with
`pytest -s`; the assertions hold what each rule promises."""
import math

import numpy as np
import pytest

import oracle as O
import workloads as W

STUDY = {  # workload, budget, q-blocks (None: all)
    "narrow-kv-8k": (W.small_workload("narrow-kv-64k", 8192, 7, 1), 0.25, None),
    "wide-head-8k-p128": (W.small_workload("wide-head-128k", 8192, 8, 1), 0.25, None),
    "gqa-32k-late": (W.small_workload("gqa-32k", 32768, 1, 1), 0.2, list(range(255, 128, -16))),
}
RULES = [  # (label, rule, eps, max_run)
    ("max eps=1e-4", "max", 1e-4, None),
    ("max eps=1e-3", "max", 1e-3, None),
    ("sum eps=1e-3", "sum", 1e-3, None),
    ("sum eps=1e-2", "sum", 1e-2, None),
    ("max eps=1e-4, break r=16", "max", 1e-4, 16),
    ("max eps=1e-4, break r=8", "max", 1e-4, 8),
    ("max eps=1e-4, break r=4", "max", 1e-4, 4),
]


def _rel_l2(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def study(name: str, seed: int = 21):
    wl, budget, qbs = STUDY[name]
    x = W.make_inputs(wl, seed=seed)
    q, kp, vp = (x[k].double().numpy() for k in ("q", "k_pool", "v_pool"))
    pt = x["page_table"].numpy()
    scale = 1 / math.sqrt(wl.head_dim)
    common = dict(num_kv_heads=wl.num_kv_heads, page_size=wl.page_size, q_block=wl.q_block,
                  qblocks=qbs)
    kap = O.kap_select(q, kp, pt, q_sub=wl.q_block // 4, k_sub=16, scale=scale, budget=budget,
                       sink_pages=1, **common)
    nqb = wl.seq_len // wl.q_block
    sel_qb = list(range(nqb)) if qbs is None else list(qbs)
    rows = np.concatenate([np.arange(b * wl.q_block, (b + 1) * wl.q_block) for b in sel_qb])
    pick = lambda o: o[:, :, rows]
    dense = pick(O.dense_attention(q, kp, vp, pt, num_kv_heads=wl.num_kv_heads, scale=scale,
                                   rows=rows)["out"])
    full = O.osk_attention(q, kp, vp, pt, kap["order"], kap["count"], eps=0.0, scale=scale,
                           **common)
    listed = int(kap["count"][:, :, sel_qb].sum())
    out = []
    for label, rule, eps, max_run in RULES:
        r = O.osk_attention(q, kp, vp, pt, kap["order"], kap["count"], eps=eps, scale=scale,
                            rule=rule, max_run=max_run, **common)
        out.append({"rule": label, "listed": listed,
                    "visited": int(r["visited"][:, :, sel_qb].sum()),
                    "computed": int(r["computed"][:, :, sel_qb].sum()),
                    "err_vs_dense": _rel_l2(pick(r["out"]), dense),
                    "err_vs_listed": _rel_l2(pick(r["out"]), pick(full["out"])),
                    "skip": r["skip"][:, :, sel_qb], "n_blocks": len(sel_qb) * wl.batch *
                    wl.num_q_heads})
    return out, _rel_l2(pick(full["out"]), dense)


@pytest.mark.parametrize("name", sorted(STUDY))
def test_skip_rule_variants(name):
    rows, listed_err = study(name)
    print(f"\n{name}: listed pages, nothing skipped: error vs dense {listed_err:.4f}")
    print(f"{'rule':28s} {'listed':>7s} {'visited':>8s} {'computed':>9s} "
          f"{'err vs dense':>13s} {'err vs listed':>14s}")
    for r in rows:
        print(f"{r['rule']:28s} {r['listed']:7d} {r['visited']:8d} {r['computed']:9d} "
              f"{r['err_vs_dense']:13.4f} {r['err_vs_listed']:14.2e}")
    by = {r["rule"]: r for r in rows}
    for r in rows:
        assert r["computed"] <= r["visited"] <= r["listed"]
        assert r["computed"] >= r["n_blocks"]  # the first listed page is always computed
    base = by["max eps=1e-4"]
    for lab in ("max eps=1e-4, break r=16", "max eps=1e-4, break r=8", "max eps=1e-4, break r=4"):
        # the break only drops pages the pages' rule would have reached later
        assert by[lab]["visited"] <= base["visited"] and by[lab]["computed"] <= base["computed"]
        assert np.all(by[lab]["skip"] >= base["skip"])
