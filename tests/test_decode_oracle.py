"""Pins for the oracle's single-query decode (osk_decode), the pages' future-work
phase ([TS] closing section) read as a q-block of one row under the same
in-kernel rule.  Pinned against torch SDPA (every page listed, eps = 0, GQA head
map), and against the closed form the decode kernel computes its decisions by:
for eps <= 1 a skipped page's local max lies below the running max, so the running
max before list position j is the maximum of the local maxima of every page
listed before j, and the decisions follow from the full logit row directly."""
import math

import numpy as np
import torch

import oracle as O
import workloads as W


def _layer(seed, N=1024, Hq=4, Hk=2, D=32, P=32):
    wl = W.small_workload("gqa-32k", N, Hq, Hk, head_dim=D, page_size=P, q_block=64,
                          shuffle_pages=True, batch=2)
    x = W.make_inputs(wl, seed=seed, keep_logical=True)
    return wl, x


def test_decode_all_pages_eps0_equals_sdpa():
    wl, x = _layer(21)
    B, Hq, N, D, P = 2, 4, 1024, 32, 32
    pos = np.array([1000, 517])
    q = x["q"][:, :, 0].double().numpy()  # any query vectors: row 0 of each head
    rng = np.random.default_rng(21)
    kc = N // P
    order = np.full((B, Hq, kc), -1, dtype=np.int32)
    count = np.zeros((B, Hq), dtype=np.int32)
    for b in range(B):
        for h in range(Hq):
            n = pos[b] // P + 1
            order[b, h, :n] = rng.permutation(n)
            count[b, h] = n
    r = O.osk_decode(q, x["k_pool"].double().numpy(), x["v_pool"].double().numpy(),
                     x["page_table"].numpy(), pos, order, count, num_kv_heads=2, page_size=P,
                     eps=0.0, scale=1 / math.sqrt(D))
    for b in range(B):
        t = int(pos[b])
        qq = torch.from_numpy(q[b])[:, None, :]                           # [H][1][D]
        k = x["k_log"][b].double().repeat_interleave(2, dim=0)[:, :t + 1]  # head h reads h // 2
        v = x["v_log"][b].double().repeat_interleave(2, dim=0)[:, :t + 1]
        want = torch.nn.functional.scaled_dot_product_attention(qq, k, v, scale=1 / math.sqrt(D))
        np.testing.assert_allclose(r["out"][b], want[:, 0].numpy(), rtol=0, atol=1e-12)
        s = (qq @ k.transpose(1, 2))[:, 0] / math.sqrt(D)
        np.testing.assert_allclose(r["lse"][b], torch.logsumexp(s, -1).numpy(), rtol=0, atol=1e-11)
    np.testing.assert_array_equal(r["computed"], count)


def test_decode_decisions_are_the_prefix_max_closed_form():
    wl, x = _layer(22)
    B, Hq, N, D, P = 2, 4, 1024, 32, 32
    pos = np.array([1023, 700])
    q = (x["q"][:, :, 5] * 2.0).double().numpy()
    kp, vp, pt = x["k_pool"].double().numpy(), x["v_pool"].double().numpy(), x["page_table"].numpy()
    rng = np.random.default_rng(22)
    kc = N // P
    n_skip = 0
    for eps in (1e-3, 1e-2, 0.3, 1.0):
        order = np.full((B, Hq, kc), -1, dtype=np.int32)
        count = np.zeros((B, Hq), dtype=np.int32)
        for b in range(B):
            for h in range(Hq):
                n = pos[b] // P + 1
                order[b, h, :n] = rng.permutation(n)
                count[b, h] = n
        r = O.osk_decode(q, kp, vp, pt, pos, order, count, num_kv_heads=2, page_size=P, eps=eps,
                         scale=1 / math.sqrt(D))
        for b in range(B):
            t = int(pos[b])
            for h in range(Hq):
                k = x["k_log"][b, h // 2].double().numpy()[:t + 1]
                s = k @ q[b, h] / math.sqrt(D)                          # the full logit row
                n = int(count[b, h])
                mloc = np.array([s[p * P:min((p + 1) * P, t + 1)].max() for p in order[b, h, :n]])
                prefix = np.maximum.accumulate(np.concatenate([[-np.inf], mloc[:-1]]))
                want = np.zeros(n, dtype=np.uint8)
                want[1:] = (mloc[1:] - prefix[1:]) < math.log(eps)
                assert np.array_equal(r["skip"][b, h, :n], want), (eps, b, h)
                n_skip += int(want.sum())
    assert n_skip > 0
