"""Pins of the grouped-query oracle (oracle.attention.forward_gqa / backward_gqa).

Grouped-query attention is not on the pages; the oracle writes out its plain
definition: query head h uses K/V head h // (H // Hkv), and the gradient of a K/V
head sums over the query heads that use it.  The pins check that against torch
float64 autograd of the same attention written with K/V repeated per query head
(the autograd of the repeat does the summing), against the multi-head oracle when
every query head has its own K/V head, and that a wrong head mapping fails.
"""
import numpy as np
import pytest
import torch

from oracle import attention as A


def _inputs(B, H, Hkv, S, D, seed):
    g = np.random.default_rng(seed)
    q = g.standard_normal((B, H, S, D))
    k = g.standard_normal((B, Hkv, S, D))
    v = g.standard_normal((B, Hkv, S, D))
    do = g.standard_normal((B, H, S, D))
    return q, k, v, do


def _autograd(q, k, v, do, causal):
    B, H, S, D = q.shape
    rep = H // k.shape[1]
    qt, kt, vt = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    kr, vr = kt.repeat_interleave(rep, dim=1), vt.repeat_interleave(rep, dim=1)
    s = (qt @ kr.transpose(-1, -2)) / np.sqrt(D)
    if causal:
        s = s.masked_fill(~torch.tril(torch.ones(S, S, dtype=torch.bool)), float("-inf"))
    o = torch.softmax(s, dim=-1) @ vr
    lse = torch.logsumexp(s, dim=-1)
    o.backward(torch.tensor(do))
    return (o.detach().numpy(), lse.detach().numpy(), qt.grad.numpy(), kt.grad.numpy(),
            vt.grad.numpy())


@pytest.mark.parametrize("B,H,Hkv,S,D,causal", [
    (2, 4, 2, 16, 8, False), (1, 8, 2, 12, 4, True), (1, 6, 1, 10, 8, True), (2, 4, 4, 9, 4, False),
])
def test_gqa_oracle_matches_autograd(B, H, Hkv, S, D, causal):
    q, k, v, do = _inputs(B, H, Hkv, S, D, seed=B * 100 + H * 10 + Hkv)
    o, lse = A.forward_gqa(q, k, v, causal)
    dq, dk, dv = A.backward_gqa(q, k, v, do, causal)
    want = _autograd(q, k, v, do, causal)
    for got, ref in zip((o, lse, dq, dk, dv), want):
        assert got.shape == ref.shape
        np.testing.assert_allclose(got, ref, rtol=1e-10, atol=1e-12)


def test_gqa_with_one_query_head_per_kv_head_is_multi_head():
    q, k, v, do = _inputs(2, 3, 3, 11, 8, seed=5)
    for causal in (False, True):
        o1, l1 = A.forward_gqa(q, k, v, causal)
        o2, l2 = A.forward(q, k, v, causal)
        assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
        g = A.backward_gqa(q, k, v, do, causal)
        m = A.backward(q, k, v, do, causal)[:3]
        for a, b in zip(g, m):
            assert np.array_equal(a, b)


def test_a_wrong_head_mapping_fails_the_pin():
    """Query head h paired with K/V head h % Hkv instead of h // (H / Hkv)."""
    q, k, v, do = _inputs(1, 4, 2, 10, 4, seed=9)
    want = _autograd(q, k, v, do, False)
    k_wrong = k[:, [0, 1, 0, 1]]  # what h % Hkv would use
    v_wrong = v[:, [0, 1, 0, 1]]
    dq_wrong = A.backward(q, k_wrong, v_wrong, do, False)[0]
    assert not np.allclose(dq_wrong, want[2], rtol=1e-6)
