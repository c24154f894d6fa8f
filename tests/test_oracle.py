"""Pins of the fp64 attention oracle against facts fixed outside it.

Each check below is independent of how ``oracle.attention`` is written:
central finite differences of the forward, torch float64 autograd of
softmax(scale*QK^T + mask) V, closed forms of uniform attention, invariants of
the softmax gradient, and the S = 1 special case.  ``test_pins_catch_planted_mistakes``
plants typical mistakes into a copy of the oracle and checks that the pins
reject every one of them.
"""
import numpy as np
import pytest
import torch

from oracle import attention as A

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _rand(shape, seed, sigma=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * sigma


def _loss_grads_fd(q, k, v, do, causal, scale, fwd=A.head_forward, h=1e-6):
    """Central finite differences of L = sum(dO * O) with respect to q, k, v."""
    grads = []
    for which in range(3):
        args = [q.copy(), k.copy(), v.copy()]
        g = np.zeros_like(args[which])
        for idx in np.ndindex(*g.shape):
            plus = [a.copy() for a in args]
            minus = [a.copy() for a in args]
            plus[which][idx] += h
            minus[which][idx] -= h
            lp = (do * fwd(*plus, causal, scale)[0]).sum()
            lm = (do * fwd(*minus, causal, scale)[0]).sum()
            g[idx] = (lp - lm) / (2 * h)
        grads.append(g)
    return grads


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("S,D", [(1, 2), (3, 2), (5, 4), (8, 3)])
def test_backward_matches_finite_differences(S, D, causal):
    q, k, v, do = (_rand((S, D), 10 + i + 7 * S + D) for i in range(4))
    scale = 0.7
    dq, dk, dv, _ = A.head_backward(q, k, v, do, causal, scale)
    fq, fk, fv = _loss_grads_fd(q, k, v, do, causal, scale)
    for got, ref in ((dq, fq), (dk, fk), (dv, fv)):
        err = np.abs(got - ref).max() / max(1.0, np.abs(ref).max())
        assert err < 1e-7


def _torch_autograd(q, k, v, do, causal, scale):
    q, k, v = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    S = q.shape[-2]
    s = scale * q @ k.transpose(-1, -2)
    if causal:
        s = s.masked_fill(torch.ones(S, S, dtype=torch.bool).triu(1), float("-inf"))
    o = torch.softmax(s, dim=-1) @ v
    lse = torch.logsumexp(s, dim=-1)
    o.backward(torch.tensor(do, dtype=torch.float64))
    return o.detach().numpy(), lse.detach().numpy(), q.grad.numpy(), k.grad.numpy(), v.grad.numpy()


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,H,S,D", [(1, 1, 64, 16), (2, 2, 33, 8), (1, 3, 17, 32)])
def test_matches_torch_float64_autograd(B, H, S, D, causal):
    q, k, v, do = (_rand((B, H, S, D), 100 + i + S) for i in range(4))
    scale = 1.0 / np.sqrt(D)
    o, lse = A.forward(q, k, v, causal, scale)
    dq, dk, dv, _ = A.backward(q, k, v, do, causal, scale)
    to, tl, tq, tk, tv = _torch_autograd(q, k, v, do, causal, scale)
    for got, ref in ((o, to), (lse, tl), (dq, tq), (dk, tk), (dv, tv)):
        assert np.abs(got - ref).max() <= 1e-11 * max(1.0, np.abs(ref).max())


@pytest.mark.parametrize("causal", [False, True])
def test_uniform_attention_closed_forms(causal):
    """All key rows equal: every allowed key gets weight 1/n_i, so dQ = 0 and
    dK, dV, O have closed forms; the dK and dQ row sums follow."""
    S, D = 24, 8
    rng = np.random.default_rng(5)
    q, v, do = (rng.standard_normal((S, D)) for _ in range(3))
    kappa = rng.standard_normal(D)
    k = np.tile(kappa, (S, 1))
    scale = 0.3
    o, lse = A.head_forward(q, k, v, causal, scale)
    dq, dk, dv, delta = A.head_backward(q, k, v, do, causal, scale)
    n = np.arange(1, S + 1, dtype=float) if causal else np.full(S, float(S))
    allowed = np.tril(np.ones((S, S), bool)) if causal else np.ones((S, S), bool)
    o_ref = np.array([v[allowed[i]].mean(axis=0) for i in range(S)])
    dv_ref = np.array([(do[allowed[:, j]] / n[allowed[:, j], None]).sum(axis=0) for j in range(S)])
    d_ref = np.array([(do[i] @ v[allowed[i]].T).sum() / n[i] for i in range(S)])
    dk_ref = np.zeros((S, D))
    for j in range(S):
        for i in range(S):
            if allowed[i, j]:
                dk_ref[j] += scale * (do[i] @ v[j] - d_ref[i]) / n[i] * q[i]
    assert np.abs(o - o_ref).max() < 1e-12
    assert np.abs(lse - (scale * q @ kappa + np.log(n))).max() < 1e-12
    assert np.abs(dq).max() < 1e-12                      # dQ row sums: zero
    assert np.abs(dv - dv_ref).max() < 1e-12
    assert np.abs(delta - d_ref).max() < 1e-12
    assert np.abs(dk - dk_ref).max() < 1e-12
    assert np.abs(dk.sum(axis=1) - dk_ref.sum(axis=1)).max() < 1e-12   # dK row sums


@pytest.mark.parametrize("causal", [False, True])
def test_softmax_gradient_invariants(causal):
    S, D = 40, 16
    q, k, v, do = (_rand((S, D), 200 + i) for i in range(4))
    scale = 1 / 4
    dq, dk, dv, delta = A.head_backward(q, k, v, do, causal, scale)
    # sum_j dS_ij = 0 for every row, so the key gradients sum to zero
    assert np.abs(dk.sum(axis=0)).max() < 1e-11
    # adding the same vector to every key row shifts each score row by a
    # constant: O, LSE - scale*q.c, dQ and dV are unchanged
    c = _rand(D, 9)
    o1, lse1 = A.head_forward(q, k, v, causal, scale)
    o2, lse2 = A.head_forward(q, k + c, v, causal, scale)
    dq2, dk2, dv2, _ = A.head_backward(q, k + c, v, do, causal, scale)
    assert np.abs(o1 - o2).max() < 1e-12
    assert np.abs((lse2 - lse1) - scale * q @ c).max() < 1e-11
    assert np.abs(dq - dq2).max() < 1e-11 and np.abs(dv - dv2).max() < 1e-12
    # Delta_i = dO_i . O_i equals sum_j P_ij dP_ij
    o, lse = A.head_forward(q, k, v, causal, scale)
    s = scale * q @ k.T
    if causal:
        s = np.where(np.tril(np.ones((S, S), bool)), s, -np.inf)
    p = np.exp(s - lse[:, None])
    assert np.abs(delta - (p * (do @ v.T)).sum(axis=1)).max() < 1e-12


def test_single_key_special_case():
    """S = 1: the only weight is 1, so O = v, dV = dO and dQ = dK = 0."""
    q, k, v, do = (_rand((1, 5), 300 + i) for i in range(4))
    o, lse = A.head_forward(q, k, v, False, 0.5)
    dq, dk, dv, _ = A.head_backward(q, k, v, do, False, 0.5)
    assert np.allclose(o, v) and np.allclose(lse, 0.5 * q @ k.T)
    assert np.allclose(dv, do) and np.abs(dq).max() == 0 and np.abs(dk).max() == 0


def test_rel_fro_metric():
    ref = np.array([3.0, 4.0])
    assert A.rel_fro(ref, ref) == 0
    assert abs(A.rel_fro(ref + np.array([0.3, 0.4]), ref) - 0.1) < 1e-15


# ---------------------------------------------------------------------------
# Planted mistakes: each mutant of the backward must fail at least one pin.

def _mutants():
    def drop_delta(q, k, v, do, causal, scale):
        S = q.shape[0]
        m = A._mask(S, causal)
        o, lse = A.head_forward(q, k, v, causal, scale)
        p = np.where(m, np.exp(np.where(m, scale * q @ k.T, -np.inf) - lse[:, None]), 0)
        ds = p * (do @ v.T)
        return scale * ds @ k, scale * ds.T @ q, p.T @ do, None

    def wrong_sign(q, k, v, do, causal, scale):
        dq, dk, dv, d = A.head_backward(q, k, v, do, causal, scale)
        return -dq, dk, dv, d

    def transposed_dk(q, k, v, do, causal, scale):
        S = q.shape[0]
        m = A._mask(S, causal)
        o, lse = A.head_forward(q, k, v, causal, scale)
        p = np.where(m, np.exp(np.where(m, scale * q @ k.T, -np.inf) - lse[:, None]), 0)
        ds = p * (do @ v.T - (do * o).sum(1)[:, None])
        return scale * ds @ k, scale * ds @ q, p.T @ do, None

    def missing_scale(q, k, v, do, causal, scale):
        dq, dk, dv, d = A.head_backward(q, k, v, do, causal, scale)
        return dq / scale, dk, dv, d

    def dv_untransposed(q, k, v, do, causal, scale):
        dq, dk, dv, d = A.head_backward(q, k, v, do, causal, scale)
        S = q.shape[0]
        m = A._mask(S, causal)
        o, lse = A.head_forward(q, k, v, causal, scale)
        p = np.where(m, np.exp(np.where(m, scale * q @ k.T, -np.inf) - lse[:, None]), 0)
        return dq, dk, p @ do, d

    def mask_off_by_one(q, k, v, do, causal, scale):
        S = q.shape[0]
        m = np.tril(np.ones((S, S), bool), -1) if causal else np.ones((S, S), bool)
        m[0, 0] = True
        s = np.where(m, scale * q @ k.T, -np.inf)
        lse = np.log(np.exp(s).sum(1))
        p = np.where(m, np.exp(s - lse[:, None]), 0)
        o = p @ v
        ds = p * (do @ v.T - (do * o).sum(1)[:, None])
        return scale * ds @ k, scale * ds.T @ q, p.T @ do, None

    return [drop_delta, wrong_sign, transposed_dk, missing_scale, dv_untransposed,
            mask_off_by_one]


@pytest.mark.parametrize("mutant", _mutants(), ids=lambda f: f.__name__)
def test_pins_catch_planted_mistakes(mutant):
    rejected = False
    for causal in (False, True):
        S, D = 6, 3
        q, k, v, do = (_rand((S, D), 400 + i) for i in range(4))
        scale = 0.6
        dq, dk, dv, _ = mutant(q, k, v, do, causal, scale)
        to, tl, tq, tk, tv = _torch_autograd(q, k, v, do, causal, scale)
        if max(np.abs(dq - tq).max(), np.abs(dk - tk).max(), np.abs(dv - tv).max()) > 1e-9:
            rejected = True
    assert rejected


@pytest.mark.parametrize("causal", [False, True])
def test_row_sampled_forward_matches_torch_softmax(causal):
    """The row-sampled forward used at full workload sizes equals torch float64
    softmax and logsumexp on the sampled rows."""
    import torch
    S, D = 96, 16
    q, k, v = (_rand((S, D), 600 + i) for i in range(3))
    scale = 0.25
    rows = np.array([0, 1, 31, 32, 63, 95])
    o, lse = A.head_forward_rows(q, k, v, causal, scale, rows)
    s = scale * (torch.from_numpy(q) @ torch.from_numpy(k).T)
    if causal:
        s = s.masked_fill(torch.ones(S, S, dtype=torch.bool).triu(1), float("-inf"))
    want_o = (torch.softmax(s, dim=1) @ torch.from_numpy(v)).numpy()
    want_lse = torch.logsumexp(s, dim=1).numpy()
    assert np.abs(o - want_o[rows]).max() < 1e-12
    assert np.abs(lse - want_lse[rows]).max() < 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_row_sampled_backward_matches_autograd(causal):
    """The row-sampled backward used at full workload sizes equals torch
    float64 autograd on the sampled rows."""
    S, D = 96, 16
    q, k, v, do = (_rand((S, D), 500 + i) for i in range(4))
    scale = 0.25
    rq = np.array([0, 5, 31, 32, 95])
    rk = np.array([0, 1, 64, 94, 95])
    dq, dk, dv = A.head_backward_rows(q, k, v, do, causal, scale, rq, rk, chunk=40)
    _, _, tq, tk, tv = _torch_autograd(q, k, v, do, causal, scale)
    assert np.abs(dq - tq[rq]).max() < 1e-11
    assert np.abs(dk - tk[rk]).max() < 1e-11
    assert np.abs(dv - tv[rk]).max() < 1e-11
