"""fp64 CPU oracle of softmax attention, forward and backward.

Test infrastructure only (see the package docstring): the product path never
imports this module.

What it computes.  DASH summary §1 fixes the object of the method: the attention
backward pass, whose dQ gradient must be accumulated in a fixed order to be
bit-reproducible.  The pages print no formulas, so this module writes out the
textbook definition of softmax attention and its gradient, per (batch, head),
in float64, with no tiling, blocking or reordering:

  forward   s_ij  = scale * q_i . k_j          (masked to -inf if causal and j > i)
            LSE_i = log sum_j exp(s_ij)        (natural log)
            P_ij  = exp(s_ij - LSE_i)
            O_i   = sum_j P_ij v_j
  backward  dV_j  = sum_i P_ij dO_i
            dP_ij = dO_i . v_j
            Delta_i = dO_i . O_i               (= sum_j P_ij dP_ij)
            dS_ij = P_ij (dP_ij - Delta_i)
            dQ_i  = scale * sum_j dS_ij k_j
            dK_j  = scale * sum_i dS_ij q_i

Causal masking is top-left aligned with equal query and key lengths: query row
i attends to keys j <= i.  Inputs may be any float dtype (e.g. bf16 values held
in float32); they are widened exactly to float64.  A matrix product (numpy's
``@``) serves as a library step.
"""
from __future__ import annotations

import numpy as np


def _f64(x) -> np.ndarray:
    """Widen to float64 (exact for bf16 / fp16 / fp32 inputs)."""
    if hasattr(x, "detach"):  # a torch tensor: go through float32 (exact for bf16)
        x = x.detach().to("cpu").float().numpy()
    return np.asarray(x, dtype=np.float64)


def _mask(S: int, causal: bool) -> np.ndarray:
    """Boolean [S,S] matrix of allowed (query i, key j) pairs."""
    if not causal:
        return np.ones((S, S), dtype=bool)
    return np.tril(np.ones((S, S), dtype=bool))


def head_forward(q, k, v, causal: bool, scale: float):
    """Forward of one head: returns (O [S,D], LSE [S]) from the definition."""
    S = q.shape[0]
    s = scale * (q @ k.T)
    allowed = _mask(S, causal)
    s = np.where(allowed, s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    lse = (m + np.log(np.exp(s - m).sum(axis=1, keepdims=True)))[:, 0]
    p = np.where(allowed, np.exp(s - lse[:, None]), 0.0)
    return p @ v, lse


def head_backward(q, k, v, do, causal: bool, scale: float):
    """Backward of one head: returns (dQ, dK, dV, Delta) from the definition.

    O and LSE are recomputed here in float64; the backward's own formula
    Delta_i = dO_i . O_i uses that O.
    """
    S = q.shape[0]
    allowed = _mask(S, causal)
    o, lse = head_forward(q, k, v, causal, scale)
    s = np.where(allowed, scale * (q @ k.T), -np.inf)
    p = np.where(allowed, np.exp(s - lse[:, None]), 0.0)
    dv = p.T @ do
    dp = do @ v.T
    delta = (do * o).sum(axis=1)
    ds = p * (dp - delta[:, None])
    dq = scale * (ds @ k)
    dk = scale * (ds.T @ q)
    return dq, dk, dv, delta


def forward(q, k, v, causal: bool, scale: float | None = None, heads=None):
    """Batched forward over [B,H,S,D] inputs.

    heads: optional iterable of (b, h) to compute; other heads are left NaN.
    Returns (O [B,H,S,D] float64, LSE [B,H,S] float64).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, S, D = q.shape
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    o = np.full((B, H, S, D), np.nan)
    lse = np.full((B, H, S), np.nan)
    for b, h in (heads if heads is not None else np.ndindex(B, H)):
        o[b, h], lse[b, h] = head_forward(q[b, h], k[b, h], v[b, h], causal, scale)
    return o, lse


def backward(q, k, v, do, causal: bool, scale: float | None = None, heads=None):
    """Batched backward over [B,H,S,D] inputs.

    heads: optional iterable of (b, h) to compute; other heads are left NaN.
    Returns (dQ, dK, dV [B,H,S,D], Delta [B,H,S]) in float64.
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    B, H, S, D = q.shape
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    dq = np.full((B, H, S, D), np.nan)
    dk = np.full((B, H, S, D), np.nan)
    dv = np.full((B, H, S, D), np.nan)
    delta = np.full((B, H, S), np.nan)
    for b, h in (heads if heads is not None else np.ndindex(B, H)):
        dq[b, h], dk[b, h], dv[b, h], delta[b, h] = head_backward(
            q[b, h], k[b, h], v[b, h], do[b, h], causal, scale)
    return dq, dk, dv, delta


def forward_gqa(q, k, v, causal: bool, scale: float | None = None):
    """Grouped-query forward: q [B,H,S,D], k and v [B,Hkv,S,D]; query head h attends
    with K/V head h // (H // Hkv).  Returns (O [B,H,S,D], LSE [B,H,S]) in float64."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, S, D = q.shape
    g = H // k.shape[1]
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    o = np.empty((B, H, S, D))
    lse = np.empty((B, H, S))
    for b, h in np.ndindex(B, H):
        o[b, h], lse[b, h] = head_forward(q[b, h], k[b, h // g], v[b, h // g], causal, scale)
    return o, lse


def backward_gqa(q, k, v, do, causal: bool, scale: float | None = None):
    """Grouped-query backward: dQ [B,H,S,D] per query head; dK and dV [B,Hkv,S,D],
    each the sum over the K/V head's query heads of that head's dK, dV (the
    gradient of a K/V head used by several query heads).  float64."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    B, H, S, D = q.shape
    Hkv = k.shape[1]
    g = H // Hkv
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    dq = np.empty((B, H, S, D))
    dk = np.zeros((B, Hkv, S, D))
    dv = np.zeros((B, Hkv, S, D))
    for b, h in np.ndindex(B, H):
        dq[b, h], dk_h, dv_h, _ = head_backward(q[b, h], k[b, h // g], v[b, h // g], do[b, h],
                                                causal, scale)
        dk[b, h // g] += dk_h
        dv[b, h // g] += dv_h
    return dq, dk, dv


def rel_fro(x, ref) -> float:
    """Relative Frobenius error ||x - ref||_F / ||ref||_F (the parity metric)."""
    x, ref = _f64(x), _f64(ref)
    den = np.linalg.norm(ref.ravel())
    num = np.linalg.norm((x - ref).ravel())
    return float(num / den) if den > 0 else float(num)


def head_forward_rows(q, k, v, causal: bool, scale: float, rows):
    """The forward of one head evaluated only at chosen query rows, for heads too large
    to hold S x S matrices: (O [len(rows), D], LSE [len(rows)]), each row from the same
    definitions as ``head_forward`` (row i sees keys j <= i under the causal mask)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    S = k.shape[0]
    rows = np.asarray(rows)
    keys = np.arange(S)
    allowed = (keys[None, :] <= rows[:, None]) if causal else np.ones((len(rows), S), bool)
    s = np.where(allowed, scale * (q[rows] @ k.T), -np.inf)
    m = s.max(axis=1, keepdims=True)
    lse = (m + np.log(np.exp(s - m).sum(axis=1, keepdims=True)))[:, 0]
    p = np.where(allowed, np.exp(s - lse[:, None]), 0.0)
    return p @ v, lse


def head_backward_rows(q, k, v, do, causal: bool, scale: float, rows_q, rows_kv, chunk=1024):
    """The backward of one head evaluated only at chosen rows, for heads too
    large to hold S x S matrices: dQ at query rows ``rows_q`` and dK, dV at
    key rows ``rows_kv``, each row from the same definitions as
    ``head_backward``.

    dK_j and dV_j sum over every query i, so O_i, LSE_i and Delta_i are first
    formed for all rows; those per-row quantities are independent of one
    another and are computed ``chunk`` rows at a time only to bound memory.
    Returns (dq [len(rows_q), D], dk, dv [len(rows_kv), D]).
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    S, D = q.shape
    rows_q = np.asarray(rows_q)
    rows_kv = np.asarray(rows_kv)
    keys = np.arange(S)
    lse = np.empty(S)
    o = np.empty((S, D))
    for a in range(0, S, chunk):
        i = np.arange(a, min(S, a + chunk))
        allowed = (keys[None, :] <= i[:, None]) if causal else np.ones((len(i), S), bool)
        s = np.where(allowed, scale * (q[i] @ k.T), -np.inf)
        m = s.max(axis=1, keepdims=True)
        lse[i] = (m + np.log(np.exp(s - m).sum(axis=1, keepdims=True)))[:, 0]
        o[i] = np.where(allowed, np.exp(s - lse[i][:, None]), 0.0) @ v
    delta = (do * o).sum(axis=1)
    # dQ rows
    allowed = (keys[None, :] <= rows_q[:, None]) if causal else np.ones((len(rows_q), S), bool)
    s = np.where(allowed, scale * (q[rows_q] @ k.T), -np.inf)
    p = np.where(allowed, np.exp(s - lse[rows_q][:, None]), 0.0)
    ds = p * (do[rows_q] @ v.T - delta[rows_q][:, None])
    dq = scale * (ds @ k)
    # dK, dV rows (columns j of P for all queries i)
    allowed = (keys[:, None] >= rows_kv[None, :]) if causal else np.ones((S, len(rows_kv)), bool)
    s = np.where(allowed, scale * (q @ k[rows_kv].T), -np.inf)
    p = np.where(allowed, np.exp(s - lse[:, None]), 0.0)
    dv = p.T @ do
    ds = p * (do @ v[rows_kv].T - delta[:, None])
    dk = scale * (ds.T @ q)
    return dq, dk, dv
