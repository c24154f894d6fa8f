"""Helpers shared by the GPU tests: inputs, library calls, oracle comparison."""
import numpy as np
import torch

from oracle import attention as A
from persistent_sm_attn_b200 import binding
from persistent_sm_attn_b200.inputs import draw

TOL = 5e-3  # relative Frobenius error bound on dQ, dK, dV (and O)

# (label, {"dq": err, "dk": err, "dv": err}) of every parity check that ran; the
# terminal summary prints them, so a run shows its margin to the bound
MARGINS = []


def log_margin(label, errs):
    MARGINS.append((label, dict(errs)))


def need_cuda():
    import pytest
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def make_case(B, H, S, D, causal, sigma=1.0, seed=0):
    q, k, v, do = draw(B, H, S, D, sigma, seed, device="cuda")
    o, lse = binding.dash_attn_fwd(q, k, v, causal)
    torch.cuda.synchronize()
    return dict(q=q, k=k, v=v, do=do, o=o, lse=lse, causal=causal)


def bwd(case, schedule):
    dq, dk, dv = binding.dash_attn_bwd(case["q"], case["k"], case["v"], case["o"], case["do"],
                                       case["lse"], case["causal"], schedule)
    st = binding.dash_attn_sync_status()
    assert st == 0, binding.dash_status_string(st)
    return dq, dk, dv


def oracle_full(case):
    q, k, v, do = (case[n].float().cpu().numpy() for n in ("q", "k", "v", "do"))
    o, lse = A.forward(q, k, v, case["causal"])
    dq, dk, dv, _ = A.backward(q, k, v, do, case["causal"])
    return o, lse, dq, dk, dv


def check_full(case, outs, ref):
    o, lse, rdq, rdk, rdv = ref
    errs = {}
    for name, got, want in (("dq", outs[0], rdq), ("dk", outs[1], rdk), ("dv", outs[2], rdv)):
        errs[name] = A.rel_fro(got.float().cpu().numpy(), want)
    return errs


def oracle_rows(case, heads, rows_q, rows_kv):
    """Per sampled head: (dq rows, dk rows, dv rows) from the oracle."""
    out = {}
    scale = 1.0 / np.sqrt(case["q"].shape[-1])
    for b, h in heads:
        args = [case[n][b, h].float().cpu().numpy() for n in ("q", "k", "v", "do")]
        out[(b, h)] = A.head_backward_rows(*args, case["causal"], scale, rows_q, rows_kv)
    return out


def check_rows(outs, ref, rows_q, rows_kv):
    errs = {"dq": 0.0, "dk": 0.0, "dv": 0.0}
    for (b, h), (rq, rk, rv) in ref.items():
        gq = outs[0][b, h][rows_q].float().cpu().numpy()
        gk = outs[1][b, h][rows_kv].float().cpu().numpy()
        gv = outs[2][b, h][rows_kv].float().cpu().numpy()
        errs["dq"] = max(errs["dq"], A.rel_fro(gq, rq))
        errs["dk"] = max(errs["dk"], A.rel_fro(gk, rk))
        errs["dv"] = max(errs["dv"], A.rel_fro(gv, rv))
    return errs


def sample_rows(S, n, seed):
    g = np.random.default_rng(seed)
    rows = set(g.choice(S, size=min(n, S), replace=False).tolist())
    rows |= {0, 127 % S, S - 1, S // 2}        # tile edges and the ends
    return np.array(sorted(rows))
