"""Grouped-query attention on the CUDA path (through the C ABI) against the fp64
oracle: H query heads share Hkv K/V heads, query head h reading K/V head
h // (H / Hkv); dK and dV sum over each K/V head's query heads.

Element-wise parity of O, LSE, dQ, dK, dV on small shapes (several tiles, both
masks, D = 64 and 128, every schedule the mask allows), including shapes with
more K/V heads than CTAs so that every CTA runs several dK/dV runs back to back;
the deterministic schedules must repeat bit for bit.
"""
import numpy as np
import pytest
import torch

from oracle import attention as A
from persistent_sm_attn_b200 import binding
from persistent_sm_attn_b200.inputs import draw
from tests import gpu_util as G

pytestmark = pytest.mark.gpu


def _schedules(S, causal):
    N = S // 128
    out = ["naive_asc", "descending", "atomic"]
    if not causal:
        out.append("shift")
    elif N % 2 == 0:
        out.append("sym_shift")
    return out


def _case(B, H, Hkv, S, D, causal, seed):
    q, _, _, do = draw(B, H, S, D, 1.0, seed, device="cuda")
    _, k, v, _ = draw(B, Hkv, S, D, 1.0, seed + 1, device="cuda")
    o, lse = binding.dash_attn_fwd_gqa(q, k, v, causal)
    torch.cuda.synchronize()
    return dict(q=q, k=k, v=v, do=do, o=o, lse=lse, causal=causal)


def _bwd(c, sched):
    out = binding.dash_attn_bwd_gqa(c["q"], c["k"], c["v"], c["o"], c["do"], c["lse"],
                                    c["causal"], sched)
    st = binding.dash_attn_sync_status()
    assert st == 0, binding.dash_status_string(st)
    return out


CASES = [
    (1, 4, 2, 256, 64, False),
    (1, 4, 2, 256, 128, False),
    (2, 4, 1, 512, 64, True),      # four query heads per K/V head
    (1, 8, 2, 512, 128, True),
    (2, 8, 4, 640, 128, False),    # odd tile count
    (1, 8, 1, 384, 64, True),      # eight query heads per K/V head, odd tile count
    # more (K/V head, KV tile) runs than CTAs: each CTA reloads K/V and drains dK/dV
    # between runs
    (4, 80, 40, 256, 64, False),
    (4, 80, 40, 256, 128, True),
]


@pytest.mark.parametrize("B,H,Hkv,S,D,causal", CASES)
def test_gqa_small_shapes_all_schedules(B, H, Hkv, S, D, causal):
    G.need_cuda()
    c = _case(B, H, Hkv, S, D, causal, seed=11 + S + D + H)
    q, k, v, do = (c[n].float().cpu().numpy() for n in ("q", "k", "v", "do"))
    o_ref, lse_ref = A.forward_gqa(q, k, v, causal)
    ref = A.backward_gqa(q, k, v, do, causal)
    assert A.rel_fro(c["o"].float().cpu().numpy(), o_ref) < G.TOL
    assert np.abs(c["lse"].cpu().numpy() - lse_ref).max() < 1e-3
    for sched in _schedules(S, causal):
        out = _bwd(c, sched)
        assert out[1].shape == c["k"].shape and out[2].shape == c["v"].shape
        errs = {n: A.rel_fro(g.float().cpu().numpy(), r)
                for n, g, r in zip(("dq", "dk", "dv"), out, ref)}
        assert max(errs.values()) < G.TOL, (sched, errs)
        if sched != "atomic":
            again = _bwd(c, sched)
            for a, b in zip(out, again):
                assert torch.equal(a, b), sched


def test_group_of_one_is_the_multi_head_path():
    G.need_cuda()
    c = _case(2, 3, 3, 384, 64, True, seed=5)
    o, lse = binding.dash_attn_fwd(c["q"], c["k"], c["v"], True)
    assert torch.equal(o, c["o"]) and torch.equal(lse, c["lse"])
    mha = binding.dash_attn_bwd(c["q"], c["k"], c["v"], c["o"], c["do"], c["lse"], True,
                                "descending")
    for a, b in zip(mha, _bwd(c, "descending")):
        assert torch.equal(a, b)
