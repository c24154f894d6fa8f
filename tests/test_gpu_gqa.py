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


# Split groups: sub-group s adds its dK/dV partials after sub-group s - 1 (fp32,
# ordered), so every split is deterministic and agrees with the oracle; split 1 is
# the un-split path (the group's sum accumulates in one CTA).
SPLIT_CASES = [
    (1, 8, 1, 512, 64, False, "shift"),
    (1, 8, 2, 512, 128, True, "sym_shift"),
    (2, 16, 2, 384, 64, True, "descending"),
    (1, 4, 1, 640, 128, False, "naive_asc"),   # odd tile count
    (1, 8, 1, 256, 128, False, "atomic"),      # dQ atomic, dK/dV still ordered
    # more runs than CTAs: CTAs hold runs of several sub-groups one after another
    (4, 64, 8, 256, 64, True, "descending"),
]


@pytest.mark.parametrize("B,H,Hkv,S,D,causal,sched", SPLIT_CASES)
def test_gqa_split_matches_oracle_and_repeats(B, H, Hkv, S, D, causal, sched):
    G.need_cuda()
    c = _case(B, H, Hkv, S, D, causal, seed=29 + S + D + H)
    q, k, v, do = (c[n].float().cpu().numpy() for n in ("q", "k", "v", "do"))
    ref = A.backward_gqa(q, k, v, do, causal)
    g = H // Hkv
    split = 1
    while split <= g:
        args = (c["q"], c["k"], c["v"], c["o"], c["do"], c["lse"], c["causal"], sched)
        out = binding.dash_attn_bwd_gqa(*args, split=split)
        st = binding.dash_attn_sync_status()
        assert st == 0, (split, binding.dash_status_string(st))
        errs = {n: A.rel_fro(x.float().cpu().numpy(), r)
                for n, x, r in zip(("dq", "dk", "dv"), out, ref)}
        G.log_margin(f"gqa B{B} H{H} Hkv{Hkv} S{S} D{D} {sched} split{split}", errs)
        assert max(errs.values()) < G.TOL, (split, errs)
        again = binding.dash_attn_bwd_gqa(*args, split=split)
        assert binding.dash_attn_sync_status() == 0
        for i, (a, b) in enumerate(zip(out, again)):
            if sched == "atomic" and i == 0:
                continue
            assert torch.equal(a, b), (split, i)
        split *= 2


def test_gqa_split_at_a_workload_shape():
    """32 query heads over 2 K/V heads at S = 4096, D = 128 (the full-mask workload's
    shape): every split agrees with the un-split path to within bf16 rounding, is
    deterministic, and the default call is the library's own choice."""
    G.need_cuda()
    B, H, Hkv, S, D, causal, sched = 1, 32, 2, 4096, 128, False, "shift"
    c = _case(B, H, Hkv, S, D, causal, seed=404)
    args = (c["q"], c["k"], c["v"], c["o"], c["do"], c["lse"], causal, sched)
    base = [x.float() for x in binding.dash_attn_bwd_gqa(*args, split=1)]
    assert binding.dash_attn_sync_status() == 0
    auto = binding.dash_bwd_gqa_split_for(binding.dash_bwd_num_ctas(0, D), B, Hkv, H // Hkv,
                                          S, causal, sched)
    assert auto in (1, 2, 4, 8, 16)
    for split in (2, 4, 16):
        out = binding.dash_attn_bwd_gqa(*args, split=split)
        assert binding.dash_attn_sync_status() == 0
        # dQ's order may change too: the split moves units across the grid's rounds
        for x, y in zip(out, base):
            rel = (torch.linalg.vector_norm(x.float() - y) / torch.linalg.vector_norm(y)).item()
            assert rel < 4e-3, (split, rel)
        again = binding.dash_attn_bwd_gqa(*args, split=split)
        for x, y in zip(out, again):
            assert torch.equal(x, y), split
    dflt = binding.dash_attn_bwd_gqa(*args)
    want = binding.dash_attn_bwd_gqa(*args, split=auto)
    for x, y in zip(dflt, want):
        assert torch.equal(x, y)
