"""The two ways the ordered dQ chains add a middle position's partial: with red in
L2 once the ticket grants the position (mode 1), or load-add-store on the SM
(mode 2).  The additions and their order are the same, so both must give the same
bits, agree with the fp64 oracle, and repeat bit for bit; mode 0 (the library's
per-launch choice) must equal both.  Shapes span several tiles, both masks, both
head dims, every deterministic schedule, and 64 tiles where mode 0 takes red.
"""
import pytest
import torch

from oracle import attention as A
from persistent_sm_attn_b200 import binding
from tests import gpu_util as G

pytestmark = pytest.mark.gpu


def _run(case, sched, mode):
    binding.dash_set_dq_chain_mode(mode)
    try:
        return G.bwd(case, sched)
    finally:
        binding.dash_set_dq_chain_mode(0)


SMALL = [
    (1, 2, 640, 64, False, "shift"),
    (2, 2, 512, 128, False, "descending"),
    (1, 3, 384, 64, True, "naive_asc"),
    (1, 2, 768, 128, True, "sym_shift"),
    (2, 1, 1024, 64, True, "descending"),
]


@pytest.mark.parametrize("B,H,S,D,causal,sched", SMALL)
def test_red_chain_matches_oracle_and_load_add_store(B, H, S, D, causal, sched):
    G.need_cuda()
    case = G.make_case(B, H, S, D, causal, seed=500 + S + D)
    _, _, *ref = G.oracle_full(case)
    red = _run(case, sched, 1)
    errs = {n: A.rel_fro(x.float().cpu().numpy(), r) for n, x, r in zip(("dq", "dk", "dv"), red, ref)}
    G.log_margin(f"red chain B{B} H{H} S{S} D{D} {'causal' if causal else 'full'} {sched}", errs)
    assert max(errs.values()) < G.TOL, errs
    lds = _run(case, sched, 2)
    for a, b in zip(red, lds):
        assert torch.equal(a, b)
    again = _run(case, sched, 1)
    for a, b in zip(red, again):
        assert torch.equal(a, b)


@pytest.mark.parametrize("D,causal,sched", [(64, True, "descending"), (128, False, "naive_asc"),
                                            (128, True, "descending"), (64, False, "shift")])
def test_modes_agree_at_64_tiles(D, causal, sched):
    """S = 8192 (64 tiles): mode 0 takes red for descending and naive ascending; the
    three modes give the same bits."""
    G.need_cuda()
    case = G.make_case(1, 4, 8192, D, causal, seed=77 + D)
    outs = [_run(case, sched, m) for m in (0, 1, 2)]
    for other in outs[1:]:
        for a, b in zip(outs[0], other):
            assert torch.equal(a, b)


def test_mode_argument_errors():
    with pytest.raises(binding.DashError):
        binding.dash_set_dq_chain_mode(3)
    with pytest.raises(binding.DashError):
        binding.dash_set_dq_chain_mode(-1)
    binding.dash_set_dq_chain_mode(0)
