"""Failure detection without a GPU fault: a schedule table whose first dQ
contributor never arrives (made on the host) must end with DASH_ERR_TIMEOUT
after a short spin limit, and the context must stay usable."""
import pytest

from persistent_sm_attn_b200 import binding
from tests import gpu_util as G


@pytest.mark.gpu
@pytest.mark.parametrize("D,causal,sched", [(64, False, "shift"), (128, True, "descending")])
def test_missing_contributor_times_out_then_recovers(D, causal, sched):
    G.need_cuda()
    case = G.make_case(1, 2, 512, D, causal, seed=31)
    binding.dash_set_spin_limit_us(2000)  # 2 ms
    try:
        binding.dash_inject_fault(1)
        binding.dash_attn_bwd(case["q"], case["k"], case["v"], case["o"], case["do"], case["lse"],
                              causal, sched)
        assert binding.dash_attn_sync_status() == 4  # DASH_ERR_TIMEOUT
    finally:
        binding.dash_inject_fault(0)
        binding.dash_set_spin_limit_us(0)
    # the same stream and context keep working
    ref = G.oracle_full(case)
    assert max(G.check_full(case, G.bwd(case, sched), ref).values()) < G.TOL


def test_inject_fault_rejects_unknown_modes():
    with pytest.raises(binding.DashError):
        binding.dash_inject_fault(7)


@pytest.mark.gpu
@pytest.mark.parametrize("D,sched", [(64, "sym_shift"), (128, "descending")])
def test_timeout_with_red_chains_interleave_and_placement(D, sched):
    """The same planted fault with every per-launch choice switched on: red chains,
    two heads per unit and slots placed by SM id (whose start-up exchange is a bounded
    wait of its own).  The timeout is reported and the next call is correct again."""
    G.need_cuda()
    case = G.make_case(1, 2, 512, D, True, seed=37)
    modes = ((binding.dash_set_dq_chain_mode, 1), (binding.dash_set_head_interleave, 2),
             (binding.dash_set_slot_placement, 1))
    try:
        for f, m in modes:
            f(m)
        binding.dash_set_spin_limit_us(2000)  # 2 ms
        binding.dash_inject_fault(1)
        binding.dash_attn_bwd(case["q"], case["k"], case["v"], case["o"], case["do"], case["lse"],
                              True, sched)
        assert binding.dash_attn_sync_status() == 4  # DASH_ERR_TIMEOUT
        binding.dash_inject_fault(0)
        binding.dash_set_spin_limit_us(0)
        ref = G.oracle_full(case)
        assert max(G.check_full(case, G.bwd(case, sched), ref).values()) < G.TOL
    finally:
        binding.dash_inject_fault(0)
        binding.dash_set_spin_limit_us(0)
        for f, _ in modes:
            f(0)
