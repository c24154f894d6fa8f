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
