"""No backward launch writes outside dQ, dK and dV.

The outputs are carved out of one buffer with guard bands filled with a
sentinel before and after each of them; every schedule (deterministic and
atomic) must leave the guards untouched and still match the oracle.
"""
import pytest
import torch

from tests import gpu_util as G
from persistent_sm_attn_b200 import binding

pytestmark = pytest.mark.gpu

GUARD = 4096  # bf16 elements before, between and after the outputs
SENTINEL = -12345.0


@pytest.mark.parametrize("B,H,S,D,causal", [(1, 2, 256, 128, False), (2, 1, 384, 64, True),
                                            (1, 3, 512, 128, True), (2, 2, 256, 64, False)])
def test_outputs_stay_in_bounds(B, H, S, D, causal):
    G.need_cuda()
    case = G.make_case(B, H, S, D, causal, seed=21 + S)
    n = B * H * S * D
    big = torch.full((4 * GUARD + 3 * n,), SENTINEL, dtype=torch.bfloat16, device="cuda")
    views = [big[GUARD + i * (n + GUARD): GUARD + i * (n + GUARD) + n].view(B, H, S, D)
             for i in range(3)]
    ref = G.oracle_full(case)
    N = S // 128
    scheds = ["naive_asc", "descending", "atomic"]
    scheds.append("shift" if not causal else ("sym_shift" if N % 2 == 0 else "naive_asc"))
    for sched in scheds:
        big.fill_(SENTINEL)
        binding.dash_attn_bwd(case["q"], case["k"], case["v"], case["o"], case["do"], case["lse"],
                              causal, sched, *views)
        assert binding.dash_attn_sync_status() == 0
        torch.cuda.synchronize()
        for i in range(4):
            g = big[i * (n + GUARD): i * (n + GUARD) + GUARD]
            assert bool((g == SENTINEL).all()), (sched, "guard", i)
        errs = G.check_full(case, views, ref)
        assert max(errs.values()) < G.TOL, (sched, errs)
