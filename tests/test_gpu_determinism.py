"""Bitwise reproducibility of every deterministic schedule: 50 launches, and
launches racing a concurrent load on another stream, on every workload at its
full size (best schedule and the descending order, plus naive ascending where
it is one of the workload's compared schedules), on a reduced causal D = 64
shape, and for the CTA-pair schedules on a full-mask D = 64 shape, the causal 16k
workload and the two D = 128 configurations (full 4k, causal 8k)."""
import pytest
import torch

from persistent_sm_attn_b200.inputs import WORKLOADS, seed_of
from tests import gpu_util as G

pytestmark = pytest.mark.gpu


def _det(w):
    return tuple(s for s in w.schedules if s != "atomic")


# (label, (B, H, S, D, causal, sigma, seed), schedules)
CASES = [(w.name, (w.B, w.H, w.S, w.D, w.causal, w.sigma, seed_of(i)), _det(w))
         for i, w in enumerate(WORKLOADS) if i >= 1]
CASES.append(("causal_b2_h8_s4096_d64", (2, 8, 4096, 64, True, 1.0, 11),
              ("sym_shift", "descending", "naive_asc")))
# the CTA-pair schedules (D = 64): a full-mask shape, and the causal 16k workload
CASES.append(("full_b2_h16_s4096_d64_pairs", (2, 16, 4096, 64, False, 1.0, 12), ("shift_pairs",)))
_w3 = WORKLOADS[3]
CASES.append((_w3.name + "_pairs", (_w3.B, _w3.H, _w3.S, _w3.D, _w3.causal, _w3.sigma, seed_of(3)),
              ("sym_shift_pairs",)))
# and at D = 128, on the full-mask 4k and causal 8k configurations
for _i, _sched in ((1, "shift_pairs"), (2, "sym_shift_pairs")):
    _w = WORKLOADS[_i]
    CASES.append((_w.name + "_pairs", (_w.B, _w.H, _w.S, _w.D, _w.causal, _w.sigma, seed_of(_i)),
                  (_sched,)))
IDS = [c[0] for c in CASES]


def _same(a, b):
    # torch.equal compares on the device
    return all(torch.equal(x, y) for x, y in zip(a, b))


def _case(shape):
    B, H, S, D, causal, sigma, seed = shape
    return G.make_case(B, H, S, D, causal, sigma, seed)


@pytest.mark.parametrize("label,shape,schedules", CASES, ids=IDS)
def test_fifty_launches_bit_identical(label, shape, schedules):
    G.need_cuda()
    case = _case(shape)
    for sched in schedules:
        first = [t.clone() for t in G.bwd(case, sched)]
        for rep in range(49):
            assert _same(first, G.bwd(case, sched)), (label, sched, rep)
        del first


@pytest.mark.parametrize("label,shape,schedules", CASES, ids=IDS)
def test_bit_identical_under_concurrent_load(label, shape, schedules):
    G.need_cuda()
    case = _case(shape)
    side = torch.cuda.Stream()
    sizes = (1024, 3072, 8192)
    mats = {n: torch.randn(n, n, device="cuda", dtype=torch.bfloat16) for n in sizes}
    for sched in schedules:
        first = [t.clone() for t in G.bwd(case, sched)]
        for rep in range(6):
            n = sizes[rep % len(sizes)]
            with torch.cuda.stream(side):
                for _ in range(4):
                    mats[n] = (mats[n] @ mats[n]).clamp_(-1, 1)
            assert _same(first, G.bwd(case, sched)), (label, sched, rep)
        torch.cuda.synchronize()
        del first


def test_atomic_variant_runs_and_is_accurate():
    """The nondeterministic comparison variant: correct to the same bound
    (bitwise differences between its runs are allowed, not required)."""
    G.need_cuda()
    case = G.make_case(1, 2, 512, 64, False, seed=13)
    ref = G.oracle_full(case)
    errs = G.check_full(case, G.bwd(case, "atomic"), ref)
    G.log_margin("B1 H2 S512 D64 full atomic", errs)
    assert max(errs.values()) < G.TOL
