"""The backward from host buffers: pipelined over parts of the heads, through
the same C ABI, with results bitwise equal to the device entry point's."""
import pytest
import torch

from persistent_sm_attn_b200 import binding
from tests import gpu_util as G

pytestmark = pytest.mark.gpu

NAMES = ("q", "k", "v", "o", "do", "lse")


@pytest.mark.parametrize("shape,sched,pinned", [
    ((2, 16, 4096, 128, False), "shift", True),     # parts straddle the persistent grid's rounds
    ((2, 8, 2048, 64, True), "sym_shift", True),
    ((3, 5, 640, 128, True), "descending", False),   # pageable host memory, uneven last part
    ((1, 2, 256, 64, False), "naive_asc", True),     # fewer heads than parts
])
def test_host_path_bitwise_equals_device_path(shape, sched, pinned):
    G.need_cuda()
    B, H, S, D, causal = shape
    case = G.make_case(B, H, S, D, causal, seed=11 + S + D)
    want = G.bwd(case, sched)
    host = [case[n].cpu() for n in NAMES]
    if pinned:
        host = [t.pin_memory() for t in host]
    got = binding.dash_attn_bwd_host(*host, causal, sched)
    assert binding.dash_attn_sync_status() == 0
    for a, b in zip(want, got):
        assert torch.equal(a.cpu(), b)


def test_host_path_atomic_is_accurate():
    G.need_cuda()
    case = G.make_case(2, 3, 512, 64, True, seed=5)
    ref = G.oracle_full(case)
    host = [case[n].cpu().pin_memory() for n in NAMES]
    got = binding.dash_attn_bwd_host(*host, True, "atomic")
    assert binding.dash_attn_sync_status() == 0
    errs = G.check_full(case, [t.cuda() for t in got], ref)
    assert max(errs.values()) < G.TOL, errs
