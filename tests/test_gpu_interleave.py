"""Head-interleaved multi-head tables on the GPU: every interleave (1, 2, 4 heads per
unit) agrees with the fp64 oracle and repeats bit for bit; the host-buffer and
no-allocation entry points give the allocating entry point's bits under the same
interleave; and the library's own choice at the default workload's shape is taken by
all three (checked through the choice query, then through equal results)."""
import pytest
import torch

from oracle import attention as A
from persistent_sm_attn_b200 import binding
from tests import gpu_util as G

pytestmark = pytest.mark.gpu

NAMES = ("q", "k", "v", "o", "do", "lse")


def _with_mode(mode, fn):
    binding.dash_set_head_interleave(mode)
    try:
        return fn()
    finally:
        binding.dash_set_head_interleave(0)


@pytest.mark.parametrize("B,H,S,D,causal,sched", [
    (2, 2, 512, 64, True, "sym_shift"),
    (1, 4, 640, 128, False, "shift"),
    (1, 8, 384, 64, True, "descending"),
])
def test_interleave_matches_oracle_and_repeats(B, H, S, D, causal, sched):
    G.need_cuda()
    case = G.make_case(B, H, S, D, causal, seed=900 + S + D)
    _, _, *ref = G.oracle_full(case)
    for mode in (1, 2, 4):
        out = _with_mode(mode, lambda: G.bwd(case, sched))
        errs = {n: A.rel_fro(x.float().cpu().numpy(), r)
                for n, x, r in zip(("dq", "dk", "dv"), out, ref)}
        G.log_margin(f"interleave {mode} B{B} H{H} S{S} D{D} {sched}", errs)
        assert max(errs.values()) < G.TOL, (mode, errs)
        again = _with_mode(mode, lambda: G.bwd(case, sched))
        for a, b in zip(out, again):
            assert torch.equal(a, b), mode


@pytest.mark.parametrize("mode", [2, 4])
def test_entry_points_agree_under_interleave(mode):
    G.need_cuda()
    B, H, S, D, causal, sched = 2, 4, 512, 64, True, "sym_shift"
    case = G.make_case(B, H, S, D, causal, seed=321)
    want = _with_mode(mode, lambda: G.bwd(case, sched))
    host = [case[n].cpu().pin_memory() for n in NAMES]
    got = _with_mode(mode, lambda: binding.dash_attn_bwd_host(*host, causal, sched))
    assert binding.dash_attn_sync_status() == 0
    for a, b in zip(want, got):
        assert torch.equal(a.cpu(), b)
    outs = [torch.empty_like(case["q"]) for _ in range(3)]
    _with_mode(mode, lambda: binding.dash_attn_bwd_noalloc(
        case["q"], case["k"], case["v"], case["o"], case["do"], case["lse"], causal, sched,
        *outs))
    assert binding.dash_attn_noalloc_sync_status() == 0
    for a, b in zip(want, outs):
        assert torch.equal(a, b)


def test_default_choice_at_the_default_workload():
    """At the default workload's shape (causal 16k D=64, 128 heads) the library
    interleaves two heads; the launch gives the bits of mode 2 and differs from mode 1
    at most by rounding."""
    G.need_cuda()
    ctas = binding.dash_bwd_num_ctas(0, 64)
    assert binding.dash_bwd_head_interleave(ctas, 64, "sym_shift", 128, 16384, True) == 2
    # a quarter of the heads keeps the test short; the choice there is the same
    assert binding.dash_bwd_head_interleave(ctas, 64, "sym_shift", 32, 16384, True) == 2
    case = G.make_case(1, 32, 16384, 64, True, seed=4242)
    auto = G.bwd(case, "sym_shift")
    two = _with_mode(2, lambda: G.bwd(case, "sym_shift"))
    one = _with_mode(1, lambda: G.bwd(case, "sym_shift"))
    for a, b, c in zip(auto, two, one):
        assert torch.equal(a, b)
        rel = (torch.linalg.vector_norm(a.float() - c.float()) /
               torch.linalg.vector_norm(c.float())).item()
        assert rel < 4e-3
