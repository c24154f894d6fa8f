"""The forward (O and LSE, the backward's inputs) against the fp64 oracle: every element
at small sizes (even and odd tile counts, one and several waves of CTAs) and sampled
rows at the configurations' full sizes (the launch the bench's inputs come from).  The
bar: relative Frobenius error 5e-3 on O, maximum absolute error 1e-3 on LSE."""
import numpy as np
import pytest

from oracle import attention as A
from persistent_sm_attn_b200 import binding
from persistent_sm_attn_b200.inputs import WORKLOADS, sample_heads, seed_of
from tests import gpu_util as G

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,H,S,D,causal", [
    (1, 2, 256, 64, False), (1, 2, 256, 64, True),
    (2, 3, 1024, 128, False), (2, 3, 1024, 128, True),
    (4, 40, 512, 64, True),                               # 640 CTAs: several waves
    (1, 2, 384, 64, True), (2, 3, 640, 128, False),      # odd tile counts
    (1, 1, 128, 64, True),
])
def test_forward_small(B, H, S, D, causal):
    G.need_cuda()
    q, k, v, _ = G.draw(B, H, S, D, 1.0, 91 + S + D, device="cuda")
    o, lse = binding.dash_attn_fwd(q, k, v, causal)
    assert binding.dash_attn_sync_status() == 0
    ro, rl = A.forward(q, k, v, causal)
    o_err = A.rel_fro(o.float().cpu().numpy(), ro)
    l_err = float(np.abs(lse.cpu().numpy() - rl).max())
    G.log_margin(f"forward B{B} H{H} S{S} D{D} {'causal' if causal else 'full'}",
                 {"o": o_err, "lse_abs": l_err})
    assert o_err < G.TOL and l_err < 1e-3, (o_err, l_err)


@pytest.mark.parametrize("index", [1, 2, 3, 4])
def test_forward_workloads_sampled(index):
    """Full sizes: the configurations' seeded inputs, 4 seeded heads and ~100 seeded
    query rows each, against the row-sampled oracle."""
    G.need_cuda()
    w = WORKLOADS[index]
    q, k, v, _ = G.draw(w.B, w.H, w.S, w.D, w.sigma, seed_of(index), device="cuda")
    o, lse = binding.dash_attn_fwd(q, k, v, w.causal)
    assert binding.dash_attn_sync_status() == 0
    rows = G.sample_rows(w.S, 96, 200 + index)
    scale = 1.0 / np.sqrt(w.D)
    o_err = l_err = 0.0
    for b, h in sample_heads(w.B, w.H, 4, seed_of(index)):
        ro, rl = A.head_forward_rows(q[b, h], k[b, h], v[b, h], w.causal, scale, rows)
        o_err = max(o_err, A.rel_fro(o[b, h][rows].float().cpu().numpy(), ro))
        l_err = max(l_err, float(np.abs(lse[b, h][rows].cpu().numpy() - rl).max()))
    G.log_margin(f"forward {w.name} (4 heads, sampled rows)", {"o": o_err, "lse_abs": l_err})
    assert o_err < G.TOL and l_err < 1e-3, (o_err, l_err)


def test_forward_repeats_bitwise():
    G.need_cuda()
    q, k, v, _ = G.draw(2, 8, 2048, 64, 1.0, 5, device="cuda")
    o1, l1 = binding.dash_attn_fwd(q, k, v, True)
    o2, l2 = binding.dash_attn_fwd(q, k, v, True)
    assert (o1 == o2).all() and (l1 == l2).all()
