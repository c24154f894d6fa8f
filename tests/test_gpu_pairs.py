"""CTA pairs that pre-sum dQ (DASH_SCHED_SHIFT_PAIRS for the full mask,
DASH_SCHED_SYM_SHIFT_PAIRS for the causal one; D = 64 and 128): the two dQ partials of a
pair's step are added before the ordered accumulation, each CTA taking half of the columns.
Against the fp64 oracle on shapes with one or several rounds of CTA pairs (and, causal,
on sampled rows of the full 16k workload), bitwise repeats, and the refusals for shapes
the pairs do not serve."""
import pytest
import torch

from oracle import attention as A
from persistent_sm_attn_b200 import binding
from persistent_sm_attn_b200.inputs import WORKLOADS, sample_heads, seed_of
from tests import gpu_util as G

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,H,S", [
    (1, 2, 256),     # one pair unit per head
    (2, 3, 1024),    # 8 tiles: 4 pair units per head
    (4, 40, 256),    # 160 pair units: more than one round of CTA pairs
    (1, 4, 2048),
])
def test_pairs_match_oracle_and_repeat(B, H, S):
    G.need_cuda()
    case = G.make_case(B, H, S, 64, False, seed=700 + S + H)
    _, _, *ref = G.oracle_full(case)
    out = G.bwd(case, "shift_pairs")
    errs = {n: A.rel_fro(x.float().cpu().numpy(), r) for n, x, r in zip(("dq", "dk", "dv"), out, ref)}
    G.log_margin(f"shift_pairs B{B} H{H} S{S} D64 full", errs)
    assert max(errs.values()) < G.TOL, errs
    again = G.bwd(case, "shift_pairs")
    for a, b in zip(out, again):
        assert torch.equal(a, b)


@pytest.mark.parametrize("S,D,causal,sched", [
    (512, 64, True, "shift_pairs"), (384, 64, False, "shift_pairs"),
    (384, 128, False, "shift_pairs"), (512, 64, False, "sym_shift_pairs"),
    (768, 64, True, "sym_shift_pairs"), (768, 128, True, "sym_shift_pairs")])
def test_pairs_refuse_other_shapes(S, D, causal, sched):
    G.need_cuda()
    case = G.make_case(1, 2, S, D, causal, seed=5)
    with pytest.raises(binding.DashError):
        binding.dash_attn_bwd(case["q"], case["k"], case["v"], case["o"], case["do"],
                              case["lse"], causal, sched)


def test_host_path_gives_the_same_bits():
    """The host-buffer path runs each part on a slice of the same pair table."""
    G.need_cuda()
    case = G.make_case(2, 8, 1024, 64, False, seed=19)
    want = G.bwd(case, "shift_pairs")
    host = [case[n].cpu().pin_memory() for n in ("q", "k", "v", "o", "do", "lse")]
    got = binding.dash_attn_bwd_host(*host, False, "shift_pairs")
    assert binding.dash_attn_sync_status() == 0
    for a, b in zip(want, got):
        assert torch.equal(a.cpu(), b)


def test_other_entry_points_refuse_pairs():
    """The no-allocation and grouped-query entry points refuse SHIFT_PAIRS
    (DASH_ERR_UNSUPPORTED)."""
    G.need_cuda()
    case = G.make_case(1, 2, 512, 64, False, seed=9)
    args = (case["q"], case["k"], case["v"], case["o"], case["do"], case["lse"], False,
            "shift_pairs")
    for call in (lambda: binding.dash_attn_bwd_noalloc(*args, *[torch.empty_like(case["q"])
                                                               for _ in range(3)]),
                 lambda: binding.dash_attn_bwd_gqa(*args)):
        with pytest.raises(binding.DashError) as e:
            call()
        assert e.value.status == 2, e.value   # DASH_ERR_UNSUPPORTED


def test_pairs_repeat_at_a_larger_shape():
    """20 launches at B=2 H=16 S=4096 D=64 (several rounds of CTA pairs) give the same
    bits, and agree with the shift schedule to within rounding."""
    G.need_cuda()
    case = G.make_case(2, 16, 4096, 64, False, seed=808)
    first = G.bwd(case, "shift_pairs")
    for _ in range(19):
        again = G.bwd(case, "shift_pairs")
        for a, b in zip(first, again):
            assert torch.equal(a, b)
    plain = G.bwd(case, "shift")
    for a, b in zip(first, plain):
        rel = (torch.linalg.vector_norm(a.float() - b.float()) /
               torch.linalg.vector_norm(b.float())).item()
        assert rel < 4e-3


# ---------------------------------------------------------------- causal CTA pairs

@pytest.mark.parametrize("B,H,S", [
    (1, 2, 512),     # N = 4: one pair unit per head, every pair-tile on or below the diagonal
    (2, 3, 1024),    # N = 8: two pair units per head
    (4, 40, 512),    # 160 pair units: more than one round of CTA pairs
    (1, 4, 2048),
])
def test_causal_pairs_match_oracle_and_repeat(B, H, S):
    G.need_cuda()
    case = G.make_case(B, H, S, 64, True, seed=900 + S + H)
    _, _, *ref = G.oracle_full(case)
    out = G.bwd(case, "sym_shift_pairs")
    errs = {n: A.rel_fro(x.float().cpu().numpy(), r) for n, x, r in zip(("dq", "dk", "dv"), out, ref)}
    G.log_margin(f"sym_shift_pairs B{B} H{H} S{S} D64 causal", errs)
    assert max(errs.values()) < G.TOL, errs
    again = G.bwd(case, "sym_shift_pairs")
    for a, b in zip(out, again):
        assert torch.equal(a, b)


def test_causal_pairs_host_path_gives_the_same_bits():
    G.need_cuda()
    case = G.make_case(2, 8, 1024, 64, True, seed=23)
    want = G.bwd(case, "sym_shift_pairs")
    host = [case[n].cpu().pin_memory() for n in ("q", "k", "v", "o", "do", "lse")]
    got = binding.dash_attn_bwd_host(*host, True, "sym_shift_pairs")
    assert binding.dash_attn_sync_status() == 0
    for a, b in zip(want, got):
        assert torch.equal(a.cpu(), b)


def test_causal_pairs_repeat_at_a_larger_shape():
    """20 launches at B=2 H=16 S=4096 D=64 causal give the same bits, and agree with
    the symmetric shift to within rounding."""
    G.need_cuda()
    case = G.make_case(2, 16, 4096, 64, True, seed=818)
    first = G.bwd(case, "sym_shift_pairs")
    for _ in range(19):
        again = G.bwd(case, "sym_shift_pairs")
        for a, b in zip(first, again):
            assert torch.equal(a, b)
    plain = G.bwd(case, "sym_shift")
    for a, b in zip(first, plain):
        rel = (torch.linalg.vector_norm(a.float() - b.float()) /
               torch.linalg.vector_norm(b.float())).item()
        assert rel < 4e-3


def test_causal_pairs_full_workload_sampled():
    """The causal 16k workload (B=4 H=32 S=16384 D=64) with the causal pairs, on the
    configuration's own seeded inputs, heads and rows (those of the sampled workload
    parity test): against the oracle row by row, and against the symmetric shift on the
    whole tensors, from which the pairs differ only in the order of fp32 additions."""
    G.need_cuda()
    w = WORKLOADS[3]
    assert (w.B, w.H, w.S, w.D, w.causal) == (4, 32, 16384, 64, True)
    case = G.make_case(w.B, w.H, w.S, w.D, w.causal, w.sigma, seed_of(3))
    heads = sample_heads(w.B, w.H, 4, seed_of(3))
    rows_q = G.sample_rows(w.S, 96, 3)
    rows_kv = G.sample_rows(w.S, 96, 103)
    ref = G.oracle_rows(case, heads, rows_q, rows_kv)
    out = G.bwd(case, "sym_shift_pairs")
    errs = G.check_rows(out, ref, rows_q, rows_kv)
    G.log_margin(f"{w.name} sym_shift_pairs ({len(heads)} heads, sampled rows)", errs)
    assert max(errs.values()) < G.TOL, errs
    plain = G.bwd(case, "sym_shift")
    for a, b in zip(out, plain):
        rel = (torch.linalg.vector_norm(a.float() - b.float()) /
               torch.linalg.vector_norm(b.float())).item()
        assert rel < 1e-4, rel


@pytest.mark.parametrize("causal,sched", [(False, "shift_pairs"), (True, "sym_shift_pairs")])
def test_pairs_with_two_heads_per_unit(causal, sched):
    """dash_set_head_interleave(2) builds the pair table with two heads per unit: parity
    with the oracle on a multi-round grid, bitwise repeats, and the host-buffer path's
    bits."""
    G.need_cuda()
    case = G.make_case(4, 40, 512, 64, causal, seed=31 + causal)
    _, _, *ref = G.oracle_full(case)
    binding.dash_set_head_interleave(2)
    try:
        out = G.bwd(case, sched)
        again = G.bwd(case, sched)
        host = [case[n].cpu().pin_memory() for n in ("q", "k", "v", "o", "do", "lse")]
        got = binding.dash_attn_bwd_host(*host, causal, sched)
        assert binding.dash_attn_sync_status() == 0
    finally:
        binding.dash_set_head_interleave(0)
    errs = {n: A.rel_fro(x.float().cpu().numpy(), r) for n, x, r in zip(("dq", "dk", "dv"), out, ref)}
    G.log_margin(f"{sched} B4 H40 S512 D64, two heads per unit", errs)
    assert max(errs.values()) < G.TOL, errs
    for a, b, c in zip(out, again, got):
        assert torch.equal(a, b)
        assert torch.equal(a.cpu(), c)


# ---------------------------------------------------------------- D = 128
# dQp stays in TMEM at D = 128; the pair exchanges the other half of each row through a
# 16 KiB buffer in the peer's shared memory, 32 columns a round.

@pytest.mark.parametrize("B,H,S,causal,sched", [
    (1, 2, 256, False, "shift_pairs"),
    (2, 3, 1024, False, "shift_pairs"),
    (4, 40, 256, False, "shift_pairs"),      # more than one round of CTA pairs
    (1, 2, 512, True, "sym_shift_pairs"),
    (2, 3, 1024, True, "sym_shift_pairs"),
    (4, 40, 512, True, "sym_shift_pairs"),
])
def test_pairs_d128_match_oracle_and_repeat(B, H, S, causal, sched):
    G.need_cuda()
    case = G.make_case(B, H, S, 128, causal, seed=1300 + S + H)
    _, _, *ref = G.oracle_full(case)
    out = G.bwd(case, sched)
    errs = {n: A.rel_fro(x.float().cpu().numpy(), r) for n, x, r in zip(("dq", "dk", "dv"), out, ref)}
    G.log_margin(f"{sched} B{B} H{H} S{S} D128 {'causal' if causal else 'full'}", errs)
    assert max(errs.values()) < G.TOL, errs
    again = G.bwd(case, sched)
    for a, b in zip(out, again):
        assert torch.equal(a, b)


@pytest.mark.parametrize("causal,sched", [(False, "shift_pairs"), (True, "sym_shift_pairs")])
def test_pairs_d128_host_path_and_repeats(causal, sched):
    """20 launches at B=2 H=16 S=4096 D=128 give the same bits, and the host-buffer path
    gives dash_attn_bwd's bits.  Against the one-CTA schedule the pairs differ only in the
    order of the fp32 additions (partials pre-summed in pairs), which flips the rounding of
    a few bf16 outputs: about 1e-4 relative, bounded here by 1e-3."""
    G.need_cuda()
    case = G.make_case(2, 16, 4096, 128, causal, seed=1700 + causal)
    first = G.bwd(case, sched)
    for _ in range(19):
        again = G.bwd(case, sched)
        for a, b in zip(first, again):
            assert torch.equal(a, b)
    plain = G.bwd(case, "sym_shift" if causal else "shift")
    for a, b in zip(first, plain):
        rel = (torch.linalg.vector_norm(a.float() - b.float()) /
               torch.linalg.vector_norm(b.float())).item()
        assert rel < 1e-3, rel
    host = [case[n].cpu().pin_memory() for n in ("q", "k", "v", "o", "do", "lse")]
    got = binding.dash_attn_bwd_host(*host, causal, sched)
    assert binding.dash_attn_sync_status() == 0
    for a, b in zip(first, got):
        assert torch.equal(a.cpu(), b)
