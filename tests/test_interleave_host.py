"""Head interleaving of multi-head tables, on the host (no GPU): the choice rule, the
forced modes, argument errors, and the interleaved table's invariants (each head's
KV segment is a chain of its own, each dQ block's positions are 0..n-1, and the
oracle's event graph has no cycle)."""
from collections import defaultdict

import pytest

from oracle import dag
from persistent_sm_attn_b200 import binding


def _acyclic(n_nodes, edges):
    indeg = [0] * n_nodes
    out = defaultdict(list)
    for u, v, _ in edges:
        out[u].append(v)
        indeg[v] += 1
    ready = [x for x in range(n_nodes) if indeg[x] == 0]
    seen = 0
    while ready:
        x = ready.pop()
        seen += 1
        for v in out[x]:
            indeg[v] -= 1
            if indeg[v] == 0:
                ready.append(v)
    return seen == n_nodes


def test_choice():
    f = binding.dash_bwd_head_interleave
    binding.dash_set_head_interleave(0)
    # causal 16k D=64, 128 heads x 64 units: 8192 or 4096 units fill 0.988 of the rounds
    assert f(148, 64, "sym_shift", 128, 16384, True) == 2
    assert f(148, 128, "sym_shift", 128, 16384, True) == 1       # D=128: no
    assert f(148, 64, "descending", 128, 16384, True) == 1       # other schedules: no
    assert f(148, 64, "sym_shift", 127, 16384, True) == 1        # odd head count
    # 16 heads x 8 units: 128/148 against 64/148 -> the fill decides against it
    assert f(148, 64, "sym_shift", 16, 2048, True) == 1


def test_forced_modes():
    f = binding.dash_bwd_head_interleave
    try:
        binding.dash_set_head_interleave(1)
        assert f(148, 64, "sym_shift", 128, 16384, True) == 1
        binding.dash_set_head_interleave(2)
        assert f(148, 128, "shift", 6, 1024, False) == 2
        assert f(148, 128, "shift", 5, 1024, False) == 1
        binding.dash_set_head_interleave(4)
        assert f(148, 64, "descending", 8, 512, True) == 4
        assert f(148, 64, "descending", 6, 512, True) == 1
    finally:
        binding.dash_set_head_interleave(0)


def test_argument_errors():
    for bad in (lambda: binding.dash_set_head_interleave(3),
                lambda: binding.dash_set_head_interleave(-1),
                lambda: binding.dash_bwd_head_interleave(0, 64, "shift", 4, 512, False),
                lambda: binding.dash_bwd_head_interleave(148, 96, "shift", 4, 512, False),
                lambda: binding.dash_bwd_head_interleave(148, 64, "shift", 0, 512, False),
                lambda: binding.dash_bwd_head_interleave(148, 64, "shift", 4, 500, False)):
        with pytest.raises(binding.DashError):
            bad()


@pytest.mark.parametrize("sched,N,causal,heads,il,ctas", [
    ("sym_shift", 4, True, 4, 2, 3), ("sym_shift", 8, True, 8, 4, 5),
    ("shift", 4, False, 6, 2, 4), ("descending", 5, True, 4, 2, 148),
    ("naive_asc", 3, False, 8, 4, 2)])
def test_interleaved_table(sched, N, causal, heads, il, ctas):
    """The table a multi-head launch uses with il heads per unit is the grouped table
    of group il; with K/V per head, every (head, KV tile) must be exactly one chain,
    the il heads of a unit's segment in order on one CTA."""
    rows = binding.dash_sched_table_gqa(heads, il, N, causal, sched, ctas)
    chains = {}
    order = []
    for cta, h, kv, q, p, ci in rows:
        if ci not in chains:
            chains[ci] = (cta, h, kv)
            order.append(ci)
    seg = defaultdict(list)
    for ci in order:
        cta, h, kv = chains[ci]
        seg[(h, kv)].append(cta)
    assert all(len(v) == 1 for v in seg.values())                # one chain per (head, kv)
    assert len(seg) == heads * N
    for i in range(len(order) - 1):
        c0, h0, kv0 = chains[order[i]]
        c1, h1, kv1 = chains[order[i + 1]]
        if c0 == c1 and kv0 == kv1 and h0 // il == h1 // il:
            assert h1 == h0 + 1                                     # the unit's heads in turn
    pos = defaultdict(list)
    for _, h, kv, q, p, _ in rows:
        pos[(h, q)].append(p)
    for (h, q), ps in pos.items():
        assert sorted(ps) == list(range(q + 1 if causal else N))
    slots = [[] for _ in range(ctas)]
    for cta, h, kv, q, p, _ in rows:
        slots[cta].append((h, kv, q, p, q + 1 if causal else N))
    for chains_per_block in (1, 2):
        n, edges, _ = dag.schedule_graph(slots, 1.0, 0.3, None, chains_per_block)
        assert _acyclic(n, edges)


def test_slot_placement_choice():
    """Slots are placed by SM id from 128 tiles by default; modes 1 and 2 force it."""
    f = binding.dash_slot_placement_by_smid
    try:
        binding.dash_set_slot_placement(0)
        assert f(16384) and f(32768) and not f(8192) and not f(128)
        binding.dash_set_slot_placement(1)
        assert f(128) and f(16384)
        binding.dash_set_slot_placement(2)
        assert not f(16384)
        for bad in (lambda: binding.dash_set_slot_placement(3),
                    lambda: binding.dash_set_slot_placement(-1),
                    lambda: f(100), lambda: f(0)):
            with pytest.raises(binding.DashError):
                bad()
    finally:
        binding.dash_set_slot_placement(0)
