"""The paired shift schedule (DASH_SCHED_SHIFT_PAIRS), on the host: CTA pairs run KV
tiles 2m and 2m + 1 over the same Q tiles at the same steps and pre-sum their dQ
partials, so each dQ block receives N / 2 contributions.  Checked without a GPU:
- the oracle's units: every KV pair visits every Q tile once, and every step touches
  N / 2 distinct dQ blocks (conflict-free);
- the library's half table equals the oracle's packed table, and its event graph
  (one or two accumulation chains per block) has no cycle;
- the grid's table: slot 2i runs KV tile 2m and slot 2i + 1 KV tile 2m + 1 with the
  same Q tiles and positions; every (head, kv, q) appears once; each dQ block's
  positions are 0..N/2-1, each held by exactly one CTA pair;
- the simulator accepts the schedule, and unsupported shapes are refused.
"""
from collections import defaultdict

import pytest

from oracle import dag, schedules as sc
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


@pytest.mark.parametrize("N", [2, 4, 6, 8, 16])
def test_oracle_units(N):
    us = sc.units(sc.SHIFT_PAIRS, N, False)
    assert len(us) == N // 2
    for m, seq in enumerate(us):
        assert [kv for kv, _ in seq] == [m] * N
        assert sorted(q for _, q in seq) == list(range(N))
    for t in range(N):
        qs = [us[m][t][1] for m in range(N // 2)]
        assert len(set(qs)) == N // 2          # conflict-free step
    assert not sc.supported(sc.SHIFT_PAIRS, 5, False)
    assert not sc.supported(sc.SHIFT_PAIRS, 4, True)


@pytest.mark.parametrize("heads,N,slots", [(1, 4, 2), (3, 4, 5), (2, 8, 3), (5, 6, 7), (4, 16, 74)])
def test_half_table_equals_oracle_and_has_no_cycle(heads, N, slots):
    rows = binding.dash_sched_table(heads, N, False, "shift_pairs", slots)
    got = [[] for _ in range(slots)]
    for cta, h, kv, q, p, _ in rows:
        got[cta].append((h, kv, q, p))
    want = sc.packed_table(sc.SHIFT_PAIRS, heads, N, False, slots)
    assert got == [[e[:4] for e in slot] for slot in want]
    for chains in (1, 2):
        n, edges, _ = dag.schedule_graph(want, 1.0, 0.3, None, chains)
        assert _acyclic(n, edges)


@pytest.mark.parametrize("heads,N,ctas", [(1, 4, 4), (3, 4, 10), (2, 8, 6), (4, 16, 148)])
def test_grid_table(heads, N, ctas):
    rows = binding.dash_sched_table_pairs(heads, N, ctas)
    assert len(rows) == heads * N * N
    per_slot = defaultdict(list)
    for cta, h, kv, q, p, _ in rows:
        per_slot[cta].append((h, kv, q, p))
    for i in range(ctas // 2):
        a, b = per_slot[2 * i], per_slot[2 * i + 1]
        assert len(a) == len(b)
        for (ha, ka, qa, pa), (hb, kb, qb, pb) in zip(a, b):
            assert (ha, qa, pa) == (hb, qb, pb) and ka % 2 == 0 and kb == ka + 1
    assert sorted((h, kv, q) for _, h, kv, q, _, _ in rows) == \
        sorted((h, kv, q) for h in range(heads) for kv in range(N) for q in range(N))
    holders = defaultdict(set)
    for cta, h, kv, q, p, _ in rows:
        holders[(h, q, p)].add(cta // 2)
    for h in range(heads):
        for q in range(N):
            for p in range(N // 2):
                assert len(holders[(h, q, p)]) == 1
    assert all(p < N // 2 for _, _, _, _, p, _ in rows)


def test_simulator_and_refusals():
    cp, mk, bub, st = binding.dash_sched_simulate(4, 8, False, "shift_pairs", 3, 1.0, 0.3, 0, 2)
    assert cp > 0 and mk > 0
    with pytest.raises(binding.DashError):
        binding.dash_sched_table(2, 5, False, "shift_pairs", 2)     # odd N
    with pytest.raises(binding.DashError):
        binding.dash_sched_table(2, 4, True, "shift_pairs", 2)      # causal
    with pytest.raises(binding.DashError):
        binding.dash_sched_table_pairs(2, 4, 3)                     # odd CTA count
