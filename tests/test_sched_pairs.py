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


def test_oracle_units_small_case_by_hand():
    # N = 4: KV pairs 0 and 1; pair m starts at Q tile m and shifts by one per step
    assert sc.units(sc.SHIFT_PAIRS, 4, False) == [
        [(0, 0), (0, 1), (0, 2), (0, 3)],
        [(1, 1), (1, 2), (1, 3), (1, 0)]]
    # one round: each block's two contributions in step order.  Block q meets pair 0 at
    # step q and pair 1 at step q - 1 mod 4, so pair 1 comes first except at block 0.
    order = sc.accumulation_order(sc.SHIFT_PAIRS, 4, False)
    assert order == {0: [(0, 0), (1, 3)], 1: [(1, 0), (0, 1)], 2: [(1, 1), (0, 2)],
                     3: [(1, 2), (0, 3)]}


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
    rows = binding.dash_sched_table_pairs(heads, N, False, ctas)
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
        binding.dash_sched_table_pairs(2, 4, False, 3)              # odd CTA count


# ---------------------------------------------------------------- causal CTA pairs
# DASH_SCHED_SYM_SHIFT_PAIRS: the symmetric shift over N/2 x N/2 pair-tiles (KV pair m,
# Q pair j, present when j >= m), each pair-tile run as Q tile 2j then 2j + 1.

@pytest.mark.parametrize("N", [4, 8, 12, 16, 32])
def test_oracle_units_causal(N):
    us = sc.units(sc.SYM_SHIFT_PAIRS, N, True)
    assert len(us) == N // 4
    visits = defaultdict(list)
    for seq in us:
        assert len(seq) == N + 2                       # N/2 + 1 pair-tiles, two steps each
        for t, (m, q) in enumerate(seq):
            visits[m].append(q)
            assert q >= 2 * m                          # never a pair-tile above the diagonal
            if t % 2 == 1:                             # a pair-tile's steps: 2j, then 2j + 1
                assert seq[t - 1] == (m, q - 1) and q % 2 == 1
    # every KV pair visits its Q tiles 2m .. N-1 exactly once
    assert sorted(visits) == list(range(N // 2))
    for m, qs in visits.items():
        assert sorted(qs) == list(range(2 * m, N))
    # conflict-free: the units' Q tiles at one step are distinct
    for t in range(N + 2):
        qs = [seq[t][1] for seq in us]
        assert len(set(qs)) == len(qs)
    order = sc.accumulation_order(sc.SYM_SHIFT_PAIRS, N, True)
    assert {q: len(v) for q, v in order.items()} == {q: q // 2 + 1 for q in range(N)}
    assert not sc.supported(sc.SYM_SHIFT_PAIRS, 6, True)      # N not a multiple of 4
    assert not sc.supported(sc.SYM_SHIFT_PAIRS, 8, False)     # full mask


def test_oracle_units_causal_small_case_by_hand():
    # N = 4: one unit, KV pairs 0 and 1.  The half-size symmetric shift (2 x 2 pair-tiles)
    # runs the dense pair-tile (0, 1), then the diagonal pair-tile (0, 0), then (1, 1).
    assert sc.units(sc.SYM_SHIFT_PAIRS, 4, True) == [
        [(0, 2), (0, 3), (0, 0), (0, 1), (1, 2), (1, 3)]]
    # blocks 0 and 1 hear from KV pair 0 only; blocks 2 and 3 from pair 0 (steps 0, 1)
    # and then pair 1 (steps 4, 5)
    assert sc.accumulation_order(sc.SYM_SHIFT_PAIRS, 4, True) == {
        0: [(0, 2)], 1: [(0, 3)], 2: [(0, 0), (0, 4)], 3: [(0, 1), (0, 5)]}


@pytest.mark.parametrize("heads,N,slots", [(1, 4, 1), (3, 4, 2), (2, 8, 3), (5, 12, 7),
                                           (4, 16, 74), (2, 32, 5)])
def test_half_table_causal_equals_oracle_and_has_no_cycle(heads, N, slots):
    rows = binding.dash_sched_table(heads, N, True, "sym_shift_pairs", slots)
    got = [[] for _ in range(slots)]
    for cta, h, kv, q, p, _ in rows:
        got[cta].append((h, kv, q, p))
    want = sc.packed_table(sc.SYM_SHIFT_PAIRS, heads, N, True, slots)
    assert got == [[e[:4] for e in slot] for slot in want]
    for chains in (1, 2):
        n, edges, _ = dag.schedule_graph(want, 1.0, 0.3, None, chains)
        assert _acyclic(n, edges)


@pytest.mark.parametrize("heads,N,ctas", [(1, 4, 2), (3, 8, 10), (2, 16, 6), (4, 32, 148)])
def test_grid_table_causal(heads, N, ctas):
    rows = binding.dash_sched_table_pairs(heads, N, True, ctas)
    per_slot = defaultdict(list)
    for cta, h, kv, q, p, _ in rows:
        per_slot[cta].append((h, kv, q, p))
    for i in range(ctas // 2):
        a, b = per_slot[2 * i], per_slot[2 * i + 1]
        assert len(a) == len(b)
        for (ha, ka, qa, pa), (hb, kb, qb, pb) in zip(a, b):
            assert (ha, qa, pa) == (hb, qb, pb) and ka % 2 == 0 and kb == ka + 1
    # the causal pairs, plus one step above the diagonal per diagonal pair-tile
    got = sorted((h, kv, q) for _, h, kv, q, _, _ in rows)
    want = sorted([(h, kv, q) for h in range(heads) for kv in range(N) for q in range(kv, N)] +
                  [(h, 2 * m + 1, 2 * m) for h in range(heads) for m in range(N // 2)])
    assert got == want
    holders = defaultdict(set)
    for cta, h, kv, q, p, _ in rows:
        holders[(h, q, p)].add(cta // 2)
    for h in range(heads):
        for q in range(N):
            for p in range(q // 2 + 1):
                assert len(holders[(h, q, p)]) == 1
    assert all(p <= q // 2 for _, _, _, q, p, _ in rows)


def test_simulator_and_refusals_causal():
    cp, mk, bub, st = binding.dash_sched_simulate(4, 8, True, "sym_shift_pairs", 3, 1.0, 0.3, 0, 2)
    assert cp > 0 and mk > 0
    with pytest.raises(binding.DashError):
        binding.dash_sched_table(2, 6, True, "sym_shift_pairs", 2)      # N not a multiple of 4
    with pytest.raises(binding.DashError):
        binding.dash_sched_table(2, 8, False, "sym_shift_pairs", 2)     # full mask
    with pytest.raises(binding.DashError):
        binding.dash_sched_table_pairs(2, 6, True, 4)                   # N not a multiple of 4
    with pytest.raises(binding.DashError):
        binding.dash_sched_table_pairs(2, 8, 2, 4)                      # causal not 0 / 1
