"""Pins of the schedule and DAG oracles.

The schedule oracle is pinned to the sequences the pages print (golden files),
to coverage / conflict-freedom / permutation properties, and the brute-force
DAG oracle to closed forms of the critical path and to the lemma of DASH
summary §2.2.B.
"""
import itertools
import os
import random

import pytest

from oracle import dag, schedules as sc

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    units = []
    for line in open(os.path.join(GOLD, name)):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        head, rest = line.split(":", 1)
        toks = rest.split()
        if all(":" in t for t in toks):
            units.append([tuple(int(x) for x in t.split(":")) for t in toks])
        else:
            units.append([(int(head), int(t)) for t in toks])
    return units


@pytest.mark.parametrize("fname,name,causal", [
    ("shift_n4_full.txt", sc.SHIFT, False),
    ("descending_n4_full.txt", sc.DESCENDING, False),
    ("descending_n4_causal.txt", sc.DESCENDING, True),
    ("sym_shift_n4_causal.txt", sc.SYM_SHIFT, True),
])
def test_units_match_golden(fname, name, causal):
    assert sc.units(name, 4, causal) == _read_golden(fname)


def _all_cases(maxN=12):
    for N in range(1, maxN + 1):
        for causal in (False, True):
            for name in sc.ALL:
                if sc.supported(name, N, causal):
                    yield name, N, causal


@pytest.mark.parametrize("name,N,causal", list(_all_cases()))
def test_schedule_properties(name, N, causal):
    us = sc.units(name, N, causal)
    pairs = [p for u in us for p in u]
    want = {(kv, q) for kv in range(N) for q in range(N) if (q >= kv or not causal)}
    assert len(pairs) == len(want) and set(pairs) == want          # coverage, once each
    # each KV tile runs as one unbroken chain inside its unit
    for u in us:
        kvs = [kv for kv, _ in u]
        runs = [k for i, k in enumerate(kvs) if i == 0 or kvs[i - 1] != k]
        assert len(runs) == len(set(runs))
    # positions form a permutation of 0..n-1 for each dQ block
    order = sc.accumulation_order(name, N, causal)
    for q, lst in order.items():
        n = N - 0 if not causal else q + 1
        assert len(lst) == n
    tab = sc.positions(name, N, causal)
    for q in range(N):
        ps = sorted(e[2] for u in tab for e in u if e[1] == q)
        assert ps == list(range(len(ps)))
    if name in (sc.SHIFT, sc.SYM_SHIFT):
        # conflict-free: no two units touch the same dQ block at the same step
        width = max(len(u) for u in us)
        for t in range(width):
            qs = [u[t][1] for u in us if t < len(u)]
            assert len(qs) == len(set(qs))
        # the accumulation order never goes back in steps (depth-monotone)
        for q, lst in order.items():
            steps = [t for _, t in lst]
            assert steps == sorted(steps) and len(set(steps)) == len(steps)
    if name == sc.SYM_SHIFT:
        h = N // 2
        assert len(us) == h and all(len(u) == N + 1 for u in us)
        phase1 = {p for u in us for p in u[:h]}
        assert phase1 == {(kv, q) for kv in range(h) for q in range(h, N)}


def test_packed_table_round_robin():
    tab = sc.packed_table(sc.SHIFT, 3, 4, False, 5)
    assert len(tab) == 5
    # 12 units on 5 slots: slot 0 runs global units 0, 5, 10
    heads_kv = [(e[0], e[1]) for e in tab[0]]
    assert heads_kv[:4] == [(0, 0)] * 4 and heads_kv[4:8] == [(1, 1)] * 4
    assert heads_kv[8:] == [(2, 2)] * 4


# ---------------------------------------------------------------------------
# DAG oracle

def _dp_longest(n, edges):
    """Independent check used only to cross-validate the brute force on
    random graphs: Bellman-style relaxation to a fixed point."""
    d = [0.0] * n
    for _ in range(n):
        for u, v, w in edges:
            d[v] = max(d[v], d[u] + w)
    return max(d) if d else 0.0, d


def test_bruteforce_on_a_hand_graph():
    #  0 -2-> 1 -3-> 3 ;  0 -4-> 2 -0.5-> 3 ; 2 -> 1 (1.0)
    edges = [(0, 1, 2.0), (1, 3, 3.0), (0, 2, 4.0), (2, 3, 0.5), (2, 1, 1.0)]
    cp, depth, height = dag.paths_longest(4, edges)
    assert cp == 8.0 and depth == [0.0, 5.0, 4.0, 8.0] and height == [8.0, 3.0, 4.0, 0.0]


def _random_dag(rng, n, p):
    edges = []
    for u in range(n):
        for v in range(u + 1, n):
            if rng.random() < p:
                edges.append((u, v, float(rng.randint(0, 5))))
    return edges


def test_bruteforce_matches_relaxation_on_random_graphs():
    rng = random.Random(7)
    for _ in range(200):
        n = rng.randint(1, 9)
        edges = _random_dag(rng, n, 0.35)
        cp, depth, _ = dag.paths_longest(n, edges)
        cp2, d2 = _dp_longest(n, edges)
        assert cp == cp2 and depth == d2


def test_lemma_zero_weight_edge():
    """DASH summary §2.2.B: adding a zero-weight edge u -> v keeps the critical
    path iff depth(u) <= depth(v).  Exact form checked: the path is kept iff
    depth(u) + height(v) <= CP; depth(u) <= depth(v) always suffices, and is
    also necessary when v lies on a critical path."""
    rng = random.Random(11)
    checked_only_if = 0
    for _ in range(300):
        n = rng.randint(2, 9)
        edges = _random_dag(rng, n, 0.3)
        cp, depth, height = dag.paths_longest(n, edges)
        for u in range(n):
            for v in range(u + 1, n):
                cp2, _, _ = dag.paths_longest(n, edges + [(u, v, 0.0)])
                kept = cp2 == cp
                assert kept == (depth[u] + height[v] <= cp)
                if depth[u] <= depth[v]:
                    assert kept
                if depth[v] + height[v] == cp:           # v is critical
                    assert kept == (depth[u] <= depth[v])
                    checked_only_if += 1
    assert checked_only_if > 100


def _one_head(name, N, causal):
    us = sc.units(name, N, causal)
    return sc.packed_table(name, 1, N, causal, len(us))


@pytest.mark.parametrize("N", [1, 2, 3, 4])
def test_dag_closed_forms(N):
    c, r = 1.0, 0.15
    cp, *_ = dag.simulate(_one_head(sc.NAIVE_ASC, N, False), c, r, None)
    assert abs(cp - (N * c + N * r)) < 1e-12
    cp, *_ = dag.simulate(_one_head(sc.SHIFT, N, False), c, r, None)
    assert abs(cp - (N * c + r)) < 1e-12
    cp, *_ = dag.simulate(_one_head(sc.DESCENDING, N, True), c, r, None)
    assert abs(cp - (N * c + r)) < 1e-12
    if N % 2 == 0:
        cp, *_ = dag.simulate(_one_head(sc.SYM_SHIFT, N, True), c, r, None)
        assert abs(cp - ((N + 1) * c + r)) < 1e-12


def test_shift_is_optimal_over_all_visiting_orders():
    """DASH summary §2.2.B calls shift scheduling optimal for full masks.  For N
    = 3, try every visiting order of every chain, with each dQ block
    accumulating in (step, kv) order, and compare with the shift's CP."""
    N, c, r = 3, 1.0, 0.3
    best = None
    for orders in itertools.product(itertools.permutations(range(N)), repeat=N):
        units = [[(k, q) for q in orders[k]] for k in range(N)]
        rank = {}
        for q in range(N):
            lst = sorted((t, k) for k in range(N) for t, (_, qq) in enumerate(units[k]) if qq == q)
            for p, (t, k) in enumerate(lst):
                rank[(k, t)] = p
        table = [[(0, kv, q, rank[(k, t)], N) for t, (kv, q) in enumerate(units[k])]
                 for k in range(N)]
        cp, *_ = dag.simulate(table, c, r, None)
        best = cp if best is None else min(best, cp)
    shift_cp, *_ = dag.simulate(_one_head(sc.SHIFT, N, False), c, r, None)
    assert abs(shift_cp - best) < 1e-12 and abs(best - (N * c + r)) < 1e-12


def test_buffer_depth_one_serialises_naive_order():
    """With one dQ buffer per slot a chain waits for its own reduction; the
    naive ascending order then stalls, the shift order does not."""
    N, c, r = 4, 1.0, 0.4
    _, _, _, st_naive = dag.simulate(_one_head(sc.NAIVE_ASC, N, False), c, r, 1)
    _, _, _, st_shift = dag.simulate(_one_head(sc.SHIFT, N, False), c, r, 1)
    assert st_naive > 0 and st_shift == 0


# ---------------------------------------------------------------------------
# Pins of the multi-chain accumulation order, the simulator's other outputs and
# the multi-round positions

def _closed_form(name, causal, N, c, r, chains):
    """Critical path of one head, one CTA slot per unit, unbounded buffers,
    r <= c / 2, derived by hand from the event graph's arcs:

    * shift (full) and symmetric shift (causal): each reduction starts when its
      own partial is ready, so the path is the longest chain plus one
      reduction, N c + r and (N + 1) c + r, for any number of chains.
    * descending, causal: every contributor of block q arrives at step N-1-q
      (positions ascend in KV), the reductions of block q queue behind each
      other, and block 0 (one contributor, last step) ends the path: N c + r.
    * naive ascending (both masks) and descending (full): the reductions of the
      last block queue at the end.  One chain: N c + N r.  Two chains: the
      block's positions split into even and odd runs of ceil(N/2) and
      floor(N/2) reductions; the last position waits for the other run, so
      the path holds floor(N/2) + 1 reductions after N c.
    """
    if name == sc.SYM_SHIFT:
        return (N + 1) * c + r
    if name == sc.SHIFT or (name == sc.DESCENDING and causal):
        return N * c + r
    return N * c + (N * r if chains == 1 else (N // 2 + 1) * r)


def _closed_forms_hold(chains_list=(1, 2)):
    for c, r in ((1.0, 0.15), (1.0, 0.4)):
        for N in range(1, 7):
            for name in sc.ALL:
                for causal in (False, True):
                    if not sc.supported(name, N, causal):
                        continue
                    tab = _one_head(name, N, causal)
                    for K in chains_list:
                        cp, makespan, bubble, stalls = dag.simulate(tab, c, r, None, K)
                        L = max(len(u) for u in tab)
                        if abs(cp - _closed_form(name, causal, N, c, r, K)) > 1e-9:
                            return False
                        # unbounded buffers: compute never waits, and each slot
                        # idles for the critical path minus its own compute
                        if stalls != 0 or abs(makespan - L * c) > 1e-9:
                            return False
                        want_bubble = sum(cp - c * len(u) for u in tab if u)
                        if abs(bubble - want_bubble) > 1e-9:
                            return False
    return True


def test_dag_closed_forms_one_and_two_chains():
    assert _closed_forms_hold()


# Hand-worked: naive ascending, full mask, N = 2, c = 1, r = 1.5, one dQ buffer
# per slot (beta = 1), two accumulation chains.  Slot k holds KV tile k and
# visits Q tiles 0, 1; its pairs have position k in both blocks.  Position 0
# has no predecessor; position 1 is the last of its block and waits for
# position 0 (the other chain's last).  Event times (a, b, s, d):
#   slot 0, q0: a 0, b 1, s 1, d 2.5
#   slot 0, q1: a 1, b max(2, d_prev 2.5) = 2.5 (stall), s 2.5, d 4
#   slot 1, q0: a 0, b 1, s max(1, d(slot 0, q0) 2.5) = 2.5, d 4
#   slot 1, q1: a 1, b max(2, d_prev 4) = 4 (stall), s max(4, 4, d(slot 0, q1) 4) = 4, d 5.5
# critical path 5.5; makespan (last compute end) max(2.5, 4) = 4;
# bubble (5.5 - 2) + (5.5 - 2) = 7; stalls 2.
HAND_NAIVE_N2 = ((1.0, 1.5, 1, 2), (5.5, 4.0, 7.0, 2))
# Hand-worked: naive ascending, full mask, N = 3, c = 1, r = 0.4, beta = 1, two
# chains.  Positions 0 and 1 start their reductions as soon as their partials
# are ready: d = t + 1.4 at step t.  Position 2 (last) waits for positions 0
# and 1: s = t + 1.4, d = t + 1.8; its own previous reduction (d = t + 0.8) never
# holds up its next partial (b = t + 1), so nothing stalls.
# critical path 3.8; makespan 3; bubble 3 x (3.8 - 3) = 2.4; stalls 0.
HAND_NAIVE_N3 = ((1.0, 0.4, 1, 2), (3.8, 3.0, 2.4, 0))


def _hand_tables_hold():
    for N, ((c, r, beta, K), want) in ((2, HAND_NAIVE_N2), (3, HAND_NAIVE_N3)):
        got = dag.simulate(_one_head(sc.NAIVE_ASC, N, False), c, r, beta, K)
        if any(abs(g - w) > 1e-9 for g, w in zip(got, want)):
            return False
    return True


def test_dag_hand_worked_tables():
    assert _hand_tables_hold()


@pytest.mark.parametrize("mutant", ["chain_pred_is_p_minus_1", "last_skips_other_chain",
                                    "last_waits_only_first", "no_chain_pred"])
def test_dag_pins_reject_planted_order_mistakes(monkeypatch, mutant):
    """Each plausible mistake in the accumulation-order rule must fail a pin."""
    real = dag.order_preds

    def m_p1(p, nc, K):          # waits for the position one ahead, not K ahead
        return ([p - 1] if p >= 1 else []) + \
            ([q for q in range(max(0, p - K + 1), p) if q != p - 1] if p == nc - 1 else [])

    def m_last(p, nc, K):        # the last contributor forgets the other chains
        return [p - K] if p >= K else []

    def m_first(p, nc, K):       # the last contributor waits for position 0 only
        return ([p - K] if p >= K else []) + ([0] if p == nc - 1 and p > 0 else [])

    def m_none(p, nc, K):        # no order within a chain
        return list(range(max(0, p - K + 1), p)) if p == nc - 1 else []

    fn = {"chain_pred_is_p_minus_1": m_p1, "last_skips_other_chain": m_last,
          "last_waits_only_first": m_first, "no_chain_pred": m_none}[mutant]
    assert real(5, 6, 2) == [3, 4]
    monkeypatch.setattr(dag, "order_preds", fn)
    assert not (_closed_forms_hold() and _hand_tables_hold())


def _read_positions(name):
    slots = []
    for line in open(os.path.join(GOLD, name)):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        _, rest = line.split(":", 1)
        slots.append([tuple(int(x) for x in t.split(":")) for t in rest.split()])
    return slots


@pytest.mark.parametrize("fname,name,heads,N,causal,slots", [
    ("shift_n4_3slots_positions.txt", sc.SHIFT, 1, 4, False, 3),
    ("sym_shift_n4_2heads_3slots_positions.txt", sc.SYM_SHIFT, 2, 4, True, 3),
])
def test_multi_round_positions_match_golden(fname, name, heads, N, causal, slots):
    """Units that run in a later round come after every unit of an earlier
    round in each dQ block's order (hand-worked tables)."""
    got = sc.packed_table(name, heads, N, causal, slots)
    want = _read_positions(fname)
    assert [[e[:4] for e in s] for s in got] == want
    for s in got:
        for hd, kv, q, pos, nc in s:
            assert nc == (q + 1 if causal else N)
