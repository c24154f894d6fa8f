"""The library's schedule tables and DAG simulator against the oracle.

Tables must equal the oracle's packed tables bit for bit (integer work); the
simulator must reproduce the brute-force critical paths on tiny tables, the
closed forms on larger ones, and the zero-weight-edge lemma of DASH summary
§2.2.B through its general longest-path entry point.
"""
import random

import pytest

from oracle import dag, schedules as sc
from persistent_sm_attn_b200 import binding

SID = {sc.NAIVE_ASC: "naive_asc", sc.DESCENDING: "descending", sc.SHIFT: "shift",
       sc.SYM_SHIFT: "sym_shift"}


def _lib_table(name, heads, N, causal, ctas):
    rows = binding.dash_sched_table(heads, N, causal, SID[name], ctas)
    slots = [[] for _ in range(ctas)]
    for cta, hd, kv, q, pos, _chain in rows:
        ncontrib = q + 1 if causal else N
        slots[cta].append((hd, kv, q, pos, ncontrib))
    return slots


CASES = [(name, N, causal, heads, ctas)
         for name in sc.ALL
         for causal in (False, True)
         for N in (1, 2, 3, 4, 7, 8, 16)
         for heads, ctas in ((1, 148), (3, 5), (5, 16), (2, 7))
         if sc.supported(name, N, causal)
         and len(sc.units(name, N, causal)) <= ctas]


@pytest.mark.parametrize("name,N,causal,heads,ctas", CASES)
def test_table_equals_oracle(name, N, causal, heads, ctas):
    assert _lib_table(name, heads, N, causal, ctas) == sc.packed_table(name, heads, N, causal, ctas)


def test_full_size_tables_validate():
    # the workload shapes on a 148-SM grid
    for heads, N, causal, name in ((32, 32, False, "shift"), (32, 32, False, "descending"),
                                   (32, 32, False, "naive_asc"), (64, 64, True, "descending"),
                                   (64, 64, True, "sym_shift"), (128, 128, True, "sym_shift"),
                                   (24, 128, False, "shift")):
        rows = binding.dash_sched_table(heads, N, causal, name, 148)
        assert len(rows) == heads * (N * (N + 1) // 2 if causal else N * N)


@pytest.mark.parametrize("heads,N,causal,name,ctas,chunk", [
    (32, 32, False, "shift", 148, 4),        # parts straddle rounds (32 chains per head)
    (13, 6, False, "naive_asc", 7, 3),       # uneven last part, several rounds per CTA
    (10, 8, True, "sym_shift", 9, 4),
    (9, 5, True, "descending", 6, 2),
])
def test_table_parts_keep_every_position(heads, N, causal, name, ctas, chunk):
    """The host-buffer path launches parts of the whole table: each part holds
    exactly the whole table's rows of its heads (renumbered), with the same CTA,
    KV tile, Q tile and dQ position, in the same per-CTA order."""
    full = binding.dash_sched_table(heads, N, causal, name, ctas)
    seen = 0
    for h0 in range(0, heads, chunk):
        h1 = min(heads, h0 + chunk)
        part = binding.dash_sched_table_part(heads, N, causal, name, ctas, h0, h1)
        want = [(c, h - h0, kv, q, pos) for c, h, kv, q, pos, _ in full if h0 <= h < h1]
        assert [r[:5] for r in part] == want
        seen += len(part)
    assert seen == len(full)


def test_more_units_than_ctas_never_deadlock():
    # a shift head of 8 chains on 4 CTAs runs in two rounds; its dQ blocks
    # accumulate round by round, so the table is valid
    rows = binding.dash_sched_table(1, 8, False, "shift", 4)
    assert len(rows) == 64
    assert binding.dash_sched_check(1, 8, False, 4, rows) == 0
    # the descending order only waits on lower KV tiles
    assert len(binding.dash_sched_table(1, 8, False, "descending", 4)) == 64


def _step_ordered_shift_rows(N, ctas):
    """Shift visiting order with every dQ block accumulated in step order
    regardless of rounds: with fewer CTAs than chains a CTA of the first round
    waits for a partial that only a chain of the second round produces."""
    rows = []
    for g in range(N):  # global unit g = KV tile g of head 0
        for t in range(N):
            rows.append((g % ctas, g // ctas, g, (g + t) % N, t))
    out = []
    for c in range(ctas):
        for rnd, kv, t, q in sorted((r[1], r[2], r[4], r[3]) for r in rows if r[0] == c):
            out.append((c, 0, kv, q, t, kv))
    return out


def test_deadlock_detected():
    rows = _step_ordered_shift_rows(8, 4)
    assert binding.dash_sched_check(1, 8, False, 4, rows) == 6
    # with one CTA per chain the same order is valid
    assert binding.dash_sched_check(1, 8, False, 8, _step_ordered_shift_rows(8, 8)) == 0


def test_check_rejects_coverage_and_position_errors():
    rows = binding.dash_sched_table(1, 4, False, "shift", 4)
    assert binding.dash_sched_check(1, 4, False, 4, rows) == 0
    assert binding.dash_sched_check(1, 4, False, 4, rows[:-1]) == 6        # a pair missing
    bad = [list(r) for r in rows]
    bad[0][4], bad[1][4] = bad[1][4], bad[0][4]    # two blocks' positions swapped
    a, b = rows[0], rows[1]
    if a[3] != b[3]:
        assert binding.dash_sched_check(1, 4, False, 4, bad) == 6
    assert binding.dash_sched_check(1, 4, False, 4, [(5, 0, 0, 0, 0, 0)]) == 1   # CTA out of range


def test_check_bounds_its_scratch_by_the_rows_given():
    """A caller's table that claims a million heads of 32767 tiles is rejected by its
    pair count before any per-block scratch is sized from the claim."""
    rows = binding.dash_sched_table(1, 4, False, "shift", 4)
    assert binding.dash_sched_check(10**6, 32767, False, 4, rows) == 6
    assert binding.dash_sched_check(1, 4, False, 4, rows + rows[-1:]) == 6   # an extra pair


@pytest.mark.parametrize("name,N,causal,heads,ctas", [
    (sc.SHIFT, 3, False, 1, 3), (sc.SHIFT, 4, False, 2, 5), (sc.NAIVE_ASC, 3, False, 1, 3),
    (sc.NAIVE_ASC, 4, True, 2, 3), (sc.DESCENDING, 4, True, 1, 4), (sc.DESCENDING, 3, False, 2, 4),
    (sc.SYM_SHIFT, 4, True, 2, 3), (sc.SYM_SHIFT, 2, True, 3, 2)])
@pytest.mark.parametrize("beta", [None, 1, 2])
@pytest.mark.parametrize("chains", [1, 2])
def test_simulator_matches_bruteforce(name, N, causal, heads, ctas, beta, chains):
    c, r = 1.0, 0.35
    table = sc.packed_table(name, heads, N, causal, ctas)
    want = dag.simulate(table, c, r, beta, chains)
    got = binding.dash_sched_simulate(heads, N, causal, SID[name], ctas, c, r, beta or 0, chains)
    assert got[3] == want[3]
    for g, w in zip(got[:3], want[:3]):
        assert abs(g - w) < 1e-9


@pytest.mark.parametrize("N", [8, 16, 32, 64])
def test_simulator_closed_forms(N):
    """One head, one CTA per unit, unbounded buffers, r <= c."""
    c, r = 1.0, 0.15
    cp = lambda name, causal: binding.dash_sched_simulate(1, N, causal, name, 148, c, r, 0)[0]
    assert abs(cp("naive_asc", False) - (N * c + N * r)) < 1e-9
    assert abs(cp("shift", False) - (N * c + r)) < 1e-9
    assert abs(cp("descending", True) - (N * c + r)) < 1e-9
    assert abs(cp("sym_shift", True) - ((N + 1) * c + r)) < 1e-9


def test_predicted_ordering_on_workload_shapes():
    """The simulator's ranking of schedules on the benchmark shapes (148 CTAs,
    a partial-buffer depth of 2 as in the kernel, reduction ~ 1/4 of compute)."""
    c, r = 1.0, 0.25
    f = lambda heads, N, causal, name: binding.dash_sched_simulate(
        heads, N, causal, name, 148, c, r, 2)[0]
    # full mask: shift is never worse than the serialised orders
    assert f(32, 32, False, "shift") <= f(32, 32, False, "descending")
    assert f(32, 32, False, "shift") <= f(32, 32, False, "naive_asc")
    # causal: descending beats the ascending baseline
    assert f(64, 64, True, "descending") < f(64, 64, True, "naive_asc")


def test_longest_path_matches_bruteforce_and_lemma():
    rng = random.Random(3)
    for _ in range(150):
        n = rng.randint(2, 8)
        edges = [(u, v, float(rng.randint(0, 4))) for u in range(n) for v in range(u + 1, n)
                 if rng.random() < 0.35]
        cp, depth, height = binding.dash_dag_longest_path(n, edges)
        bcp, bdepth, bheight = dag.paths_longest(n, edges)
        assert cp == bcp and depth == bdepth and height == bheight
        for u in range(n):
            for v in range(u + 1, n):
                cp2, _, _ = binding.dash_dag_longest_path(n, edges + [(u, v, 0.0)])
                if depth[u] <= depth[v]:
                    assert cp2 == cp
                if depth[v] + height[v] == cp:
                    assert (cp2 == cp) == (depth[u] <= depth[v])


def test_table_cta_count_is_bounded():
    lib = binding.load()
    assert lib.dash_sched_table(2, 4, 0, 2, 65536, None, 0) == 32
    assert lib.dash_sched_table(2, 4, 0, 2, 65537, None, 0) == -2
    assert lib.dash_sched_table(2, 4, 0, 2, 2**31 - 1, None, 0) == -2
    assert binding.dash_sched_check(1, 4, False, 2**31 - 1, []) == 1
