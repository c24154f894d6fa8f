"""Grouped-query schedule tables (dash_sched_table_gqa).

With a group of g query heads per K/V head, a CTA runs each KV segment of a unit
for the g query heads in turn, so the dK/dV tile of that segment stays on one SM
for the whole group.  These tests check, without a GPU:
- group 1 gives the multi-head table;
- every (query head, kv, q) pair of the mask appears once, and every dQ block's
  positions are 0..n-1;
- each K/V head's KV tile is one run of consecutive chains on one CTA, the group's
  query heads in order, each with the multi-head unit's Q tiles for that segment;
- the table's dependence graph (the oracle's event graph, two accumulation
  chains per block as the kernel runs it) has no cycle, so no CTA waits forever;
- the library's own validator accepts the rows.
"""
from collections import defaultdict

import pytest

from oracle import dag, schedules as sc
from persistent_sm_attn_b200 import binding

SID = {sc.NAIVE_ASC: "naive_asc", sc.DESCENDING: "descending", sc.SHIFT: "shift",
       sc.SYM_SHIFT: "sym_shift"}


def _mask_pairs(N, causal):
    return [(kv, q) for kv in range(N) for q in range(N) if not causal or q >= kv]


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


@pytest.mark.parametrize("name,N,causal,heads,ctas", [
    (sc.SHIFT, 4, False, 3, 5), (sc.NAIVE_ASC, 3, True, 2, 7), (sc.DESCENDING, 5, True, 4, 6),
    (sc.SYM_SHIFT, 4, True, 3, 4), (sc.SHIFT, 32, False, 32, 148)])
def test_group_one_is_the_multi_head_table(name, N, causal, heads, ctas):
    assert (binding.dash_sched_table_gqa(heads, 1, N, causal, SID[name], ctas)
            == binding.dash_sched_table(heads, N, causal, SID[name], ctas))


GQA_CASES = [(name, N, causal, heads, group, ctas)
             for name in sc.ALL
             for causal in (False, True)
             for N, heads, group, ctas in ((4, 4, 2, 3), (6, 8, 4, 5), (4, 6, 2, 16),
                                           (8, 4, 4, 2), (2, 2, 2, 1), (8, 16, 8, 148))
             if sc.supported(name, N, causal)]


@pytest.mark.parametrize("name,N,causal,heads,group,ctas", GQA_CASES)
def test_grouped_table_invariants(name, N, causal, heads, group, ctas):
    rows = binding.dash_sched_table_gqa(heads, group, N, causal, SID[name], ctas)
    # coverage: each pair of every query head once
    got = sorted((h, kv, q) for _, h, kv, q, _, _ in rows)
    assert got == sorted((h, kv, q) for h in range(heads) for kv, q in _mask_pairs(N, causal))
    # positions of each dQ block are a permutation of its contributors
    pos = defaultdict(list)
    for _, h, kv, q, p, _ in rows:
        pos[(h, q)].append(p)
    for (h, q), ps in pos.items():
        assert sorted(ps) == list(range(q + 1 if causal else N))
    # chains: consecutive rows of one chain index; runs of one (K/V head, kv) per CTA
    chains = []  # (cta, chain, head, kv, [q...]) in table order
    for cta, h, kv, q, _, ci in rows:
        if not chains or chains[-1][1] != ci:
            chains.append((cta, ci, h, kv, []))
        chains[-1][4].append(q)
    runs = []
    for c in chains:
        cta, _, h, kv, qs = c
        if runs and runs[-1][0] == cta and runs[-1][1] == h // group and runs[-1][2] == kv:
            runs[-1][3].append((h, qs))
        else:
            runs.append((cta, h // group, kv, [(h, qs)]))
    keys = [(r[1], r[2]) for r in runs]
    assert len(keys) == len(set(keys)) == (heads // group) * N   # one run per KV tile
    mha = {}
    for slot in sc.packed_table(name, 1, N, causal, len(sc.units(name, N, causal))):
        for _, kv, q, _, _ in slot:
            mha.setdefault(kv, []).append(q)
    for _, kvh, kv, members in runs:
        assert [h for h, _ in members] == [kvh * group + i for i in range(group)]
        for _, qs in members:
            assert qs == mha[kv]        # the multi-head unit's Q tiles of that segment
    # no dependence cycle (two accumulation chains per block, as the kernel runs)
    slots = [[] for _ in range(ctas)]
    for cta, h, kv, q, p, _ in rows:
        slots[cta].append((h, kv, q, p, q + 1 if causal else N))
    for chains_per_block in (1, 2):
        n, edges, _ = dag.schedule_graph(slots, 1.0, 0.3, None, chains_per_block)
        assert _acyclic(n, edges)
    assert binding.dash_sched_check(heads, N, causal, ctas, rows) == 0


def test_grouped_tables_at_workload_shapes_validate():
    # 32 query heads over 8 K/V heads (B=2 H=16 at S=4096 full; B=2 H=32 at S=8192 causal)
    for heads, group, N, causal, name in ((32, 4, 32, False, "shift"),
                                          (32, 4, 32, False, "descending"),
                                          (64, 8, 64, True, "sym_shift"),
                                          (64, 2, 64, True, "descending")):
        rows = binding.dash_sched_table_gqa(heads, group, N, causal, name, 148)
        assert len(rows) == heads * (N * (N + 1) // 2 if causal else N * N)


def test_grouped_table_argument_errors():
    with pytest.raises(binding.DashError):
        binding.dash_sched_table_gqa(6, 4, 4, False, "shift", 4)     # 4 does not divide 6
    with pytest.raises(binding.DashError):
        binding.dash_sched_table_gqa(4, 0, 4, False, "shift", 4)


@pytest.mark.parametrize("name,N,causal,heads,group,ctas", [
    (sc.SHIFT, 3, False, 2, 2, 3), (sc.SHIFT, 2, False, 4, 2, 3), (sc.NAIVE_ASC, 3, True, 2, 2, 2),
    (sc.DESCENDING, 3, True, 2, 2, 2), (sc.DESCENDING, 2, False, 4, 4, 3),
    (sc.SYM_SHIFT, 2, True, 4, 2, 3),
    (sc.SYM_SHIFT, 4, True, 2, 2, 2)])
@pytest.mark.parametrize("beta", [None, 1, 2])
@pytest.mark.parametrize("chains", [1, 2])
def test_grouped_simulator_matches_bruteforce(name, N, causal, heads, group, ctas, beta, chains):
    c, r = 1.0, 0.35
    rows = binding.dash_sched_table_gqa(heads, group, N, causal, SID[name], ctas)
    slots = [[] for _ in range(ctas)]
    for cta, h, kv, q, p, _ in rows:
        slots[cta].append((h, kv, q, p, q + 1 if causal else N))
    want = dag.simulate(slots, c, r, beta, chains)
    got = binding.dash_sched_simulate_gqa(heads, group, N, causal, SID[name], ctas, c, r,
                                          0 if beta is None else beta, chains)
    assert got[0] == pytest.approx(want[0], abs=1e-9)
    assert got[1] == pytest.approx(want[1], abs=1e-9)
    assert got[2] == pytest.approx(want[2], abs=1e-9)
    assert got[3] == want[3]


def test_grouped_simulator_group_one_is_multi_head():
    for name, N, causal in (("shift", 8, False), ("sym_shift", 8, True), ("descending", 6, True)):
        assert (binding.dash_sched_simulate_gqa(12, 1, N, causal, name, 20, 1.0, 0.8, 2, 2)
                == binding.dash_sched_simulate(12, N, causal, name, 20, 1.0, 0.8, 2, 2))


@pytest.mark.parametrize("kv_heads,group,N", [(1, 4, 8), (3, 2, 16), (2, 8, 5)])
def test_grouped_shift_closed_form(kv_heads, group, N):
    """Full-mask shift with every unit in one round and r <= c: each dQ block's
    contributors arrive one step apart, so nothing waits, and the last reduction
    ends at g*N*c + r (g*N pairs per CTA)."""
    c, r = 1.0, 0.6
    ctas = kv_heads * N
    cp, mk, bt, st = binding.dash_sched_simulate_gqa(kv_heads * group, group, N, False, "shift",
                                                     ctas, c, r, 0, 1)
    assert cp == pytest.approx(group * N * c + r)
    assert mk == pytest.approx(group * N * c)
    assert bt == pytest.approx(ctas * r)
    assert st == 0


def test_grouped_simulator_argument_errors():
    for args in ((6, 4), (4, 0)):
        with pytest.raises(binding.DashError):
            binding.dash_sched_simulate_gqa(args[0], args[1], 4, False, "shift", 4, 1.0, 0.5)


def test_units_longer_than_two_to_the_sixteen_steps():
    """512 query heads on one K/V head at N = 128, causal symmetric shift: each grouped
    unit runs 512 * 129 pairs, more than a 16-bit step field holds.  The table still
    builds and passes validation (positions, runs, deadlock)."""
    lib = binding.load()
    assert lib.dash_sched_table_gqa(512, 512, 128, 1, 3, 148, None, 0) == 512 * 128 * 129 // 2


def test_tables_beyond_int32_pairs_are_refused_before_building():
    lib = binding.load()
    # 256 heads x 4096^2 pairs > 2^31 - 1: refused as unsupported, without building
    assert lib.dash_sched_table_gqa(256, 1, 4096, 0, 2, 148, None, 0) == -2
    assert lib.dash_sched_table(256, 4096, 0, 2, 148, None, 0) == -2


# ---------------------------------------------------------------------------
# Split groups: each K/V head's group of g query heads cut into `split` sub-groups
# of g / split consecutive heads, each a unit of its own (the table of g / split
# query heads per virtual K/V head).  Sub-group s adds its dK/dV partials of a KV
# tile after sub-group s - 1 has added its own.

@pytest.mark.parametrize("name,N,causal,heads,group,split,ctas", [
    (sc.SHIFT, 4, False, 8, 4, 2, 3), (sc.SHIFT, 4, False, 8, 4, 4, 5),
    (sc.DESCENDING, 3, True, 4, 4, 2, 2), (sc.NAIVE_ASC, 5, True, 8, 8, 4, 7),
    (sc.SYM_SHIFT, 4, True, 8, 2, 2, 4), (sc.SYM_SHIFT, 6, True, 16, 8, 8, 9),
    (sc.SHIFT, 8, False, 16, 8, 4, 148), (sc.DESCENDING, 6, False, 4, 4, 4, 1)])
def test_split_group_table(name, N, causal, heads, group, split, ctas):
    """The virtual table of a split group: each (K/V head, KV tile) is one run per
    sub-group, its g / split query heads in order; and every wait (the dQ tickets with
    one or two chains per block, and sub-group s's dK/dV epilogue after s - 1's) points
    back in the grid's execution order, so no CTA waits forever."""
    sub = group // split
    rows = binding.dash_sched_table_gqa(heads, sub, N, causal, SID[name], ctas)
    slots = [[] for _ in range(ctas)]
    for cta, h, kv, q, p, _ in rows:
        slots[cta].append((h, kv, q, p, q + 1 if causal else N))
    for chains in (1, 2):
        n, edges, index = dag.schedule_graph(slots, 1.0, 0.3, None, chains)
        # a run's epilogue follows its last reduction and precedes the CTA's next one
        epi = {}
        for sl, seq in enumerate(slots):
            for i, (h, kv, _, _, _) in enumerate(seq):
                nxt = seq[i + 1] if i + 1 < len(seq) else None
                if nxt is not None and nxt[0] // sub == h // sub and nxt[1] == kv:
                    continue
                epi[(h // group, kv, (h // sub) % split)] = n
                edges.append((index[(sl, i)] + 3, n, 0.0))
                if nxt is not None:
                    edges.append((n, index[(sl, i + 1)] + 2, 0.0))
                n += 1
        for (kvh, kv, s), e in epi.items():
            if s > 0:
                edges.append((epi[(kvh, kv, s - 1)], e, 0.0))
        assert _acyclic(n, edges)
        assert len(epi) == (heads // group) * N * split
    runs = defaultdict(list)   # (K/V head, kv, sub-group) -> query heads, per chain
    prev = None
    for cta, h, kv, q, p, ci in rows:
        if ci != prev:
            runs[(h // group, kv, (h // sub) % split)].append((cta, h))
            prev = ci
    assert sorted(runs) == sorted((kvh, kv, s) for kvh in range(heads // group)
                                  for kv in range(N) for s in range(split))
    for (kvh, kv, s), members in runs.items():
        assert len({c for c, _ in members}) == 1          # one CTA
        assert [h for _, h in members] == [kvh * group + s * sub + i for i in range(sub)]


def test_split_choice():
    """dash_bwd_gqa_split_for: among the splits whose units fill the grid's rounds
    within 2 points of the best, the one closest to two query heads per run
    (hand-counted)."""
    f = binding.dash_bwd_gqa_split_for
    # 1 K/V head of 8, shift at S = 4096 (32 units per sub-group) on 148 CTAs:
    # 32/148, 64/148, 128/148, 256/296 -> splits 4 and 8 fill best; 4 runs two heads
    assert f(148, 1, 1, 8, 4096, False, "shift") == 4
    # 4 K/V heads of 8, shift at S = 4096: 128/148, 256/296, 512/592 (0.865),
    # 1024/1036 (0.988) -> only 8 fills best
    assert f(148, 2, 2, 8, 4096, False, "shift") == 8
    # 8 K/V heads of 8: 256/296, 512/592 (0.865), 1024/1036, 2048/2072 (0.988) -> 4
    assert f(148, 1, 8, 8, 4096, False, "shift") == 4
    # 4 K/V heads x 37 units (shift at S = 4736) fill every round at every split -> 4
    assert f(148, 1, 4, 8, 4736, False, "shift") == 4
    # 16 K/V heads of 8, sym_shift causal S = 16384 (64 units): 1024/1036 and up, all
    # 0.988 -> 4
    assert f(148, 4, 4, 8, 16384, True, "sym_shift") == 4
    # 2 K/V heads of 4, sym_shift causal S = 8192 (32 units): 64/148, 128/148,
    # 256/296 -> splits 2 and 4 fill best; 2 runs two heads
    assert f(148, 1, 2, 4, 8192, True, "sym_shift") == 2
    # 1 K/V head of 2, naive_asc at S = 16384: 128/148, 256/296 -> 1 (two heads a run)
    assert f(148, 1, 1, 2, 16384, False, "naive_asc") == 1
    assert f(148, 4, 8, 1, 4096, False, "shift") == 1      # no group to split
    assert f(1, 1, 1, 16, 1024, True, "descending") == 8   # one CTA: always full
    for bad in ((0, 1, 1, 2, 1024, False, "shift"), (148, 1, 1, 3, 1024, False, "shift"),
                (148, 0, 1, 2, 1024, False, "shift")):
        with pytest.raises(binding.DashError):
            f(*bad)
    with pytest.raises(binding.DashError):
        f(148, 1, 1, 2, 1000, False, "shift")               # not a multiple of 128
    with pytest.raises(binding.DashError):
        f(148, 1, 1, 2, 1024, True, "shift")                # shift needs the full mask


def test_split_argument_errors_before_the_device():
    """A bad split is refused before any device call (dummy pointers, no GPU)."""
    import ctypes
    lib = binding.load()
    buf = ctypes.create_string_buffer(64)
    al = ctypes.c_void_p((ctypes.addressof(buf) + 15) // 16 * 16)
    for split in (-1, 3, 8, 16):   # group 4: 3 not a power of two, 8 and 16 do not divide
        rc = lib.dash_attn_bwd_gqa_split(*([al] * 9), 1, 8, 2, 256, 64, 0, 2, split, None)
        assert rc == 1, split      # DASH_ERR_INVALID_ARG
