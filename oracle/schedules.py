"""Oracle of the DASH tile schedules: visiting order and dQ accumulation order.

Test infrastructure only (see the package docstring).

Vocabulary.  A head has N = S/128 key/value (KV) tiles and N query (Q) tiles.
A *pair* (kv, q) is the work of one KV tile against one Q tile; with a causal
mask only pairs with q >= kv exist.  DASH summary §2.1 requires that all pairs of
one KV tile run back to back on one SM (a *chain*), with dK/dV held on chip.  A
*unit* is the work one CTA slot does for one head: one chain, or for the
symmetric shift two chains.  Step t of a unit is its t-th pair.  Each Q tile's
dQ block receives one partial per contributing KV tile; the *position* of a
pair is the index of its partial in that block's fixed accumulation order.

Schedules (names follow the pages):

* ``naive_asc``  -- the serialised deterministic baseline of DASH summary §1:
  every chain visits Q tiles ascending, and each dQ block accumulates its
  partials in ascending KV order.
* ``descending`` -- DASH summary §2.2.A: Q tiles visited from the last to the
  first ("N to 0" on the page, read as N-1 down to 0 for N tiles numbered from
  0).  The page does not change the accumulation order, so it stays ascending
  in KV.
* ``shift``      -- DASH summary §2.2.B, full masks: the SM holding KV tile k
  visits k, k+1, ..., N-1, 0, ..., k-1 (the page prints this sequence; with one
  KV tile per SM it is read as the sequence of Q tiles, i.e. dQ blocks, that
  chain visits).  Each dQ block accumulates in step order.
* ``shift_pairs`` -- the shift order for CTA pairs that pre-sum dQ (the "2-CTA
  pairs" the pages' register-pressure remark in DASH summary §4 points to; the
  pages print no such schedule, so this is this library's construction): unit m
  stands for KV tiles 2m and 2m+1, run by two CTAs over the same Q tiles at the
  same steps, m + t mod N at step t, so each step touches N/2 distinct dQ blocks.
  A dQ block then receives N/2 pre-summed contributions, accumulated in step
  order.  Full mask, even N.
* ``sym_shift``  -- DASH summary §2.2.B, causal masks: KV tiles k and N-1-k are
  paired (one CTA serves both, one after the other) so the triangle of causal
  pairs folds into an N/2 x (N+1) rectangle, run in two phases: the dense
  lower-left rectangle (Q in [N/2, N) x KV in [0, N/2)) and then the folded
  upper triangle.  Accumulation follows (phase, step).  Requires even N.
* ``sym_shift_pairs`` -- the CTA pairs of ``shift_pairs`` under the causal mask
  (this library's construction, like ``shift_pairs``): KV pair m (KV tiles 2m,
  2m+1) against Q pair j (Q tiles 2j, 2j+1) is a pair-tile, present when
  j >= m; ``sym_shift`` runs over the N/2 x N/2 pair-tiles, and each visited
  pair-tile becomes two steps, Q tile 2j and then 2j+1.  A unit stands for KV
  pairs, written as m; Q tile q >= 2m is visited by KV pair m, so dQ block q
  receives q//2 + 1 pre-summed contributions, in (round, step) order.  On a
  diagonal pair-tile the step (KV 2m+1, Q 2m) lies above the diagonal and adds
  nothing.  Causal mask, N a multiple of 4.
"""
from __future__ import annotations

NAIVE_ASC, DESCENDING, SHIFT, SYM_SHIFT = "naive_asc", "descending", "shift", "sym_shift"
ALL = (NAIVE_ASC, DESCENDING, SHIFT, SYM_SHIFT)
# units stand for KV pairs; not in ALL (their units differ in kind)
SHIFT_PAIRS, SYM_SHIFT_PAIRS = "shift_pairs", "sym_shift_pairs"


def supported(name: str, N: int, causal: bool) -> bool:
    """Which (schedule, mask) combinations the pages define."""
    if name == SHIFT:
        return not causal
    if name == SYM_SHIFT:
        return causal and N % 2 == 0
    if name == SHIFT_PAIRS:
        return not causal and N % 2 == 0
    if name == SYM_SHIFT_PAIRS:
        return causal and N % 4 == 0
    return name in (NAIVE_ASC, DESCENDING)


def units(name: str, N: int, causal: bool):
    """Per-head units: a list, one entry per CTA slot of the head, each a list
    of (kv, q) pairs in visiting order."""
    if not supported(name, N, causal):
        raise ValueError(f"schedule {name} undefined for N={N} causal={causal}")
    out = []
    if name == NAIVE_ASC:
        for k in range(N):
            qs = range(k, N) if causal else range(N)
            out.append([(k, q) for q in qs])
    elif name == DESCENDING:
        for k in range(N):
            lo = k if causal else 0
            out.append([(k, q) for q in range(N - 1, lo - 1, -1)])
    elif name == SHIFT:
        for k in range(N):
            out.append([(k, (k + t) % N) for t in range(N)])
    elif name == SHIFT_PAIRS:
        # unit m: the KV pair (2m, 2m+1), written as m
        for m in range(N // 2):
            out.append([(m, (m + t) % N) for t in range(N)])
    elif name == SYM_SHIFT_PAIRS:
        # pair-tile (m, j) of the half-size symmetric shift -> steps (m, 2j), (m, 2j+1)
        for seq in units(SYM_SHIFT, N // 2, True):
            out.append([(m, 2 * j + b) for (m, j) in seq for b in (0, 1)])
    elif name == SYM_SHIFT:
        h = N // 2
        for k in range(h):
            seq = []
            # phase 1: dense lower-left rectangle Q in [h, N) x KV in [0, h)
            for t in range(h):
                seq.append((k, h + (k + t) % h))
            # phase 2: upper-left triangle of KV k, folded with the
            # 180-degree-rotated lower-right triangle of KV N-1-k
            for t in range(h):
                r = (k + t) % h
                seq.append((k, r) if r >= k else (N - 1 - k, N - 1 - r))
            seq.append((N - 1 - k, N - 1 - k))  # the shared diagonal, last
            out.append(seq)
    return out


def accumulation_order(name: str, N: int, causal: bool, rounds=None):
    """dQ accumulation order per block: dict q -> list of (unit, step), first
    partial first.

    rounds[u] is the round in which unit u of the head runs (all 0 when every
    unit of the head has a CTA slot of its own).  For the step-ordered
    schedules a block accumulates in execution order: by round, then by step
    within the round.  The pages only treat one unit per SM; taking the round
    first is the plainest extension when a head has more units than slots or
    straddles two rounds, and it keeps every wait pointing to an earlier
    (round, step), so no table deadlocks.
    """
    us = units(name, N, causal)
    if rounds is None:
        rounds = [0] * len(us)
    contrib = {q: [] for q in range(N)}
    for u, seq in enumerate(us):
        for t, (kv, q) in enumerate(seq):
            contrib[q].append((u, t, kv))
    order = {}
    for q, lst in contrib.items():
        if name in (NAIVE_ASC, DESCENDING):
            lst = sorted(lst, key=lambda e: e[2])                 # ascending KV
        else:
            lst = sorted(lst, key=lambda e: (rounds[e[0]], e[1]))  # (round, step)
        order[q] = [(u, t) for (u, t, _kv) in lst]
    return order


def positions(name: str, N: int, causal: bool, rounds=None):
    """Per-head table: list per unit of (kv, q, position, n_contributors)."""
    us = units(name, N, causal)
    order = accumulation_order(name, N, causal, rounds)
    pos = {}
    for q, lst in order.items():
        for p, ut in enumerate(lst):
            pos[ut] = (p, len(lst))
    return [[(kv, q) + pos[(u, t)] for t, (kv, q) in enumerate(seq)]
            for u, seq in enumerate(us)]


def packed_table(name: str, n_heads: int, N: int, causal: bool, num_slots: int):
    """Whole-grid table: per CTA slot, the list of (head, kv, q, position,
    n_contributors) it runs, in order.

    Heads are taken in order, each head's units in consecutive global unit
    numbers; global unit g runs on slot g mod num_slots, in round g div
    num_slots.  (The pages only say that later heads follow; this static
    round-robin packing is the plainest reading.)
    """
    U = len(units(name, N, causal))
    slots = [[] for _ in range(num_slots)]
    for hd in range(n_heads):
        rounds = [(hd * U + k) // num_slots for k in range(U)]
        per_head = positions(name, N, causal, rounds)
        for k in range(U):
            g = hd * U + k
            slots[g % num_slots].extend((hd,) + e for e in per_head[k])
    return slots
