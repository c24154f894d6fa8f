"""Brute-force oracle of the DASH scheduling DAG (tiny sizes only).

Test infrastructure only (see the package docstring).

DASH summary §2.1 models the deterministic backward as a DAG whose nodes are
tile-compute phases and reduction phases, whose edges are data dependencies and
the mandatory accumulation order, and whose objective is the critical-path
length; all work of one KV tile forms an unbroken chain on one SM.  The pages
give no weights or event granularity.  The reading used here (activity on arcs,
four events per pair x = (kv, q)):

  a(x) -> b(x)  weight c   tile compute (the five products and the softmax)
  b(x) -> s(x)  weight 0   the partial is ready before its reduction starts
  d(y) -> s(x)  weight 0   accumulation order: y is x's predecessor in its dQ block
  s(x) -> d(x)  weight r   the reduction of the partial into the block
  b(x_n) -> a(x_n+1)  0    next pair on the same CTA slot (chain / resource order)
  d(x_n) -> s(x_n+1)  0    one reduction at a time per slot (the SM's reducer)
  d(x_n+1-beta) -> b(x_n+1)  0   at most beta partials in flight per slot

With K accumulation chains per dQ block (the block's positions split by
position mod K, each residue class accumulating into an accumulator of its
own in position order, and the last contributor adding the K sums), the
predecessor of position p is position p - K, and the block's last contributor
also waits for the last position of every other chain.  K = 1 is the single
fixed order of the pages.

The times of events are their longest-path depths from time 0.  This module
finds them by enumerating every path explicitly, with no dynamic programming,
so it only serves tiny graphs and checks the simulator built into the product
library.
"""
from __future__ import annotations

import math


def paths_longest(n_nodes: int, edges):
    """Longest path by explicit enumeration of every path.

    edges: list of (u, v, w).  Returns (cp, depth, height): cp is the longest
    path over the whole graph, depth[x] the longest path ending at x, height[x]
    the longest path starting at x (both 0 for isolated nodes).
    """
    out = [[] for _ in range(n_nodes)]
    indeg = [0] * n_nodes
    for u, v, w in edges:
        out[u].append((v, w))
        indeg[v] += 1
    depth = [0.0] * n_nodes
    height = [0.0] * n_nodes
    cp = 0.0

    def walk(path, length):
        nonlocal cp
        x = path[-1]
        depth[x] = max(depth[x], length)
        cp = max(cp, length)
        if not out[x]:
            # a maximal path: credit every node on it with its remaining length
            acc = 0.0
            for i in range(len(path) - 1, -1, -1):
                height[path[i]] = max(height[path[i]], acc)
                if i:
                    acc += _w(path[i - 1], path[i])
            return
        for v, w in out[x]:
            path.append(v)
            walk(path, length + w)
            path.pop()

    wmap = {}
    for u, v, w in edges:
        wmap[(u, v)] = max(wmap.get((u, v), -math.inf), w)

    def _w(u, v):
        return wmap[(u, v)]

    for s in range(n_nodes):
        if indeg[s] == 0:
            walk([s], 0.0)
    return cp, depth, height


def order_preds(p: int, nc: int, chains: int):
    """Positions whose reductions must be done before position p of a dQ block
    with nc contributors starts its own (the accumulation-order arcs).

    Position p adds into chain p mod K after position p - K of the same chain.
    The block's last position also waits for the last position of every other
    chain, since it adds their sums (those are positions nc-K .. nc-2)."""
    preds = [p - chains] if p >= chains else []
    if p == nc - 1:
        preds += list(range(max(0, p - chains + 1), p))
    return preds


def schedule_graph(table, c: float, r: float, beta: int | None, chains: int = 1):
    """Build the event graph of a packed schedule table.

    table: per slot, a list of (head, kv, q, position, n_contributors) as
    returned by ``oracle.schedules.packed_table``.  beta: dQ partial buffers
    per slot, None for unbounded.  chains: accumulation chains per dQ block.
    Returns (n_nodes, edges, index) where index[(slot, n)] = node id of event
    a of the n-th pair on that slot (b, s, d follow as +1, +2, +3).
    """
    index = {}
    nid = 0
    for sl, seq in enumerate(table):
        for n in range(len(seq)):
            index[(sl, n)] = nid
            nid += 4
    by_block = {}
    for sl, seq in enumerate(table):
        for n, (hd, kv, q, p, nc) in enumerate(seq):
            by_block[(hd, q, p)] = index[(sl, n)]
    edges = []
    for sl, seq in enumerate(table):
        for n, (hd, kv, q, p, nc) in enumerate(seq):
            a = index[(sl, n)]
            edges += [(a, a + 1, c), (a + 1, a + 2, 0.0), (a + 2, a + 3, r)]
            for pp in order_preds(p, nc, chains):
                edges.append((by_block[(hd, q, pp)] + 3, a + 2, 0.0))
            if n > 0:
                prev = index[(sl, n - 1)]
                edges.append((prev + 1, a, 0.0))
                edges.append((prev + 3, a + 2, 0.0))
                if beta is not None and n - beta >= 0:
                    edges.append((index[(sl, n - beta)] + 3, a + 1, 0.0))
    return nid, edges, index


def simulate(table, c: float, r: float, beta: int | None, chains: int = 1):
    """Critical path, compute makespan, idle (bubble) time and stall count of
    a schedule table, all by brute-force path enumeration.

    critical_path: latest event time (the last reduction done).
    makespan:      latest end of a compute phase over all slots.
    bubble_time:   sum over used slots of (critical_path - that slot's compute).
    stalls:        pairs whose partial-ready event waits on a full buffer.
    """
    n, edges, index = schedule_graph(table, c, r, beta, chains)
    cp, depth, _ = paths_longest(n, edges)
    makespan = 0.0
    bubble = 0.0
    stalls = 0
    for sl, seq in enumerate(table):
        if not seq:
            continue
        for k in range(len(seq)):
            a = index[(sl, k)]
            if depth[a + 1] > depth[a] + c + 1e-12 * max(1.0, abs(depth[a])):
                stalls += 1
        makespan = max(makespan, depth[index[(sl, len(seq) - 1)] + 1])
        bubble += cp - c * len(seq)
    return cp, makespan, bubble, stalls
