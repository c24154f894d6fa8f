// Host-side DASH schedule tables, their validator and the DAG simulator.
//
// A table tells each CTA of the persistent backward kernel which chains it
// runs and, for every (KV tile, Q tile) pair of a chain, the Q tile and the
// pair's position in that dQ block's fixed accumulation order.
//
// Source: "Resumen Técnico: DASH – Programación de Atención Determinista ...",
// §2.1 (DAG formulation, one KV tile per SM as an unbroken chain) and §2.2
// (descending Q-tile iteration, shift and symmetric shift scheduling).
#pragma once
#include <cstdint>
#include <string>
#include <vector>

namespace dash {

enum Schedule { NAIVE_ASC = 0, DESCENDING = 1, SHIFT = 2, SYM_SHIFT = 3, ATOMIC = 4,
                SHIFT_PAIRS = 5, SYM_SHIFT_PAIRS = 6 };

// The CTA-pair schedules, whose tables are built as half tables (one unit per KV pair).
inline bool pair_schedule(int s) { return s == SHIFT_PAIRS || s == SYM_SHIFT_PAIRS; }

// Upper bound on a table's CTA count (the kernel's grid is the SM count times the CTAs
// resident per SM); larger requests are refused instead of sizing per-CTA lists by them.
constexpr int kMaxTableCtas = 65536;

struct Chain {           // one KV tile of one head, run back to back on one CTA
  int32_t bh;            // b * H + h
  int32_t kv;            // KV tile index
  int32_t pair_off;      // first entry in Table::pairs
  int32_t pair_cnt;      // number of pairs (Q tiles) of this chain
};

// Packed pair word: bits [0,16) Q tile, bits [16,32) position in the dQ order.
inline uint32_t pack_pair(int q, int pos) { return uint32_t(q) | (uint32_t(pos) << 16); }
inline int pair_q(uint32_t w) { return int(w & 0xffffu); }
inline int pair_pos(uint32_t w) { return int(w >> 16); }

struct Table {
  int n_heads = 0, N = 0, causal = 0, schedule = 0, num_ctas = 0;
  int group = 1;  // query heads per K/V head (grouped-query attention); 1 = one K/V head each
  // KV units per head when a unit stands for a pair of KV tiles (SHIFT_PAIRS' half table:
  // N / 2, unit m = KV tiles 2m and 2m + 1); 0: one KV tile per unit, N of them
  int kv_units = 0;
  std::vector<int32_t> cta_off;   // num_ctas + 1 offsets into chains
  std::vector<Chain> chains;      // grouped by CTA, in execution order
  std::vector<uint32_t> pairs;    // packed (q, position)
  long long n_pairs() const { return (long long)pairs.size(); }
};

// True when the pages define `schedule` for this mask and tile count.
bool schedule_supported(int schedule, int N, int causal);

// Units of one head: each a list of (kv, q) in visiting order.
std::vector<std::vector<std::pair<int, int>>> head_units(int schedule, int N, int causal);

// SYM_SHIFT_PAIRS (causal, N a multiple of 4): the same pairing under the causal mask.
// KV pair m and Q pair j (Q tiles 2j, 2j + 1) form a pair-tile, visible when j >= m; the
// half table runs SYM_SHIFT over N / 2 pair-tiles, each pair-tile as two steps (Q tiles 2j
// then 2j + 1).  On the diagonal pair-tile the odd KV tile's first step (KV 2m + 1, Q 2m)
// is fully masked: it contributes zeros, so that both CTAs keep the same steps.  A dQ
// block q receives q / 2 + 1 pre-summed contributions.
// SHIFT_PAIRS (full mask, N even): CTA pairs (2i, 2i + 1) run KV tiles 2m and 2m + 1 of
// a head over the same Q tiles at the same steps, m + t mod N at step t, and pre-sum
// their two dQ partials before the ordered accumulation, so a dQ block receives N / 2
// (pre-summed) contributions, in (round, step) order.  build_table_grouped builds the
// half table (one unit per KV pair, num_ctas / 2 slots, kv = m); expand_pair_table
// turns it into the grid's table, slot 2i running KV tile 2m and slot 2i + 1 KV tile
// 2m + 1 with the same Q tiles and positions.
// (A half table built with several heads per unit, build_table_grouped's group, expands
// the same way: each CTA's chains keep the half table's head order.)
bool expand_pair_table(const Table& half, Table* out);

// Query heads per unit of a multi-head launch's table.  With il > 1 the launch uses
// build_table_grouped(n_heads, il, ...) although every head has K/V of its own: each KV
// segment of a unit runs for il heads in turn (K/V loaded again for each), which
// spaces successive contributions to a dQ block further apart in the persistent
// grid's steps.  mode 0: the measured choice (2 for symmetric shift at D = 64 when
// the units still fill the grid's rounds within 2 points, else 1); mode 1: 1; mode 2
// or 4: that many where it divides n_heads, else 1.
int head_interleave(int D, int schedule, int n_heads, int N, int causal, int num_ctas, int mode);

// Build the whole-grid table: heads in order, unit g on CTA g mod num_ctas in
// round g / num_ctas; step-ordered schedules accumulate each dQ block in
// (round, step) order.
// Returns false (with a message) if the combination is unsupported.
bool build_table(int n_heads, int N, int causal, int schedule, int num_ctas, Table* out,
                 std::string* err);

// The same for grouped-query attention: n_heads query heads, `group` of them per
// K/V head (n_heads a multiple of group).  A unit covers one K/V head's KV tile (or
// tiles) for all its query heads: each KV segment of the unit runs for every query
// head of the group in turn, so the chains that feed one dK/dV tile run back to back
// on one CTA and the kernel carries the accumulators across them.  Positions follow
// the same keys (round, then step within the unit); group = 1 gives build_table's
// table.
bool build_table_grouped(int n_heads, int group, int N, int causal, int schedule,
                         int num_ctas, Table* out, std::string* err);

// Checks coverage (every allowed pair once), positions (a permutation per dQ
// block), unbroken chains, pair-word ranges, and deadlock freedom of the
// ticket order when all num_ctas CTAs run concurrently and each CTA performs
// its reductions in table order.  Returns false with a message on failure.
bool validate_table(const Table& t, std::string* err);

// The part of `full` that covers heads [h0, h1), renumbered to heads 0..h1-h0-1.
// Every chain keeps its CTA, its place among that CTA's chains, and its pairs'
// positions, so a launch over the part performs each dQ block's additions in
// the same order as a launch over the whole table.  Returns false if the range
// is empty or outside the table.
bool split_table(const Table& full, int h0, int h1, Table* out);

// Longest path of a general DAG (Kahn order).  Returns false on a cycle.
bool dag_longest_path(int n_nodes, int n_edges, const int* src, const int* dst,
                      const double* w, double* depth, double* height, double* cp);

struct SimResult {
  double critical_path = 0, makespan = 0, bubble_time = 0;
  long long stalls = 0;
};

// Event-graph simulation of a table: per pair, events a (start), b (partial
// ready), s (reduction start), d (reduction done); arcs a->b weight c,
// b->s 0, s->d weight r, b(prev on slot)->a 0, d(prev on slot)->s 0 (one
// reducer per CTA), with beta >= 1 buffers d(pair n-beta on slot)->b(pair n)
// (beta <= 0 = unbounded), and the accumulation order: with `chains`
// accumulators per dQ block, d(position p - chains)->s(p), and for the block's
// last contributor d(last position of every other chain)->s.  chains = 1 is
// the single fixed order.
bool simulate_table(const Table& t, double c, double r, int beta, int chains, SimResult* res,
                    std::string* err);

// A table given as rows of six ints {cta, bh, kv, q, position, chain id}, the
// format dash_sched_table writes: rows grouped by CTA in ascending order, each
// CTA's rows in execution order, consecutive rows of one chain sharing the
// chain id.  Only the shape is checked here; validate_table checks the rest.
bool table_from_rows(int n_heads, int N, int causal, int num_ctas, const int* rows,
                     long long n_rows, Table* out, std::string* err);

// Failure-detection testing: moves every partial of dQ block (head 0, Q tile 0)
// two positions later, so the block's first two positions (the first of each
// of its two accumulation chains) never arrive and the waits on them run out.
// Every index stays in range; the table no longer passes validate_table.
void plant_missing_first_partials(Table* t);

}  // namespace dash
