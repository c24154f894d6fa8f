// DASH schedule tables, validator and DAG simulator (host C++).
//
// Schedules follow "Resumen Técnico: DASH – Programación de Atención
// Determinista ..." §2.2:
//   NAIVE_ASC   serialised baseline of §1: Q tiles ascending, dQ order by KV.
//   DESCENDING  §2.2.A: Q tiles from the last to the first, dQ order by KV.
//   SHIFT       §2.2.B full masks: the chain of KV tile k visits Q tiles
//               k, k+1, ..., N-1, 0, ..., k-1; dQ blocks accumulate in
//               execution order (round, then step), so every step touches N
//               distinct blocks.
//   SYM_SHIFT   §2.2.B causal masks: KV tiles k and N-1-k share one CTA; a
//               dense phase over Q in [N/2, N) x KV in [0, N/2) is followed by
//               the folded triangle; dQ blocks accumulate in (phase, step)
//               order.  Needs even N.
//   ATOMIC      the unordered comparison variant: SHIFT's visiting order for
//               full masks, SYM_SHIFT's for causal masks (NAIVE_ASC for odd
//               N); positions are unused.
#include "sched.h"

#include <algorithm>
#include <climits>
#include <cmath>
#include <cstdio>
#include <deque>
#include <map>
#include <queue>

namespace dash {

bool schedule_supported(int schedule, int N, int causal) {
  if (N < 1 || N > 32767) return false;
  switch (schedule) {
    case NAIVE_ASC:
    case DESCENDING:
    case ATOMIC: return true;
    case SHIFT: return !causal;
    case SYM_SHIFT: return causal && (N % 2 == 0);
    case SHIFT_PAIRS: return !causal && (N % 2 == 0);
    case SYM_SHIFT_PAIRS: return causal && (N % 4 == 0);
    default: return false;
  }
}

using Units = std::vector<std::vector<std::pair<int, int>>>;

static Units units_of(int schedule, int N, int causal) {
  Units u;
  if (schedule == ATOMIC) {
    if (!causal) schedule = SHIFT;
    else schedule = (N % 2 == 0) ? SYM_SHIFT : NAIVE_ASC;
  }
  switch (schedule) {
    case NAIVE_ASC:
      for (int k = 0; k < N; ++k) {
        std::vector<std::pair<int, int>> seq;
        for (int q = causal ? k : 0; q < N; ++q) seq.push_back({k, q});
        u.push_back(seq);
      }
      break;
    case DESCENDING:
      for (int k = 0; k < N; ++k) {
        std::vector<std::pair<int, int>> seq;
        for (int q = N - 1; q >= (causal ? k : 0); --q) seq.push_back({k, q});
        u.push_back(seq);
      }
      break;
    case SHIFT:
      for (int k = 0; k < N; ++k) {
        std::vector<std::pair<int, int>> seq;
        for (int t = 0; t < N; ++t) seq.push_back({k, (k + t) % N});
        u.push_back(seq);
      }
      break;
    case SHIFT_PAIRS:
      // unit m: the pair of KV tiles 2m, 2m + 1 (written as m), Q tiles m + t mod N
      for (int m = 0; m < N / 2; ++m) {
        std::vector<std::pair<int, int>> seq;
        for (int t = 0; t < N; ++t) seq.push_back({m, (m + t) % N});
        u.push_back(seq);
      }
      break;
    case SYM_SHIFT_PAIRS: {
      // SYM_SHIFT over the N / 2 pair-tiles; each visited (KV pair, Q pair) becomes the two
      // steps of its Q tiles, in order
      const Units half = units_of(SYM_SHIFT, N / 2, 1);
      for (const auto& hs : half) {
        std::vector<std::pair<int, int>> seq;
        for (const auto& e : hs) {
          seq.push_back({e.first, 2 * e.second});
          seq.push_back({e.first, 2 * e.second + 1});
        }
        u.push_back(seq);
      }
      break;
    }
    case SYM_SHIFT: {
      const int h = N / 2;
      for (int k = 0; k < h; ++k) {
        std::vector<std::pair<int, int>> seq;
        for (int t = 0; t < h; ++t) seq.push_back({k, h + (k + t) % h});       // dense phase
        for (int t = 0; t < h; ++t) {                                            // folded phase
          const int r = (k + t) % h;
          if (r >= k) seq.push_back({k, r});
          else seq.push_back({N - 1 - k, N - 1 - r});
        }
        seq.push_back({N - 1 - k, N - 1 - k});                                   // shared diagonal
        u.push_back(seq);
      }
      break;
    }
    default: break;
  }
  return u;
}

std::vector<std::vector<std::pair<int, int>>> head_units(int schedule, int N, int causal) {
  return units_of(schedule, N, causal);
}

bool build_table(int n_heads, int N, int causal, int schedule, int num_ctas, Table* out,
                 std::string* err) {
  return build_table_grouped(n_heads, 1, N, causal, schedule, num_ctas, out, err);
}

int head_interleave(int D, int schedule, int n_heads, int N, int causal, int num_ctas, int mode) {
  if (n_heads < 1 || num_ctas < 1 || N < 1) return 1;
  if (mode == 2 || mode == 4) return n_heads % mode == 0 ? mode : 1;
  if (mode != 0 || D != 64 || schedule != SYM_SHIFT || n_heads % 2 != 0 ||
      !schedule_supported(schedule, N, causal))
    return 1;
  const long long per_head = (long long)units_of(schedule, N, causal).size();
  auto fill = [&](int il) {
    const long long u = (long long)(n_heads / il) * per_head;
    const long long rounds = (u + num_ctas - 1) / num_ctas;
    return (double)u / (double)(rounds * num_ctas);
  };
  return fill(2) >= fill(1) - 0.02 ? 2 : 1;
}

bool build_table_grouped(int n_heads, int group, int N, int causal, int schedule,
                         int num_ctas, Table* out, std::string* err) {
  if (n_heads < 1 || num_ctas < 1 || num_ctas > kMaxTableCtas || group < 1 ||
      n_heads % group != 0 || !schedule_supported(schedule, N, causal)) {
    if (err) *err = "schedule not defined for this mask / tile count / head grouping";
    return false;
  }
  // Chain offsets into the pair list are int32, and a grouped unit's step must fit the
  // 24 bits the position keys below give it: refuse larger problems before building.
  const long long per_head = causal ? (long long)N * (N + 1) / 2 : (long long)N * N;
  if ((long long)n_heads * per_head > INT32_MAX || (long long)group * (N + 1) >= (1LL << 24)) {
    if (err) *err = "table too large (more than 2^31 - 1 pairs, or 2^24 steps in a unit)";
    return false;
  }
  const Units units = units_of(schedule, N, causal);
  const int U = (int)units.size();
  // Group unit k: unit k's KV segments in order, each run for query heads 0..group-1
  // of the K/V head in turn.  Entries (query head offset, kv, q) in execution order.
  struct Step { int head, kv, q; };
  std::vector<std::vector<Step>> gunits(U);
  for (int k = 0; k < U; ++k) {
    const auto& seq = units[k];
    for (int a = 0; a < (int)seq.size();) {
      int b = a;
      while (b < (int)seq.size() && seq[b].first == seq[a].first) ++b;
      for (int h = 0; h < group; ++h)
        for (int i = a; i < b; ++i) gunits[k].push_back({h, seq[i].first, seq[i].second});
      a = b;
    }
  }
  // Positions within each dQ block, per query head.  NAIVE_ASC / DESCENDING order a
  // block by KV; SHIFT / SYM_SHIFT / ATOMIC by execution order: the round in which
  // the unit runs (global unit g runs in round g / num_ctas), then the step within
  // the unit.  The round only matters for K/V heads whose units span two rounds;
  // K/V heads with the same first-unit offset in their round share one table.
  const bool by_kv = (schedule == NAIVE_ASC || schedule == DESCENDING);
  auto head_positions = [&](long long first_g) {
    // per (query head offset, q): (key, (unit, step)); keys are distinct within a block
    // (by KV tile, or by round, step and unit, with step < 2^24 and unit < 2^16)
    std::vector<std::vector<std::pair<long long, std::pair<int, int>>>> contrib(
        (size_t)group * N);
    for (int k = 0; k < U; ++k) {
      const long long rnd = (first_g + k) / num_ctas - first_g / num_ctas;
      for (int t = 0; t < (int)gunits[k].size(); ++t) {
        const Step& st = gunits[k][t];
        const long long key = by_kv ? st.kv : (rnd << 40) + (long long)t * 65536 + k;
        contrib[(size_t)st.head * N + st.q].push_back({key, {k, t}});
      }
    }
    std::vector<std::vector<int>> pos(U);
    for (int k = 0; k < U; ++k) pos[k].assign(gunits[k].size(), -1);
    for (auto& c : contrib) {
      std::sort(c.begin(), c.end());
      for (int p = 0; p < (int)c.size(); ++p) pos[c[p].second.first][c[p].second.second] = p;
    }
    return pos;
  };
  std::map<long long, std::vector<std::vector<int>>> pos_by_offset;
  auto positions_of = [&](int kvh) -> const std::vector<std::vector<int>>& {
    const long long first_g = (long long)kvh * U;
    const long long key = by_kv ? 0 : first_g % num_ctas;
    auto f = pos_by_offset.find(key);
    if (f == pos_by_offset.end()) f = pos_by_offset.emplace(key, head_positions(first_g)).first;
    return f->second;
  };
  Table t;
  t.n_heads = n_heads; t.N = N; t.causal = causal; t.schedule = schedule; t.num_ctas = num_ctas;
  t.group = group;
  if (pair_schedule(schedule)) t.kv_units = N / 2;
  // per CTA, the global units it runs, in round order
  std::vector<std::vector<long long>> per_cta(num_ctas);
  const long long total_units = (long long)(n_heads / group) * U;
  for (long long g = 0; g < total_units; ++g) per_cta[g % num_ctas].push_back(g);
  t.cta_off.assign(num_ctas + 1, 0);
  for (int c = 0; c < num_ctas; ++c) {
    t.cta_off[c] = (int32_t)t.chains.size();
    for (long long g : per_cta[c]) {
      const int kvh = (int)(g / U), k = (int)(g % U);
      const auto& seq = gunits[k];
      const auto& pos = positions_of(kvh);
      for (int i = 0; i < (int)seq.size(); ++i) {
        const int bh = kvh * group + seq[i].head;
        if (i == 0 || seq[i].kv != seq[i - 1].kv || seq[i].head != seq[i - 1].head) {
          Chain ch{bh, seq[i].kv, (int32_t)t.pairs.size(), 0};
          t.chains.push_back(ch);
        }
        t.chains.back().pair_cnt++;
        t.pairs.push_back(pack_pair(seq[i].q, pos[k][i]));
      }
    }
  }
  t.cta_off[num_ctas] = (int32_t)t.chains.size();
  *out = std::move(t);
  return true;
}

bool table_from_rows(int n_heads, int N, int causal, int num_ctas, const int* rows,
                     long long n_rows, Table* out, std::string* err) {
  auto fail = [&](const char* m) { if (err) *err = m; return false; };
  if (n_heads < 1 || N < 1 || N > 32767 || num_ctas < 1 || num_ctas > kMaxTableCtas ||
      n_rows < 0 || (n_rows > 0 && !rows))
    return fail("bad table shape");
  Table t;
  t.n_heads = n_heads; t.N = N; t.causal = causal; t.schedule = NAIVE_ASC; t.num_ctas = num_ctas;
  t.cta_off.assign(num_ctas + 1, 0);
  int prev_cta = 0, prev_chain = -1;
  for (long long i = 0; i < n_rows; ++i) {
    const int* r = rows + 6 * i;
    const int cta = r[0], bh = r[1], kv = r[2], q = r[3], pos = r[4], chain = r[5];
    if (cta < prev_cta || cta >= num_ctas) return fail("rows not grouped by CTA in order");
    if (q < 0 || q >= N || pos < 0 || pos >= N) return fail("q tile or position out of range");
    if (t.chains.empty() || cta != prev_cta || chain != prev_chain) {
      for (int c = prev_cta + 1; c <= cta; ++c) t.cta_off[c] = (int32_t)t.chains.size();
      t.chains.push_back(Chain{bh, kv, (int32_t)t.pairs.size(), 0});
    } else if (t.chains.back().bh != bh || t.chains.back().kv != kv) {
      return fail("a chain changes head or KV tile");
    }
    t.chains.back().pair_cnt++;
    t.pairs.push_back(pack_pair(q, pos));
    prev_cta = cta;
    prev_chain = chain;
  }
  for (int c = prev_cta + 1; c <= num_ctas; ++c) t.cta_off[c] = (int32_t)t.chains.size();
  *out = std::move(t);
  return true;
}

bool split_table(const Table& full, int h0, int h1, Table* out) {
  if (h0 < 0 || h1 <= h0 || h1 > full.n_heads) return false;
  if (h0 % full.group != 0 || h1 % full.group != 0) return false;  // whole K/V heads only
  Table t;
  t.n_heads = h1 - h0;
  t.N = full.N;
  t.causal = full.causal;
  t.schedule = full.schedule;
  t.num_ctas = full.num_ctas;
  t.group = full.group;
  t.kv_units = full.kv_units;
  t.cta_off.assign(full.num_ctas + 1, 0);
  for (int c = 0; c < full.num_ctas; ++c) {
    for (int i = full.cta_off[c]; i < full.cta_off[c + 1]; ++i) {
      const Chain& ch = full.chains[i];
      if (ch.bh < h0 || ch.bh >= h1) continue;
      Chain n = ch;
      n.bh = ch.bh - h0;
      n.pair_off = (int32_t)t.pairs.size();
      t.pairs.insert(t.pairs.end(), full.pairs.begin() + ch.pair_off,
                     full.pairs.begin() + ch.pair_off + ch.pair_cnt);
      t.chains.push_back(n);
    }
    t.cta_off[c + 1] = (int32_t)t.chains.size();
  }
  *out = std::move(t);
  return true;
}

bool validate_table(const Table& t, std::string* err) {
  auto fail = [&](const char* m) { if (err) *err = m; return false; };
  const int N = t.N;
  if (t.n_heads < 1 || N < 1 || N > 32767 || t.num_ctas < 1) return fail("bad table shape");
  if ((int)t.cta_off.size() != t.num_ctas + 1 || t.cta_off[0] != 0 ||
      t.cta_off[t.num_ctas] != (long long)t.chains.size())
    return fail("bad cta offsets");
  // the pair count is fixed by the mask; checking it first bounds the scratch below by
  // the table's own size, whatever n_heads a caller-supplied table claims
  // KV units per head: N, or N / 2 KV pairs for a pair schedule's half table
  const int kvn = t.kv_units > 0 ? t.kv_units : N;
  const bool half = t.kv_units > 0;  // a pair schedule's half table: kv is a KV pair
  if (kvn > N || (half && (!pair_schedule(t.schedule) || 2 * kvn != N ||
                           t.causal != (t.schedule == SYM_SHIFT_PAIRS))))
    return fail("bad KV unit count");
  // pairs per head: causal half tables hold Q tiles 2m .. N-1 for KV pair m
  const long long per_head = !t.causal ? (long long)kvn * N
                             : half    ? (long long)kvn * N - (long long)kvn * (kvn - 1)
                                       : (long long)N * (N + 1) / 2;
  if ((long long)t.n_pairs() != (long long)t.n_heads * per_head)
    return fail("table has missing or extra pairs");
  const long long nblk = (long long)t.n_heads * N;
  std::vector<uint8_t> seen((size_t)nblk * N, 0);       // (bh, kv, q)
  std::vector<uint8_t> chain_seen((size_t)nblk, 0);     // (bh, kv)
  std::vector<int> n_contrib(nblk, 0);
  std::vector<uint8_t> pos_seen((size_t)nblk * N, 0);   // (bh, q, pos)
  for (int c = 0; c < t.num_ctas; ++c) {
    if (t.cta_off[c] > t.cta_off[c + 1]) return fail("cta offsets not monotone");
    for (int ci = t.cta_off[c]; ci < t.cta_off[c + 1]; ++ci) {
      const Chain& ch = t.chains[ci];
      if (ch.bh < 0 || ch.bh >= t.n_heads || ch.kv < 0 || ch.kv >= kvn || ch.pair_cnt < 1)
        return fail("chain out of range");
      if (ch.pair_off < 0 || (long long)ch.pair_off + ch.pair_cnt > t.n_pairs())
        return fail("chain pair range out of bounds");
      uint8_t& cs = chain_seen[(size_t)ch.bh * N + ch.kv];
      if (cs) return fail("KV tile split over two chains");
      cs = 1;
      for (int i = 0; i < ch.pair_cnt; ++i) {
        const uint32_t w = t.pairs[ch.pair_off + i];
        const int q = pair_q(w), p = pair_pos(w);
        if (q < 0 || q >= N) return fail("q tile out of range");
        if (t.causal && q < (half ? 2 * ch.kv : ch.kv)) return fail("pair above the causal diagonal");
        uint8_t& s = seen[((size_t)ch.bh * N + ch.kv) * N + q];
        if (s) return fail("pair visited twice");
        s = 1;
        const long long blk = (long long)ch.bh * N + q;
        if (p < 0 || p >= N) return fail("position out of range");
        uint8_t& ps = pos_seen[(size_t)blk * N + p];
        if (ps) return fail("position used twice in a dQ block");
        ps = 1;
        n_contrib[blk]++;
      }
    }
  }
  if (t.group < 1 || t.n_heads % t.group != 0) return fail("bad head grouping");
  if (t.group > 1) {
    // the chains of one dK/dV tile (K/V head, KV tile) must run back to back on one CTA
    std::vector<uint8_t> run_done((size_t)(t.n_heads / t.group) * N, 0);
    for (int c = 0; c < t.num_ctas; ++c)
      for (int ci = t.cta_off[c]; ci < t.cta_off[c + 1]; ++ci) {
        const Chain& ch = t.chains[ci];
        const size_t key = (size_t)(ch.bh / t.group) * N + ch.kv;
        const bool cont = ci > t.cta_off[c] && t.chains[ci - 1].bh / t.group == ch.bh / t.group &&
                          t.chains[ci - 1].kv == ch.kv;
        if (!cont) {
          if (run_done[key]) return fail("chains of one dK/dV tile split into two runs");
          run_done[key] = 1;
        }
      }
  }
  for (long long blk = 0; blk < nblk; ++blk) {
    const int q = (int)(blk % N);
    const int want = t.causal ? (half ? q / 2 + 1 : q + 1) : kvn;
    if (n_contrib[blk] != want) return fail("dQ block has missing or extra contributors");
    for (int p = 0; p < want; ++p)
      if (!pos_seen[(size_t)blk * N + p]) return fail("positions are not a permutation");
  }
  if (t.schedule == ATOMIC) return true;  // no ordering to deadlock on
  // Deadlock freedom: every CTA reduces its pairs in table order and waits for
  // the block's ticket to equal the pair's position.
  std::vector<int> ticket(nblk, 0);
  std::vector<long long> next(t.num_ctas), end(t.num_ctas);
  std::vector<std::vector<int>> waiters(nblk);
  // flatten each CTA's pairs as (chain index, pair index) via a cursor
  std::vector<int> cur_chain(t.num_ctas), cur_pair(t.num_ctas);
  for (int c = 0; c < t.num_ctas; ++c) { cur_chain[c] = t.cta_off[c]; cur_pair[c] = 0; }
  std::deque<int> work;
  for (int c = 0; c < t.num_ctas; ++c) work.push_back(c);
  long long done = 0;
  while (!work.empty()) {
    const int c = work.front();
    work.pop_front();
    while (cur_chain[c] < t.cta_off[c + 1]) {
      const Chain& ch = t.chains[cur_chain[c]];
      const uint32_t w = t.pairs[ch.pair_off + cur_pair[c]];
      const long long blk = (long long)ch.bh * N + pair_q(w);
      if (ticket[blk] != pair_pos(w)) { waiters[blk].push_back(c); break; }
      ticket[blk]++;
      ++done;
      for (int wc : waiters[blk]) work.push_back(wc);
      waiters[blk].clear();
      if (++cur_pair[c] == ch.pair_cnt) { cur_pair[c] = 0; ++cur_chain[c]; }
    }
  }
  if (done != t.n_pairs()) return fail("ticket order deadlocks with this many CTAs");
  return true;
}

bool dag_longest_path(int n, int m, const int* src, const int* dst, const double* w,
                      double* depth, double* height, double* cp) {
  std::vector<int> indeg(n, 0), head(n + 1, 0), order;
  for (int e = 0; e < m; ++e) {
    if (src[e] < 0 || src[e] >= n || dst[e] < 0 || dst[e] >= n) return false;
    indeg[dst[e]]++;
    head[src[e] + 1]++;
  }
  for (int i = 0; i < n; ++i) head[i + 1] += head[i];
  std::vector<int> adj(m), fill(head.begin(), head.end() - 1);
  for (int e = 0; e < m; ++e) adj[fill[src[e]]++] = e;
  std::vector<int> deg = indeg;
  std::queue<int> qu;
  for (int i = 0; i < n; ++i) if (!deg[i]) qu.push(i);
  std::vector<double> d(n, 0.0), h(n, 0.0);
  while (!qu.empty()) {
    const int u = qu.front(); qu.pop();
    order.push_back(u);
    for (int j = head[u]; j < head[u + 1]; ++j) {
      const int e = adj[j];
      d[dst[e]] = std::max(d[dst[e]], d[u] + w[e]);
      if (--deg[dst[e]] == 0) qu.push(dst[e]);
    }
  }
  if ((int)order.size() != n) return false;  // cycle
  for (int i = n - 1; i >= 0; --i) {
    const int u = order[i];
    for (int j = head[u]; j < head[u + 1]; ++j) {
      const int e = adj[j];
      h[u] = std::max(h[u], w[e] + h[dst[e]]);
    }
  }
  double best = 0.0;
  for (int i = 0; i < n; ++i) best = std::max(best, d[i]);
  if (depth) std::copy(d.begin(), d.end(), depth);
  if (height) std::copy(h.begin(), h.end(), height);
  if (cp) *cp = best;
  return true;
}

bool simulate_table(const Table& t, double c, double r, int beta, int chains, SimResult* res,
                    std::string* err) {
  if (chains < 1) { if (err) *err = "chains must be >= 1"; return false; }
  const long long P = t.n_pairs();
  if (P * 4 > (1LL << 31) - 1) { if (err) *err = "table too large to simulate"; return false; }
  const int N = t.N;
  // node id of event a of each pair, in CTA order
  std::vector<int> a_of(P);
  std::vector<int> blk_pos_node((size_t)t.n_heads * N * N, -1);
  int nid = 0;
  std::vector<int> src, dst;
  std::vector<double> wt;
  auto edge = [&](int u, int v, double w) { src.push_back(u); dst.push_back(v); wt.push_back(w); };
  std::vector<std::vector<int>> cta_nodes(t.num_ctas);
  for (int cta = 0; cta < t.num_ctas; ++cta)
    for (int ci = t.cta_off[cta]; ci < t.cta_off[cta + 1]; ++ci) {
      const Chain& ch = t.chains[ci];
      for (int i = 0; i < ch.pair_cnt; ++i) {
        const uint32_t w = t.pairs[ch.pair_off + i];
        const size_t key = ((size_t)ch.bh * N + pair_q(w)) * N + pair_pos(w);
        blk_pos_node[key] = nid;
        cta_nodes[cta].push_back(nid);
        nid += 4;
      }
    }
  for (int cta = 0; cta < t.num_ctas; ++cta) {
    const auto& nodes = cta_nodes[cta];
    size_t n = 0;
    for (int ci = t.cta_off[cta]; ci < t.cta_off[cta + 1]; ++ci) {
      const Chain& ch = t.chains[ci];
      for (int i = 0; i < ch.pair_cnt; ++i, ++n) {
        const int a = nodes[n];
        const uint32_t w = t.pairs[ch.pair_off + i];
        edge(a, a + 1, c);
        edge(a + 1, a + 2, 0.0);
        edge(a + 2, a + 3, r);
        const int p = pair_pos(w);
        const int nc = t.causal ? pair_q(w) + 1 : N;
        // accumulation order: position p - chains of the same chain, and for the
        // block's last contributor the last position of every other chain
        auto pred = [&](int pp) {
          const size_t key = ((size_t)ch.bh * N + pair_q(w)) * N + pp;
          const int y = blk_pos_node[key];
          if (y < 0) return false;
          edge(y + 3, a + 2, 0.0);
          return true;
        };
        if (p >= chains && !pred(p - chains)) {
          if (err) *err = "missing predecessor in dQ order";
          return false;
        }
        if (p == nc - 1)
          for (int pp = std::max(0, p - chains + 1); pp < p; ++pp)
            if (!pred(pp)) { if (err) *err = "missing predecessor in dQ order"; return false; }
        if (n > 0) {
          edge(nodes[n - 1] + 1, a, 0.0);
          edge(nodes[n - 1] + 3, a + 2, 0.0);  // one reduction at a time per CTA
          if (beta >= 1 && (long long)n - beta >= 0) edge(nodes[n - beta] + 3, a + 1, 0.0);
        }
      }
    }
  }
  std::vector<double> depth(nid);
  double cp = 0;
  if (!dag_longest_path(nid, (int)src.size(), src.data(), dst.data(), wt.data(), depth.data(),
                        nullptr, &cp)) {
    if (err) *err = "schedule graph has a cycle (ticket deadlock)";
    return false;
  }
  SimResult out;
  out.critical_path = cp;
  for (int cta = 0; cta < t.num_ctas; ++cta) {
    const auto& nodes = cta_nodes[cta];
    if (nodes.empty()) continue;
    for (int a : nodes)
      if (depth[a + 1] > depth[a] + c + 1e-12 * std::max(1.0, std::fabs(depth[a]))) out.stalls++;
    out.makespan = std::max(out.makespan, depth[nodes.back() + 1]);
    out.bubble_time += cp - c * (double)nodes.size();
  }
  *res = out;
  return true;
}

bool expand_pair_table(const Table& half, Table* out) {
  if (!pair_schedule(half.schedule) || half.kv_units * 2 != half.N ||
      half.causal != (half.schedule == SYM_SHIFT_PAIRS) || half.group < 1 ||
      (long long)half.num_ctas * 2 > kMaxTableCtas)
    return false;
  Table t;
  t.n_heads = half.n_heads; t.N = half.N; t.causal = half.causal; t.schedule = half.schedule;
  t.num_ctas = 2 * half.num_ctas;
  t.group = half.group;  // heads per unit: each KV segment runs for `group` heads in turn
  t.kv_units = 0;  // the grid's table holds every KV tile
  t.cta_off.assign(t.num_ctas + 1, 0);
  for (int c = 0; c < half.num_ctas; ++c)
    for (int r = 0; r < 2; ++r) {
      t.cta_off[2 * c + r] = (int32_t)t.chains.size();
      for (int ci = half.cta_off[c]; ci < half.cta_off[c + 1]; ++ci) {
        const Chain& h = half.chains[ci];
        t.chains.push_back(Chain{h.bh, 2 * h.kv + r, (int32_t)t.pairs.size(), h.pair_cnt});
        for (int i = 0; i < h.pair_cnt; ++i) t.pairs.push_back(half.pairs[h.pair_off + i]);
      }
    }
  t.cta_off[t.num_ctas] = (int32_t)t.chains.size();
  *out = std::move(t);
  return true;
}

void plant_missing_first_partials(Table* t) {
  for (const Chain& ch : t->chains)
    if (ch.bh == 0)
      for (int i = 0; i < ch.pair_cnt; ++i) {
        uint32_t& w = t->pairs[ch.pair_off + i];
        if (pair_q(w) == 0) w = pack_pair(0, pair_pos(w) + 2);
      }
}

}  // namespace dash
