// C ABI of the deterministic attention backward: argument checks, workspace
// and schedule-table caches, TMA descriptors and launches.  The operation
// itself is documented in include/dash_attn.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <array>
#include <atomic>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <map>
#include <mutex>
#include <new>
#include <string>
#include <tuple>
#include <vector>

#include "../../include/dash_attn.h"
#include "aux_kernels.cuh"
#include "bwd_kernel.cuh"
#include "fwd_kernel.cuh"
#include "internal.h"
#include "sched.h"

namespace {

using dash::BwdCfg;
using dash::BwdParams;

// ------------------------------------------------------------------ settings
long long default_spin_us() {
  const char* e = std::getenv("DASH_SPIN_LIMIT_US");
  if (e) {
    const long long v = std::atoll(e);
    if (v > 0) return v;
  }
  return 10LL * 1000 * 1000;
}
std::atomic<long long> g_spin_us{0};
std::atomic<int> g_fault{0};  // host-side fault injection for the next backward (tests only)
long long spin_us() {
  long long v = g_spin_us.load();
  return v > 0 ? v : default_spin_us();
}

// ------------------------------------------------------------------ caches
struct Workspace {
  float* acc = nullptr;
  size_t acc_bytes = 0;
  uint32_t* tickets = nullptr;
  size_t tk_bytes = 0;
  float* rowbuf = nullptr;  // per-row column terms of the backward, 16 bytes per row
  size_t rows_cap = 0;
  float* dkv = nullptr;     // fp32 dK/dV accumulators of split grouped-query sub-groups
  size_t dkv_bytes = 0;
  unsigned* err = nullptr;   // [0] error word, [1] per-launch abort flag
};

struct DevTable {
  int* cta_off = nullptr;
  int4* chains = nullptr;
  uint32_t* pairs = nullptr;
  int group = 1;  // query heads per unit of the table it came from
};

std::mutex g_mu;
std::map<std::pair<int, uintptr_t>, Workspace> g_ws;                  // (device, stream)
// device, heads, N, causal, sched, ctas, group, run_group
std::map<std::tuple<int, int, int, int, int, int, int, int>, DevTable> g_tables;
std::map<std::pair<int, int>, int> g_num_ctas;                        // (device, D)

// Optional per-launch device timing: while enabled, each backward records four
// events (before the Delta kernel, before and after the main kernel, after the
// last auxiliary kernel) on its stream.
std::atomic<bool> g_prof_on{false};
std::mutex g_prof_mu;
std::vector<std::array<cudaEvent_t, 4>> g_prof;

bool prof_record(int slot, std::array<cudaEvent_t, 4>* ev, cudaStream_t st) {
  if (!g_prof_on.load()) return true;
  if (slot == 0)
    for (auto& e : *ev)
      if (cudaEventCreate(&e) != cudaSuccess) return false;
  return cudaEventRecord((*ev)[slot], st) == cudaSuccess;
}

#define DASH_CUDA(call)                    \
  do {                                     \
    if ((call) != cudaSuccess) return DASH_ERR_CUDA; \
  } while (0)

int grow(void** p, size_t* have, size_t need) {
  if (*have >= need) return DASH_OK;
  if (*p) {
    if (cudaDeviceSynchronize() != cudaSuccess) return DASH_ERR_CUDA;
    cudaFree(*p);
    *p = nullptr;
    *have = 0;
  }
  if (cudaMalloc(p, need) != cudaSuccess) {
    cudaGetLastError();
    return DASH_ERR_OOM;
  }
  *have = need;
  return DASH_OK;
}

int get_workspace(int dev, void* stream, size_t acc_bytes, size_t tk_bytes, size_t rows,
                  Workspace** out, size_t dkv_bytes = 0) {
  Workspace& w = g_ws[{dev, reinterpret_cast<uintptr_t>(stream)}];
  int rc;
  if ((rc = grow(reinterpret_cast<void**>(&w.acc), &w.acc_bytes, acc_bytes))) return rc;
  if ((rc = grow(reinterpret_cast<void**>(&w.dkv), &w.dkv_bytes, dkv_bytes))) return rc;
  if ((rc = grow(reinterpret_cast<void**>(&w.tickets), &w.tk_bytes, tk_bytes))) return rc;
  size_t rb = w.rows_cap * 16;
  if (rows > w.rows_cap) {
    if ((rc = grow(reinterpret_cast<void**>(&w.rowbuf), &rb, rows * 16))) return rc;
    w.rows_cap = rows;
  }
  if (!w.err) {
    if (cudaMalloc(&w.err, 2 * sizeof(unsigned)) != cudaSuccess) {
      cudaGetLastError();
      w.err = nullptr;
      return DASH_ERR_OOM;
    }
    if (cudaMemset(w.err, 0, 2 * sizeof(unsigned)) != cudaSuccess) {
      cudaFree(w.err);  // never keep an error word that was not cleared
      w.err = nullptr;
      return DASH_ERR_CUDA;
    }
  }
  *out = &w;
  return DASH_OK;
}

void free_table(DevTable* d) {
  cudaFree(d->cta_off);
  cudaFree(d->chains);
  cudaFree(d->pairs);
  *d = DevTable{};
}

// The device copy of a table's chains: the pair count of each chain carries the
// kernel's run flags (a run: consecutive chains of one CTA that feed one dK/dV tile,
// which only grouped-query tables have).  run_group: query heads that share a K/V
// head (the table's group, or 1 for a multi-head table that interleaves heads).
std::vector<dash::Chain> device_chains(const dash::Table& t, int run_group) {
  std::vector<dash::Chain> c = t.chains;
  auto same = [&](int a, int b) {
    return t.chains[a].bh / run_group == t.chains[b].bh / run_group &&
           t.chains[a].kv == t.chains[b].kv;
  };
  for (int k = 0; k < t.num_ctas; ++k)
    for (int i = t.cta_off[k]; i < t.cta_off[k + 1]; ++i) {
      if (i > t.cta_off[k] && same(i - 1, i)) c[i].pair_cnt |= dash::kChainContPrev;
      if (i + 1 < t.cta_off[k + 1] && same(i, i + 1)) c[i].pair_cnt |= dash::kChainContNext;
    }
  return c;
}

int upload_table(const dash::Table& t, DevTable* out, int run_group) {
  DevTable d;
  d.group = t.group;
  const std::vector<dash::Chain> chains = device_chains(t, run_group);
  // an empty chain or pair list still gets a valid (unused) allocation
  const size_t nc = t.chains.empty() ? 1 : t.chains.size();
  const size_t np = t.pairs.empty() ? 1 : t.pairs.size();
  if (cudaMalloc(&d.cta_off, t.cta_off.size() * sizeof(int)) != cudaSuccess ||
      cudaMalloc(&d.chains, nc * sizeof(int4)) != cudaSuccess ||
      cudaMalloc(&d.pairs, np * sizeof(uint32_t)) != cudaSuccess) {
    cudaGetLastError();
    free_table(&d);
    return DASH_ERR_OOM;
  }
  static_assert(sizeof(dash::Chain) == sizeof(int4), "chain layout");
  if (cudaMemcpy(d.cta_off, t.cta_off.data(), t.cta_off.size() * sizeof(int),
                 cudaMemcpyHostToDevice) != cudaSuccess ||
      (!chains.empty() &&
       cudaMemcpy(d.chains, chains.data(), chains.size() * sizeof(int4),
                  cudaMemcpyHostToDevice) != cudaSuccess) ||
      (!t.pairs.empty() && cudaMemcpy(d.pairs, t.pairs.data(), t.pairs.size() * sizeof(uint32_t),
                                      cudaMemcpyHostToDevice) != cudaSuccess)) {
    free_table(&d);
    return DASH_ERR_CUDA;
  }
  *out = d;
  return DASH_OK;
}

// group: query heads per unit of the table; run_group: query heads per K/V head
// (group for a grouped-query table, 1 for a multi-head table that interleaves heads)
int get_table(int dev, int heads, int N, int causal, int sched, int ctas, DevTable** out,
              int group, int run_group) {
  auto key = std::make_tuple(dev, heads, N, causal, sched, ctas, group, run_group);
  auto itb = g_tables.find(key);
  if (itb != g_tables.end()) {
    *out = &itb->second;
    return DASH_OK;
  }
  dash::Table t;
  std::string err;
  if (!dash::build_table_grouped(heads, group, N, causal, sched, ctas, &t, &err))
    return DASH_ERR_UNSUPPORTED;
  if (!dash::validate_table(t, &err)) return DASH_ERR_SCHEDULE;
  DevTable d;
  int rc = upload_table(t, &d, run_group);
  if (rc) return rc;
  auto res = g_tables.emplace(key, d);
  *out = &res.first->second;
  return DASH_OK;
}

// Tables of the host-buffer path: the whole grid's table split into parts of
// `chunk` heads (split_table keeps every dQ block's order), one per part.
std::map<std::tuple<int, int, int, int, int, int, int, int>, std::vector<DevTable>> g_chunk_tables;

int get_chunk_tables(int dev, int heads, int N, int causal, int sched, int ctas, int chunk,
                     int il, std::vector<DevTable>** out) {
  auto key = std::make_tuple(dev, heads, N, causal, sched, ctas, chunk, il);
  auto itc = g_chunk_tables.find(key);
  if (itc != g_chunk_tables.end()) {
    *out = &itc->second;
    return DASH_OK;
  }
  dash::Table full;
  std::string err;
  if (!dash::build_table_grouped(heads, il, N, causal, sched, ctas, &full, &err))
    return DASH_ERR_UNSUPPORTED;
  if (!dash::validate_table(full, &err)) return DASH_ERR_SCHEDULE;
  std::vector<DevTable> parts;
  int rc = DASH_OK;
  for (int h0 = 0; h0 < heads && rc == DASH_OK; h0 += chunk) {
    dash::Table t;
    const int h1 = h0 + chunk < heads ? h0 + chunk : heads;
    if (!dash::split_table(full, h0, h1, &t) || !dash::validate_table(t, &err)) {
      rc = DASH_ERR_SCHEDULE;
      break;
    }
    DevTable d;
    if ((rc = upload_table(t, &d, 1)) == DASH_OK) parts.push_back(d);
  }
  if (rc) {
    for (DevTable& d : parts) free_table(&d);
    return rc;
  }
  auto res = g_chunk_tables.emplace(key, std::move(parts));
  *out = &res.first->second;
  return DASH_OK;
}

// The host-buffer path's parts of a CTA-pair launch (SHIFT_PAIRS, or SYM_SHIFT_PAIRS when
// causal): the half table (one unit per KV pair, ctas / 2 slots) split by heads, each
// part validated and expanded to the grid's table, so every part keeps the whole
// launch's dQ orders.
std::map<std::tuple<int, int, int, int, int, int, int>, std::vector<DevTable>>
    g_pair_chunk_tables;

int pair_sched_of(int causal) { return causal ? dash::SYM_SHIFT_PAIRS : dash::SHIFT_PAIRS; }

int get_pair_chunk_tables(int dev, int heads, int N, int causal, int ctas, int chunk, int il,
                          std::vector<DevTable>** out) {
  auto key = std::make_tuple(dev, heads, N, causal, ctas, chunk, il);
  auto itc = g_pair_chunk_tables.find(key);
  if (itc != g_pair_chunk_tables.end()) {
    *out = &itc->second;
    return DASH_OK;
  }
  dash::Table half;
  std::string err;
  if (!dash::build_table_grouped(heads, il, N, causal, pair_sched_of(causal), ctas / 2, &half,
                                 &err))
    return DASH_ERR_UNSUPPORTED;
  if (!dash::validate_table(half, &err)) return DASH_ERR_SCHEDULE;
  std::vector<DevTable> parts;
  int rc = DASH_OK;
  for (int h0 = 0; h0 < heads && rc == DASH_OK; h0 += chunk) {
    dash::Table t, g;
    const int h1 = h0 + chunk < heads ? h0 + chunk : heads;
    if (!dash::split_table(half, h0, h1, &t) || !dash::validate_table(t, &err) ||
        !dash::expand_pair_table(t, &g)) {
      rc = DASH_ERR_SCHEDULE;
      break;
    }
    DevTable d;
    if ((rc = upload_table(g, &d, 1)) == DASH_OK) parts.push_back(d);
  }
  if (rc) {
    for (DevTable& d : parts) free_table(&d);
    return rc;
  }
  auto res = g_pair_chunk_tables.emplace(key, std::move(parts));
  *out = &res.first->second;
  return DASH_OK;
}

// A deliberately broken table for failure-detection tests: every partial of
// dQ block (head 0, Q tile 0) moves one position later, so its first position
// is never filled and the waits on it must run out.  All indices stay in range.
DevTable g_fault_table;
int get_fault_table(int dev, int heads, int N, int causal, int sched, int ctas, int il,
                    DevTable** out) {
  dash::Table t;
  std::string err;
  if (!dash::build_table_grouped(heads, il, N, causal, sched, ctas, &t, &err))
    return DASH_ERR_UNSUPPORTED;
  dash::plant_missing_first_partials(&t);
  cudaFree(g_fault_table.cta_off);
  cudaFree(g_fault_table.chains);
  cudaFree(g_fault_table.pairs);
  g_fault_table = DevTable{};
  DevTable& d = g_fault_table;
  if (cudaMalloc(&d.cta_off, t.cta_off.size() * sizeof(int)) != cudaSuccess ||
      cudaMalloc(&d.chains, t.chains.size() * sizeof(int4)) != cudaSuccess ||
      cudaMalloc(&d.pairs, t.pairs.size() * sizeof(uint32_t)) != cudaSuccess) {
    cudaGetLastError();
    return DASH_ERR_OOM;
  }
  DASH_CUDA(cudaMemcpy(d.cta_off, t.cta_off.data(), t.cta_off.size() * sizeof(int),
                       cudaMemcpyHostToDevice));
  DASH_CUDA(cudaMemcpy(d.chains, t.chains.data(), t.chains.size() * sizeof(int4),
                       cudaMemcpyHostToDevice));
  DASH_CUDA(cudaMemcpy(d.pairs, t.pairs.data(), t.pairs.size() * sizeof(uint32_t),
                       cudaMemcpyHostToDevice));
  (void)dev;
  *out = &d;
  return DASH_OK;
}

// ------------------------------------------------------------------ TMA descriptors
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// [rows][D] bf16 viewed with a 64-column x box_rows box and the 128-byte swizzle.
int make_tmap(CUtensorMap* m, const void* base, long long rows, int D, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return DASH_ERR_CUDA;
  cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? DASH_OK : DASH_ERR_CUDA;
}

// [rows][8] bf16 column terms viewed with an 8 x 128 box, no swizzle: the box lands as
// 8-row x 16-byte core matrices, the layout of the backward's extra K-step operand.
int make_tmap_cols(CUtensorMap* m, const void* base, long long rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return DASH_ERR_CUDA;
  cuuint64_t dims[2] = {8, (cuuint64_t)rows};
  cuuint64_t strides[1] = {16};
  cuuint32_t box[2] = {8, 128};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? DASH_OK : DASH_ERR_CUDA;
}

// ------------------------------------------------------------------ helpers
bool aligned16(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool pair_sched(int schedule) {
  return schedule == DASH_SCHED_SHIFT_PAIRS || schedule == DASH_SCHED_SYM_SHIFT_PAIRS;
}

int check_shape(int B, int H, int S, int D) {
  if (B < 0 || H < 0 || S < 0 || D < 0) return DASH_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return DASH_ERR_UNSUPPORTED;
  if (S == 0 || S % 128 != 0 || S / 128 > 32767) return DASH_ERR_UNSUPPORTED;
  if ((long long)B * H * S >= (1LL << 31)) return DASH_ERR_UNSUPPORTED;
  return DASH_OK;
}

// The backward kernel of one launch: the deterministic path takes the red chain
// variant when `red` is set.
template <int D, bool kAtomic, bool kTrace>
auto bwd_kernel_for(bool red) {
  if constexpr (kAtomic)
    return dash::dash_bwd_kernel<D, true, kTrace, false>;
  else
    return red ? dash::dash_bwd_kernel<D, false, kTrace, true>
               : dash::dash_bwd_kernel<D, false, kTrace, false>;
}

// Whether a deterministic launch adds its chains' middle positions with red in L2
// (bitwise the same results): measured faster on B200 where consecutive positions of
// a block have slack between them, i.e. descending and naive ascending from 64 tiles,
// and at D = 64 tables that run two or more query heads per unit (interleaved
// multi-head tables, grouped-query sub-groups); slower or equal for the step-ordered
// schedules otherwise and for short sequences.  dash_set_dq_chain_mode overrides it.
std::atomic<int> g_chain_mode{0};  // 0 by schedule, length, head dim and heads per unit
std::atomic<int> g_il_mode{0};     // dash_set_head_interleave: 0 the library's choice
// dash_set_slot_placement: 0 by SM id from 128 tiles on (measured faster there: the
// best schedules of causal 16k D=64 and full 16k D=128 gained 3-4 %, shorter sequences
// lost up to 5 %), 1 by SM id, 2 launch order
std::atomic<int> g_place_mode{0};
bool place_by_smid(int N) {
  const int m = g_place_mode.load();
  return m == 1 || (m == 0 && N >= 128);
}
bool red_chain_for(int sched, int N, int D, int heads_per_unit) {
  const int m = g_chain_mode.load();
  if (m == 1) return true;
  if (m == 2) return false;
  // CTA pairs: red measured slower (2-5 % at D = 64, full 4k to 16k)
  if (pair_sched(sched)) return false;
  return ((sched == DASH_SCHED_DESCENDING || sched == DASH_SCHED_NAIVE_ASC) && N >= 64) ||
         (D == 64 && heads_per_unit > 1);
}

// The kernel moves registers between warpgroups with setmaxnreg; the split adds up
// to exactly kLaunchRegs per thread, so refuse any other allocation.
template <int D, bool kAtomic, bool kTrace>
int prepare_kernel(bool red) {
  using C = BwdCfg<D>;
  auto kern = bwd_kernel_for<D, kAtomic, kTrace>(red);
  DASH_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes));
  cudaFuncAttributes fa;
  DASH_CUDA(cudaFuncGetAttributes(&fa, kern));
  if (fa.numRegs != C::kLaunchRegs) return DASH_ERR_UNSUPPORTED;
  return DASH_OK;
}

template <int D, bool kAtomic>
int num_ctas_for(int dev, int* out) {
  using C = BwdCfg<D>;
  auto key = std::make_pair(dev, D * 2 + (kAtomic ? 1 : 0));
  auto itn = g_num_ctas.find(key);
  if (itn != g_num_ctas.end()) {
    *out = itn->second;
    return DASH_OK;
  }
  int rc;
  if ((rc = prepare_kernel<D, kAtomic, false>(false))) return rc;
  if (!kAtomic && (rc = prepare_kernel<D, kAtomic, false>(true))) return rc;
  auto kern = bwd_kernel_for<D, kAtomic, false>(false);
  int per_sm = 0, sms = 0;
  DASH_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, C::kThreads, C::kSmemBytes));
  DASH_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  if (per_sm < 1) return DASH_ERR_UNSUPPORTED;
  *out = per_sm * sms;
  g_num_ctas[key] = *out;
  return DASH_OK;
}

// Sub-groups per K/V head for a grouped-query backward (split = 0 asks for this choice).
// Each K/V head contributes `per_head` units per sub-group; a round is `ctas` units.
// Two measured effects decide: a split whose units fill the grid's rounds better wins;
// among splits that fill them equally (within 2 points), runs of two query heads are
// fastest (longer runs stretch the schedule's dQ order, one-head runs send every dK/dV
// tile through the ordered fp32 reduction).
int choose_split(long long kv_heads, int group, long long per_head, int ctas) {
  auto fill = [&](int sp) {
    const long long u = kv_heads * sp * per_head;
    const long long rounds = (u + ctas - 1) / ctas;
    return (double)u / (double)(rounds * ctas);
  };
  double best_fill = 0.0;
  for (int sp = 1; sp <= group; sp *= 2) best_fill = std::max(best_fill, fill(sp));
  int best = 1, best_dist = 1 << 30;
  for (int sp = 1; sp <= group; sp *= 2) {
    if (fill(sp) < best_fill - 0.02) continue;
    const int heads_log2 = __builtin_ctz((unsigned)(group / sp));  // log2 heads per run
    const int dist = heads_log2 > 1 ? heads_log2 - 1 : 1 - heads_log2;
    if (dist < best_dist) {
      best = sp;
      best_dist = dist;
    }
  }
  return best;
}

template <int D, bool kAtomic, bool kTrace = false>
int launch_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
               const float* lse, void* dq, void* dk, void* dv, int B, int H, int S, int causal,
               int sched, cudaStream_t stream, int dev, unsigned long long* trace = nullptr,
               int trace_rows = 0, const DevTable* tab_override = nullptr, int group = 1,
               int split = 1) {
  using C = BwdCfg<D>;
  const int N = S / 128;
  const long long rows = (long long)B * H * S;
  int ctas = 0;
  int rc = num_ctas_for<D, kAtomic>(dev, &ctas);
  if (rc) return rc;
  if (split == 0)
    split = group > 1 ? choose_split((long long)B * (H / group), group,
                                     (long long)dash::head_units(sched, N, causal).size(), ctas)
                      : 1;
  // the table's query heads per unit, and per K/V head (a multi-head launch may
  // interleave heads in its units; each head keeps its own K/V)
  const int tgroup = group > 1 ? group / split
                               : dash::head_interleave(D, sched, B * H, N, causal, ctas,
                                                       g_il_mode.load());
  const int rgroup = group > 1 ? group / split : 1;
  // a split group runs as group / split query heads per (virtual) K/V head in the table;
  // the kernel still reads K/V of head / group
  const long long dqn = dash::dq_units<D>((long long)B * H * N);
  const long long dkvn = split > 1 ? (long long)B * (H / group) * N : 0;
  DevTable* tab = nullptr;
  Workspace* ws = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    // an armed fault is kept for a multi-head call (its table has no run flags)
    const int fault = (tab_override || group > 1) ? 0 : g_fault.exchange(0);
    if (tab_override) {
      tab = const_cast<DevTable*>(tab_override);
    } else if (fault == 1 && !kAtomic) {
      if ((rc = get_fault_table(dev, B * H, N, causal, sched, ctas, tgroup, &tab))) return rc;
    } else if ((rc = get_table(dev, B * H, N, causal, sched, ctas, &tab, tgroup, rgroup))) {
      return rc;
    }
    if ((rc = get_workspace(dev, stream, 2 * (size_t)rows * D * sizeof(float),
                            (size_t)(dqn + dkvn + 1 + ctas) * sizeof(uint32_t), (size_t)rows, &ws,
                            2 * (size_t)(rows / group) * D * sizeof(float) * (split > 1))))
      return rc;
  }
  CUtensorMap tq, tk, tv, tdo, tc;
  if ((rc = make_tmap(&tq, q, rows, D, C::kQRows)) ||
      (rc = make_tmap(&tk, k, rows / group, D, C::kKVRows)) ||
      (rc = make_tmap(&tv, v, rows / group, D, C::kKVRows)) ||
      (rc = make_tmap(&tdo, dout, rows, D, C::kQRows)) ||
      (rc = make_tmap_cols(&tc, ws->rowbuf, rows)))
    return rc;
  const float scale = 1.0f / sqrtf((float)D);
  std::array<cudaEvent_t, 4> ev{};
  if (!prof_record(0, &ev, stream)) return DASH_ERR_CUDA;
  // Delta and the column terms; the same launch clears the abort flag and, on the
  // deterministic path, the tickets
  // (the dQ tickets on the deterministic path, the dK/dV tickets of a split group)
  dash::dash_delta_kernel<D><<<dash::delta_grid<D>(rows, ctas), 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dout), lse,
      reinterpret_cast<uint4*>(ws->rowbuf), rows, 1.0f / scale, ws->tickets + (kAtomic ? dqn : 0),
      (kAtomic ? 0LL : dqn) + dkvn + 1, ws->err + 1, 1);
  if (kAtomic) DASH_CUDA(cudaMemsetAsync(ws->acc, 0, (size_t)rows * D * sizeof(float), stream));
  BwdParams p;
  p.cta_off = tab->cta_off;
  p.chains = tab->chains;
  p.pairs = tab->pairs;
  p.acc = ws->acc;
  p.tickets = ws->tickets;
  p.err = ws->err;
  p.abort_flag = ws->err + 1;
  p.dq = static_cast<__nv_bfloat16*>(dq);
  p.dk = static_cast<__nv_bfloat16*>(dk);
  p.dv = static_cast<__nv_bfloat16*>(dv);
  p.S = S;
  p.N = N;
  p.causal = causal;
  p.group_log2 = __builtin_ctz((unsigned)group);
  p.split_log2 = __builtin_ctz((unsigned)split);
  p.dkv_acc = ws->dkv;
  p.dkv_tickets = ws->tickets + dqn;
  // tickets: [dQ][dK/dV of split groups][placement counter][placement SM ids]
  if (place_by_smid(N)) {
    p.slot_arrive = ws->tickets + dqn + dkvn;
    p.slot_smid = reinterpret_cast<int*>(ws->tickets + dqn + dkvn + 1);
  }
  p.scale = scale;
  p.scale_log2 = p.scale * 1.4426950408889634f;
  p.spin_ns = (unsigned long long)spin_us() * 1000ull;
  p.trace = trace;
  p.trace_rows = trace_rows;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ctas);
  cfg.blockDim = dim3(C::kThreads);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (!prof_record(1, &ev, stream)) return DASH_ERR_CUDA;
  // query heads per unit of the table (the host-buffer path passes the parts of one)
  const int hpu = tab_override ? tab_override->group : tgroup;
  const bool red = !kAtomic && red_chain_for(sched, N, D, hpu);
  if (kTrace && (rc = prepare_kernel<D, kAtomic, true>(red))) return rc;
  DASH_CUDA(cudaLaunchKernelEx(&cfg, bwd_kernel_for<D, kAtomic, kTrace>(red), tq, tk, tv, tdo,
                               tc, p));
  if (!prof_record(2, &ev, stream)) return DASH_ERR_CUDA;
  if (kAtomic) {
    const long long n_blocks = (long long)B * H * N;  // 128-row accumulator blocks
    const long long threads = n_blocks * 32 * D;
    dash::dash_dq_convert<D><<<(int)((threads + 255) / 256), 256, 0, stream>>>(
        ws->acc, static_cast<__nv_bfloat16*>(dq), n_blocks, p.scale);
  }
  if (!prof_record(3, &ev, stream)) return DASH_ERR_CUDA;
  if (g_prof_on.load()) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    g_prof.push_back(ev);
  }
  DASH_CUDA(cudaGetLastError());
  return DASH_OK;
}

// ------------------------------------------------------------------ CTA pairs
// SHIFT_PAIRS / SYM_SHIFT_PAIRS: the kernel runs in clusters of two CTAs, with as many
// clusters as fit on the device at once (cooperative, so all are resident).
std::map<std::pair<int, int>, int> g_pair_ctas;  // (device, D) -> CTAs of the pair launch
template <int D>
int pair_ctas(int dev, int* out) {
  auto it = g_pair_ctas.find({dev, D});
  if (it != g_pair_ctas.end()) {
    *out = it->second;
    return DASH_OK;
  }
  using C = BwdCfg<D>;
  auto kern = dash::dash_bwd_kernel<D, false, false, false, true>;
  for (auto k2 : {kern, dash::dash_bwd_kernel<D, false, false, true, true>}) {
    DASH_CUDA(cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   C::kSmemPairBytes));
    cudaFuncAttributes fa;
    DASH_CUDA(cudaFuncGetAttributes(&fa, k2));
    if (fa.numRegs != C::kLaunchRegs) return DASH_ERR_UNSUPPORTED;
  }
  int sms = 0;
  DASH_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(2 * sms));
  cfg.blockDim = dim3(C::kThreads);
  cfg.dynamicSmemBytes = C::kSmemPairBytes;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int clusters = 0;
  DASH_CUDA(cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg));
  if (clusters < 1) return DASH_ERR_UNSUPPORTED;
  *out = 2 * clusters;
  g_pair_ctas[{dev, D}] = *out;
  return DASH_OK;
}

template <int D>
int launch_bwd_pairs(const void* q, const void* k, const void* v, const void* o,
                     const void* dout, const float* lse, void* dq, void* dk, void* dv, int B,
                     int H, int S, int causal, cudaStream_t stream, int dev,
                     const DevTable* tab_override = nullptr) {
  using C = BwdCfg<D>;
  const int N = S / 128;
  const long long rows = (long long)B * H * S;
  int ctas = 0;
  int rc;
  // tickets per (block, half of the columns, chain)
  const long long dqn = 2 * dash::dq_units<D>((long long)B * H * N);
  DevTable* tab = nullptr;
  Workspace* ws = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if ((rc = pair_ctas<D>(dev, &ctas))) return rc;
    // heads per unit of the half table (1 unless dash_set_head_interleave forces more)
    const int il = dash::head_interleave(D, pair_sched_of(causal), B * H, N, causal, ctas / 2,
                                         g_il_mode.load());
    auto key = std::make_tuple(dev, B * H, N, causal, pair_sched_of(causal), ctas, il, 1);
    auto itb = g_tables.find(key);
    if (tab_override) {
      tab = const_cast<DevTable*>(tab_override);
    } else if (itb != g_tables.end()) {
      tab = &itb->second;
    } else {
      dash::Table half, t;
      std::string err;
      if (!dash::build_table_grouped(B * H, il, N, causal, pair_sched_of(causal), ctas / 2,
                                     &half, &err))
        return DASH_ERR_UNSUPPORTED;
      if (!dash::validate_table(half, &err) || !dash::expand_pair_table(half, &t))
        return DASH_ERR_SCHEDULE;
      DevTable d;
      if ((rc = upload_table(t, &d, 1))) return rc;
      tab = &g_tables.emplace(key, d).first->second;
    }
    if ((rc = get_workspace(dev, stream, 2 * (size_t)rows * D * sizeof(float),
                            (size_t)(dqn + 1) * sizeof(uint32_t), (size_t)rows, &ws)))
      return rc;
  }
  CUtensorMap tq, tk, tv, tdo, tc;
  if ((rc = make_tmap(&tq, q, rows, D, C::kQRows)) ||
      (rc = make_tmap(&tk, k, rows, D, C::kKVRows)) ||
      (rc = make_tmap(&tv, v, rows, D, C::kKVRows)) ||
      (rc = make_tmap(&tdo, dout, rows, D, C::kQRows)) ||
      (rc = make_tmap_cols(&tc, ws->rowbuf, rows)))
    return rc;
  const float scale = 1.0f / sqrtf((float)D);
  std::array<cudaEvent_t, 4> ev{};
  if (!prof_record(0, &ev, stream)) return DASH_ERR_CUDA;
  dash::dash_delta_kernel<D><<<dash::delta_grid<D>(rows, ctas), 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dout), lse,
      reinterpret_cast<uint4*>(ws->rowbuf), rows, 1.0f / scale, ws->tickets, dqn, ws->err + 1,
      1);
  BwdParams p;
  p.cta_off = tab->cta_off;
  p.chains = tab->chains;
  p.pairs = tab->pairs;
  p.acc = ws->acc;
  p.tickets = ws->tickets;
  p.err = ws->err;
  p.abort_flag = ws->err + 1;
  p.dq = static_cast<__nv_bfloat16*>(dq);
  p.dk = static_cast<__nv_bfloat16*>(dk);
  p.dv = static_cast<__nv_bfloat16*>(dv);
  p.S = S;
  p.N = N;
  p.causal = causal;
  p.group_log2 = 0;
  p.scale = scale;
  p.scale_log2 = p.scale * 1.4426950408889634f;
  p.spin_ns = (unsigned long long)spin_us() * 1000ull;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)ctas);
  cfg.blockDim = dim3(C::kThreads);
  cfg.dynamicSmemBytes = C::kSmemPairBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 2;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  if (!prof_record(1, &ev, stream)) return DASH_ERR_CUDA;
  // middle links with red in L2 only where the chain mode forces it (bitwise the same)
  const bool red = red_chain_for(pair_sched_of(causal), N, D, 1);
  DASH_CUDA(cudaLaunchKernelEx(&cfg,
                               red ? dash::dash_bwd_kernel<D, false, false, true, true>
                                   : dash::dash_bwd_kernel<D, false, false, false, true>,
                               tq, tk, tv, tdo, tc, p));
  if (!prof_record(2, &ev, stream) || !prof_record(3, &ev, stream)) return DASH_ERR_CUDA;
  if (g_prof_on.load()) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    g_prof.push_back(ev);
  }
  DASH_CUDA(cudaGetLastError());
  return DASH_OK;
}

// ------------------------------------------------------------------ forward
template <int D>
int launch_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
               int S, int causal, cudaStream_t stream, int dev, int group = 1) {
  using C = dash::FwdCfg<D>;
  const int N = S / 128;
  const long long rows = (long long)B * H * S;
  if ((long long)N * B * H > 0x7fffffffLL) return DASH_ERR_UNSUPPORTED;
  Workspace* ws = nullptr;
  int rc;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if ((rc = get_workspace(dev, stream, 0, 0, 0, &ws))) return rc;
  }
  CUtensorMap tq, tk, tv;
  if ((rc = make_tmap(&tq, q, rows, D, 128)) || (rc = make_tmap(&tk, k, rows / group, D, 128)) ||
      (rc = make_tmap(&tv, v, rows / group, D, 128)))
    return rc;
  auto kern = dash::dash_fwd_tc_kernel<D>;
  DASH_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes));
  dash::FwdParams p;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.err = ws->err;
  p.abort_flag = ws->err + 1;
  p.S = S;
  p.N = N;
  p.BH = B * H;
  p.group = group;
  p.causal = causal;
  p.scale_log2 = (1.0f / sqrtf((float)D)) * 1.4426950408889634f;
  p.spin_ns = (unsigned long long)spin_us() * 1000ull;
  DASH_CUDA(cudaMemsetAsync(ws->err + 1, 0, sizeof(unsigned), stream));
  kern<<<(unsigned)(N * B * H), C::kThreads, C::kSmemBytes, stream>>>(tq, tk, tv, p);
  DASH_CUDA(cudaGetLastError());
  return DASH_OK;
}

// ------------------------------------------------------------------ host-buffer path
// Per (device, caller stream): two copy streams, events, and two slots of device
// staging for one part's inputs and outputs.
struct HostPipe {
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t entry = nullptr;
  cudaEvent_t in_ready[2] = {}, comp_done[2] = {}, out_done[2] = {};
  unsigned char* buf = nullptr;
  size_t cap = 0;
};
std::map<std::pair<int, uintptr_t>, HostPipe> g_pipes;

void free_pipe(HostPipe* hp);

int get_pipe(int dev, void* stream, size_t bytes, HostPipe** out) {
  HostPipe& hp = g_pipes[{dev, reinterpret_cast<uintptr_t>(stream)}];
  if (!hp.h2d) {
    bool ok = cudaStreamCreateWithFlags(&hp.h2d, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&hp.d2h, cudaStreamNonBlocking) == cudaSuccess &&
              cudaEventCreateWithFlags(&hp.entry, cudaEventDisableTiming) == cudaSuccess;
    for (int i = 0; i < 2 && ok; ++i)
      ok = cudaEventCreateWithFlags(&hp.in_ready[i], cudaEventDisableTiming) == cudaSuccess &&
           cudaEventCreateWithFlags(&hp.comp_done[i], cudaEventDisableTiming) == cudaSuccess &&
           cudaEventCreateWithFlags(&hp.out_done[i], cudaEventDisableTiming) == cudaSuccess;
    if (!ok) {
      cudaGetLastError();
      free_pipe(&hp);  // a later call starts from scratch, not from a half-made pipe
      return DASH_ERR_CUDA;
    }
  }
  int rc = grow(reinterpret_cast<void**>(&hp.buf), &hp.cap, bytes);
  if (rc) return rc;
  *out = &hp;
  return DASH_OK;
}

void free_pipe(HostPipe* hp) {
  if (hp->buf) cudaFree(hp->buf);
  for (int i = 0; i < 2; ++i) {
    if (hp->in_ready[i]) cudaEventDestroy(hp->in_ready[i]);
    if (hp->comp_done[i]) cudaEventDestroy(hp->comp_done[i]);
    if (hp->out_done[i]) cudaEventDestroy(hp->out_done[i]);
  }
  if (hp->entry) cudaEventDestroy(hp->entry);
  if (hp->h2d) cudaStreamDestroy(hp->h2d);
  if (hp->d2h) cudaStreamDestroy(hp->d2h);
  *hp = HostPipe{};
}

constexpr int kHostParts = 8;  // parts the heads are split into on the host-buffer path

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Backward from host buffers: the heads are split into parts; part p's inputs are
// copied in on one stream while part p-1 computes on the caller's stream and the
// results of part p-2 are copied out on a third, through two staging slots.
template <int D, bool kAtomic>
int host_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
             const float* lse, void* dq, void* dk, void* dv, int B, int H, int S, int causal,
             int sched, cudaStream_t stream, int dev) {
  const int BH = B * H, N = S / 128;
  const bool pairs = pair_sched(sched);  // CTA pairs
  int ctas = 0;
  int rc;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    rc = pairs ? pair_ctas<D>(dev, &ctas) : num_ctas_for<D, kAtomic>(dev, &ctas);
  }
  if (rc) return rc;
  // the parts hold whole units of the launch's table, so its interleaved heads stay
  // together and every dQ block keeps the order dash_attn_bwd gives it
  const int il = dash::head_interleave(D, sched, BH, N, causal, pairs ? ctas / 2 : ctas,
                                       g_il_mode.load());
  const int chunk = ((BH + kHostParts - 1) / kHostParts + il - 1) / il * il;
  const size_t rows_c = (size_t)chunk * S;
  const size_t tile = align256(rows_c * D * 2), lse_b = align256(rows_c * 4);
  const size_t slot_bytes = 8 * tile + lse_b;  // q k v o dO, LSE; dQ dK dV
  std::vector<DevTable>* parts = nullptr;
  HostPipe* hp = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if ((rc = pairs ? get_pair_chunk_tables(dev, BH, N, causal, ctas, chunk, il, &parts)
                    : get_chunk_tables(dev, BH, N, causal, sched, ctas, chunk, il, &parts)))
      return rc;
    if ((rc = get_pipe(dev, stream, 2 * slot_bytes, &hp))) return rc;
  }
  // the copy streams start after whatever the caller queued before this call
  DASH_CUDA(cudaEventRecord(hp->entry, stream));
  DASH_CUDA(cudaStreamWaitEvent(hp->h2d, hp->entry, 0));
  DASH_CUDA(cudaStreamWaitEvent(hp->d2h, hp->entry, 0));
  const unsigned char* hin[5] = {static_cast<const unsigned char*>(q),
                                 static_cast<const unsigned char*>(k),
                                 static_cast<const unsigned char*>(v),
                                 static_cast<const unsigned char*>(o),
                                 static_cast<const unsigned char*>(dout)};
  unsigned char* hout[3] = {static_cast<unsigned char*>(dq), static_cast<unsigned char*>(dk),
                            static_cast<unsigned char*>(dv)};
  int c = 0;
  for (int h0 = 0; h0 < BH; h0 += chunk, ++c) {
    const int nh = (BH - h0 < chunk) ? BH - h0 : chunk;
    const int slot = c & 1;
    unsigned char* base = hp->buf + slot * slot_bytes;
    unsigned char* din[5];
    for (int i = 0; i < 5; ++i) din[i] = base + i * tile;
    float* dlse = reinterpret_cast<float*>(base + 5 * tile);
    unsigned char* dout3[3];
    for (int i = 0; i < 3; ++i) dout3[i] = base + 5 * tile + lse_b + i * tile;
    const size_t off = (size_t)h0 * S * D * 2, n = (size_t)nh * S * D * 2;
    // inputs of part c, once the compute of part c - 2 has released the slot
    if (c >= 2) DASH_CUDA(cudaStreamWaitEvent(hp->h2d, hp->comp_done[slot], 0));
    for (int i = 0; i < 5; ++i)
      DASH_CUDA(cudaMemcpyAsync(din[i], hin[i] + off, n, cudaMemcpyHostToDevice, hp->h2d));
    DASH_CUDA(cudaMemcpyAsync(dlse, lse + (size_t)h0 * S, (size_t)nh * S * 4,
                              cudaMemcpyHostToDevice, hp->h2d));
    DASH_CUDA(cudaEventRecord(hp->in_ready[slot], hp->h2d));
    // compute, once the inputs are in and the results of part c - 2 are out
    DASH_CUDA(cudaStreamWaitEvent(stream, hp->in_ready[slot], 0));
    if (c >= 2) DASH_CUDA(cudaStreamWaitEvent(stream, hp->out_done[slot], 0));
    if ((rc = pairs ? launch_bwd_pairs<D>(din[0], din[1], din[2], din[3], din[4], dlse, dout3[0],
                                       dout3[1], dout3[2], 1, nh, S, causal, stream, dev,
                                       &(*parts)[c])
                    : launch_bwd<D, kAtomic>(din[0], din[1], din[2], din[3], din[4], dlse,
                                             dout3[0], dout3[1], dout3[2], 1, nh, S, causal,
                                             sched, stream, dev, nullptr, 0, &(*parts)[c])))
      return rc;
    DASH_CUDA(cudaEventRecord(hp->comp_done[slot], stream));
    // results of part c
    DASH_CUDA(cudaStreamWaitEvent(hp->d2h, hp->comp_done[slot], 0));
    for (int i = 0; i < 3; ++i)
      DASH_CUDA(cudaMemcpyAsync(hout[i] + off, dout3[i], n, cudaMemcpyDeviceToHost, hp->d2h));
    DASH_CUDA(cudaEventRecord(hp->out_done[slot], hp->d2h));
  }
  // the caller's stream completes once every result is on the host
  for (int i = 0; i < 2 && i < c; ++i) DASH_CUDA(cudaStreamWaitEvent(stream, hp->out_done[i], 0));
  return DASH_OK;
}

}  // namespace

namespace dash {

long long spin_limit_us() { return spin_us(); }
int take_armed_fault() { return g_fault.exchange(0); }
int head_interleave_mode() { return g_il_mode.load(); }

}  // namespace dash

using dash::no_throw;

extern "C" {

const char* dash_status_string(int s) {
  switch (s) {
    case DASH_OK: return "DASH_OK";
    case DASH_ERR_INVALID_ARG: return "DASH_ERR_INVALID_ARG";
    case DASH_ERR_UNSUPPORTED: return "DASH_ERR_UNSUPPORTED";
    case DASH_ERR_CUDA: return "DASH_ERR_CUDA";
    case DASH_ERR_TIMEOUT: return "DASH_ERR_TIMEOUT";
    case DASH_ERR_OOM: return "DASH_ERR_OOM";
    case DASH_ERR_SCHEDULE: return "DASH_ERR_SCHEDULE";
    default: return "DASH_ERR_UNKNOWN";
  }
}

int dash_inject_fault(int mode) {
  if (mode != 0 && mode != 1) return DASH_ERR_INVALID_ARG;
  g_fault.store(mode);
  return DASH_OK;
}

int dash_set_spin_limit_us(long long us) {
  g_spin_us.store(us > 0 ? us : 0);
  return DASH_OK;
}

int dash_set_slot_placement(int mode) {
  if (mode < 0 || mode > 2) return DASH_ERR_INVALID_ARG;
  g_place_mode.store(mode);
  return DASH_OK;
}

int dash_slot_placement_by_smid(int S, int* by_smid) {
  if (!by_smid || S < 128 || S % 128 != 0) return DASH_ERR_INVALID_ARG;
  *by_smid = place_by_smid(S / 128) ? 1 : 0;
  return DASH_OK;
}

int dash_set_head_interleave(int mode) {
  if (mode != 0 && mode != 1 && mode != 2 && mode != 4) return DASH_ERR_INVALID_ARG;
  g_il_mode.store(mode);
  return DASH_OK;
}

int dash_bwd_head_interleave(int num_ctas, int D, int schedule, int n_heads, int S, int causal,
                             int* heads_per_unit) {
  if (!heads_per_unit || num_ctas < 1 || n_heads < 1 || (D != 64 && D != 128) || S < 128 ||
      S % 128 != 0 || schedule < DASH_SCHED_NAIVE_ASC || schedule > DASH_SCHED_SYM_SHIFT_PAIRS ||
      (causal != 0 && causal != 1))
    return DASH_ERR_INVALID_ARG;
  *heads_per_unit =
      dash::head_interleave(D, schedule, n_heads, S / 128, causal, num_ctas, g_il_mode.load());
  return DASH_OK;
}

int dash_set_dq_chain_mode(int mode) {
  if (mode < 0 || mode > 2) return DASH_ERR_INVALID_ARG;
  g_chain_mode.store(mode);
  return DASH_OK;
}

int dash_dq_chain_uses_red(int schedule, int S, int D, int heads_per_unit, int* red) {
  if (!red || S < 128 || S % 128 != 0 || schedule < DASH_SCHED_NAIVE_ASC ||
      schedule > DASH_SCHED_SYM_SHIFT_PAIRS || heads_per_unit < 1 || (D != 64 && D != 128))
    return DASH_ERR_INVALID_ARG;
  // the atomic variant has no chains
  *red = (schedule != DASH_SCHED_ATOMIC && red_chain_for(schedule, S / 128, D, heads_per_unit))
             ? 1 : 0;
  return DASH_OK;
}

int dash_attn_fwd_gqa(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                      int H, int Hkv, int S, int D, int causal, void* stream) {
  return no_throw([&]() -> int {
    int rc = check_shape(B, H, S, D);
    if (rc) return rc;
    if (causal != 0 && causal != 1) return DASH_ERR_INVALID_ARG;
    if (H > 0 && (Hkv < 1 || H % Hkv != 0)) return DASH_ERR_INVALID_ARG;
    if (H > 0 && ((H / Hkv) & (H / Hkv - 1)) != 0) return DASH_ERR_UNSUPPORTED;  // 2^k per K/V head
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !lse)
      return DASH_ERR_INVALID_ARG;
    if (B == 0 || H == 0) return DASH_OK;
    int dev = 0;
    DASH_CUDA(cudaGetDevice(&dev));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    return D == 64 ? launch_fwd<64>(q, k, v, o, lse, B, H, S, causal, st, dev, H / Hkv)
                   : launch_fwd<128>(q, k, v, o, lse, B, H, S, causal, st, dev, H / Hkv);
  }, DASH_ERR_OOM, DASH_ERR_INVALID_ARG);
}

int dash_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                  int S, int D, int causal, void* stream) {
  return dash_attn_fwd_gqa(q, k, v, o, lse, B, H, H, S, D, causal, stream);
}

int dash_attn_bwd_gqa_split(const void* q, const void* k, const void* v, const void* o,
                            const void* dout, const float* lse, void* dq, void* dk, void* dv,
                            int B, int H, int Hkv, int S, int D, int causal, int schedule,
                            int split, void* stream) {
  return no_throw([&]() -> int {
    int rc = check_shape(B, H, S, D);
    if (rc) return rc;
    if (causal != 0 && causal != 1) return DASH_ERR_INVALID_ARG;
    if (H > 0 && (Hkv < 1 || H % Hkv != 0)) return DASH_ERR_INVALID_ARG;
    if (H > 0 && ((H / Hkv) & (H / Hkv - 1)) != 0) return DASH_ERR_UNSUPPORTED;  // 2^k per K/V head
    // split: 0 = chosen by the library, else a power of two dividing the group
    if (split < 0 || (split > 0 && H > 0 &&
                      ((split & (split - 1)) != 0 || (H / Hkv) % split != 0)))
      return DASH_ERR_INVALID_ARG;
    if (schedule < DASH_SCHED_NAIVE_ASC || schedule > DASH_SCHED_SYM_SHIFT_PAIRS)
      return DASH_ERR_INVALID_ARG;
    if (pair_sched(schedule)) return DASH_ERR_UNSUPPORTED;  // dash_attn_bwd only
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) ||
        !aligned16(lse) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
      return DASH_ERR_INVALID_ARG;
    if (!dash::schedule_supported(schedule, S / 128, causal)) return DASH_ERR_UNSUPPORTED;
    if (B == 0 || H == 0) return DASH_OK;
    int dev = 0;
    DASH_CUDA(cudaGetDevice(&dev));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const bool atomic = (schedule == DASH_SCHED_ATOMIC);
    const int g = H / Hkv;
    if (D == 64)
      return atomic ? launch_bwd<64, true>(q, k, v, o, dout, lse, dq, dk, dv, B, H, S, causal,
                                           schedule, st, dev, nullptr, 0, nullptr, g, split)
                    : launch_bwd<64, false>(q, k, v, o, dout, lse, dq, dk, dv, B, H, S, causal,
                                            schedule, st, dev, nullptr, 0, nullptr, g, split);
    return atomic ? launch_bwd<128, true>(q, k, v, o, dout, lse, dq, dk, dv, B, H, S, causal,
                                          schedule, st, dev, nullptr, 0, nullptr, g, split)
                  : launch_bwd<128, false>(q, k, v, o, dout, lse, dq, dk, dv, B, H, S, causal,
                                           schedule, st, dev, nullptr, 0, nullptr, g, split);
  }, DASH_ERR_OOM, DASH_ERR_INVALID_ARG);
}

int dash_attn_bwd_gqa(const void* q, const void* k, const void* v, const void* o,
                      const void* dout, const float* lse, void* dq, void* dk, void* dv, int B,
                      int H, int Hkv, int S, int D, int causal, int schedule, void* stream) {
  return dash_attn_bwd_gqa_split(q, k, v, o, dout, lse, dq, dk, dv, B, H, Hkv, S, D, causal,
                                 schedule, 0, stream);
}

int dash_bwd_gqa_split_for(int num_ctas, int B, int Hkv, int group, int S, int causal,
                           int schedule, int* split) {
  return no_throw([&]() -> int {
    if (!split || num_ctas < 1 || B < 1 || Hkv < 1 || group < 1 || (group & (group - 1)) != 0 ||
        (causal != 0 && causal != 1))
      return DASH_ERR_INVALID_ARG;
    if (S < 128 || S % 128 != 0) return DASH_ERR_UNSUPPORTED;
    if (!dash::schedule_supported(schedule, S / 128, causal)) return DASH_ERR_UNSUPPORTED;
    *split = choose_split((long long)B * Hkv, group,
                          (long long)dash::head_units(schedule, S / 128, causal).size(), num_ctas);
    return DASH_OK;
  }, DASH_ERR_OOM, DASH_ERR_INVALID_ARG);
}

int dash_attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
                  const float* lse, void* dq, void* dk, void* dv, int B, int H, int S, int D,
                  int causal, int schedule, void* stream) {
  if (pair_sched(schedule))
    return no_throw([&]() -> int {
      int rc = check_shape(B, H, S, D);
      if (rc) return rc;
      if (causal != 0 && causal != 1) return DASH_ERR_INVALID_ARG;
      if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) ||
          !aligned16(lse) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
        return DASH_ERR_INVALID_ARG;
      // CTA pairs: SHIFT_PAIRS for the full mask, SYM_SHIFT_PAIRS for the causal one
      if (!dash::schedule_supported(schedule, S / 128, causal)) return DASH_ERR_UNSUPPORTED;
      if (B == 0 || H == 0) return DASH_OK;
      int dev = 0;
      DASH_CUDA(cudaGetDevice(&dev));
      return D == 64 ? launch_bwd_pairs<64>(q, k, v, o, dout, lse, dq, dk, dv, B, H, S, causal,
                                            static_cast<cudaStream_t>(stream), dev)
                     : launch_bwd_pairs<128>(q, k, v, o, dout, lse, dq, dk, dv, B, H, S, causal,
                                             static_cast<cudaStream_t>(stream), dev);
    }, DASH_ERR_OOM, DASH_ERR_INVALID_ARG);
  return dash_attn_bwd_gqa(q, k, v, o, dout, lse, dq, dk, dv, B, H, H, S, D, causal, schedule,
                           stream);
}

int dash_attn_bwd_host(const void* q, const void* k, const void* v, const void* o,
                       const void* dout, const float* lse, void* dq, void* dk, void* dv, int B,
                       int H, int S, int D, int causal, int schedule, void* stream) {
  return no_throw([&]() -> int {
    int rc = check_shape(B, H, S, D);
    if (rc) return rc;
    if (causal != 0 && causal != 1) return DASH_ERR_INVALID_ARG;
    if (schedule < DASH_SCHED_NAIVE_ASC || schedule > DASH_SCHED_SYM_SHIFT_PAIRS)
      return DASH_ERR_INVALID_ARG;
    if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv) return DASH_ERR_INVALID_ARG;
    if (!dash::schedule_supported(schedule, S / 128, causal)) return DASH_ERR_UNSUPPORTED;
    if (B == 0 || H == 0) return DASH_OK;
    int dev = 0;
    DASH_CUDA(cudaGetDevice(&dev));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const bool atomic = (schedule == DASH_SCHED_ATOMIC);
    if (D == 64)
      return atomic ? host_bwd<64, true>(q, k, v, o, dout, lse, dq, dk, dv, B, H, S, causal,
                                         schedule, st, dev)
                    : host_bwd<64, false>(q, k, v, o, dout, lse, dq, dk, dv, B, H, S, causal,
                                          schedule, st, dev);
    return atomic ? host_bwd<128, true>(q, k, v, o, dout, lse, dq, dk, dv, B, H, S, causal,
                                        schedule, st, dev)
                  : host_bwd<128, false>(q, k, v, o, dout, lse, dq, dk, dv, B, H, S, causal,
                                         schedule, st, dev);
  }, DASH_ERR_OOM, DASH_ERR_INVALID_ARG);
}

int dash_attn_sync_status(void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return DASH_ERR_CUDA;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DASH_ERR_CUDA;
  unsigned* err = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    auto itw = g_ws.find({dev, reinterpret_cast<uintptr_t>(stream)});
    if (itw == g_ws.end()) return DASH_OK;
    err = itw->second.err;
  }
  unsigned h = 0;
  if (!err) return DASH_OK;
  if (cudaMemcpy(&h, err, sizeof(unsigned), cudaMemcpyDeviceToHost) != cudaSuccess)
    return DASH_ERR_CUDA;
  if (h) {
    if (cudaMemset(err, 0, sizeof(unsigned)) != cudaSuccess) return DASH_ERR_CUDA;
    return (h & dash::dev::ERR_TIMEOUT) ? DASH_ERR_TIMEOUT : DASH_ERR_UNSUPPORTED;
  }
  return DASH_OK;
}

int dash_bwd_num_ctas(int device, int D, int* num_ctas) {
  if (!num_ctas) return DASH_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return DASH_ERR_UNSUPPORTED;
  int prev = 0;
  DASH_CUDA(cudaGetDevice(&prev));
  DASH_CUDA(cudaSetDevice(device));
  std::lock_guard<std::mutex> lk(g_mu);
  const int rc = (D == 64) ? num_ctas_for<64, false>(device, num_ctas)
                           : num_ctas_for<128, false>(device, num_ctas);
  cudaSetDevice(prev);
  return rc;
}

int dash_profile_begin(void) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  for (auto& ev : g_prof)
    for (auto e : ev) cudaEventDestroy(e);
  g_prof.clear();
  g_prof_on.store(true);
  return DASH_OK;
}

int dash_profile_end(double* main_ms, double* aux_ms, long long* launches) {
  g_prof_on.store(false);
  std::lock_guard<std::mutex> lk(g_prof_mu);
  double m = 0, a = 0;
  int rc = DASH_OK;
  for (auto& ev : g_prof) {
    float t01 = 0, t12 = 0, t23 = 0;
    if (cudaEventSynchronize(ev[3]) != cudaSuccess ||
        cudaEventElapsedTime(&t01, ev[0], ev[1]) != cudaSuccess ||
        cudaEventElapsedTime(&t12, ev[1], ev[2]) != cudaSuccess ||
        cudaEventElapsedTime(&t23, ev[2], ev[3]) != cudaSuccess)
      rc = DASH_ERR_CUDA;
    m += t12;
    a += t01 + t23;
    for (auto e : ev) cudaEventDestroy(e);
  }
  if (main_ms) *main_ms = m;
  if (aux_ms) *aux_ms = a;
  if (launches) *launches = (long long)g_prof.size();
  g_prof.clear();
  return rc;
}

int dash_release_workspace(void) {
  int dev = 0;
  DASH_CUDA(cudaGetDevice(&dev));
  DASH_CUDA(cudaDeviceSynchronize());
  std::lock_guard<std::mutex> lk(g_mu);
  for (auto itw = g_ws.begin(); itw != g_ws.end();) {
    if (itw->first.first == dev) {
      cudaFree(itw->second.acc);
      cudaFree(itw->second.dkv);
      cudaFree(itw->second.tickets);
      cudaFree(itw->second.rowbuf);
      cudaFree(itw->second.err);
      itw = g_ws.erase(itw);
    } else {
      ++itw;
    }
  }
  for (auto itt = g_tables.begin(); itt != g_tables.end();) {
    if (std::get<0>(itt->first) == dev) {
      free_table(&itt->second);
      itt = g_tables.erase(itt);
    } else {
      ++itt;
    }
  }
  for (auto itc = g_chunk_tables.begin(); itc != g_chunk_tables.end();) {
    if (std::get<0>(itc->first) == dev) {
      for (DevTable& d : itc->second) free_table(&d);
      itc = g_chunk_tables.erase(itc);
    } else {
      ++itc;
    }
  }
  for (auto itp = g_pipes.begin(); itp != g_pipes.end();) {
    if (itp->first.first == dev) {
      free_pipe(&itp->second);
      itp = g_pipes.erase(itp);
    } else {
      ++itp;
    }
  }
  return DASH_OK;
}

int dash_trace_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
                   const float* lse, void* dq, void* dk, void* dv, int B, int H, int S, int D,
                   int causal, int schedule, void* stream, unsigned long long* host_trace,
                   long long cap, int* num_ctas, int* rows_per_cta) {
  return no_throw([&]() -> int {
    int rc = check_shape(B, H, S, D);
    if (rc) return rc;
    if (causal != 0 && causal != 1) return DASH_ERR_INVALID_ARG;
    if (schedule < DASH_SCHED_NAIVE_ASC || schedule > DASH_SCHED_SYM_SHIFT_PAIRS)
      return DASH_ERR_INVALID_ARG;
    if (pair_sched(schedule)) return DASH_ERR_UNSUPPORTED;  // dash_attn_bwd only
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) ||
        !aligned16(lse) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || !host_trace ||
        !num_ctas || !rows_per_cta)
      return DASH_ERR_INVALID_ARG;
    if (!dash::schedule_supported(schedule, S / 128, causal)) return DASH_ERR_UNSUPPORTED;
    if (B == 0 || H == 0) return DASH_ERR_INVALID_ARG;
    int dev = 0;
    DASH_CUDA(cudaGetDevice(&dev));
    const bool atomic = (schedule == DASH_SCHED_ATOMIC);
    int ctas = 0;
    {
      std::lock_guard<std::mutex> lk(g_mu);
      if (D == 64)
        rc = atomic ? num_ctas_for<64, true>(dev, &ctas) : num_ctas_for<64, false>(dev, &ctas);
      else
        rc = atomic ? num_ctas_for<128, true>(dev, &ctas) : num_ctas_for<128, false>(dev, &ctas);
    }
    if (rc) return rc;
    dash::Table t;
    std::string err;
    const int il = dash::head_interleave(D, schedule, B * H, S / 128, causal, ctas,
                                         g_il_mode.load());
    if (!dash::build_table_grouped(B * H, il, S / 128, causal, schedule, ctas, &t, &err))
      return DASH_ERR_UNSUPPORTED;
    int rows = 0;
    for (int c = 0; c < ctas; ++c) {
      int n = 0;
      for (int ci = t.cta_off[c]; ci < t.cta_off[c + 1]; ++ci) n += t.chains[ci].pair_cnt;
      rows = n > rows ? n : rows;
    }
    const size_t n_entries = (size_t)ctas * rows * dash::kTraceEvents;
    unsigned long long* dtrace = nullptr;
    if (cudaMalloc(&dtrace, n_entries * sizeof(unsigned long long)) != cudaSuccess)
      return DASH_ERR_OOM;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    rc = cudaMemsetAsync(dtrace, 0, n_entries * sizeof(unsigned long long), st) == cudaSuccess
             ? DASH_OK : DASH_ERR_CUDA;
    if (!rc) {
      if (D == 64)
        rc = atomic ? launch_bwd<64, true, true>(q, k, v, o, dout, lse, dq, dk, dv, B, H, S,
                                                 causal, schedule, st, dev, dtrace, rows)
                    : launch_bwd<64, false, true>(q, k, v, o, dout, lse, dq, dk, dv, B, H, S,
                                                  causal, schedule, st, dev, dtrace, rows);
      else
        rc = atomic ? launch_bwd<128, true, true>(q, k, v, o, dout, lse, dq, dk, dv, B, H, S,
                                                  causal, schedule, st, dev, dtrace, rows)
                    : launch_bwd<128, false, true>(q, k, v, o, dout, lse, dq, dk, dv, B, H, S,
                                                   causal, schedule, st, dev, dtrace, rows);
    }
    if (!rc && cudaStreamSynchronize(st) != cudaSuccess) rc = DASH_ERR_CUDA;
    if (!rc) {
      const size_t n = n_entries < (size_t)cap ? n_entries : (size_t)cap;
      if (cudaMemcpy(host_trace, dtrace, n * sizeof(unsigned long long), cudaMemcpyDeviceToHost) !=
          cudaSuccess)
        rc = DASH_ERR_CUDA;
    }
    cudaFree(dtrace);
    *num_ctas = ctas;
    *rows_per_cta = rows;
    return rc;
  }, DASH_ERR_OOM, DASH_ERR_INVALID_ARG);
}

long long dash_sched_table_gqa(int n_heads, int group, int N, int causal, int schedule,
                               int num_ctas, int* rows, long long cap) {
  return no_throw([&]() -> long long {
    dash::Table t;
    std::string err;
    if (group < 1 || n_heads < 1 || n_heads % group != 0) return -DASH_ERR_INVALID_ARG;
    if (!dash::build_table_grouped(n_heads, group, N, causal, schedule, num_ctas, &t, &err))
      return -DASH_ERR_UNSUPPORTED;
    if (!dash::validate_table(t, &err)) return -DASH_ERR_SCHEDULE;
    long long n = 0;
    for (int c = 0; c < t.num_ctas; ++c)
      for (int ci = t.cta_off[c]; ci < t.cta_off[c + 1]; ++ci) {
        const dash::Chain& ch = t.chains[ci];
        for (int i = 0; i < ch.pair_cnt; ++i, ++n) {
          if (rows && n < cap) {
            const uint32_t w = t.pairs[ch.pair_off + i];
            int* r = rows + 6 * n;
            r[0] = c;
            r[1] = ch.bh;
            r[2] = ch.kv;
            r[3] = dash::pair_q(w);
            r[4] = dash::pair_pos(w);
            r[5] = ci;
          }
        }
      }
    return n;
  }, -DASH_ERR_OOM, -DASH_ERR_INVALID_ARG);
}

long long dash_sched_table_part(int n_heads, int N, int causal, int schedule, int num_ctas,
                                int h0, int h1, int* rows, long long cap) {
  return no_throw([&]() -> long long {
    dash::Table full, t;
    std::string err;
    if (!dash::build_table(n_heads, N, causal, schedule, num_ctas, &full, &err))
      return -DASH_ERR_UNSUPPORTED;
    if (!dash::validate_table(full, &err)) return -DASH_ERR_SCHEDULE;
    if (!dash::split_table(full, h0, h1, &t)) return -DASH_ERR_INVALID_ARG;
    if (!dash::validate_table(t, &err)) return -DASH_ERR_SCHEDULE;
    long long n = 0;
    for (int c = 0; c < t.num_ctas; ++c)
      for (int ci = t.cta_off[c]; ci < t.cta_off[c + 1]; ++ci) {
        const dash::Chain& ch = t.chains[ci];
        for (int i = 0; i < ch.pair_cnt; ++i, ++n) {
          if (rows && n < cap) {
            const uint32_t w = t.pairs[ch.pair_off + i];
            int* r = rows + 6 * n;
            r[0] = c;
            r[1] = ch.bh;
            r[2] = ch.kv;
            r[3] = dash::pair_q(w);
            r[4] = dash::pair_pos(w);
            r[5] = ci;
          }
        }
      }
    return n;
  }, -DASH_ERR_OOM, -DASH_ERR_INVALID_ARG);
}

long long dash_sched_table(int n_heads, int N, int causal, int schedule, int num_ctas, int* rows,
                           long long cap) {
  return no_throw([&]() -> long long {
    dash::Table t;
    std::string err;
    if (!dash::build_table(n_heads, N, causal, schedule, num_ctas, &t, &err))
      return -DASH_ERR_UNSUPPORTED;
    if (!dash::validate_table(t, &err)) return -DASH_ERR_SCHEDULE;
    long long n = 0;
    for (int c = 0; c < t.num_ctas; ++c)
      for (int ci = t.cta_off[c]; ci < t.cta_off[c + 1]; ++ci) {
        const dash::Chain& ch = t.chains[ci];
        for (int i = 0; i < ch.pair_cnt; ++i, ++n) {
          if (rows && n < cap) {
            const uint32_t w = t.pairs[ch.pair_off + i];
            int* r = rows + 6 * n;
            r[0] = c;
            r[1] = ch.bh;
            r[2] = ch.kv;
            r[3] = dash::pair_q(w);
            r[4] = dash::pair_pos(w);
            r[5] = ci;
          }
        }
      }
    return n;
  }, -DASH_ERR_OOM, -DASH_ERR_INVALID_ARG);
}

long long dash_sched_table_pairs(int n_heads, int N, int causal, int num_ctas, int* rows,
                                 long long cap) {
  return no_throw([&]() -> long long {
    if (num_ctas < 2 || num_ctas % 2 != 0 || (causal != 0 && causal != 1))
      return -DASH_ERR_INVALID_ARG;
    dash::Table half, t;
    std::string err;
    if (!dash::build_table(n_heads, N, causal, pair_sched_of(causal), num_ctas / 2, &half,
                           &err))
      return -DASH_ERR_UNSUPPORTED;
    if (!dash::validate_table(half, &err)) return -DASH_ERR_SCHEDULE;
    if (!dash::expand_pair_table(half, &t)) return -DASH_ERR_SCHEDULE;
    long long n = 0;
    for (int c = 0; c < t.num_ctas; ++c)
      for (int ci = t.cta_off[c]; ci < t.cta_off[c + 1]; ++ci) {
        const dash::Chain& ch = t.chains[ci];
        for (int i = 0; i < ch.pair_cnt; ++i, ++n) {
          if (rows && n < cap) {
            const uint32_t w = t.pairs[ch.pair_off + i];
            int* r = rows + 6 * n;
            r[0] = c;
            r[1] = ch.bh;
            r[2] = ch.kv;
            r[3] = dash::pair_q(w);
            r[4] = dash::pair_pos(w);
            r[5] = ci;
          }
        }
      }
    return n;
  }, -DASH_ERR_OOM, -DASH_ERR_INVALID_ARG);
}

int dash_sched_simulate(int n_heads, int N, int causal, int schedule, int num_ctas,
                        double w_compute, double w_reduce, int dq_buffers, int dq_chains,
                        double* critical_path, double* makespan, double* bubble_time,
                        long long* stalls) {
  return dash_sched_simulate_gqa(n_heads, 1, N, causal, schedule, num_ctas, w_compute, w_reduce,
                                 dq_buffers, dq_chains, critical_path, makespan, bubble_time,
                                 stalls);
}

int dash_sched_simulate_gqa(int n_heads, int group, int N, int causal, int schedule,
                            int num_ctas, double w_compute, double w_reduce, int dq_buffers,
                            int dq_chains, double* critical_path, double* makespan,
                            double* bubble_time, long long* stalls) {
  return no_throw([&]() -> int {
    if (w_compute < 0 || w_reduce < 0 || dq_chains < 1) return DASH_ERR_INVALID_ARG;
    if (group < 1 || n_heads < 1 || n_heads % group != 0) return DASH_ERR_INVALID_ARG;
    dash::Table t;
    std::string err;
    if (!dash::build_table_grouped(n_heads, group, N, causal, schedule, num_ctas, &t, &err))
      return DASH_ERR_UNSUPPORTED;
    if (!dash::validate_table(t, &err)) return DASH_ERR_SCHEDULE;
    dash::SimResult r;
    if (!dash::simulate_table(t, w_compute, w_reduce, dq_buffers, dq_chains, &r, &err))
      return DASH_ERR_SCHEDULE;
    if (critical_path) *critical_path = r.critical_path;
    if (makespan) *makespan = r.makespan;
    if (bubble_time) *bubble_time = r.bubble_time;
    if (stalls) *stalls = r.stalls;
    return DASH_OK;
  }, DASH_ERR_OOM, DASH_ERR_INVALID_ARG);
}

int dash_sched_check(int n_heads, int N, int causal, int num_ctas, const int* rows,
                     long long n_rows) {
  return no_throw([&]() -> int {
    if (causal != 0 && causal != 1) return DASH_ERR_INVALID_ARG;
    dash::Table t;
    std::string err;
    if (!dash::table_from_rows(n_heads, N, causal, num_ctas, rows, n_rows, &t, &err))
      return DASH_ERR_INVALID_ARG;
    return dash::validate_table(t, &err) ? DASH_OK : DASH_ERR_SCHEDULE;
  }, DASH_ERR_OOM, DASH_ERR_INVALID_ARG);
}

int dash_dag_longest_path(int n_nodes, int n_edges, const int* src, const int* dst, const double* w,
                          double* depth, double* height, double* cp) {
  return no_throw([&]() -> int {
    if (n_nodes < 0 || n_edges < 0 || (n_edges > 0 && (!src || !dst || !w)))
      return DASH_ERR_INVALID_ARG;
    if (!dash::dag_longest_path(n_nodes, n_edges, src, dst, w, depth, height, cp))
      return DASH_ERR_INVALID_ARG;
    return DASH_OK;
  }, DASH_ERR_OOM, DASH_ERR_INVALID_ARG);
}

}  // extern "C"
