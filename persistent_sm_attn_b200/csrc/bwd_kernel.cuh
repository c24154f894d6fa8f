// Persistent deterministic attention backward for sm_100a.
//
// One CTA per SM runs the chains its schedule table lists ("Resumen Técnico:
// DASH ..." §2.1: all pairs of one KV tile run back to back on one SM, with the
// dK/dV accumulators on chip).  Per (KV tile j, Q tile i) pair of 128 x 128:
//
//   S^T  = K_j Q_i^T                  tcgen05.mma (smem x smem) -> TMEM [0, 128)
//   dP^T = V_j dO_i^T                 tcgen05.mma (smem x smem) -> TMEM [128, 256)
//   P^T  = exp(scale S^T - LSE_i)     softmax warps, packed bf16 back into S^T's columns
//   dV_j += P^T dO_i                  tcgen05.mma with A in TMEM, as soon as P^T is packed
//   dS^T = P^T (dP^T - Delta_i)       softmax warps, into shared memory (and at D = 128
//                                     into S^T's columns)
//   dK_j += dS^T Q_i                  tcgen05.mma, A in TMEM (D = 128) or smem (D = 64)
//   dQp  = dS K_j                     tcgen05.mma (smem x smem) -> TMEM
//   ordered reduction of dQp into an fp32 accumulator of block (b,h,i): wait
//   until the accumulator's ticket says it is this pair's turn, add with plain
//   loads and stores, publish, bump the ticket (§1: a fixed accumulation order
//   makes dQ bitwise reproducible; §2.2 chooses the order).  Each block has two
//   accumulators, one for the even and one for the odd positions of its order,
//   so a contributor waits on the one two positions ahead of it; the last
//   contributor adds the two sums, rounds once to bf16 and writes dQ.
//
// D = 128: the MMA issuer queues S^T and dP^T of the next tile right behind dK
// and dQp, so the exponentials of tile i+1 run while the tensor pipe finishes
// tile i, and dV of tile i+1 runs while its dS is formed.  Taking P^T and dS^T
// from TMEM keeps two of the five products off the shared-memory read path.
// D = 64: TMEM has room for two S^T buffers, so the two softmax warpgroups take
// alternate tiles: one computes the exponentials of tile i+1 (bound by the MUFU
// unit) while the other forms dS of tile i (bound by instruction issue).  A
// tile's P^T goes into the upper half of its S^T buffer and its dQp into the
// lower half; dK reads dS^T from shared memory (one buffer per warpgroup).
//
// Warp roles (512 threads, four warpgroups):
//   WG0, WG1  softmax / dS (96 registers at D = 128, 104 at D = 64); D = 128: WG0 owns
//             Q columns 0-63 of every tile, WG1 columns 64-127; D = 64: WG0 takes the
//             even tiles, WG1 the odd ones, all 128 columns, and stages each tile's dQp
//             out of TMEM into its dS buffer
//   WG2       dQ reduction and the dK/dV epilogue (224 registers at D = 128, 208 at D = 64)
//   WG3       warp 12 TMA producer (K, V, Q; dO too at D = 64), warp 13 MMA issuer and
//             TMEM owner (at D = 64 of the score products S^T, dP^T, dV only), warp 14
//             publisher of the ordered reduction (D = 64), warp 15 TMA producer of dO
//             (D = 128) or issuer of the gradient products dQp, dK (D = 64); 96 registers
// TMEM lane quarter of a warp is (warp % 4), so each warpgroup covers the 128 lanes.
//
// TMEM columns (512).  D = 128: S^T [0,128) then packed P^T/dS^T, dP^T
// [128,256) then dQp, dV [256,384), dK [384,512).  D = 64: S^T of even tiles
// [0,128), of odd tiles [128,256), each then holding the packed P^T in its upper
// 64 columns and that tile's dQp in its lower 64; dP^T [256,384), dV [384,448),
// dK [448,512).  Packed layout after the softmax, two bf16 per column: D = 128,
// the 32 fp32 columns of chunk c (Q columns 32c..32c+31) hold P^T of those
// columns in 32c..32c+15 and dS^T in 32c+16..32c+31; D = 64, P^T of chunk c is
// in the 16 columns at p_col64(c).
//
// Shared-memory tiles are [128 rows][D] bf16 stored as D/64 column blocks of
// 128 rows x 128 bytes with the 128-byte swizzle (the layout a TMA load with
// SWIZZLE_128B and a 64 x 128 box produces).  The same bytes serve as a
// K-major operand (rows = M or N, contiguous along K) or as an MN-major one
// (rows = K, contiguous along M or N): leading byte offset 16 KiB between
// 64-element column blocks, stride byte offset 1 KiB between 8-row groups.
// A descriptor's start address field holds (address >> 4) in its low 14 bits;
// every tile here ends below 256 KiB, so adding (byte offset >> 4) to a base
// descriptor moves its start without carrying into the other fields.
#pragma once
#include <type_traits>

#include "ptx.cuh"

namespace dash {

// Chain word w (pair count) as uploaded: the count in the low 16 bits and two flags for
// grouped-query attention runs (chains that share one dK/dV tile on one CTA).
constexpr int kChainCountMask = 0xffff;
constexpr int kChainContPrev = 1 << 29;
constexpr int kChainContNext = 1 << 30;

struct BwdParams {
  const int* cta_off;     // [grid + 1]
  const int4* chains;     // {bh, kv, pair_off, pair_cnt}
  const uint32_t* pairs;  // q | position << 16
  float* acc;             // fp32 dQ accumulators, [D/4][128][4] each: two per 128-row block
                          // (the atomic variant uses the first per block)
  uint32_t* tickets;      // one per accumulator
  unsigned* err;          // device error word (accumulates until read by the host)
  unsigned* abort_flag;   // per-launch: set by the first timeout, cleared before each launch
  __nv_bfloat16* dq;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  int S, N, causal;
  int group_log2;         // log2 of the query heads per K/V head (0: one K/V head each)
  // Grouped-query attention with each K/V head's group split into 2^split_log2 sub-groups
  // that run as separate units: the sub-groups' dK/dV partials of a (K/V head, KV tile)
  // add, in sub-group order, into fp32 accumulators [dV, dK][D/4][128][4] under one
  // ticket each; the last sub-group writes bf16.  split_log2 = 0: dK/dV go straight
  // to bf16.
  int split_log2 = 0;
  float* dkv_acc = nullptr;
  uint32_t* dkv_tickets = nullptr;
  float scale, scale_log2;
  unsigned long long spin_ns;
  // Placement of the table's slots on the SMs.  nullptr: CTA b runs slot b.  Else CTA
  // b runs the slot equal to the rank of its SM id among the grid's (slot_smid holds
  // gridDim.x ints, slot_arrive a counter that starts at 0), so consecutive slots, which
  // hold a head's consecutive units, run on SMs with consecutive ids.  Which CTA runs a
  // slot changes no result: the table fixes every order.
  int* slot_smid = nullptr;
  uint32_t* slot_arrive = nullptr;
  // Optional %globaltimer trace (kernels instantiated with kTrace only):
  // trace[(cta * trace_rows + pair) * 8 + event], events listed at kTrace.
  unsigned long long* trace = nullptr;
  int trace_rows = 0;
};

template <int D>
struct BwdCfg {
  static constexpr int kThreads = 512;
  static constexpr int kLaunchRegs = 65536 / kThreads;   // 128: the setmaxnreg split below
  // D = 64: the softmax also stages dQp (64 fp32 per thread) out of TMEM
  static constexpr int kRegsSoftmax = (D == 64) ? 104 : 96;  // WG0, WG1
  static constexpr int kRegsReduce = (D == 64) ? 208 : 224;  // WG2
  static constexpr int kRegsCtrl = 96;                       // WG3
  static_assert(2 * kRegsSoftmax + kRegsReduce + kRegsCtrl == 4 * kLaunchRegs,
                "register split must equal the launch allocation");
  static constexpr int kKVRows = 128;                    // TMA box rows of K and V
  static constexpr int kQRows = 128;                     // TMA box rows of Q and dO
  static constexpr int kTile = 128 * D * 2;              // one [128][D] bf16 tile
  // D = 128: Q is double-buffered (the next S^T follows dK right away) and dO has one
  // buffer, refilled between dV of a tile and dP^T of the next, to fit the smem budget.
  // D = 64: three stages each; S^T runs two tiles ahead and dP^T one.
  static constexpr int kStagesQ = (D == 64) ? 3 : 2;
  static constexpr int kStagesDO = (D == 64) ? 3 : 1;
  // LSE and Delta enter the S^T and dP^T products as one extra K-step each: a per-Q-row
  // column tile ([128 rows][8] bf16, loaded with Q) against a constant tile of ones.
  // Each tile is 2 KiB of core matrices (8 rows x 16 bytes, no swizzle) followed by
  // 2 KiB of zeros for the K-step's second half.  They sit first in shared memory.
  static constexpr int kColTile = 4096;
  static constexpr int OFF_ONES = 0;                       // ones for S^T, then for dP^T
  static constexpr int OFF_COL = OFF_ONES + 2 * kColTile;  // kStagesQ column tiles
  static constexpr int OFF_K = OFF_COL + kStagesQ * kColTile;
  static_assert(OFF_K % 1024 == 0, "swizzled tiles need 1 KiB alignment");
  static constexpr int OFF_V = OFF_K + kTile;
  static constexpr int OFF_Q = OFF_V + kTile;
  static constexpr int OFF_DO = OFF_Q + kStagesQ * kTile;
  // dS^T [128 kv][128 q]: one buffer per softmax warpgroup at D = 64, where the two
  // warpgroups take alternate tiles; one at D = 128
  static constexpr int kDsBufs = (D == 64) ? 2 : 1;
  static constexpr int OFF_DST = OFF_DO + kStagesDO * kTile;
  static constexpr int OFF_BAR = OFF_DST + kDsBufs * 32768;
  static constexpr int kBars = 26 + 2 * kStagesQ + 2 * kStagesDO;
  static constexpr int OFF_TMEM_SLOT = OFF_BAR + kBars * 8;
  // The swizzled tiles need a 1 KiB aligned base; the kernel checks it.
  static constexpr int kSmemBytes = OFF_TMEM_SLOT + 16;
  static_assert(kSmemBytes <= 232448, "shared memory per block exceeded");
  // CTA pairs at D = 128: a 16 KiB buffer into which the peer writes 32 columns of its dQp
  // rows at a time ([8 float4 groups][128 rows][float4]); pair launches only
  static constexpr int OFF_XB = (kSmemBytes + 1023) / 1024 * 1024;
  static constexpr int kSmemPairBytes = (D == 64) ? kSmemBytes : OFF_XB + 16384;
  static_assert(kSmemPairBytes <= 232448, "shared memory per block exceeded (pairs)");
  // TMEM columns.  D = 128: S^T [0,128), dP^T [128,256), dV, dK; dQp reuses dP^T's
  // columns and dK takes dS^T from S^T's columns.  D = 64: S^T has two buffers [0,128)
  // and [128,256), one per softmax warpgroup (they take alternate tiles), dP^T
  // [256,384), dV, dK.  The softmax packs a tile's P^T into the upper 64 columns of its
  // S^T buffer, and the tile's dQp goes into the lower 64; dK takes dS^T from shared
  // memory.
  static constexpr bool kSDouble = (D == 64);
  static constexpr uint32_t TM_S = 0, TM_DP = kSDouble ? 256 : 128;
  static constexpr uint32_t TM_DV = TM_DP + 128, TM_DK = TM_DV + D;
  static_assert(TM_DK + D == 512, "TMEM columns");
  static constexpr bool kDqInDp = !kSDouble;
  // D = 64: a publisher warp releases the tickets, taking the release's wait for the
  // stores off the reducers (at D = 128 the extra hand-off lengthens each link of the
  // accumulation chains more than it saves)
  static constexpr bool kPublisher = kSDouble;
};

// Number of dQ accumulation chains (tickets, and fp32 accumulators of 128 x D):
// two per 128-row block.
template <int D>
constexpr long long dq_units(long long bh_times_n) {
  return 2 * bh_times_n;
}

// barrier indices
enum {
  B_KV_FULL = 0, B_KV_EMPTY, B_S_FULL, B_DP_FULL, B_DS_READY, B_DS_FREE, B_DQ_FULL0, B_DQ_FULL1,
  B_DQ_EMPTY0, B_DQ_EMPTY1, B_DVDK_DONE, B_DKDV_FULL, B_DKDV_EMPTY, B_FINAL, B_P_READY,
  B_S_FULL1, B_P_READY1, B_PEER0,  // the second S^T buffer's barriers (D = 64); see B_PEER1
  B_PUB_READY0, B_PUB_READY1, B_PUB_FREE0, B_PUB_FREE1,  // reducers -> publisher hand-off
  B_DS_READY1, B_DP_FULL1, B_DS_FREE1,  // odd tiles' barriers (D = 64)
  B_PEER1,  // CTA pairs: the peer's tile of this parity is staged (with B_PEER0)
  B_STAGE0 = 26
};

// D = 64: the TMEM column (within a tile's S^T buffer) where the softmax packs the
// bf16 P^T of Q columns 32c..32c+31.  Chunks are packed in the order 2, 3, 0, 1 into
// columns 64, 80, 96, 112, so each store lands on S^T columns already read.
__host__ __device__ constexpr uint32_t p_col64(int c) { return 64u + 16u * (uint32_t)((c + 2) & 3); }

// kTrace: record %globaltimer per pair of this CTA, kTraceEvents slots per pair:
//   0 S^T issued              1 softmax done (seen by the MMA issuer)
//   2 tile MMAs issued        3 softmax start (S^T seen)
//   4 dQ partial ready (seen by the reducers)       5 partial drained from TMEM
//   6 ticket granted          7 reduction published (or dQ written)
//   8 P^T packed (softmax, phase 1 end)             9 softmax phase 2 start
//  10 dS ready (softmax, phase 2 end)              11 P^T seen by the MMA issuer
//  12 MMA issuer starts waiting for the S^T buffer 13 load-add-store (or atomics) done
//  14 reducers start waiting for the ticket        15 dP^T issued
constexpr int kTraceEvents = 16;
// kRed (deterministic only): a chain's middle positions add their partial into the
// accumulator with red (fp32 addition performed in L2, no read back) once the ticket
// grants them, instead of a load-add-store from the SM.  The additions and their order
// are the same, so the results are bitwise the same; only the traffic and the latency
// of each link differ.
// kPair (deterministic): the grid runs in clusters of two
// CTAs, 2i and 2i + 1, with a SHIFT_PAIRS or SYM_SHIFT_PAIRS table: the pair runs KV tiles
// 2m and 2m + 1 over the same Q tiles at the same steps.  Each CTA's reducers add the two
// dQ partials of a step (its own and the peer's) for half of the columns, CTA 2i + r taking
// columns [rD/2, (r + 1)D/2), and run the ordered accumulation of that half: one
// contribution per pair and step, so N / 2 per block (q / 2 + 1 for block q under the
// causal mask) and half the accumulator bytes per CTA.  D = 64: each reducer reads the
// peer's staged tile over distributed shared memory, and both CTAs free a staged tile only
// after both have read it.  D = 128 (dQp only in TMEM): each reducer thread writes the
// peer's half of its row into the peer's exchange buffer, 32 columns a round, two rounds
// per step, and adds what the peer wrote into its own.  Under the causal mask CTA 2i + 1
// meets one tile wholly above the diagonal per diagonal pair-tile (KV 2m + 1, Q 2m): every
// probability of it is masked to zero, so its partials are zeros.
template <int D, bool kAtomic, bool kTrace = false, bool kRed = false, bool kPair = false>
__global__ void __launch_bounds__(512, 1)
    dash_bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                    const __grid_constant__ CUtensorMap tmC, const BwdParams p) {
  using namespace dev;
  using C = BwdCfg<D>;
  static_assert(!kPair || !kAtomic, "CTA pairs: deterministic only");
  constexpr int ST = C::kStagesQ, SD = C::kStagesDO;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t sb = smem_u32(smem_raw);
  if (sb & 1023u) {  // the launch gave an unaligned base: refuse rather than misread
    if (threadIdx.x == 0) {
      atomicOr(p.err, ERR_MISALIGNED);
      atomicOr(p.abort_flag, 1u);
    }
    if constexpr (kPair) cluster_sync_all();  // the peer takes the same branch
    return;
  }
  if constexpr (kPair) {
    // every CTA must sit in a cluster of two with the rank of its slot's parity; a launch
    // without that (a tool that drops the cluster attribute, say) computes nothing and
    // reports it, instead of reading a peer that is not there
    if (cluster_nctarank() != 2u || cluster_ctarank() != (blockIdx.x & 1u)) {
      if (threadIdx.x == 0) {
        atomicOr(p.err, ERR_NO_CLUSTER);
        atomicOr(p.abort_flag, 1u);
      }
      return;
    }
  }
  uint8_t* gb = smem_raw;
  const uint32_t sK = sb + C::OFF_K, sV = sb + C::OFF_V, sQ = sb + C::OFF_Q, sDO = sb + C::OFF_DO;
  const uint32_t sDSt = sb + C::OFF_DST;
  const uint32_t bar0 = sb + C::OFF_BAR;
  auto BAR = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  auto Q_FULL = [&](int s) { return BAR(B_STAGE0 + s); };
  auto Q_EMPTY = [&](int s) { return BAR(B_STAGE0 + ST + s); };
  auto DO_FULL = [&](int s) { return BAR(B_STAGE0 + 2 * ST + s); };
  auto DO_EMPTY = [&](int s) { return BAR(B_STAGE0 + 2 * ST + SD + s); };
  // Per-tile buffers: tile i's S^T columns and the barriers reporting them full and P^T
  // packed; its dQp columns and the barriers reporting them full and drained.  With two
  // buffers (D = 64) each barrier serves every other tile, so its phase parity is
  // (i / 2) mod 2.
  auto s_col = [&](int i) { return C::kSDouble ? 128u * (uint32_t)(i & 1) : 0u; };
  auto S_FULL = [&](int i) { return BAR(C::kSDouble && (i & 1) ? B_S_FULL1 : B_S_FULL); };
  auto P_READY = [&](int i) { return BAR(C::kSDouble && (i & 1) ? B_P_READY1 : B_P_READY); };
  auto s_phase = [&](int i) { return C::kSDouble ? (i >> 1) & 1 : i & 1; };
  // D = 64 keeps one barrier per tile parity for dS ready, dP^T full and dS^T free, since
  // the two softmax warpgroups take alternate tiles; D = 128 has one of each
  auto DS_READY = [&](int i) { return BAR(C::kSDouble && (i & 1) ? B_DS_READY1 : B_DS_READY); };
  auto DP_FULL = [&](int i) { return BAR(C::kSDouble && (i & 1) ? B_DP_FULL1 : B_DP_FULL); };
  auto DS_FREE = [&](int i) { return BAR(C::kSDouble && (i & 1) ? B_DS_FREE1 : B_DS_FREE); };
  auto dq_col = [&](int i) { return C::kDqInDp ? C::TM_DP : 128u * (uint32_t)(i & 1); };
  auto DQ_FULL = [&](int i) { return BAR(C::kDqInDp ? B_DQ_FULL0 : B_DQ_FULL0 + (i & 1)); };
  auto DQ_EMPTY = [&](int i) { return BAR(C::kDqInDp ? B_DQ_EMPTY0 : B_DQ_EMPTY0 + (i & 1)); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gb + C::OFF_TMEM_SLOT);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint64_t lim = p.spin_ns;
  auto trace = [&](int row, int ev) {
    if constexpr (kTrace) {
      if (row < p.trace_rows)
        p.trace[((size_t)tmem_slot[1] * p.trace_rows + row) * kTraceEvents + ev] = globaltimer();
    }
  };
  auto wait = [&](uint32_t bar, uint32_t phase) { mbar_wait(bar, phase, lim, p.err, p.abort_flag); };
  auto drain = [&](uint32_t bar, uint32_t phase) {
    mbar_wait_drain(bar, phase, lim, p.err, p.abort_flag);
  };

  if (threadIdx.x == 0) {
    mbar_init(BAR(B_KV_FULL), 1);
    mbar_init(BAR(B_KV_EMPTY), C::kSDouble ? 2u : 1u);
    mbar_init(BAR(B_S_FULL), 1);
    mbar_init(BAR(B_S_FULL1), 1);
    // D = 64: one softmax warpgroup (128 threads) per tile, D = 128: both
    constexpr uint32_t kSoftmaxArrive = C::kSDouble ? 128u : 256u;
    mbar_init(BAR(B_DP_FULL), 1);
    mbar_init(BAR(B_DP_FULL1), 1);
    mbar_init(BAR(B_DS_READY), kSoftmaxArrive);
    mbar_init(BAR(B_DS_READY1), kSoftmaxArrive);
    // D = 64: the reducers (128 threads) free a dS buffer once they have read the dQp
    // staged there; D = 128: the commit of dQp and dK frees it
    // CTA pairs at D = 64: both CTAs' reducers read each staged tile (128 + 128 arrivals)
    constexpr uint32_t kDsFree = C::kSDouble ? (kPair ? 256u : 128u) : 1u;
    mbar_init(BAR(B_DS_FREE), kDsFree);
    mbar_init(BAR(B_DS_FREE1), kDsFree);
    // CTA pairs: D = 64, the peer's softmax warpgroup (128 threads) has staged its tile's
    // dQp; D = 128, the peer's reducers (128 threads) have filled this CTA's exchange
    // buffer (B_PEER0), or have read theirs, so this CTA may write it again (B_PEER1)
    mbar_init(BAR(B_PEER0), 128);
    mbar_init(BAR(B_PEER1), 128);
    for (int b = 0; b < 2; ++b) {
      mbar_init(BAR(B_DQ_FULL0 + b), 1);
      mbar_init(BAR(B_DQ_EMPTY0 + b), 128);
    }
    mbar_init(BAR(B_DVDK_DONE), 1);
    // D = 64: two threads issue the products (scores and gradients), and each commits
    // its share of the shared barriers
    constexpr uint32_t kIssuers = C::kSDouble ? 2u : 1u;
    mbar_init(BAR(B_DKDV_FULL), kIssuers);
    mbar_init(BAR(B_DKDV_EMPTY), 128);
    mbar_init(BAR(B_FINAL), kIssuers);
    mbar_init(BAR(B_P_READY), kSoftmaxArrive);
    mbar_init(BAR(B_P_READY1), kSoftmaxArrive);
    for (int b = 0; b < 2; ++b) {
      mbar_init(BAR(B_PUB_READY0 + b), 128);
      mbar_init(BAR(B_PUB_FREE0 + b), 1);
    }
    for (int s = 0; s < ST; ++s) {
      mbar_init(Q_FULL(s), 1);
      mbar_init(Q_EMPTY(s), kIssuers);
    }
    for (int s = 0; s < SD; ++s) {
      mbar_init(DO_FULL(s), 1);
      mbar_init(DO_EMPTY(s), 1);
    }
    fence_mbar_init();
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    prefetch_tmap(&tmDO);
    prefetch_tmap(&tmC);
  }
  // the constant tiles of the extra K-step: row r of the first holds bf16 ones in columns
  // 0-2 (they meet the LSE terms), of the second in columns 3-5 (the Delta terms); the
  // second 2 KiB of every column tile and of both constant tiles stay zero
  for (int i = threadIdx.x; i < 128; i += blockDim.x) {
    const uint32_t one = 0x3F80u;  // bf16 1.0
    st_shared_v4(sb + C::OFF_ONES + i * 16, one | (one << 16), one, 0u, 0u);
    st_shared_v4(sb + C::OFF_ONES + C::kColTile + i * 16, 0u, one << 16, one | (one << 16), 0u);
  }
  for (int i = threadIdx.x; i < 128 * (2 + ST); i += blockDim.x)
    st_shared_v4(sb + C::OFF_ONES + (i >> 7) * C::kColTile + 2048 + (i & 127) * 16, 0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
  if (warp == 13) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    int slot = (int)blockIdx.x;
    if (!kPair && p.slot_smid) {  // a pair's slots are its cluster's CTAs
      // every CTA of the cooperative grid is resident: enter this SM's id, count in
      // (release), wait (bounded) for all entries, and take the rank of this id
      const int my = (int)smid_u32();
      p.slot_smid[blockIdx.x] = my;
      red_add_release_gpu(p.slot_arrive, 1u);
      const uint64_t t0 = globaltimer();
      bool all = false;
      while (!(all = (ld_acquire_gpu(p.slot_arrive) >= gridDim.x))) {
        if (aborted(p.abort_flag) || globaltimer() - t0 > lim) {
          if (!aborted(p.abort_flag)) raise_timeout(p.err, p.abort_flag, ERR_WHERE_PIPE);
          break;
        }
      }
      if (all) {
        int rank = 0;
        for (int j = 0; j < (int)gridDim.x; ++j) {
          const int o = ld_cg_s32(p.slot_smid + j);
          rank += (o < my || (o == my && j < (int)blockIdx.x)) ? 1 : 0;
        }
        slot = rank;
      }
    }
    reinterpret_cast<volatile uint32_t*>(tmem_slot)[1] = (uint32_t)slot;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // CTA pairs: the peer's barriers are initialised before anything arrives on them
  if constexpr (kPair) cluster_sync_all();
  const uint32_t tmem = *tmem_slot;
  const int slot = (int)tmem_slot[1];  // the table slot this CTA runs
  const uint32_t prank = kPair ? cluster_ctarank() : 0u;  // this CTA's rank in its pair

  const int cbeg = p.cta_off[slot], cend = p.cta_off[slot + 1];
  const int S = p.S, N = p.N;
  // Grouped-query attention: the chains of one dK/dV tile (K/V head, KV tile) run back
  // to back on this CTA; such a run loads K/V once and carries dK/dV in TMEM from one
  // chain to the next.  With one K/V head per query head every run is one chain.
  // The library marks this in the chain's pair-count word (kChainContPrev: the chain
  // continues the previous chain's run, kChainContNext: the next chain continues its run).
  const int gl2 = p.group_log2;
  auto n_pairs = [](int w) { return w & kChainCountMask; };
  auto cont_prev = [&](int ci) { return (p.chains[ci].w & kChainContPrev) != 0; };
  auto cont_next = [&](int ci) { return (p.chains[ci].w & kChainContNext) != 0; };

  if (warp >= 12) {
    setmaxnreg_dec<C::kRegsCtrl>();
    if (warp == 12 && lane == 0) {
      // ---------------------------------------------------------- TMA producer: K, V, Q
      // K/V once per run; per pair Q with its column tile (LSE and Delta terms, read by
      // S^T and dP^T, which finish before dK frees the stage), and at D = 64 dO.  At
      // D = 128 dO has a producer of its own (warp 15), so a Q load never queues behind
      // the wait for the single dO stage.
      int it = 0, kn = 0;  // kn: K/V loads so far
      const uint64_t pol_first = policy_evict_first();  // K/V: one chain's use only
      for (int ci = cbeg; ci < cend; ++ci) {
        const int4 ch = p.chains[ci];
        if (!(ch.w & kChainContPrev)) {
          if (kn > 0) wait(BAR(B_KV_EMPTY), (kn - 1) & 1);
          mbar_expect_tx(BAR(B_KV_FULL), 2 * C::kTile);
          const int row_kv = (ch.x >> gl2) * S + ch.y * 128;
#pragma unroll
          for (int cb = 0; cb < D / 64; ++cb) {
            tma_load_2d_hint(sK + cb * 16384, &tmK, cb * 64, row_kv, BAR(B_KV_FULL), pol_first);
            tma_load_2d_hint(sV + cb * 16384, &tmV, cb * 64, row_kv, BAR(B_KV_FULL), pol_first);
          }
          ++kn;
        }
        for (int t = 0; t < n_pairs(ch.w); ++t, ++it) {
          const int q = (int)(p.pairs[ch.z + t] & 0xffffu);
          const int s = it % ST;
          const int row_q = ch.x * S + q * 128;
          if (it >= ST) wait(Q_EMPTY(s), ((it / ST) - 1) & 1);
          mbar_expect_tx(Q_FULL(s), C::kTile + 2048);
#pragma unroll
          for (int cb = 0; cb < D / 64; ++cb)
            tma_load_2d(sQ + s * C::kTile + cb * 16384, &tmQ, cb * 64, row_q, Q_FULL(s));
          tma_load_2d(sb + C::OFF_COL + s * C::kColTile, &tmC, 0, row_q, Q_FULL(s));
          if constexpr (C::kSDouble) {
            const int sd = it % SD;
            if (it >= SD) wait(DO_EMPTY(sd), ((it / SD) - 1) & 1);
            mbar_expect_tx(DO_FULL(sd), C::kTile);
#pragma unroll
            for (int cb = 0; cb < D / 64; ++cb)
              tma_load_2d(sDO + sd * C::kTile + cb * 16384, &tmDO, cb * 64, row_q, DO_FULL(sd));
          }
        }
      }
      // drain: every issued load has landed before the CTA can exit
      for (int s = 0; s < ST && s < it; ++s) {
        const int last_use = ((it - 1 - s) / ST) * ST + s;
        drain(Q_FULL(s), (last_use / ST) & 1);
      }
      if constexpr (C::kSDouble) {
        for (int s = 0; s < SD && s < it; ++s) {
          const int last_use = ((it - 1 - s) / SD) * SD + s;
          drain(DO_FULL(s), (last_use / SD) & 1);
        }
      }
      if (kn > 0) drain(BAR(B_KV_FULL), (kn - 1) & 1);
    } else if (warp == 15 && lane == 0 && !C::kSDouble) {
      // ---------------------------------------------------------- TMA producer: dO
      int it = 0;
      for (int ci = cbeg; ci < cend; ++ci) {
        const int4 ch = p.chains[ci];
        for (int t = 0; t < n_pairs(ch.w); ++t, ++it) {
          const int q = (int)(p.pairs[ch.z + t] & 0xffffu);
          const int sd = it % SD;
          const int row_q = ch.x * S + q * 128;
          if (it >= SD) wait(DO_EMPTY(sd), ((it / SD) - 1) & 1);
          mbar_expect_tx(DO_FULL(sd), C::kTile);
#pragma unroll
          for (int cb = 0; cb < D / 64; ++cb)
            tma_load_2d(sDO + sd * C::kTile + cb * 16384, &tmDO, cb * 64, row_q, DO_FULL(sd));
        }
      }
      for (int s = 0; s < SD && s < it; ++s) {
        const int last_use = ((it - 1 - s) / SD) * SD + s;
        drain(DO_FULL(s), (last_use / SD) & 1);
      }
    } else if (warp == 13 && lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      // One thread issues every MMA at D = 128; at D = 64 this one issues the score
      // products and warp 15 the gradient products.  An MMA is accepted only about as
      // fast as the tensor core runs it, so a waiting issuer idles the tensor core:
      // the loops are unrolled with constant operand offsets added to descriptor
      // words, and each product is written out once.
      constexpr uint32_t ID_SS = idesc_bf16_f32(128, 128, 0, 0);  // S^T, dP^T
      constexpr uint32_t ID_KV = idesc_bf16_f32(128, D, 0, 1);    // dV, dK (A in TMEM)
      constexpr uint32_t ID_Q = idesc_bf16_f32(128, D, 1, 1);     // dQ
      const uint32_t tS = tmem + C::TM_S, tDP = tmem + C::TM_DP, tDV = tmem + C::TM_DV,
                     tDK = tmem + C::TM_DK;
      const uint32_t hi = sdesc_hi(1024);  // every operand here: 1 KiB between 8-row groups
      const uint32_t kK = sdesc_lo(sK, 16), kV = sdesc_lo(sV, 16);            // K-major
      const uint32_t mK = sdesc_lo(sK, 16384), mDS = sdesc_lo(sDSt, 16384);  // MN-major
      // the extra K-step's operands: K-major core matrices without swizzle, 2 KiB
      // between the two 8-column halves of the step, 128 bytes between 8-row groups
      const uint32_t hi_none = sdesc_hi_none(128);
      const uint32_t kOnesS = sdesc_lo_none(sb + C::OFF_ONES, 2048);
      const uint32_t kOnesDP = sdesc_lo_none(sb + C::OFF_ONES + C::kColTile, 2048);
      if constexpr (C::kSDouble) {
        // D = 64, the score products (S^T, dP^T, dV).  The two softmax warpgroups take
        // alternate tiles, so tile i's S^T lives in buffer i mod 2 and two tiles are in
        // flight: while one warpgroup forms dS of tile i, the other computes the
        // exponentials of tile i+1.
        int it = 0, kn = 0;  // kn: runs started (K/V loads consumed)
        // S'^T = K Q^T - LSE/scale of tile i into its buffer, once the softmax has
        // staged out the dQp that tile i - 2 left there
        auto issue_s = [&](int i) {
          const int s = i % ST;
          const uint32_t kQ = sdesc_lo(sQ + s * C::kTile, 16);
          const uint32_t kCol = sdesc_lo_none(sb + C::OFF_COL + s * C::kColTile, 2048);
          const uint32_t tSi = tS + s_col(i);
          wait(Q_FULL(s), (i / ST) & 1);
          trace(i, 12);
          if (i >= 2) wait(DQ_EMPTY(i - 2), s_phase(i - 2));
          tc_fence_after();
          trace(i, 0);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (uint32_t)(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
            tc_mma_ss_w(tSi, kK + off, kQ + off, hi, ID_SS, kk > 0 ? 1u : 0u);
          }
          tc_mma_ss_w(tSi, kOnesS, kCol, hi_none, ID_SS, 1u);  // - LSE / scale
          tc_commit(S_FULL(i));
        };
        // dP'^T = V dO^T - Delta of tile i (the issuer has already seen the softmax
        // finish with tile i - 1's dP'^T)
        auto issue_dp = [&](int i) {
          const int s = i % ST, sd = i % SD;
          const uint32_t kDO = sdesc_lo(sDO + sd * C::kTile, 16);
          const uint32_t kCol = sdesc_lo_none(sb + C::OFF_COL + s * C::kColTile, 2048);
          wait(DO_FULL(sd), (i / SD) & 1);
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (uint32_t)(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
            tc_mma_ss_w(tDP, kV + off, kDO + off, hi, ID_SS, kk > 0 ? 1u : 0u);
          }
          tc_mma_ss_w(tDP, kOnesDP, kCol, hi_none, ID_SS, 1u);  // - Delta
          tc_commit(DP_FULL(i));
          tc_commit(Q_EMPTY(s));  // S'^T(i) and dP'^T(i) have read Q and the column tile
          trace(i, 15);
        };
        // dV += P^T dO of tile i (A = P^T from the upper half of its S^T buffer), once
        // P^T is packed; a run's first chain waits for the previous run's read-out
        auto issue_dv = [&](int i, bool first_of_run, uint32_t acc0) {
          const int sd = i % SD;
          const uint32_t mDO = sdesc_lo(sDO + sd * C::kTile, 16384);
          const uint32_t tSi = tS + s_col(i);
          wait(P_READY(i), s_phase(i));
          trace(i, 11);
          if (first_of_run && kn >= 2) wait(BAR(B_DKDV_EMPTY), (kn - 2) & 1);
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            tc_mma_ts_w(tDV, tSi + p_col64(kk >> 1) + 8 * (kk & 1), mDO + kk * 128, hi, ID_KV,
                        kk > 0 ? 1u : acc0);
          tc_commit(DO_EMPTY(sd));  // dP'^T and dV have read dO
        };
        // the score products' loop: dP'^T(it + 1) once the softmax has read dP'^T(it),
        // dV(it + 1) once P^T(it + 1) is packed, S'^T(it + 2) once the softmax has
        // staged dQp(it) out of S^T buffer it mod 2.  The gradient products (dQp, dK)
        // come from warp 15, so none of these waits holds them up.
        for (int ci = cbeg; ci < cend; ++ci) {
          const int cnt = n_pairs(p.chains[ci].w);
          const bool cprev = cont_prev(ci);
          if (!cprev) wait(BAR(B_KV_FULL), (kn++) & 1);
          tc_fence_after();
          if (cnt > 0) {
            issue_s(it);
            if (cnt > 1) issue_s(it + 1);
            issue_dp(it);
            issue_dv(it, !cprev, cprev ? 1u : 0u);
          }
          for (int t = 0; t < cnt; ++t, ++it) {
            wait(DS_READY(it), s_phase(it));
            trace(it, 1);
            tc_fence_after();
            if (t + 1 < cnt) {
              issue_dp(it + 1);
              issue_dv(it + 1, false, 1u);
            }
            if (t + 2 < cnt) issue_s(it + 2);
            trace(it, 2);
          }
          // the run's last chain: its dV are all issued, and S^T / dP^T are done with K/V
          if (!cont_next(ci)) {
            tc_commit(BAR(B_DKDV_FULL));
            tc_commit(BAR(B_KV_EMPTY));
          }
        }
      } else {
        int it = 0, kn = 0;  // kn: runs started (K/V loads consumed)
        for (int ci = cbeg; ci < cend; ++ci) {
          const int cnt = n_pairs(p.chains[ci].w);
          const bool cprev = cont_prev(ci);
          if (!cprev) wait(BAR(B_KV_FULL), (kn++) & 1);
          tc_fence_after();
          // t = -1 only issues the chain's first S^T/dP^T; each later step finishes
          // tile `it` and then issues S^T/dP^T of the next tile behind it
          for (int t = -1; t < cnt; ++t) {
            if (t >= 0) {
              const int s = it % ST, sd = it % SD;
              const uint32_t mQ = sdesc_lo(sQ + s * C::kTile, 16384);
              const uint32_t mDO = sdesc_lo(sDO + sd * C::kTile, 16384);
              // dV += P^T dO : M = kv, N = D, K = q (A in TMEM, B MN-major), once P is packed
              wait(BAR(B_P_READY), it & 1);
              trace(it, 11);
              // a run's first chain: the previous run's dV/dK must have been read out
              if (t == 0 && !cprev && kn >= 2) wait(BAR(B_DKDV_EMPTY), (kn - 2) & 1);
              tc_fence_after();
              const uint32_t acc0 = (t > 0 || cprev) ? 1u : 0u;
  #pragma unroll
              for (int kk = 0; kk < 8; ++kk)
                tc_mma_ts_w(tDV, tS + 32 * (kk >> 1) + 8 * (kk & 1), mDO + kk * 128, hi, ID_KV,
                            kk > 0 ? 1u : acc0);
              tc_commit(DO_EMPTY(sd));
              // dK += dS^T Q
              wait(BAR(B_DS_READY), it & 1);
              trace(it, 1);
              tc_fence_after();
  #pragma unroll
              for (int kk = 0; kk < 8; ++kk)
                tc_mma_ts_w(tDK, tS + 32 * (kk >> 1) + 16 + 8 * (kk & 1), mQ + kk * 128, hi, ID_KV,
                            kk > 0 ? 1u : acc0);
              tc_commit(Q_EMPTY(s));
              tc_commit(BAR(B_DVDK_DONE));
              if (t == cnt - 1 && !cont_next(ci)) tc_commit(BAR(B_DKDV_FULL));
              // dQp = dS K : M = q, N = D, K = kv (both operands MN-major)
              const int buf = C::kDqInDp ? 0 : (it & 1);
              if (!C::kDqInDp && it >= 2) {
                wait(BAR(B_DQ_EMPTY0 + buf), ((it - 2) >> 1) & 1);
                tc_fence_after();
              }
              const uint32_t tDQ = tmem + dq_col(it);
  #pragma unroll
              for (int kk = 0; kk < 8; ++kk)
                tc_mma_ss_w(tDQ, mDS + kk * 128, mK + kk * 128, hi, ID_Q, kk > 0 ? 1u : 0u);
              tc_commit(BAR(B_DQ_FULL0 + buf));
              tc_commit(BAR(B_DS_FREE));
              trace(it, 2);
              ++it;
            }
            if (t + 1 < cnt) {
              // S^T = K Q^T of tile `it`: M = kv, N = q, K = D (both K-major), once dV/dK
              // of the previous tile have read packed P^T/dS^T out of these columns
              const int s = it % ST, sd = it % SD;
              const uint32_t kQ = sdesc_lo(sQ + s * C::kTile, 16);
              const uint32_t kDO = sdesc_lo(sDO + sd * C::kTile, 16);
              const uint32_t kCol = sdesc_lo_none(sb + C::OFF_COL + s * C::kColTile, 2048);
              wait(Q_FULL(s), (it / ST) & 1);
              trace(it, 12);
              if (it > 0) wait(BAR(B_DVDK_DONE), (it - 1) & 1);
              tc_fence_after();
              trace(it, 0);
  #pragma unroll
              for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t off = (uint32_t)(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
                tc_mma_ss_w(tS, kK + off, kQ + off, hi, ID_SS, kk > 0 ? 1u : 0u);
              }
              // S'^T = S^T - LSE / scale, so the softmax takes P = 2^(scale log2e S')
              tc_mma_ss_w(tS, kOnesS, kCol, hi_none, ID_SS, 1u);
              tc_commit(BAR(B_S_FULL));
              // dP^T = V dO^T; at D = 128 these columns hold dQp of the previous tile
              // until the reducers have drained it
              wait(DO_FULL(sd), (it / SD) & 1);
              if (C::kDqInDp && it > 0) wait(BAR(B_DQ_EMPTY0), (it - 1) & 1);
              tc_fence_after();
  #pragma unroll
              for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t off = (uint32_t)(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
                tc_mma_ss_w(tDP, kV + off, kDO + off, hi, ID_SS, kk > 0 ? 1u : 0u);
              }
              // dP'^T = dP^T - Delta, so the softmax forms dS = P dP'
              tc_mma_ss_w(tDP, kOnesDP, kCol, hi_none, ID_SS, 1u);
              tc_commit(BAR(B_DP_FULL));
              trace(it, 15);
            }
          }
          // the run's last chain: K/V are done with
          if (!cont_next(ci)) tc_commit(BAR(B_KV_EMPTY));
        }
      }
      // drain: all issued MMAs complete before TMEM is released
      tc_commit(BAR(B_FINAL));
      drain(BAR(B_FINAL), 0);
    } else if (warp == 15 && lane == 0 && C::kSDouble) {
      // ---------------------------------------------------------- gradient products (D = 64)
      // dQp(it) = dS K into the lower half of S^T buffer it mod 2 and dK += dS^T Q, once
      // dS(it) is ready; their commit tells the softmax that dQp is ready to stage and
      // that dS has been read.
      constexpr uint32_t ID_KV = idesc_bf16_f32(128, D, 0, 1);  // dK (B = Q MN-major)
      constexpr uint32_t ID_Q = idesc_bf16_f32(128, D, 1, 1);   // dQp
      const uint32_t tDK = tmem + C::TM_DK;
      const uint32_t hi = sdesc_hi(1024);
      const uint32_t mK = sdesc_lo(sK, 16384);
      int it = 0, kn = 0;  // kn: runs started
      for (int ci = cbeg; ci < cend; ++ci) {
        const int cnt = n_pairs(p.chains[ci].w);
        const bool cprev = cont_prev(ci);
        if (!cprev) wait(BAR(B_KV_FULL), (kn++) & 1);
        for (int t = 0; t < cnt; ++t, ++it) {
          const int s = it % ST;
          const uint32_t dsb = sDSt + 32768u * (uint32_t)(it & 1);
          const uint32_t mQ = sdesc_lo(sQ + s * C::kTile, 16384);
          const uint32_t mDSi = sdesc_lo(dsb, 16384);  // dS MN-major (dQp)
          const uint32_t kDSi = sdesc_lo(dsb, 16);     // dS^T K-major (dK)
          wait(DS_READY(it), s_phase(it));
          // a run's first chain: the previous run's dK must have been read out
          if (t == 0 && !cprev && kn >= 2) wait(BAR(B_DKDV_EMPTY), (kn - 2) & 1);
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            tc_mma_ss_w(tmem + dq_col(it), mDSi + kk * 128, mK + kk * 128, hi, ID_Q,
                        kk > 0 ? 1u : 0u);
          const uint32_t acc0 = (t > 0 || cprev) ? 1u : 0u;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (uint32_t)(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
            tc_mma_ss_w(tDK, kDSi + off, mQ + kk * 128, hi, ID_KV, kk > 0 ? 1u : acc0);
          }
          tc_commit(DQ_FULL(it));
          tc_commit(Q_EMPTY(s));  // dK(it) has read Q
        }
        if (!cont_next(ci)) {
          tc_commit(BAR(B_DKDV_FULL));
          tc_commit(BAR(B_KV_EMPTY));  // dQp has read K
        }
      }
      tc_commit(BAR(B_FINAL));
      drain(BAR(B_FINAL), 0);
    } else if (warp == 14 && lane == 0 && !kAtomic && C::kPublisher) {
      // ---------------------------------------------------------- publisher
      // Publishes the reducers' load-add-store results in their place: once all 128
      // reducer threads have arrived after their stores (release at CTA scope,
      // acquired here), a release store at gpu scope advances the chain's ticket and
      // makes those stores visible with it.  The reducers go on to the next pair
      // without waiting for the release.  Hand-off slot k mod 2; the reducers take a
      // slot again only after this warp has freed it.
      int it = 0, k = 0;
      for (int ci = cbeg; ci < cend; ++ci) {
        const int4 ch = p.chains[ci];
        for (int t = 0; t < n_pairs(ch.w); ++t, ++it) {
          const uint32_t w = p.pairs[ch.z + t];
          const int q = (int)(w & 0xffffu), pos = (int)(w >> 16);
          // CTA pairs: N / 2 (causal: q / 2 + 1) contributions per block, tickets per
          // (block, half, chain)
          const int ncontrib = kPair ? (p.causal ? q / 2 + 1 : N / 2) : (p.causal ? q + 1 : N);
          if (pos == ncontrib - 1) continue;  // the last contributor writes dQ itself
          const long long unit =
              kPair ? (((long long)ch.x * N + q) * 2 + prank) * 2 + (pos & 1)
                    : ((long long)ch.x * N + q) * 2 + (pos & 1);
          wait(BAR(B_PUB_READY0 + (k & 1)), (k >> 1) & 1);
          st_release_gpu(p.tickets + unit, (uint32_t)((pos >> 1) + 1));
          mbar_arrive(BAR(B_PUB_FREE0 + (k & 1)));
          trace(it, 7);
          ++k;
        }
      }
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------ softmax / dS
    // Two phases per tile: P first (all the exponentials), published so that the
    // MMA issuer can start dV while dS is computed; then dS once dP^T is in TMEM.
    setmaxnreg_dec<C::kRegsSoftmax>();
    const int quarter = warp & 3, half = warp >> 2;
    const int r = quarter * 32 + lane;  // KV row of the tile = TMEM lane
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t rowoff =
        (uint32_t)half * 16384 + (uint32_t)(r >> 3) * 1024 + (uint32_t)(r & 7) * 128;
    const uint32_t tS0 = tmem + lane_off + C::TM_S, tDP = tmem + lane_off + C::TM_DP;
    const float sl2 = p.scale_log2;
    // P^T of 32 Q columns from S'^T: 2^(scale log2e S'), zero above the causal diagonal
    // (Q column qc < lim_c), packed as bf16 pairs
    auto exp_chunk = [&](const uint32_t (&sv)[32], uint32_t (&pk)[16], int c, int lim_c) {
      auto body = [&](auto masked) {
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          const int qc = 32 * c + j;
          // S'^T already has LSE / scale taken off by the tensor core
          float p0 = ex2_approx(__uint_as_float(sv[j]) * sl2);
          float p1 = ex2_approx(__uint_as_float(sv[j + 1]) * sl2);
          if constexpr (decltype(masked)::value) {
            if (qc < lim_c) p0 = 0.f;
            if (qc + 1 < lim_c) p1 = 0.f;
          }
          pk[j >> 1] = pack_bf16x2(p0, p1);
        }
      };
      // the causal mask only touches chunks that reach the diagonal
      if (lim_c > 32 * c) body(std::true_type{});
      else body(std::false_type{});
    };
    // dS = P dP' of 32 Q columns from packed P and fp32 dP'^T (Delta already taken off
    // by the tensor core), packed as bf16 pairs
    auto ds_chunk = [&](const uint32_t (&pk)[16], const uint32_t (&dv)[32], uint32_t (&dk)[16]) {
#pragma unroll
      for (int j = 0; j < 32; j += 2) {
        const float p0 = __uint_as_float(pk[j >> 1] << 16);
        const float p1 = __uint_as_float(pk[j >> 1] & 0xffff0000u);
        dk[j >> 1] = pack_bf16x2(p0 * __uint_as_float(dv[j]), p1 * __uint_as_float(dv[j + 1]));
      }
    };
    if constexpr (C::kSDouble) {
      // D = 64: warpgroup `half` takes the tiles of parity `half`, all 128 Q columns of
      // them, so one warpgroup's exponentials (MUFU-bound) run beside the other's dS
      // (issue-bound).  S'^T of its tiles is in buffer `half`; P^T goes into that
      // buffer's upper 64 columns (p_col64), dS^T into shared-memory buffer `half`.
      const uint32_t tS = tS0 + 128u * (uint32_t)half;
      const uint32_t sDS = sDSt + 32768u * (uint32_t)half;
      const uint32_t rowbase = (uint32_t)(r >> 3) * 1024 + (uint32_t)(r & 7) * 128;
      const bool tracer = threadIdx.x == 128 * half;
      int it = 0;
      for (int ci = cbeg; ci < cend; ++ci) {
        const int4 ch = p.chains[ci];
        for (int t = 0; t < n_pairs(ch.w); ++t, ++it) {
          if ((it & 1) != half) continue;
          const int q = (int)(p.pairs[ch.z + t] & 0xffffu);
          wait(S_FULL(it), s_phase(it));
          if (tracer) trace(it, 3);
          tc_fence_after();
          // causal: on the diagonal tile Q column qc sees KV row r only if qc >= r; a CTA
          // pair's tile above the diagonal (q < kv) is masked whole
          const int lim_c = !p.causal ? -1 : q == ch.y ? r : (kPair && q < ch.y) ? 128 : -1;
          // chunks 2, 3, 0, 1 into columns 64, 80, 96, 112: each store lands on columns
          // this thread has already read
#pragma unroll 1
          for (int cc = 0; cc < 4; ++cc) {
            const int c = (cc + 2) & 3;
            uint32_t sv[32], pk[16];
            tmem_ld32(tS + 32 * c, sv);
            exp_chunk(sv, pk, c, lim_c);
            tmem_st16(tS + 64 + 16 * cc, pk);
          }
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(P_READY(it));
          if (tracer) trace(it, 8);
          wait(DP_FULL(it), s_phase(it));
          // the reducers have read tile it - 2's dQp out of this buffer
          if (it >= 2) wait(DS_FREE(it - 2), s_phase(it - 2));
          tc_fence_after();
          if (tracer) trace(it, 9);
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t pk[16], dv[32], dk[16];
            tmem_ld16(tS + p_col64(c), pk);
            tmem_ld32(tDP + 32 * c, dv);
            ds_chunk(pk, dv, dk);
            // 128-byte swizzle, 64-column block c / 2
#pragma unroll
            for (int m = 0; m < 4; ++m) {
              const uint32_t unit = (uint32_t)((((c & 1) * 4 + m) ^ (r & 7)) * 16);
              st_shared_v4(sDS + (uint32_t)(c >> 1) * 16384 + rowbase + unit, dk[4 * m],
                           dk[4 * m + 1], dk[4 * m + 2], dk[4 * m + 3]);
            }
          }
          fence_proxy_async_smem();
          tc_fence_before();
          mbar_arrive(DS_READY(it));
          if (tracer) trace(it, 10);
          // Stage this tile's dQp: once dQp and dK have read dS (their commit), move dQp
          // out of the lower half of the S^T buffer into this warpgroup's dS buffer as
          // fp32 [D/4][128 rows][4], the reducers' layout.  The S^T buffer is then free
          // for tile it + 2 whatever the reducers are doing; they have until this
          // warpgroup's next dS to read the staged copy.
          wait(DQ_FULL(it), s_phase(it));
          tc_fence_after();
          {
            uint32_t v[32];
#pragma unroll
            for (int c2 = 0; c2 < 2; ++c2) {
              tmem_ld32(tS + 32 * c2, v);
#pragma unroll
              for (int j = 0; j < 8; ++j)
                st_shared_v4(sDS + (uint32_t)(((c2 * 8 + j) * 128 + r) * 16), v[4 * j],
                             v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
            }
          }
          tc_fence_before();
          mbar_arrive(DQ_EMPTY(it));
          // CTA pairs: tell the peer's reducers that this tile's dQp is staged here
          if constexpr (kPair)
            mbar_arrive_cluster(mapa_shared(BAR((it & 1) ? B_PEER1 : B_PEER0), prank ^ 1u));
        }
      }
    } else {
    int it = 0;
    for (int ci = cbeg; ci < cend; ++ci) {
      const int4 ch = p.chains[ci];
      for (int t = 0; t < n_pairs(ch.w); ++t, ++it) {
        const int q = (int)(p.pairs[ch.z + t] & 0xffffu);
        const uint32_t tS = tS0 + s_col(it);
        wait(S_FULL(it), s_phase(it));
        if (threadIdx.x == 0) trace(it, 3);
        tc_fence_after();
        // causal: on the diagonal tile Q column qc sees KV row r only if qc >= r; a CTA
        // pair's tile above the diagonal (q < kv) is masked whole
        const int lim_c = !p.causal ? -1 : q == ch.y ? r : (kPair && q < ch.y) ? 128 : -1;
#pragma unroll 1
        for (int cc = 0; cc < 2; ++cc) {
          const int c = half * 2 + cc;  // 32-column chunk of the tile
          uint32_t sv[32];
          tmem_ld32(tS + 32 * c, sv);
          uint32_t pk[16];
          exp_chunk(sv, pk, c, lim_c);
          // P^T into the first 16 columns of chunk c (this lane's own row)
          tmem_st16(tS + 32 * c, pk);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(P_READY(it));
        if (threadIdx.x == 0) trace(it, 8);
        wait(BAR(B_DP_FULL), it & 1);
        if (it > 0) wait(BAR(B_DS_FREE), (it - 1) & 1);
        tc_fence_after();
        if (threadIdx.x == 0) trace(it, 9);
        // dS from the bf16 P just packed: the registers are not there to keep P in
        // fp32 across the wait, and the extra rounding stays far inside the error bound
        // in sub-chunks of 16 Q columns (h = 0..3 of this warpgroup's 64), the next
        // sub-chunk's P and dP' loads in flight while this one is formed; dS^T goes into
        // the last 16 columns of its 32-column chunk, where dK reads it from TMEM, and to
        // shared memory (128-byte swizzle, 64-column block `half`)
        {
          uint32_t pa[8], da[16], pb[8], db[16];
          auto load = [&](int h, uint32_t (&pp)[8], uint32_t (&dd)[16]) {
            const int c = half * 2 + (h >> 1);
            tmem_ld8_async(tS + 32 * c + 8 * (h & 1), pp);
            tmem_ld16_async(tDP + 32 * c + 16 * (h & 1), dd);
          };
          auto form = [&](int h, const uint32_t (&pp)[8], const uint32_t (&dd)[16]) {
            const int c = half * 2 + (h >> 1);
            uint32_t dk[8];
#pragma unroll
            for (int j = 0; j < 16; j += 2) {
              const float p0 = __uint_as_float(pp[j >> 1] << 16);
              const float p1 = __uint_as_float(pp[j >> 1] & 0xffff0000u);
              dk[j >> 1] =
                  pack_bf16x2(p0 * __uint_as_float(dd[j]), p1 * __uint_as_float(dd[j + 1]));
            }
            tmem_st8(tS + 32 * c + 16 + 8 * (h & 1), dk);
#pragma unroll
            for (int m = 0; m < 2; ++m) {
              const uint32_t unit = (uint32_t)(((2 * h + m) ^ (r & 7)) * 16);
              st_shared_v4(sDSt + rowoff + unit, dk[4 * m], dk[4 * m + 1], dk[4 * m + 2],
                           dk[4 * m + 3]);
            }
          };
          load(0, pa, da);
          tmem_wait_ld();
          load(1, pb, db);
          form(0, pa, da);
          tmem_wait_ld();
          load(2, pa, da);
          form(1, pb, db);
          tmem_wait_ld();
          load(3, pb, db);
          form(2, pa, da);
          tmem_wait_ld();
          form(3, pb, db);
        }
        tmem_wait_st();
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(BAR(B_DS_READY));
        if (threadIdx.x == 0) trace(it, 10);
      }
    }
    }
  } else {
    // ------------------------------------------------------------ dQ reduction + dK/dV epilogue
    setmaxnreg_inc<C::kRegsReduce>();
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // Q row for dQ, KV row for dK/dV
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    constexpr int NV = D / 4;           // float4 per row
    // float4 per row of this CTA's share of a dQ block: all of it, or half for CTA pairs
    constexpr int NA = kPair ? NV / 2 : NV;
    constexpr int G = 24;               // loads in flight per group
    int it = 0, fn = 0;  // fn: dK/dV runs written out
    int npub = 0;        // pairs handed to the publisher
    const uint64_t pol_last = policy_evict_last();  // dQ accumulators: live for a whole head
    // D = 64, deterministic: once this pair is handed off, the accumulator loads of the
    // next pair go out if its ticket is already granted (checked once, never waited
    // for here), so their round trip overlaps the wait for the next partial and its
    // drain.  The values loaded and the order of the additions are the same either way.
    constexpr bool kLook = !kAtomic && D == 64 && !kRed && !kPair;
    float4 pre[NV];
    bool pre_ok = false;  // pre holds this pair's accumulator, loaded ahead
    for (int ci = cbeg; ci < cend; ++ci) {
      const int4 ch = p.chains[ci];
      for (int t = 0; t < n_pairs(ch.w); ++t, ++it) {
        const uint32_t w = p.pairs[ch.z + t];
        const int q = (int)(w & 0xffffu), pos = (int)(w >> 16);
        // CTA pairs: N / 2 (causal: q / 2 + 1) pre-summed contributions per block
        const int ncontrib = kPair ? (p.causal ? q / 2 + 1 : N / 2) : (p.causal ? q + 1 : N);
        const bool last = (pos == ncontrib - 1);
        float a[D];
        if constexpr (kPair && C::kSDouble) {
          // this CTA's half of the columns of the two partials staged for this step, its
          // own and the peer's (read over distributed shared memory once the peer says it
          // is staged), added: a + b is the same sum in either CTA
          wait(DQ_EMPTY(it), s_phase(it));
          mbar_wait_cluster(BAR((it & 1) ? B_PEER1 : B_PEER0), s_phase(it), lim, p.err,
                            p.abort_flag);
          if (threadIdx.x == 256) trace(it, 4);
          const uint32_t stage = sDSt + 32768u * (uint32_t)(it & 1);
          const uint32_t pstage = mapa_shared(stage, prank ^ 1u);
#pragma unroll
          for (int j = 0; j < NA; ++j) {
            const uint32_t off = (uint32_t)((((int)prank * NA + j) * 128 + r) * 16);
            const float4 u = ld_shared_f4(stage + off);
            const float4 v = ld_shared_cluster_f4(pstage + off);
            a[4 * j] = u.x + v.x;
            a[4 * j + 1] = u.y + v.y;
            a[4 * j + 2] = u.z + v.z;
            a[4 * j + 3] = u.w + v.w;
          }
          // both CTAs read both staged tiles: each frees both
          mbar_arrive(DS_FREE(it));
          mbar_arrive_cluster(mapa_shared(DS_FREE(it), prank ^ 1u));
        } else if constexpr (C::kSDouble) {
          // D = 64: the softmax warpgroup of this tile has staged dQp in its dS buffer
          wait(DQ_EMPTY(it), s_phase(it));
          if (threadIdx.x == 256) trace(it, 4);
          const uint32_t stage = sDSt + 32768u * (uint32_t)(it & 1);
#pragma unroll
          for (int j = 0; j < D / 4; ++j) {
            const float4 v = ld_shared_f4(stage + (uint32_t)((j * 128 + r) * 16));
            a[4 * j] = v.x;
            a[4 * j + 1] = v.y;
            a[4 * j + 2] = v.z;
            a[4 * j + 3] = v.w;
          }
          mbar_arrive(DS_FREE(it));
        } else {
          wait(DQ_FULL(it), s_phase(it));
          if (threadIdx.x == 256) trace(it, 4);
          tc_fence_after();
#pragma unroll
          for (int c2 = 0; c2 < D / 32; ++c2) {
            uint32_t v[32];
            tmem_ld32(tmem + lane_off + dq_col(it) + c2 * 32, v);
#pragma unroll
            for (int j = 0; j < 32; ++j) a[c2 * 32 + j] = __uint_as_float(v[j]);
          }
          tc_fence_before();
          mbar_arrive(DQ_EMPTY(it));
          if constexpr (kPair) {
            // this CTA's half of the row in a[0, D/2), the peer's half in a[D/2, D)
#pragma unroll
            for (int j = 0; j < D / 2; ++j) {
              const float lo = a[j], hi = a[D / 2 + j];
              a[j] = prank ? hi : lo;
              a[D / 2 + j] = prank ? lo : hi;
            }
            const uint32_t xb = sb + C::OFF_XB;
            const uint32_t pxb = mapa_shared(xb, prank ^ 1u);
#pragma unroll
            for (int k = 0; k < D / 64; ++k) {
              const int R = (D / 64) * it + k;  // exchange round
              // the peer has read round R - 1 out of its buffer
              if (R >= 1)
                mbar_wait_cluster(BAR(B_PEER1), (uint32_t)((R - 1) & 1), lim, p.err,
                                  p.abort_flag);
#pragma unroll
              for (int g = 0; g < 8; ++g) {
                const float* x = a + D / 2 + 32 * k + 4 * g;
                st_shared_cluster_f4(pxb + (uint32_t)((g * 128 + r) * 16),
                                     make_float4(x[0], x[1], x[2], x[3]));
              }
              mbar_arrive_cluster(mapa_shared(BAR(B_PEER0), prank ^ 1u));
              // the peer's columns of this CTA's half, round R
              mbar_wait_cluster(BAR(B_PEER0), (uint32_t)(R & 1), lim, p.err, p.abort_flag);
#pragma unroll
              for (int g = 0; g < 8; ++g) {
                const float4 v = ld_shared_f4(xb + (uint32_t)((g * 128 + r) * 16));
                float* x = a + 32 * k + 4 * g;
                x[0] = x[0] + v.x;
                x[1] = x[1] + v.y;
                x[2] = x[2] + v.z;
                x[3] = x[3] + v.w;
              }
              mbar_arrive_cluster(mapa_shared(BAR(B_PEER1), prank ^ 1u));
            }
          }
        }
        if (threadIdx.x == 256) trace(it, 5);
        const long long blk = (long long)ch.x * N + q;
        if constexpr (!kAtomic) {
          // Two accumulation chains per dQ block: the contributions at even and at
          // odd positions each add, in position order, into an fp32 accumulator of
          // their own, so consecutive contributors to a block do not wait on each
          // other.  The block's last contributor adds the two chain sums.
          const int chain = pos & 1, idx = pos >> 1;
          // CTA pairs: one chain per (block, half of the columns, parity), 128 x D/2 fp32
          auto unit_of = [&](int ch_) -> long long {
            return kPair ? (blk * 2 + (long long)prank) * 2 + ch_ : blk * 2 + ch_;
          };
          const long long unit = unit_of(chain);
          float4* accp = reinterpret_cast<float4*>(p.acc) + unit * (128 * NA);
          // wait (bounded) until a chain's ticket reaches `want`.  Lane 0 acquires
          // (its acquire pairs with the publisher's release) and the warp barrier
          // orders the other lanes' accumulator loads after it.  `seen` is a value
          // lane 0 already acquired (~0u: none).
          auto ticket_wait = [&](uint32_t* tk, uint32_t want, uint32_t seen) {
            if (lane == 0) {
              if (seen != want && ld_acquire_gpu(tk) != want) {
                const uint64_t t0 = globaltimer();
                bool ok = false;
                while (!ok) {
#pragma unroll 1
                  for (int i = 0; i < 32 && !ok; ++i) ok = (ld_acquire_gpu(tk) == want);
                  if (!ok && (aborted(p.abort_flag) || globaltimer() - t0 > lim)) {
                    if (!aborted(p.abort_flag)) raise_timeout(p.err, p.abort_flag, ERR_WHERE_TICKET);
                    break;
                  }
                }
              }
            }
            __syncwarp();
          };
          // a = acc + a over this thread's NA slots, up to G loads in flight before their
          // adds (the last group holds the remaining NA mod G slots)
          auto add_from = [&](const float4* src) {
#pragma unroll
            for (int g0 = 0; g0 < NA; g0 += G) {
              float4 old[G];
#pragma unroll
              for (int j = 0; j < G; ++j)
                if (g0 + j < NA) old[j] = ld_cg_f4_hint(src + (g0 + j) * 128 + r, pol_last);
#pragma unroll
              for (int j = 0; j < G; ++j) {
                if (g0 + j < NA) {
                  float* x = a + 4 * (g0 + j);
                  x[0] = old[j].x + x[0];
                  x[1] = old[j].y + x[1];
                  x[2] = old[j].z + x[2];
                  x[3] = old[j].w + x[3];
                }
              }
            }
          };
          if constexpr (kRed) {
            // middle positions add with red in L2 below; only the last one loads
            if (idx > 0 && last) {
              if (threadIdx.x == 256) trace(it, 14);
              ticket_wait(p.tickets + unit, (uint32_t)idx, ~0u);
              if (threadIdx.x == 256) trace(it, 6);
              add_from(accp);
            }
          } else if constexpr (kLook) {
            if (idx > 0) {
              if (!pre_ok) {
                if (threadIdx.x == 256) trace(it, 14);
                ticket_wait(p.tickets + unit, (uint32_t)idx, ~0u);
                if (threadIdx.x == 256) trace(it, 6);
#pragma unroll
                for (int j = 0; j < NV; ++j) pre[j] = ld_cg_f4_hint(accp + j * 128 + r, pol_last);
              }
#pragma unroll
              for (int j = 0; j < NV; ++j) {
                float* x = a + 4 * j;
                x[0] = pre[j].x + x[0];
                x[1] = pre[j].y + x[1];
                x[2] = pre[j].z + x[2];
                x[3] = pre[j].w + x[3];
              }
            }
          } else if (idx > 0) {
            if (threadIdx.x == 256) trace(it, 14);
            ticket_wait(p.tickets + unit, (uint32_t)idx, ~0u);
            if (threadIdx.x == 256) trace(it, 6);
            add_from(accp);
          }
          if (last) {
            if (ncontrib > 1) {
              // the other chain is complete once its ticket counts all its positions
              const int other = chain ^ 1;
              const long long ounit = unit_of(other);
              ticket_wait(p.tickets + ounit, (uint32_t)((ncontrib + 1 - other) / 2), ~0u);
              add_from(reinterpret_cast<const float4*>(p.acc) + ounit * (128 * NA));
            }
            // CTA pairs: this CTA's half of the columns
            __nv_bfloat16* out = p.dq + ((size_t)ch.x * S + (size_t)q * 128 + r) * D +
                                 (kPair ? (size_t)prank * (D / 2) : 0);
            const float sc = p.scale;
#pragma unroll
            for (int c8 = 0; c8 < NA / 2; ++c8) {
              const float* x = a + 8 * c8;
              uint4 pk;
              pk.x = pack_bf16x2(x[0] * sc, x[1] * sc);
              pk.y = pack_bf16x2(x[2] * sc, x[3] * sc);
              pk.z = pack_bf16x2(x[4] * sc, x[5] * sc);
              pk.w = pack_bf16x2(x[6] * sc, x[7] * sc);
              *reinterpret_cast<uint4*>(out + 8 * c8) = pk;
            }
          } else {
            if (kRed && idx > 0) {
              // Once the ticket shows every earlier position's additions performed, this
              // partial is added in L2 (red, no read back); the release below waits for
              // these additions to be performed, so the chain's order is kept.
              if (threadIdx.x == 256) trace(it, 14);
              ticket_wait(p.tickets + unit, (uint32_t)idx, ~0u);
              if (threadIdx.x == 256) trace(it, 6);
#pragma unroll
              for (int c4 = 0; c4 < NA; ++c4)
                red_add_f4_hint(accp + c4 * 128 + r,
                                make_float4(a[4 * c4], a[4 * c4 + 1], a[4 * c4 + 2], a[4 * c4 + 3]),
                                pol_last);
            } else {
#pragma unroll
              for (int c4 = 0; c4 < NA; ++c4)
                st_cg_f4_hint(accp + c4 * 128 + r,
                              make_float4(a[4 * c4], a[4 * c4 + 1], a[4 * c4 + 2], a[4 * c4 + 3]),
                              pol_last);
            }
            if (threadIdx.x == 256) trace(it, 13);
            if constexpr (C::kPublisher) {
              // hand the publication of these stores to the publisher warp (slot k mod 2,
              // free again once it has published pair k - 2)
              if (npub >= 2) wait(BAR(B_PUB_FREE0 + (npub & 1)), ((npub - 2) >> 1) & 1);
              mbar_arrive(BAR(B_PUB_READY0 + (npub & 1)));
              ++npub;
            } else {
              // the barrier orders every thread's stores before thread 256's release,
              // which publishes them at gpu scope
              named_bar_sync(1, 128);
              if (threadIdx.x == 256) st_release_gpu(p.tickets + unit, (uint32_t)(idx + 1));
            }
          }
          if constexpr (kLook) {
            // the next pair (possibly in a later chain of this CTA): if its ticket is
            // already granted, its accumulator loads go out now
            pre_ok = false;
            int nci = ci, nt = t + 1;
            while (nci < cend && nt >= n_pairs(p.chains[nci].w)) {
              ++nci;
              nt = 0;
            }
            if (nci < cend) {
              const int4 nch = p.chains[nci];
              const uint32_t nw = p.pairs[nch.z + nt];
              const int npos = (int)(nw >> 16);
              if ((npos >> 1) > 0) {
                const long long nunit =
                    ((long long)nch.x * N + (int)(nw & 0xffffu)) * 2 + (npos & 1);
                // lane 0 acquires (pairing with the publisher's release); the warp
                // barrier orders the other lanes' loads after it
                uint32_t okw = 0;
                if (lane == 0)
                  okw = ld_acquire_gpu(p.tickets + nunit) == (uint32_t)(npos >> 1) ? 1u : 0u;
                pre_ok = __shfl_sync(0xffffffffu, okw, 0) != 0u;
                __syncwarp();
                if (pre_ok) {
                  const float4* nacc = reinterpret_cast<const float4*>(p.acc) + nunit * (32 * D);
#pragma unroll
                  for (int j = 0; j < NV; ++j) pre[j] = ld_cg_f4_hint(nacc + j * 128 + r, pol_last);
                }
              }
            }
          }
        } else {
          float4* accp = reinterpret_cast<float4*>(p.acc + blk * 128 * D);
#pragma unroll
          for (int c4 = 0; c4 < NV; ++c4)
            atomicAdd(accp + c4 * 128 + r,
                      make_float4(a[4 * c4], a[4 * c4 + 1], a[4 * c4 + 2], a[4 * c4 + 3]));
          if (threadIdx.x == 256) trace(it, 13);
        }
        if (threadIdx.x == 256 && (kAtomic || last || !C::kPublisher)) trace(it, 7);
      }
      // run epilogue: dV_j and scale * dK_j (rows of KV tile ch.y of the chain's K/V
      // head) to global bf16, after the run's last chain
      if (ch.w & kChainContNext) continue;
      wait(BAR(B_DKDV_FULL), (fn++) & 1);
      tc_fence_after();
      const size_t row = (size_t)(ch.x >> gl2) * S + (size_t)ch.y * 128 + r;
      if (p.split_log2 > 0) {
        // This run is sub-group s of its K/V head's group: it adds its dK/dV partials
        // to the fp32 accumulator after sub-group s - 1 (an ordered load-add-store
        // under the tile's ticket, as for dQ), and sub-group sp - 1 rounds to bf16.
        // (A wait-free variant, where the last sub-group to finish adds every slot,
        // made the whole kernel slower, also without a split.)
        const int sp = 1 << p.split_log2;
        const int s = (ch.x >> (gl2 - p.split_log2)) & (sp - 1);
        const long long unit = (long long)(ch.x >> gl2) * N + ch.y;
        float4* acc = reinterpret_cast<float4*>(p.dkv_acc) + unit * (2 * 32 * D);
        uint32_t* tk = p.dkv_tickets + unit;
        if (s > 0) {
          // bounded wait: lane 0 acquires, the warp barrier orders the lanes' loads
          if (lane == 0 && ld_acquire_gpu(tk) != (uint32_t)s) {
            const uint64_t t0 = globaltimer();
            bool ok = false;
            while (!ok) {
#pragma unroll 1
              for (int i = 0; i < 32 && !ok; ++i) ok = (ld_acquire_gpu(tk) == (uint32_t)s);
              if (!ok && (aborted(p.abort_flag) || globaltimer() - t0 > lim)) {
                if (!aborted(p.abort_flag)) raise_timeout(p.err, p.abort_flag, ERR_WHERE_TICKET);
                break;
              }
            }
          }
          __syncwarp();
        }
#pragma unroll 1
        for (int which = 0; which < 2; ++which) {
          const uint32_t col = which ? C::TM_DK : C::TM_DV;
          const float sc = which ? p.scale : 1.0f;
          __nv_bfloat16* out = (which ? p.dk : p.dv) + row * D;
          float4* a = acc + which * 32 * D;
#pragma unroll
          for (int c2 = 0; c2 < D / 32; ++c2) {
            uint32_t v[32];
            tmem_ld32(tmem + lane_off + col + c2 * 32, v);
            float x[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) x[j] = __uint_as_float(v[j]);
            if (s > 0) {
              float4 old[8];
#pragma unroll
              for (int j = 0; j < 8; ++j) old[j] = ld_cg_f4(a + (c2 * 8 + j) * 128 + r);
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                x[4 * j] = old[j].x + x[4 * j];
                x[4 * j + 1] = old[j].y + x[4 * j + 1];
                x[4 * j + 2] = old[j].z + x[4 * j + 2];
                x[4 * j + 3] = old[j].w + x[4 * j + 3];
              }
            }
            if (s < sp - 1) {
#pragma unroll
              for (int j = 0; j < 8; ++j)
                st_cg_f4(a + (c2 * 8 + j) * 128 + r,
                         make_float4(x[4 * j], x[4 * j + 1], x[4 * j + 2], x[4 * j + 3]));
            } else {
#pragma unroll
              for (int c8 = 0; c8 < 4; ++c8) {
                uint4 pk;
                pk.x = pack_bf16x2(x[8 * c8] * sc, x[8 * c8 + 1] * sc);
                pk.y = pack_bf16x2(x[8 * c8 + 2] * sc, x[8 * c8 + 3] * sc);
                pk.z = pack_bf16x2(x[8 * c8 + 4] * sc, x[8 * c8 + 5] * sc);
                pk.w = pack_bf16x2(x[8 * c8 + 6] * sc, x[8 * c8 + 7] * sc);
                *reinterpret_cast<uint4*>(out + c2 * 32 + c8 * 8) = pk;
              }
            }
          }
        }
        tc_fence_before();
        mbar_arrive(BAR(B_DKDV_EMPTY));
        if (s < sp - 1) {
          // every reducer's stores precede thread 256's release, which publishes them
          named_bar_sync(1, 128);
          if (threadIdx.x == 256) st_release_gpu(tk, (uint32_t)(s + 1));
        }
        continue;
      }
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        const uint32_t col = which ? C::TM_DK : C::TM_DV;
        const float sc = which ? p.scale : 1.0f;
        __nv_bfloat16* out = (which ? p.dk : p.dv) + row * D;
#pragma unroll
        for (int c2 = 0; c2 < D / 32; ++c2) {
          uint32_t v[32];
          tmem_ld32(tmem + lane_off + col + c2 * 32, v);
#pragma unroll
          for (int c8 = 0; c8 < 4; ++c8) {
            uint4 pk;
            pk.x = pack_bf16x2(__uint_as_float(v[8 * c8]) * sc, __uint_as_float(v[8 * c8 + 1]) * sc);
            pk.y = pack_bf16x2(__uint_as_float(v[8 * c8 + 2]) * sc, __uint_as_float(v[8 * c8 + 3]) * sc);
            pk.z = pack_bf16x2(__uint_as_float(v[8 * c8 + 4]) * sc, __uint_as_float(v[8 * c8 + 5]) * sc);
            pk.w = pack_bf16x2(__uint_as_float(v[8 * c8 + 6]) * sc, __uint_as_float(v[8 * c8 + 7]) * sc);
            *reinterpret_cast<uint4*>(out + c2 * 32 + c8 * 8) = pk;
          }
        }
      }
      tc_fence_before();
      mbar_arrive(BAR(B_DKDV_EMPTY));
    }
  }

  tc_fence_before();
  __syncthreads();
  // CTA pairs: neither CTA leaves while the other may still read its shared memory or
  // arrive on its barriers
  if constexpr (kPair) cluster_sync_all();
  if (warp == 13) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace dash
