// Attention forward for sm_100a: O = softmax(scale Q K^T + mask) V and the row
// log-sum-exp, which the backward takes as inputs.
//
// One CTA per (head, 128-row Q tile), launched heaviest tile first.  Per KV tile j
// of 128 rows:
//
//   S_j  = Q K_j^T        tcgen05.mma (smem x smem) -> TMEM, two buffers [0,128) [128,256)
//   P_j  = 2^(s S_j - m)  softmax warpgroup, thread = Q row = TMEM lane, packed bf16 back
//                         into S_j's columns (the layout the backward uses for P^T)
//   O   += P_j V_j        tcgen05.mma with A = P_j in TMEM -> TMEM [256, 256 + D)
//
// with s = scale log2(e) and m the row's running maximum of s S in the log2 domain.
// The running maximum is moved (and O and the running sum rescaled) only when the
// new maximum exceeds the current one by more than kRescaleLog2, so every P stays
// at most 2^kRescaleLog2; the final O / l and LSE = (m + log2 l) ln 2 use the same
// m as the P that were summed, so the result does not depend on when m moved.
//
// Warp roles (256 threads): warp 0 TMA producer, warp 1 MMA issuer and TMEM owner,
// warps 4-7 softmax, rescale and epilogue.  S_j is issued while the softmax works on
// tile j - 1, so the exponentials and the two products overlap.
#pragma once
#include "ptx.cuh"

namespace dash {

struct FwdParams {
  __nv_bfloat16* o;
  float* lse;
  unsigned* err;         // device error word (shared with the backward's workspace)
  unsigned* abort_flag;  // cleared before each launch
  int S, N, BH, causal;
  int group;             // query heads per K/V head
  float scale_log2;      // scale * log2(e)
  unsigned long long spin_ns;
};

template <int D>
struct FwdCfg {
  static constexpr int kThreads = 256;
  static constexpr int kTile = 128 * D * 2;               // one [128][D] bf16 tile
  static constexpr int kStages = 3;                         // K/V stages (224 KiB at D = 128)
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + kTile;
  static constexpr int OFF_V = OFF_K + kStages * kTile;
  static constexpr int OFF_BAR = OFF_V + kStages * kTile;
  static constexpr int kBars = 8 + 2 * kStages;
  static constexpr int OFF_TMEM_SLOT = OFF_BAR + kBars * 8;
  // at least 120 KiB, so one CTA runs per SM and its 512 TMEM columns are free
  static constexpr int kNeed = OFF_TMEM_SLOT + 16;
  static constexpr int kSmemBytes = kNeed > 122880 ? kNeed : 122880;
  static_assert(kSmemBytes <= 232448, "shared memory per block exceeded");
  static constexpr uint32_t TM_S = 0, TM_O = 256;
  static constexpr float kRescaleLog2 = 8.0f;
};

enum {
  F_Q_FULL = 0, F_S_FULL0, F_S_FULL1, F_P_READY0, F_P_READY1, F_PV_DONE0, F_PV_DONE1, F_O_FINAL,
  F_STAGE0 = 8
};

template <int D>
__global__ void __launch_bounds__(256, 1)
    dash_fwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  using namespace dev;
  using C = FwdCfg<D>;
  constexpr int KST = C::kStages;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t sb = smem_u32(smem_raw);
  if (sb & 1023u) {
    if (threadIdx.x == 0) {
      atomicOr(p.err, ERR_MISALIGNED);
      atomicOr(p.abort_flag, 1u);
    }
    return;
  }
  const uint32_t sQ = sb + C::OFF_Q, sK = sb + C::OFF_K, sV = sb + C::OFF_V;
  const uint32_t bar0 = sb + C::OFF_BAR;
  auto BAR = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  auto KV_FULL = [&](int s) { return BAR(F_STAGE0 + s); };
  auto KV_EMPTY = [&](int s) { return BAR(F_STAGE0 + KST + s); };
  auto S_FULL = [&](int j) { return BAR(F_S_FULL0 + (j & 1)); };
  auto P_READY = [&](int j) { return BAR(F_P_READY0 + (j & 1)); };
  auto PV_DONE = [&](int j) { return BAR(F_PV_DONE0 + (j & 1)); };
  auto ph2 = [&](int j) { return (uint32_t)((j >> 1) & 1); };  // parity of a two-buffer barrier
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem_raw + C::OFF_TMEM_SLOT);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint64_t lim = p.spin_ns;
  auto wait = [&](uint32_t bar, uint32_t phase) { mbar_wait(bar, phase, lim, p.err, p.abort_flag); };

  const int S = p.S, N = p.N;
  // block t * BH + bh: Q tile N - 1 - t of head bh, so the heaviest (causal) tiles of
  // every head start first
  const int qt = N - 1 - (int)(blockIdx.x / (unsigned)p.BH);
  const int bh = (int)(blockIdx.x % (unsigned)p.BH);
  const int nkv = p.causal ? qt + 1 : N;
  const int row_q = bh * S + qt * 128;

  if (threadIdx.x == 0) {
    mbar_init(BAR(F_Q_FULL), 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(BAR(F_S_FULL0 + b), 1);
      mbar_init(BAR(F_P_READY0 + b), 128);
      mbar_init(BAR(F_PV_DONE0 + b), 1);
    }
    mbar_init(BAR(F_O_FINAL), 1);
    for (int s = 0; s < KST; ++s) {
      mbar_init(KV_FULL(s), 1);
      mbar_init(KV_EMPTY(s), 1);
    }
    fence_mbar_init();
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------------- TMA producer
    mbar_expect_tx(BAR(F_Q_FULL), C::kTile);
#pragma unroll
    for (int cb = 0; cb < D / 64; ++cb) tma_load_2d(sQ + cb * 16384, &tmQ, cb * 64, row_q, BAR(F_Q_FULL));
    for (int j = 0; j < nkv; ++j) {
      const int s = j % KST;
      if (j >= KST) wait(KV_EMPTY(s), (uint32_t)(((j / KST) - 1) & 1));
      mbar_expect_tx(KV_FULL(s), 2 * C::kTile);
      const int row_kv = (bh / p.group) * S + j * 128;
#pragma unroll
      for (int cb = 0; cb < D / 64; ++cb) {
        tma_load_2d(sK + s * C::kTile + cb * 16384, &tmK, cb * 64, row_kv, KV_FULL(s));
        tma_load_2d(sV + s * C::kTile + cb * 16384, &tmV, cb * 64, row_kv, KV_FULL(s));
      }
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------------- MMA issuer
    constexpr uint32_t ID_S = idesc_bf16_f32(128, 128, 0, 0);  // S = Q K^T, both K-major
    constexpr uint32_t ID_PV = idesc_bf16_f32(128, D, 0, 1);   // O += P V, V MN-major
    const uint32_t hi = sdesc_hi(1024);
    const uint32_t kQ = sdesc_lo(sQ, 16);
    const uint32_t tO = tmem + C::TM_O;
    // O += P_i V_i, once the softmax has packed P_i (and rescaled O if it had to)
    auto issue_pv = [&](int i) {
      const int s = i % KST;
      const uint32_t mV = sdesc_lo(sV + s * C::kTile, 16384);
      const uint32_t tP = tmem + C::TM_S + 128u * (uint32_t)(i & 1);
      wait(P_READY(i), ph2(i));
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        tc_mma_ts_w(tO, tP + 32 * (kk >> 1) + 8 * (kk & 1), mV + kk * 128, hi, ID_PV,
                    (i > 0 || kk > 0) ? 1u : 0u);
      tc_commit(PV_DONE(i));
      tc_commit(KV_EMPTY(s));  // K_i (read by S_i, issued earlier) and V_i are free
    };
    wait(BAR(F_Q_FULL), 0);
    for (int j = 0; j < nkv; ++j) {
      const int s = j % KST;
      const uint32_t kK = sdesc_lo(sK + s * C::kTile, 16);
      const uint32_t tSj = tmem + C::TM_S + 128u * (uint32_t)(j & 1);
      wait(KV_FULL(s), (uint32_t)((j / KST) & 1));
      // S_j's buffer held P_{j-2}, which P V_{j-2} must have read
      if (j >= 2) wait(PV_DONE(j - 2), ph2(j - 2));
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (uint32_t)(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
        tc_mma_ss_w(tSj, kQ + off, kK + off, hi, ID_S, kk > 0 ? 1u : 0u);
      }
      tc_commit(S_FULL(j));
      if (j >= 1) issue_pv(j - 1);
    }
    if (nkv > 0) issue_pv(nkv - 1);
    tc_commit(BAR(F_O_FINAL));
    mbar_wait_drain(BAR(F_O_FINAL), 0, lim, p.err, p.abort_flag);
  } else if (warp >= 4) {
    // ---------------------------------------------------------------- softmax
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // Q row of the tile = TMEM lane
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t tO = tmem + lane_off + C::TM_O;
    const float sl2 = p.scale_log2;
    float m = -INFINITY, l = 0.f;
    for (int j = 0; j < nkv; ++j) {
      const uint32_t tS = tmem + lane_off + C::TM_S + 128u * (uint32_t)(j & 1);
      wait(S_FULL(j), ph2(j));
      tc_fence_after();
      // causal: on the diagonal tile KV column c is visible to row r only if c <= r
      const int vis = (p.causal && j == qt) ? r : 127;
      // the row's 128 scores, loaded two chunks at a time with one wait for each pair, and
      // kept in registers for both passes
      uint32_t sv[4][32];
      tmem_ld32x2(tS, tS + 32, sv[0], sv[1]);
      tmem_ld32x2(tS + 64, tS + 96, sv[2], sv[3]);
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int k = 0; k < 32; ++k)
          if (32 * c + k <= vis) mx = fmaxf(mx, __uint_as_float(sv[c][k]));
      const float mt = mx * sl2;
      // move the running maximum when this tile would push P above 2^kRescaleLog2;
      // the decision is per warp (TMEM loads and stores are warp-wide), each lane
      // with its own factor
      if (__any_sync(0xffffffffu, mt > m + C::kRescaleLog2)) {
        const float mn = fmaxf(m, mt);
        if (j > 0) {
          const float f = ex2_approx(m - mn);
          l *= f;
          wait(PV_DONE(j - 1), ph2(j - 1));  // O holds every earlier tile
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t ov[32];
            tmem_ld32(tO + 32 * c, ov);
            uint32_t lo[16], up[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) {
              lo[k] = __float_as_uint(__uint_as_float(ov[k]) * f);
              up[k] = __float_as_uint(__uint_as_float(ov[16 + k]) * f);
            }
            tmem_st16(tO + 32 * c, lo);
            tmem_st16(tO + 32 * c + 16, up);
          }
        }
        m = mn;
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int k = 0; k < 32; k += 2) {
          float p0 = (32 * c + k <= vis) ? ex2_approx(__uint_as_float(sv[c][k]) * sl2 - m) : 0.f;
          float p1 = (32 * c + k + 1 <= vis)
                         ? ex2_approx(__uint_as_float(sv[c][k + 1]) * sl2 - m)
                         : 0.f;
          l += p0 + p1;
          pk[k >> 1] = pack_bf16x2(p0, p1);
        }
        // P_j into the first 16 columns of chunk c of its own buffer (chunk c's scores
        // are already in registers)
        tmem_st16(tS + 32 * c, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(P_READY(j));
    }
    // epilogue: O / l to bf16, LSE = (m + log2 l) ln 2
    wait(BAR(F_O_FINAL), 0);
    tc_fence_after();
    const float inv = 1.0f / l;
    __nv_bfloat16* out = p.o + ((size_t)row_q + r) * D;
#pragma unroll 1
    for (int c = 0; c < D / 32; ++c) {
      uint32_t ov[32];
      tmem_ld32(tO + 32 * c, ov);
#pragma unroll
      for (int c8 = 0; c8 < 4; ++c8) {
        uint4 pk;
        const float* x = reinterpret_cast<const float*>(ov + 8 * c8);
        pk.x = pack_bf16x2(x[0] * inv, x[1] * inv);
        pk.y = pack_bf16x2(x[2] * inv, x[3] * inv);
        pk.z = pack_bf16x2(x[4] * inv, x[5] * inv);
        pk.w = pack_bf16x2(x[6] * inv, x[7] * inv);
        *reinterpret_cast<uint4*>(out + 32 * c + 8 * c8) = pk;
      }
    }
    p.lse[(size_t)row_q + r] = (m + log2f(l)) * 0.69314718055994531f;
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace dash
