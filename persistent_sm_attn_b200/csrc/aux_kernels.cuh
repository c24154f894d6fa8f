// Supporting kernels of the backward path:
//   dash_delta_kernel   Delta_i = sum_d dO_id O_id (fp32), and per row the column
//                       terms the backward's S^T and dP^T products add (LSE_i / scale
//                       and Delta_i, each as three bf16 parts)
//   dash_dq_convert     fp32 accumulator -> bf16 dQ (atomic comparison variant only)
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

namespace dash {

__device__ __forceinline__ void bf16x8_to_f32(uint4 v, float* f) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __bfloat1622float2(h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

// x as three bf16 parts whose fp32 sum is x to about 24 bits: hi = bf16(x),
// mid = bf16(x - hi), lo = bf16(x - hi - mid).
__device__ __forceinline__ void split3_bf16(float x, __nv_bfloat16* part) {
  part[0] = __float2bfloat16_rn(x);
  const float r1 = x - __bfloat162float(part[0]);
  part[1] = __float2bfloat16_rn(r1);
  part[2] = __float2bfloat16_rn(r1 - __bfloat162float(part[1]));
}

// One group of L = D/8 lanes per row; 16-byte loads of O and dO.  Writes cols[row] =
// 8 bf16: -(LSE_row / scale) in three parts, -Delta_row in three parts, two zeros.
// The backward adds them to S^T and dP^T through one extra K-step of each product
// (against constant ones), so S' = S - LSE/scale and dP' = dP - Delta.
// Each thread takes kDeltaRows rows one grid-width apart and issues all their loads
// before any arithmetic, so a grid of a few CTAs per SM keeps enough bytes in flight
// to stream HBM.  The same launch clears the words the backward needs at zero:
// `clear[0..n_clear)` (error words, block 0) and `tickets[0..n_tickets)`.
constexpr int kDeltaRows = 4;
template <int D>
__global__ void __launch_bounds__(256) dash_delta_kernel(const __nv_bfloat16* __restrict__ o,
                                                         const __nv_bfloat16* __restrict__ dout,
                                                         const float* __restrict__ lse,
                                                         uint4* __restrict__ cols, long long rows,
                                                         float inv_scale,
                                                         uint32_t* __restrict__ tickets,
                                                         long long n_tickets,
                                                         unsigned* __restrict__ clear,
                                                         int n_clear) {
  constexpr int L = D / 8;  // lanes per row
  static_assert(32 % L == 0, "a warp holds whole rows");
  const long long nthreads = (long long)gridDim.x * blockDim.x;
  const long long gt = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (blockIdx.x == 0 && threadIdx.x < n_clear) clear[threadIdx.x] = 0u;
  for (long long i = gt; i < n_tickets; i += nthreads) tickets[i] = 0u;
  const long long per_pass = nthreads / L;  // rows one pass covers (blockDim is a multiple of 32)
  const int sub = (int)(gt % L);
  // the loop bound is taken from the warp's first row, so every lane of a warp runs the
  // same iterations and the shuffles below see full warps
  const long long row0 = gt / L, warp_row0 = (gt & ~31LL) / L;
  for (long long base = 0; warp_row0 + base < rows; base += kDeltaRows * per_pass) {
    uint4 ov[kDeltaRows], dv[kDeltaRows];
#pragma unroll
    for (int u = 0; u < kDeltaRows; ++u) {
      const long long row = row0 + base + u * per_pass;
      if (row < rows) {
        ov[u] = reinterpret_cast<const uint4*>(o + row * D)[sub];
        dv[u] = reinterpret_cast<const uint4*>(dout + row * D)[sub];
      } else {
        ov[u] = make_uint4(0u, 0u, 0u, 0u);
        dv[u] = ov[u];
      }
    }
#pragma unroll
    for (int u = 0; u < kDeltaRows; ++u) {
      const long long row = row0 + base + u * per_pass;
      float fo[8], fd[8], acc = 0.f;
      bf16x8_to_f32(ov[u], fo);
      bf16x8_to_f32(dv[u], fd);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc = fmaf(fo[i], fd[i], acc);
#pragma unroll
      for (int m = L / 2; m >= 1; m >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m);
      if (row < rows && sub == 0) {
        __align__(16) __nv_bfloat16 part[8];
        split3_bf16(-lse[row] * inv_scale, part);
        split3_bf16(-acc, part + 3);
        part[6] = part[7] = __float2bfloat16_rn(0.f);
        cols[row] = *reinterpret_cast<const uint4*>(part);
      }
    }
  }
}

// Grid of the Delta kernel: enough CTAs for kDeltaRows rows per thread, at most four
// per SM (what its 64 registers a thread leave resident), so it runs as one wave.
template <int D>
inline int delta_grid(long long rows, int num_sms) {
  const long long need = (rows * (D / 8) + 256LL * kDeltaRows - 1) / (256LL * kDeltaRows);
  const long long cap = 4LL * (num_sms > 0 ? num_sms : 1);
  return (int)(need < 1 ? 1 : (need < cap ? need : cap));
}

// fp32 accumulator -> bf16 dQ.  One accumulator block per 128-row Q tile,
// laid out [D/4][128][4]: slot (c4, r) holds head dims 4*c4..4*c4+3 of row r.
// One thread per float4 slot.
template <int D>
__global__ void __launch_bounds__(256) dash_dq_convert(const float* __restrict__ acc,
                                                       __nv_bfloat16* __restrict__ dq,
                                                       long long n_blocks, float scale) {
  const long long gt = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (gt >= n_blocks * 32 * D) return;
  const int r = (int)(gt % 128);
  const int c4 = (int)((gt / 128) % (D / 4));
  const long long blk = gt / (32 * D);
  const float4 v = reinterpret_cast<const float4*>(acc)[gt];
  __nv_bfloat162 lo = __floats2bfloat162_rn(v.x * scale, v.y * scale);
  __nv_bfloat162 hi = __floats2bfloat162_rn(v.z * scale, v.w * scale);
  uint2 pk;
  pk.x = *reinterpret_cast<uint32_t*>(&lo);
  pk.y = *reinterpret_cast<uint32_t*>(&hi);
  *reinterpret_cast<uint2*>(dq + (blk * 128 + r) * D + 4 * c4) = pk;
}

}  // namespace dash
