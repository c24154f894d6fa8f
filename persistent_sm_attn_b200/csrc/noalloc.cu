// dash_attn_bwd_noalloc: the backward pass without any device allocation.
//
// Some callers cannot call cudaMalloc: runtimes that own all device memory
// through their own pool and forbid allocations outside it, and embedded or
// certified deployments that must fix their whole device footprint before
// they start.  This entry point runs the same kernels as dash_attn_bwd, but
// takes every byte of scratch memory (the fp32 dQ accumulators, the tickets,
// the per-row LSE and Delta terms, the error words and the schedule table)
// from one statically allocated device array of kNoallocScratchBytes.  Every
// device that loads the library holds that array until the process exits.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <string>

#include "../../include/dash_attn.h"
#include "aux_kernels.cuh"
#include "bwd_kernel.cuh"
#include "internal.h"
#include "sched.h"

namespace {

constexpr size_t kNoallocScratchBytes = size_t(DASH_NOALLOC_SCRATCH_BYTES);
constexpr int kMaxDevices = 64;

// The scratch array.  In host code `g_noalloc_scratch` names a host-side
// stand-in, not device memory: its device address is obtained once per device
// with cudaGetSymbolAddress and passed to the kernels.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

struct DeviceState {
  bool ready = false;
  unsigned char* base = nullptr;  // device address of g_noalloc_scratch on this device
  int ctas[2][2] = {{0, 0}, {0, 0}};  // [D==128][atomic]
  // key of the schedule table currently held in the scratch array
  long long table_key[7] = {-1, -1, -1, -1, -1, -1, -1};
};
DeviceState g_dev[kMaxDevices];
std::mutex g_noalloc_mu;

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn noalloc_encode_fn() {
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

// [rows][8] bf16 column terms: an 8 x 128 box without swizzle (core-matrix layout).
int noalloc_tmap_cols(CUtensorMap* m, const void* base, long long rows) {
  EncodeTiledFn fn = noalloc_encode_fn();
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

int noalloc_tmap(CUtensorMap* m, const void* base, long long rows, int D, int box_rows) {
  EncodeTiledFn fn = noalloc_encode_fn();
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

template <int D, bool kAtomic>
int noalloc_ctas(int dev) {
  using C = dash::BwdCfg<D>;
  auto kern = dash::dash_bwd_kernel<D, kAtomic>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) !=
      cudaSuccess)
    return -DASH_ERR_CUDA;
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return -DASH_ERR_CUDA;
  if (fa.numRegs != C::kLaunchRegs) return -DASH_ERR_UNSUPPORTED;
  int per_sm = 0, sms = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, C::kThreads, C::kSmemBytes) !=
          cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return -DASH_ERR_CUDA;
  if (per_sm < 1) return -DASH_ERR_UNSUPPORTED;
  return per_sm * sms;
}

// Once per device, with that device current: the scratch array's device
// address and the persistent grid sizes.
int noalloc_setup(int dev, DeviceState** out) {
  DeviceState& st = g_dev[dev];
  if (!st.ready) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) {
      cudaGetLastError();
      return DASH_ERR_CUDA;
    }
    st.base = static_cast<unsigned char*>(ptr);
    const int c[4] = {noalloc_ctas<64, false>(dev), noalloc_ctas<64, true>(dev),
                      noalloc_ctas<128, false>(dev), noalloc_ctas<128, true>(dev)};
    for (int i = 0; i < 4; ++i)
      if (c[i] < 0) return -c[i];
    st.ctas[0][0] = c[0];
    st.ctas[0][1] = c[1];
    st.ctas[1][0] = c[2];
    st.ctas[1][1] = c[3];
    st.ready = true;
  }
  *out = &st;
  return DASH_OK;
}


// Scratch bytes a call needs, table excluded.
size_t fixed_scratch(long long rows, int D, long long blocks) {
  return 256                                         // error word + abort flag
         + align256((size_t)blocks * 4)              // tickets
         + align256((size_t)rows * 16)               // per-row column terms (LSE, Delta)
         + align256(2 * (size_t)rows * D * 4);       // fp32 dQ accumulators (two per block)
}

template <int D, bool kAtomic>
int noalloc_launch(const void* q, const void* k, const void* v, const void* o, const void* dout,
                   const float* lse, void* dq, void* dk, void* dv, int B, int H, int S,
                   int causal, int sched, cudaStream_t stream, DeviceState* st) {
  using C = dash::BwdCfg<D>;
  const int N = S / 128;
  const long long rows = (long long)B * H * S;
  const long long blocks = dash::dq_units<D>((long long)B * H * N);  // tickets (reduction units)
  const int ctas = st->ctas[D == 128][kAtomic ? 1 : 0];
  // lay out the scratch array
  unsigned char* p0 = st->base;
  unsigned* err = reinterpret_cast<unsigned*>(p0);
  size_t off = 256;
  uint32_t* tickets = reinterpret_cast<uint32_t*>(p0 + off);
  off += align256((size_t)blocks * 4);
  uint4* cols = reinterpret_cast<uint4*>(p0 + off);
  off += align256((size_t)rows * 16);
  float* acc = reinterpret_cast<float*>(p0 + off);
  off += align256(2 * (size_t)rows * D * 4);
  // the schedule table, built and checked on the host, then copied in.  A fault armed
  // with dash_inject_fault replaces it, for this call only, by a table whose dQ block
  // (head 0, Q tile 0) never receives its first partials.
  // the allocating entry point's table (heads interleaved the same way), so the two
  // add every dQ block in the same order
  const int il =
      dash::head_interleave(D, sched, B * H, N, causal, ctas, dash::head_interleave_mode());
  const long long key[7] = {B * (long long)H, N, causal, sched, ctas, (long long)off, il};
  const int fault = kAtomic ? 0 : dash::take_armed_fault();
  dash::Table t;
  std::string msg;
  if (!dash::build_table_grouped(B * H, il, N, causal, sched, ctas, &t, &msg))
    return DASH_ERR_UNSUPPORTED;
  if (fault == 1) dash::plant_missing_first_partials(&t);
  const size_t off_cta = off;
  const size_t off_chain = off_cta + align256(t.cta_off.size() * sizeof(int));
  const size_t off_pair = off_chain + align256(t.chains.size() * sizeof(int4));
  const size_t end = off_pair + align256(t.pairs.size() * sizeof(uint32_t));
  if (end > kNoallocScratchBytes) return DASH_ERR_OOM;
  if (fault == 1 || std::memcmp(key, st->table_key, sizeof(key)) != 0) {
    // A capturing stream would record the upload as a copy from host memory that is
    // gone when the graph runs: a new table is only uploaded outside capture.
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) {
      cudaGetLastError();
      return DASH_ERR_CUDA;
    }
    if (cap != cudaStreamCaptureStatusNone) return DASH_ERR_UNSUPPORTED;
    if (fault != 1 && !dash::validate_table(t, &msg)) return DASH_ERR_SCHEDULE;
    if (cudaMemcpyAsync(p0 + off_cta, t.cta_off.data(), t.cta_off.size() * sizeof(int),
                        cudaMemcpyHostToDevice, stream) != cudaSuccess ||
        cudaMemcpyAsync(p0 + off_chain, t.chains.data(), t.chains.size() * sizeof(int4),
                        cudaMemcpyHostToDevice, stream) != cudaSuccess ||
        cudaMemcpyAsync(p0 + off_pair, t.pairs.data(), t.pairs.size() * sizeof(uint32_t),
                        cudaMemcpyHostToDevice, stream) != cudaSuccess)
      return DASH_ERR_CUDA;
    // after a planted fault the next call uploads its table again
    if (fault == 1)
      for (long long& x : st->table_key) x = -1;
    else
      std::memcpy(st->table_key, key, sizeof(key));
  }
  CUtensorMap tq, tk, tv, tdo, tc;
  int rc;
  if ((rc = noalloc_tmap(&tq, q, rows, D, C::kQRows)) ||
      (rc = noalloc_tmap(&tk, k, rows, D, C::kKVRows)) ||
      (rc = noalloc_tmap(&tv, v, rows, D, C::kKVRows)) ||
      (rc = noalloc_tmap(&tdo, dout, rows, D, C::kQRows)) ||
      (rc = noalloc_tmap_cols(&tc, cols, rows)))
    return rc;
  const float scale = 1.0f / sqrtf((float)D);
  // The array keeps the previous call's contents: the Delta launch clears the abort
  // flag and (deterministic path) the tickets; the atomic variant's accumulator is
  // cleared here.  The error word (err[0]) keeps what earlier calls recorded until
  // dash_attn_noalloc_sync_status reads and clears it.
  if (kAtomic && cudaMemsetAsync(acc, 0, (size_t)rows * D * 4, stream) != cudaSuccess)
    return DASH_ERR_CUDA;
  dash::dash_delta_kernel<D><<<dash::delta_grid<D>(rows, ctas), 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dout), lse, cols,
      rows, 1.0f / scale, tickets, kAtomic ? 0LL : blocks, err + 1, 1);
  dash::BwdParams p;
  p.cta_off = reinterpret_cast<const int*>(p0 + off_cta);
  p.chains = reinterpret_cast<const int4*>(p0 + off_chain);
  p.pairs = reinterpret_cast<const uint32_t*>(p0 + off_pair);
  p.acc = acc;
  p.tickets = tickets;
  p.err = err;
  p.abort_flag = err + 1;
  p.dq = static_cast<__nv_bfloat16*>(dq);
  p.dk = static_cast<__nv_bfloat16*>(dk);
  p.dv = static_cast<__nv_bfloat16*>(dv);
  p.S = S;
  p.N = N;
  p.causal = causal;
  p.group_log2 = 0;
  p.scale = scale;
  p.scale_log2 = p.scale * 1.4426950408889634f;
  p.spin_ns = (unsigned long long)dash::spin_limit_us() * 1000ull;
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
  if (cudaLaunchKernelEx(&cfg, dash::dash_bwd_kernel<D, kAtomic>, tq, tk, tv, tdo, tc, p) !=
      cudaSuccess)
    return DASH_ERR_CUDA;
  if (kAtomic) {
    const long long n_blocks = (long long)B * H * N;  // 128-row accumulator blocks
    const long long threads = n_blocks * 32 * D;
    dash::dash_dq_convert<D><<<(int)((threads + 255) / 256), 256, 0, stream>>>(
        acc, static_cast<__nv_bfloat16*>(dq), n_blocks, p.scale);
  }
  return cudaGetLastError() == cudaSuccess ? DASH_OK : DASH_ERR_CUDA;
}

bool aligned16(const void* ptr) { return ptr && (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

}  // namespace

extern "C" int dash_attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                                     const void* dout, const float* lse, void* dq, void* dk,
                                     void* dv, int B, int H, int S, int D, int causal,
                                     int schedule, void* stream) {
  if (B < 0 || H < 0 || S < 0 || D < 0) return DASH_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return DASH_ERR_INVALID_ARG;
  if (schedule < DASH_SCHED_NAIVE_ASC || schedule > DASH_SCHED_SYM_SHIFT_PAIRS)
    return DASH_ERR_INVALID_ARG;
  if (schedule == DASH_SCHED_SHIFT_PAIRS || schedule == DASH_SCHED_SYM_SHIFT_PAIRS)
    return DASH_ERR_UNSUPPORTED;  // dash_attn_bwd only
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) ||
      !aligned16(lse) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return DASH_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return DASH_ERR_UNSUPPORTED;
  if (S == 0 || S % 128 != 0 || S / 128 > 32767) return DASH_ERR_UNSUPPORTED;
  if ((long long)B * H * S >= (1LL << 31)) return DASH_ERR_UNSUPPORTED;
  if (!dash::schedule_supported(schedule, S / 128, causal)) return DASH_ERR_UNSUPPORTED;
  if (B == 0 || H == 0) return DASH_OK;
  // reject sizes beyond the array before touching the device
  const long long rows = (long long)B * H * S, blocks = 2LL * B * H * (S / 128);
  if (fixed_scratch(rows, D, blocks) > kNoallocScratchBytes) return DASH_ERR_OOM;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DASH_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return DASH_ERR_UNSUPPORTED;
  // the table is built in host containers: no C++ exception may leave this function
  return dash::no_throw([&]() -> int {
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    DeviceState* st = nullptr;
    int rc = noalloc_setup(dev, &st);
    if (rc) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool atomic = (schedule == DASH_SCHED_ATOMIC);
    if (D == 64)
      return atomic ? noalloc_launch<64, true>(q, k, v, o, dout, lse, dq, dk, dv, B, H, S,
                                               causal, schedule, s, st)
                    : noalloc_launch<64, false>(q, k, v, o, dout, lse, dq, dk, dv, B, H, S,
                                                causal, schedule, s, st);
    return atomic ? noalloc_launch<128, true>(q, k, v, o, dout, lse, dq, dk, dv, B, H, S,
                                              causal, schedule, s, st)
                  : noalloc_launch<128, false>(q, k, v, o, dout, lse, dq, dk, dv, B, H, S,
                                               causal, schedule, s, st);
  }, DASH_ERR_OOM, DASH_ERR_INVALID_ARG);
}

extern "C" int dash_attn_noalloc_sync_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return DASH_ERR_CUDA;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DASH_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return DASH_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  const DeviceState& st = g_dev[dev];
  if (!st.ready) return DASH_OK;  // no call has run on this device
  unsigned h = 0;
  if (cudaMemcpy(&h, st.base, sizeof(unsigned), cudaMemcpyDeviceToHost) != cudaSuccess)
    return DASH_ERR_CUDA;
  if (h == 0) return DASH_OK;
  if (cudaMemset(st.base, 0, sizeof(unsigned)) != cudaSuccess) return DASH_ERR_CUDA;
  return (h & dash::dev::ERR_TIMEOUT) ? DASH_ERR_TIMEOUT : DASH_ERR_UNSUPPORTED;
}
