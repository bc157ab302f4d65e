// C-ABI launcher for the sm_100a attention forward kernel: argument checks,
// TMA tensor maps, launch configuration and the device status word.
//
// The operation and the ABI contract are documented in include/attn_b200.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <atomic>
#include <mutex>

#include "attn_b200.h"
#include "attn_fwd_kernel.cuh"

namespace attn_b200 {

// Written (first error wins) by kernels whose bounded waits ran out.
__device__ int g_attn_status = 0;

// Work-queue slots: each launch takes the next slot ({next item, CTAs
// finished}); the launch's last CTA resets it to zero.  Launches that run
// at the same time use different slots as long as fewer than kQueueSlots
// of them overlap.
constexpr int kQueueSlots = 256;
__device__ int g_attn_queue[2 * kQueueSlots];

// Scratch of attn_fwd_noalloc: a fixed array this library owns for as long
// as it is loaded (every GPU that loads it keeps these bytes until exit).
// The call needs one work-queue slot ({next item, CTAs finished}, 8 bytes)
// out of it, for any problem size.  Host code must not pass the symbol
// itself to a kernel (on the host it is only a stand-in); each device's
// address comes from cudaGetSymbolAddress in device_state().
constexpr int kNoAllocScratchBytes = 256;
constexpr int kNoAllocQueueBytes = 2 * static_cast<int>(sizeof(int));
static_assert(kNoAllocQueueBytes <= kNoAllocScratchBytes, "queue slot must fit the scratch");
static __device__ __align__(256) int g_attn_noalloc_scratch[kNoAllocScratchBytes / sizeof(int)];

namespace {

constexpr int kMaxDevices = 64;

struct DeviceState {
  bool checked = false;
  bool usable = false;
  int* status = nullptr;  // device address of g_attn_status
  int* queue = nullptr;   // device address of g_attn_queue
  int* noalloc_scratch = nullptr;  // device address of g_attn_noalloc_scratch
  int num_sms = 0;
  std::atomic<unsigned> launches{0};
};

std::mutex g_mu;
DeviceState g_dev[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

// Per-device one-time set-up: capability check and the status word address.
int device_state(DeviceState** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return ATTN_ERR_NO_DEVICE;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState& st = g_dev[dev];
  if (!st.checked) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      return ATTN_ERR_NO_DEVICE;
    }
    st.usable = (major == 10 && minor == 0);
    st.num_sms = sms;
    if (st.usable) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_attn_status) != cudaSuccess) {
        cudaGetLastError();
        return ATTN_ERR_CUDA;
      }
      st.status = static_cast<int*>(p);
      if (cudaGetSymbolAddress(&p, g_attn_queue) != cudaSuccess) {
        cudaGetLastError();
        return ATTN_ERR_CUDA;
      }
      st.queue = static_cast<int*>(p);
      if (cudaGetSymbolAddress(&p, g_attn_noalloc_scratch) != cudaSuccess) {
        cudaGetLastError();
        return ATTN_ERR_CUDA;
      }
      st.noalloc_scratch = static_cast<int*>(p);
    }
    if (!g_encode) {
      cudaDriverEntryPointQueryResult q;
      void* fn = nullptr;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
              cudaSuccess ||
          q != cudaDriverEntryPointSuccess || fn == nullptr) {
        cudaGetLastError();
        return ATTN_ERR_CUDA;
      }
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    st.checked = true;
  }
  if (!st.usable) return ATTN_ERR_NO_DEVICE;
  *out = &st;
  return ATTN_OK;
}

// 3-D view [B*H][N][d] of a [B,H,N,d] bf16 tensor; boxes of 128 rows x 64
// columns of one head, with the 128-byte swizzle the tcgen05 shared-memory
// descriptors expect.  Rows past N of a head are outside the view and read
// as zero, so a tile never picks up the next head's rows.
int make_tmap(CUtensorMap* m, const void* ptr, int BH, int N, int d) {
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                        static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                           static_cast<cuuint64_t>(N) * static_cast<cuuint64_t>(d) * 2};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ATTN_OK : ATTN_ERR_CUDA;
}

bool ranges_overlap(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

template <int D, bool CAUSAL, int kPolyPairs>
int launch(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
           int N, float scale, cudaStream_t stream, DeviceState& st, int* queue = nullptr) {
  using C = Config<D>;
  CUtensorMap tq, tk, tv;
  if (make_tmap(&tq, q, B * H, N, D) || make_tmap(&tk, k, B * H, N, D) ||
      make_tmap(&tv, v, B * H, N, D))
    return ATTN_ERR_CUDA;

  KernelArgs args;
  args.o = static_cast<__nv_bfloat16*>(o);
  args.lse = lse;
  args.N = N;
  args.n_qtiles = (N + kBlockM - 1) / kBlockM;
  args.n_qpairs = (args.n_qtiles + 1) / 2;
  args.BH = B * H;
  args.n_items = args.BH * args.n_qpairs;
  // Scheduling window: enough heads that a window holds about two rounds of
  // items (so its light tail evens out the CTAs), few enough that the
  // window's K/V stays in L2 while its CTAs run.
  {
    const int want = (2 * st.num_sms + args.n_qpairs - 1) / args.n_qpairs;
    args.win_heads = want < 1 ? 1 : (want > args.BH ? args.BH : want);
  }
  args.queue = queue != nullptr
                   ? queue
                   : st.queue + 2 * static_cast<int>(st.launches.fetch_add(1) % kQueueSlots);
  args.scale_log2 = scale * 1.4426950408889634f;
  args.status = st.status;

  auto kern = attn_fwd_kernel<D, CAUSAL, kPolyPairs>;
  // The kernel's register split (setmaxnreg) hands the softmax warpgroups
  // registers released by the producer/MMA warpgroup; it is only valid if
  // the kernel was built with the full per-thread budget it assumes.
  static const bool regs_ok = [&] {
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) {
      cudaGetLastError();
      return false;
    }
    return fa.numRegs * kThreads >= kRegSplitTotal;
  }();
  if (!regs_ok) return ATTN_ERR_CUDA;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) !=
      cudaSuccess) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof cfg);
  // Persistent: one CTA per SM (at most one per work item).
  const int grid = args.n_items < st.num_sms ? args.n_items : st.num_sms;
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = stream;
  if (cudaLaunchKernelEx(&cfg, kern, tq, tk, tv, args) != cudaSuccess) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  return ATTN_OK;
}

// Default share of exponentials computed by the FMA polynomial (pairs per 4):
// measured on B200, the special-function unit alone is fastest for this
// kernel (see the exp2 split sweep in the design notes).
constexpr int kDefaultPolyPairs = 0;

template <int D, bool CAUSAL>
int launch_poly(int poly_pairs, const void* q, const void* k, const void* v, void* o, float* lse,
                int B, int H, int N, float scale, cudaStream_t s, DeviceState& st) {
  switch (poly_pairs) {
    case 0: return launch<D, CAUSAL, 0>(q, k, v, o, lse, B, H, N, scale, s, st);
    case 2: return launch<D, CAUSAL, 2>(q, k, v, o, lse, B, H, N, scale, s, st);
    default: return launch<D, CAUSAL, 1>(q, k, v, o, lse, B, H, N, scale, s, st);
  }
}

int fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N,
             int d, int causal, float scale, int poly_pairs, attn_stream_t stream);

}  // namespace
}  // namespace attn_b200

using namespace attn_b200;

extern "C" int attn_check_args(const void* q, const void* k, const void* v, const void* o,
                               const float* lse, int B, int H, int N, int d, float scale) {
  if (!q || !k || !v || !o || !lse) return ATTN_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || N <= 0) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.f)) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  const uint64_t rows = static_cast<uint64_t>(B) * H * N;
  // Work items (B*H*ceil(N/256)) are numbered in int.
  if (rows >= (1ull << 31)) return ATTN_ERR_UNSUPPORTED;
  const uintptr_t al = reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
                       reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(o);
  if (al & 15u) return ATTN_ERR_MISALIGNED;
  if (reinterpret_cast<uintptr_t>(lse) & 3u) return ATTN_ERR_MISALIGNED;
  const size_t tb = rows * static_cast<size_t>(d) * 2, lb = rows * 4;
  if (ranges_overlap(o, tb, q, tb) || ranges_overlap(o, tb, k, tb) ||
      ranges_overlap(o, tb, v, tb) || ranges_overlap(lse, lb, q, tb) ||
      ranges_overlap(lse, lb, k, tb) || ranges_overlap(lse, lb, v, tb) ||
      ranges_overlap(lse, lb, o, tb))
    return ATTN_ERR_INVALID_ARG;
  return ATTN_OK;
}

namespace attn_b200 {
namespace {
int fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N,
             int d, int causal, float scale, int poly_pairs, attn_stream_t stream) {
  int rc = attn_check_args(q, k, v, o, lse, B, H, N, d, scale);
  if (rc != ATTN_OK) return rc;
  DeviceState* st = nullptr;
  rc = device_state(&st);
  if (rc != ATTN_OK) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (d == 128)
    return causal ? launch_poly<128, true>(poly_pairs, q, k, v, o, lse, B, H, N, scale, s, *st)
                  : launch_poly<128, false>(poly_pairs, q, k, v, o, lse, B, H, N, scale, s, *st);
  return causal ? launch_poly<64, true>(poly_pairs, q, k, v, o, lse, B, H, N, scale, s, *st)
                : launch_poly<64, false>(poly_pairs, q, k, v, o, lse, B, H, N, scale, s, *st);
}
}  // namespace
}  // namespace attn_b200

extern "C" int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                        int H, int N, int d, int causal, float scale, attn_stream_t stream) {
  return fwd_impl(q, k, v, o, lse, B, H, N, d, causal, scale, kDefaultPolyPairs, stream);
}

extern "C" int attn_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                           int H, int N, int d, int causal, float scale, const attn_opts* opts,
                           attn_stream_t stream) {
  int poly = kDefaultPolyPairs;
  if (opts) {
    if (opts->exp2_poly_pairs < -1 || opts->exp2_poly_pairs > 2) return ATTN_ERR_INVALID_ARG;
    if (opts->exp2_poly_pairs >= 0) poly = opts->exp2_poly_pairs;
  }
  return fwd_impl(q, k, v, o, lse, B, H, N, d, causal, scale, poly, stream);
}

// Allocation-free entry point (include/attn_b200.h): same kernel, work
// queue in the library's fixed scratch array, cleared on every call.
extern "C" int attn_fwd_noalloc(const void* q, const void* k, const void* v, void* o, float* lse,
                                int B, int H, int N, int d, int causal, float scale,
                                attn_stream_t stream) {
  int rc = attn_check_args(q, k, v, o, lse, B, H, N, d, scale);
  if (rc != ATTN_OK) return rc;
  DeviceState* st = nullptr;
  rc = device_state(&st);  // first call on a device: resolves the scratch address
  if (rc != ATTN_OK) return rc;
  // The queue counter is a 32-bit int that every CTA pushes once past the
  // last item: items + CTAs must stay representable.
  const int64_t items = static_cast<int64_t>(B) * H * (((N + kBlockM - 1) / kBlockM + 1) / 2);
  if (items + st->num_sms > 0x7FFFFFFFll) return ATTN_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(st->noalloc_scratch, 0, kNoAllocQueueBytes, s) != cudaSuccess) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  int* qs = st->noalloc_scratch;
  if (d == 128)
    return causal ? launch<128, true, kDefaultPolyPairs>(q, k, v, o, lse, B, H, N, scale, s, *st, qs)
                  : launch<128, false, kDefaultPolyPairs>(q, k, v, o, lse, B, H, N, scale, s, *st, qs);
  return causal ? launch<64, true, kDefaultPolyPairs>(q, k, v, o, lse, B, H, N, scale, s, *st, qs)
                : launch<64, false, kDefaultPolyPairs>(q, k, v, o, lse, B, H, N, scale, s, *st, qs);
}

extern "C" int attn_selftest_wait_timeout(int limit_us, attn_stream_t stream) {
  if (limit_us <= 0 || limit_us > 10000000) return ATTN_ERR_INVALID_ARG;
  DeviceState* st = nullptr;
  int rc = device_state(&st);
  if (rc != ATTN_OK) return rc;
  wait_timeout_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      st->status, static_cast<uint64_t>(limit_us) * 1000ull);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  return ATTN_OK;
}

extern "C" int attn_last_device_error(attn_stream_t stream) {
  DeviceState* st = nullptr;
  int rc = device_state(&st);
  if (rc != ATTN_OK) return rc;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  int val = 0;
  const int zero = 0;
  if (cudaMemcpyFromSymbol(&val, g_attn_status, sizeof(int)) != cudaSuccess ||
      cudaMemcpyToSymbol(g_attn_status, &zero, sizeof(int)) != cudaSuccess) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  return val;
}

extern "C" int attn_fwd_host(const void* q_h, const void* k_h, const void* v_h, void* o_h,
                             float* lse_h, void* q_d, void* k_d, void* v_d, void* o_d,
                             float* lse_d, int B, int H, int N, int d, int causal, float scale,
                             attn_stream_t stream) {
  if (!q_h || !k_h || !v_h || !o_h || !lse_h) return ATTN_ERR_INVALID_ARG;
  int rc = attn_check_args(q_d, k_d, v_d, o_d, lse_d, B, H, N, d, scale);
  if (rc != ATTN_OK) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t rows = static_cast<size_t>(B) * H * N;
  const size_t tb = rows * static_cast<size_t>(d) * 2;
  if (cudaMemcpyAsync(q_d, q_h, tb, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(k_d, k_h, tb, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(v_d, v_h, tb, cudaMemcpyHostToDevice, s) != cudaSuccess) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  rc = attn_fwd(q_d, k_d, v_d, o_d, lse_d, B, H, N, d, causal, scale, stream);
  if (rc != ATTN_OK) return rc;
  if (cudaMemcpyAsync(o_h, o_d, tb, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaMemcpyAsync(lse_h, lse_d, rows * 4, cudaMemcpyDeviceToHost, s) != cudaSuccess) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  return attn_last_device_error(stream);
}

extern "C" const char* attn_strerror(int status) {
  switch (status) {
    case ATTN_OK: return "ok";
    case ATTN_ERR_INVALID_ARG: return "invalid argument";
    case ATTN_ERR_UNSUPPORTED: return "unsupported shape (d must be 64 or 128; B*H*N below 2^31)";
    case ATTN_ERR_MISALIGNED: return "misaligned pointer (q, k, v, o need 16 bytes, lse 4)";
    case ATTN_ERR_CUDA: return "CUDA call failed";
    case ATTN_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case ATTN_ERR_NO_DEVICE: return "no usable sm_100 device";
    default: return "unknown status";
  }
}

#ifdef ATTN_TRACE_ENABLED
// Tracing builds only: register the device buffer (kTraceCtas x kTrNumEvents
// x kTraceSteps uint64) that kernels stamp; nullptr turns stamping off.
extern "C" int attn_trace_set_buffer(void* dev_buf) {
  unsigned long long* p = static_cast<unsigned long long*>(dev_buf);
  return cudaMemcpyToSymbol(g_trace_buf, &p, sizeof p) == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}
#endif

extern "C" int attn_version(void) { return (0 << 16) | (1 << 8) | 0; }
