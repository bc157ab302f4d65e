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
#include "attn_combine_kernel.cuh"
#include "attn_fwd_kernel.cuh"
#include "attn_fwd_wide_kernel.cuh"
#include "host_common.h"

namespace attn_b200 {

// Written (first error wins) by kernels whose bounded waits ran out.
__device__ int g_attn_status = 0;

// Work-queue slots: each launch takes the next slot ({next item, CTAs
// finished}); the launch's last CTA resets it to zero.  Launches that run
// at the same time use different slots as long as fewer than kQueueSlots
// of them overlap.
__device__ int g_attn_queue[2 * host::kQueueSlots];

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

namespace host {

namespace {
std::mutex g_mu;
DeviceState g_dev[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
}  // namespace

int* next_queue_slot(DeviceState& st) {
  return st.queue + 2 * static_cast<int>(st.launches.fetch_add(1) % kQueueSlots);
}

namespace {
// Host-side cache of encoded tensor maps.  A map is a pure function of the
// encode's arguments (type, address, extents, strides, box; the rest is
// fixed below), so a hit hands back exactly what a fresh encode would: the
// cache only saves the host time of encoding three maps per launch.  The
// least recently used entry is replaced when it is full.
struct TmapEntry {
  bool used = false;
  unsigned long long stamp = 0;
  CUtensorMapDataType type{};
  CUtensorMapSwizzle swizzle{};
  const void* ptr = nullptr;
  cuuint64_t dims[3] = {0, 0, 0};
  cuuint64_t strides[2] = {0, 0};
  cuuint32_t box[3] = {0, 0, 0};
  CUtensorMap map{};
};
constexpr int kTmapCacheEntries = 48;
std::mutex g_tmap_mu;
TmapEntry g_tmap[kTmapCacheEntries];
unsigned long long g_tmap_clock = 0;
}  // namespace

CUresult encode_tiled(CUtensorMap* m, CUtensorMapDataType type, const void* ptr,
                      const cuuint64_t* dims, const cuuint64_t* strides, const cuuint32_t* box,
                      CUtensorMapSwizzle swizzle) {
  std::lock_guard<std::mutex> lock(g_tmap_mu);
  int victim = 0;
  for (int i = 0; i < kTmapCacheEntries; ++i) {
    TmapEntry& e = g_tmap[i];
    if (e.used && e.type == type && e.swizzle == swizzle && e.ptr == ptr &&
        e.dims[0] == dims[0] && e.dims[1] == dims[1] &&
        e.dims[2] == dims[2] && e.strides[0] == strides[0] && e.strides[1] == strides[1] &&
        e.box[0] == box[0] && e.box[1] == box[1] && e.box[2] == box[2]) {
      e.stamp = ++g_tmap_clock;
      *m = e.map;
      return CUDA_SUCCESS;
    }
    if (!e.used || (g_tmap[victim].used && e.stamp < g_tmap[victim].stamp)) victim = i;
  }
  cuuint32_t estr[3] = {1, 1, 1};
  const CUresult rc = g_encode(m, type, 3, const_cast<void*>(ptr), const_cast<cuuint64_t*>(dims),
                               const_cast<cuuint64_t*>(strides), const_cast<cuuint32_t*>(box),
                               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (rc != CUDA_SUCCESS) return rc;
  TmapEntry& e = g_tmap[victim];
  e.used = true;
  e.stamp = ++g_tmap_clock;
  e.type = type;
  e.swizzle = swizzle;
  e.ptr = ptr;
  for (int k = 0; k < 3; ++k) e.dims[k] = dims[k];
  e.strides[0] = strides[0];
  e.strides[1] = strides[1];
  for (int k = 0; k < 3; ++k) e.box[k] = box[k];
  e.map = *m;
  return CUDA_SUCCESS;
}

void tmap_cache_clear() {
  std::lock_guard<std::mutex> lock(g_tmap_mu);
  for (TmapEntry& e : g_tmap) e.used = false;
}

int set_smem_once(const void* kern, int bytes, const DeviceState& st,
                  std::atomic<unsigned long long>& done) {
  const unsigned long long bit = 1ull << st.ordinal;
  if (done.load(std::memory_order_acquire) & bit) return ATTN_OK;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
      cudaSuccess) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  done.fetch_or(bit, std::memory_order_release);
  return ATTN_OK;
}

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
    st.ordinal = dev;
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

// Per-head 3-D view [Z][N][d] of a [.., N, d] bf16 tensor (Z = batch x
// heads); boxes of 128 rows x 64 columns of one head, with the 128-byte
// swizzle the tcgen05 shared-memory descriptors expect.  Rows past N of a
// head are outside the view and read as zero, so a tile never picks up the
// next head's rows.
int make_tmap_heads(CUtensorMap* m, const void* ptr, int Z, int N, int d) {
  return make_tmap_heads_rows(m, ptr, Z, N, d, 128);
}

int make_tmap_heads_rows(CUtensorMap* m, const void* ptr, int Z, int N, int d, int box_rows) {
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                        static_cast<cuuint64_t>(Z)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                           static_cast<cuuint64_t>(N) * static_cast<cuuint64_t>(d) * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  return encode_tiled(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, ptr, dims, strides, box) ==
                 CUDA_SUCCESS
             ? ATTN_OK
             : ATTN_ERR_CUDA;
}

// Token-major 3-D view [T][Hx][d] of a packed [T, Hx, d] bf16 tensor; boxes
// of 64 columns x 1 head x 128 tokens, which land in shared memory exactly
// like the per-head boxes (128 rows of 128 bytes).  Tokens past T read as
// zero; tokens of the next sequence inside a tile are masked (keys) or not
// stored (queries) by the kernel.
int make_tmap_tokens(CUtensorMap* m, const void* ptr, int T, int Hx, int d) {
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(Hx),
                        static_cast<cuuint64_t>(T)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                           static_cast<cuuint64_t>(Hx) * static_cast<cuuint64_t>(d) * 2};
  cuuint32_t box[3] = {64, 1, 128};
  return encode_tiled(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, ptr, dims, strides, box) ==
                 CUDA_SUCCESS
             ? ATTN_OK
             : ATTN_ERR_CUDA;
}

int check_on_device(const DeviceState& st, const void* const* ptrs, int n) {
  for (int i = 0; i < n; ++i) {
    if (ptrs[i] == nullptr) continue;
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, ptrs[i]) != cudaSuccess) {
      cudaGetLastError();
      return ATTN_ERR_INVALID_ARG;
    }
    if (at.type != cudaMemoryTypeDevice || at.device != st.ordinal) return ATTN_ERR_INVALID_ARG;
  }
  return ATTN_OK;
}

bool ranges_overlap(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

bool scale_ok(float scale) { return std::isfinite(scale) && scale > 0.f; }

// Output buffers must not overlap the inputs or one another.
bool outputs_disjoint(const void* const* outs, const size_t* out_bytes, int n_out,
                      const void* const* ins, const size_t* in_bytes, int n_in) {
  for (int i = 0; i < n_out; ++i) {
    for (int j = 0; j < n_in; ++j)
      if (ranges_overlap(outs[i], out_bytes[i], ins[j], in_bytes[j])) return false;
    for (int j = i + 1; j < n_out; ++j)
      if (ranges_overlap(outs[i], out_bytes[i], outs[j], out_bytes[j])) return false;
  }
  return true;
}

}  // namespace host

using namespace host;

namespace {

// Default share of exponentials computed by the FMA polynomial (pairs per 4):
// measured on B200, the special-function unit alone is fastest for this
// kernel (see the exp2 split sweep in the design notes).
constexpr int kDefaultPolyPairs = 0;

// Most key slices of one split-KV launch (and parts of one merge).
constexpr int kMaxSplits = 256;

// One attention launch, in either layout (see KernelArgs).  Checked by the
// entry points before it reaches launch().
struct Problem {
  const void* q = nullptr;
  const void* k = nullptr;
  const void* v = nullptr;
  void* o = nullptr;
  float* lse = nullptr;
  const int* cu_q = nullptr;  // packed layout when set
  const int* cu_k = nullptr;
  int B = 0, H = 0, H_kv = 0;
  int N_q = 0, N_k = 0;  // per head, or the longest sequence (packed)
  int T_q = 0, T_k = 0;  // packed: total tokens
  int d = 0;
  int causal = 0;
  int delta = 0;         // dense causal offset
  float scale = 0.f;
  int o_f32 = 0;
  int n_splits = 1;
  int split_tiles = 0;   // 0: all K/V tiles in one slice
  long long split_rows = 0;
};

// Two query heads share one work item when every head has a single Q tile
// and K/V heads are shared (up to 128 queries per head, or per sequence in
// the packed layout; H / H_kv >= 2; head dims handled by the two-tile
// kernel): both softmax groups then work, and one K/V stream feeds both.  A packed item runs two tiles per step in
// about 1.36x the step time of a one-tile item (measured on B200), so
// packing pays unless it leaves too many SMs idle: it is used when the
// packed items still number at least two thirds of the SMs.
int64_t packed_items(const Problem& p) {
  const int64_t pairs = (p.H / p.H_kv + 1) / 2;
  return static_cast<int64_t>(p.B) * p.H_kv * pairs * p.n_splits;
}
bool head_pack(const Problem& p, int num_sms) {
  return p.N_q <= kBlockM && p.H / p.H_kv >= 2 && p.d <= 128 &&
         3 * packed_items(p) >= 2 * static_cast<int64_t>(num_sms);
}

// Work items of a problem: (head, Q tile pair, key slice), or with head
// packing (K/V head, pair of its query heads, key slice).
int64_t problem_items(const Problem& p, int num_sms) {
  if (head_pack(p, num_sms)) return packed_items(p);
  const int64_t pairs = ((static_cast<int64_t>(p.N_q) + kBlockM - 1) / kBlockM + 1) / 2;
  return static_cast<int64_t>(p.B) * p.H * pairs * p.n_splits;
}

template <int D, bool CAUSAL, int kPolyPairs, int STAGES = 0>
int launch(const Problem& p, cudaStream_t stream, DeviceState& st, int* queue = nullptr,
           float tau = kRescaleTauBf16) {
  CUtensorMap tq, tk, tv, to;
  if (p.cu_q != nullptr) {
    if (make_tmap_tokens(&tq, p.q, p.T_q, p.H, D) || make_tmap_tokens(&tk, p.k, p.T_k, p.H_kv, D) ||
        make_tmap_tokens(&tv, p.v, p.T_k, p.H_kv, D))
      return ATTN_ERR_CUDA;
  } else {
    if (make_tmap_heads(&tq, p.q, p.B * p.H, p.N_q, D) ||
        make_tmap_heads(&tk, p.k, p.B * p.H_kv, p.N_k, D) ||
        make_tmap_heads(&tv, p.v, p.B * p.H_kv, p.N_k, D))
      return ATTN_ERR_CUDA;
  }
  // O's map (boxes of 32 rows, one softmax warp's share of a tile) for the
  // epilogue's TMA stores of bf16 per-head output without key slices: in
  // the wide kernel always, in the two-tile kernel without the causal mask.
  // In every other case the kernel stores rows itself and never reads it.
  to = tq;
  if constexpr (D == wide::kD || !CAUSAL) {
    if (p.cu_q == nullptr && !p.o_f32 && p.split_rows == 0 &&
        make_tmap_heads_rows(&to, p.o, p.B * p.H, p.N_q, D, 32))
      return ATTN_ERR_CUDA;
  }

  KernelArgs args;
  args.o = p.o;
  args.lse = p.lse;
  args.cu_q = p.cu_q;
  args.cu_k = p.cu_k;
  args.H = p.H;
  args.H_kv = p.H_kv;
  args.q_per_kv = p.H / p.H_kv;
  args.N_q = p.N_q;
  args.N_k = p.N_k;
  args.T_q = p.T_q;
  args.T_k = p.T_k;
  args.delta = p.delta;
  args.head_pack = head_pack(p, st.num_sms) ? 1 : 0;
  args.n_qpairs = args.head_pack ? (args.q_per_kv + 1) / 2
                                 : ((p.N_q + kBlockM - 1) / kBlockM + 1) / 2;
  args.n_splits = p.n_splits;
  args.split_tiles = p.split_tiles > 0 ? p.split_tiles : (p.N_k + kBlockN - 1) / kBlockN;
  if (args.split_tiles < 1) args.split_tiles = 1;
  args.split_rows = p.split_rows;
  args.o_f32 = p.o_f32;
  args.BH = args.head_pack ? p.B * p.H_kv : p.B * p.H;  // units of the item windows
  args.B = p.B;
  args.n_items = static_cast<int>(problem_items(p, st.num_sms));
  // Scheduling window: enough heads that a window holds about two rounds of
  // items (so its light tail evens out the CTAs), few enough that the
  // window's K/V stays in L2 while its CTAs run.  This is the largest
  // window; the kernel cuts the heads into windows of equal size to within
  // one head (item_window).
  {
    const int per_head = args.n_qpairs * args.n_splits;
    const int want = (2 * st.num_sms + per_head - 1) / per_head;
    args.win_heads = want < 1 ? 1 : (want > args.BH ? args.BH : want);
  }
  args.queue = queue != nullptr ? queue : next_queue_slot(st);
  args.scale_log2 = p.scale * 1.4426950408889634f;
  args.rescale_tau = tau;
  args.status = st.status;

  // d = 256 runs the wide kernel (one Q tile at a time, 256-column O).
  // Both kernels take the maps of Q, K, V and O.
  void (*kern)(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, KernelArgs);
  int threads, smem_bytes;
  if constexpr (D == wide::kD) {
    kern = wide::attn_fwd_wide_kernel<CAUSAL, kPolyPairs>;
    threads = wide::kThreads;
    smem_bytes = wide::kSmemBytes;
  } else {
    kern = attn_fwd_kernel<D, CAUSAL, kPolyPairs, STAGES>;
    threads = kThreads;
    smem_bytes = Config<D, STAGES, !CAUSAL>::kSmemBytes;
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
  }
  static std::atomic<unsigned long long> smem_set{0};
  if (set_smem_once(reinterpret_cast<const void*>(kern), smem_bytes, st, smem_set) != ATTN_OK)
    return ATTN_ERR_CUDA;
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof cfg);
  // Persistent: one CTA per SM (at most one per work item).
  const int grid = args.n_items < st.num_sms ? args.n_items : st.num_sms;
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(static_cast<unsigned>(threads), 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem_bytes);
  cfg.stream = stream;
  if (cudaLaunchKernelEx(&cfg, kern, tq, tk, tv, to, args) != cudaSuccess) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  return ATTN_OK;
}

// How a launch computes (attn_opts, checked): the exponential split and
// the K/V ring depth (0: the head dim's default; 2..5 at d = 128 with the
// default split).
struct Tuning {
  int poly_pairs = kDefaultPolyPairs;
  int kv_stages = 0;
  float rescale_tau = kRescaleTauBf16;
};

template <int D, bool CAUSAL>
int launch_poly(const Tuning& t, const Problem& p, cudaStream_t s, DeviceState& st, int* queue) {
  if constexpr (D == 128) {
    switch (t.kv_stages) {
      case 2: return launch<D, CAUSAL, 0, 2>(p, s, st, queue, t.rescale_tau);
      case 3: return launch<D, CAUSAL, 0, 3>(p, s, st, queue, t.rescale_tau);
      case 5: return launch<D, CAUSAL, 0, 5>(p, s, st, queue, t.rescale_tau);
      default: break;
    }
  }
  switch (t.poly_pairs) {
    case 0: return launch<D, CAUSAL, 0>(p, s, st, queue, t.rescale_tau);
    case 2: return launch<D, CAUSAL, 2>(p, s, st, queue, t.rescale_tau);
    default: return launch<D, CAUSAL, 1>(p, s, st, queue, t.rescale_tau);
  }
}

template <int D>
int launch_d(const Tuning& t, const Problem& p, cudaStream_t s, DeviceState& st, int* queue) {
  return p.causal ? launch_poly<D, true>(t, p, s, st, queue)
                  : launch_poly<D, false>(t, p, s, st, queue);
}

// Launch a checked problem on the calling thread's device.
int run_problem(const Problem& p, const Tuning& tune, attn_stream_t stream, int* queue = nullptr,
                DeviceState* st = nullptr) {
  if (st == nullptr) {
    const int rc = device_state(&st);
    if (rc != ATTN_OK) return rc;
  }
  {
    const void* ptrs[7] = {p.q, p.k, p.v, p.o, p.lse, p.cu_q, p.cu_k};
    const int rc = check_on_device(*st, ptrs, 7);
    if (rc != ATTN_OK) return rc;
  }
  if (problem_items(p, st->num_sms) + st->num_sms > 0x7FFFFFFFll) return ATTN_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  switch (p.d) {
    case 256: return launch_d<256>(tune, p, s, *st, queue);
    case 128: return launch_d<128>(tune, p, s, *st, queue);
    case 96: return launch_d<96>(tune, p, s, *st, queue);
    default: return launch_d<64>(tune, p, s, *st, queue);
  }
}

// LSE merge of G partial results (see attn_combine_kernel.cuh).
int run_combine(const float* o_parts, const float* lse_parts, int G, long long rows, int d,
                void* o, float* lse, int o_f32, attn_stream_t stream, const DeviceState& st) {
  {
    const void* ptrs[4] = {o_parts, lse_parts, o, lse};
    const int rc = check_on_device(st, ptrs, 4);
    if (rc != ATTN_OK) return rc;
  }
  const long long threads = rows * (d / 4);
  long long blocks = (threads + 255) / 256;
  const long long cap = static_cast<long long>(st.num_sms) * 8;
  if (blocks > cap) blocks = cap;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (o_f32)
    lse_combine_kernel<true><<<static_cast<unsigned>(blocks), 256, 0, s>>>(o_parts, lse_parts, G,
                                                                          rows, d, o, lse);
  else
    lse_combine_kernel<false><<<static_cast<unsigned>(blocks), 256, 0, s>>>(o_parts, lse_parts, G,
                                                                           rows, d, o, lse);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  return ATTN_OK;
}

bool head_dim_ok(int d) { return d == 64 || d == 96 || d == 128 || d == 256; }

// Checks of a dense problem with per-head layout (attn_fwd, attn_fwd_chunk).
int check_dense(const Problem& p) {
  if (!p.q || !p.k || !p.v || !p.o || !p.lse) return ATTN_ERR_INVALID_ARG;
  if (p.B <= 0 || p.H <= 0 || p.H_kv <= 0 || p.N_q <= 0 || p.N_k <= 0) return ATTN_ERR_INVALID_ARG;
  if (p.H % p.H_kv != 0) return ATTN_ERR_INVALID_ARG;
  if (!scale_ok(p.scale)) return ATTN_ERR_INVALID_ARG;
  if (p.delta < -(1 << 30) || p.delta > (1 << 30)) return ATTN_ERR_INVALID_ARG;
  if (!head_dim_ok(p.d)) return ATTN_ERR_UNSUPPORTED;
  const uint64_t rows_q = static_cast<uint64_t>(p.B) * p.H * p.N_q;
  const uint64_t rows_k = static_cast<uint64_t>(p.B) * p.H_kv * p.N_k;
  // Rows are numbered in int on the device.
  if (rows_q >= (1ull << 31) || rows_k >= (1ull << 31)) return ATTN_ERR_UNSUPPORTED;
  const uintptr_t al = reinterpret_cast<uintptr_t>(p.q) | reinterpret_cast<uintptr_t>(p.k) |
                       reinterpret_cast<uintptr_t>(p.v) | reinterpret_cast<uintptr_t>(p.o);
  if (al & 15u) return ATTN_ERR_MISALIGNED;
  if (reinterpret_cast<uintptr_t>(p.lse) & 3u) return ATTN_ERR_MISALIGNED;
  const size_t qb = rows_q * static_cast<size_t>(p.d) * 2, kb = rows_k * static_cast<size_t>(p.d) * 2;
  const size_t splits = p.n_splits > 1 ? static_cast<size_t>(p.n_splits) : 1;
  const size_t ob = splits * rows_q * static_cast<size_t>(p.d) * (p.o_f32 ? 4 : 2);
  const size_t lb = splits * rows_q * 4;
  const void* outs[2] = {p.o, p.lse};
  const size_t out_bytes[2] = {ob, lb};
  const void* ins[3] = {p.q, p.k, p.v};
  const size_t in_bytes[3] = {qb, kb, kb};
  if (!outputs_disjoint(outs, out_bytes, 2, ins, in_bytes, 3)) return ATTN_ERR_INVALID_ARG;
  return ATTN_OK;
}

Problem dense_problem(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                      int H, int N, int d, int causal, float scale) {
  Problem p;
  p.q = q;
  p.k = k;
  p.v = v;
  p.o = o;
  p.lse = lse;
  p.B = B;
  p.H = H;
  p.H_kv = H;
  p.N_q = N;
  p.N_k = N;
  p.d = d;
  p.causal = causal ? 1 : 0;
  p.scale = scale;
  return p;
}

}  // namespace
}  // namespace attn_b200

using namespace attn_b200;

extern "C" int attn_check_args(const void* q, const void* k, const void* v, const void* o,
                               const float* lse, int B, int H, int N, int d, float scale) {
  return check_dense(dense_problem(q, k, v, const_cast<void*>(o), const_cast<float*>(lse), B, H,
                                   N, d, 0, scale));
}

extern "C" int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                        int H, int N, int d, int causal, float scale, attn_stream_t stream) {
  const Problem p = dense_problem(q, k, v, o, lse, B, H, N, d, causal, scale);
  const int rc = check_dense(p);
  if (rc != ATTN_OK) return rc;
  return run_problem(p, Tuning{}, stream);
}

extern "C" attn_opts attn_opts_default(void) {
  attn_opts o;
  o.exp2_poly_pairs = -1;
  o.kv_stages = 0;
  o.rescale_tau = -1.f;
  return o;
}

extern "C" int attn_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                           int H, int N, int d, int causal, float scale, const attn_opts* opts,
                           attn_stream_t stream) {
  Tuning t;
  if (opts) {
    if (opts->exp2_poly_pairs < -1 || opts->exp2_poly_pairs > 2) return ATTN_ERR_INVALID_ARG;
    if (opts->exp2_poly_pairs >= 0) t.poly_pairs = opts->exp2_poly_pairs;
    if (opts->kv_stages < 0 || opts->kv_stages == 1 || opts->kv_stages > 5)
      return ATTN_ERR_INVALID_ARG;
    t.kv_stages = opts->kv_stages == kDefaultStagesD128 ? 0 : opts->kv_stages;
    if (t.kv_stages != 0 && (d != 128 || t.poly_pairs != kDefaultPolyPairs))
      return ATTN_ERR_UNSUPPORTED;
    if (opts->rescale_tau != -1.f) {  // -1: the default
      if (!(opts->rescale_tau >= 0.f && opts->rescale_tau <= 16.f)) return ATTN_ERR_INVALID_ARG;
      if (d > 128) return ATTN_ERR_UNSUPPORTED;
      t.rescale_tau = opts->rescale_tau;
    }
  }
  const Problem p = dense_problem(q, k, v, o, lse, B, H, N, d, causal, scale);
  const int rc = check_dense(p);
  if (rc != ATTN_OK) return rc;
  return run_problem(p, t, stream);
}

extern "C" int attn_fwd_chunk(const void* q, const void* k, const void* v, void* o, float* lse,
                              int B, int H, int H_kv, int N_q, int N_k, int d, int causal,
                              int causal_delta, float scale, int o_fp32, attn_stream_t stream) {
  Problem p = dense_problem(q, k, v, o, lse, B, H, N_q, d, causal, scale);
  p.H_kv = H_kv;
  p.N_k = N_k;
  p.delta = causal_delta;
  p.o_f32 = o_fp32 ? 1 : 0;
  const int rc = check_dense(p);
  if (rc != ATTN_OK) return rc;
  return run_problem(p, Tuning{}, stream);
}

extern "C" int attn_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                               const int* cu_seqlens_q, const int* cu_seqlens_k, int B, int H,
                               int H_kv, int max_seqlen_q, int max_seqlen_k, int total_q,
                               int total_k, int d, int causal, float scale,
                               attn_stream_t stream) {
  if (!q || !k || !v || !o || !lse || !cu_seqlens_q || !cu_seqlens_k) return ATTN_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || H_kv <= 0 || H % H_kv != 0) return ATTN_ERR_INVALID_ARG;
  if (max_seqlen_q <= 0 || max_seqlen_k <= 0 || total_q <= 0 || total_k <= 0)
    return ATTN_ERR_INVALID_ARG;
  if (!scale_ok(scale)) return ATTN_ERR_INVALID_ARG;
  if (!head_dim_ok(d)) return ATTN_ERR_UNSUPPORTED;
  const uint64_t rows_q = static_cast<uint64_t>(total_q) * H;
  const uint64_t rows_k = static_cast<uint64_t>(total_k) * H_kv;
  if (rows_q >= (1ull << 31) || rows_k >= (1ull << 31)) return ATTN_ERR_UNSUPPORTED;
  const uintptr_t al = reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
                       reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(o);
  if (al & 15u) return ATTN_ERR_MISALIGNED;
  if ((reinterpret_cast<uintptr_t>(lse) | reinterpret_cast<uintptr_t>(cu_seqlens_q) |
       reinterpret_cast<uintptr_t>(cu_seqlens_k)) & 3u)
    return ATTN_ERR_MISALIGNED;
  const size_t qb = rows_q * static_cast<size_t>(d) * 2, kb = rows_k * static_cast<size_t>(d) * 2;
  const size_t cb = (static_cast<size_t>(B) + 1) * 4;
  const void* outs[2] = {o, lse};
  const size_t out_bytes[2] = {qb, rows_q * 4};
  const void* ins[5] = {q, k, v, cu_seqlens_q, cu_seqlens_k};
  const size_t in_bytes[5] = {qb, kb, kb, cb, cb};
  if (!outputs_disjoint(outs, out_bytes, 2, ins, in_bytes, 5)) return ATTN_ERR_INVALID_ARG;
  Problem p = dense_problem(q, k, v, o, lse, B, H, max_seqlen_q, d, causal, scale);
  p.H_kv = H_kv;
  p.N_k = max_seqlen_k;
  p.cu_q = cu_seqlens_q;
  p.cu_k = cu_seqlens_k;
  p.T_q = total_q;
  p.T_k = total_k;
  return run_problem(p, Tuning{}, stream);
}

extern "C" int attn_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse,
                                int B, int H, int H_kv, int N_q, int N_k, int d, int causal,
                                int causal_delta, float scale, int n_splits, float* ws_o,
                                float* ws_lse, attn_stream_t stream) {
  if (n_splits < 1 || n_splits > kMaxSplits) return ATTN_ERR_INVALID_ARG;
  Problem p = dense_problem(q, k, v, o, lse, B, H, N_q, d, causal, scale);
  p.H_kv = H_kv;
  p.N_k = N_k;
  p.delta = causal_delta;
  int rc = check_dense(p);
  if (rc != ATTN_OK) return rc;
  const int tiles = (N_k + kBlockN - 1) / kBlockN;
  const int split_tiles = (tiles + n_splits - 1) / n_splits;
  const int used = (tiles + split_tiles - 1) / split_tiles;  // slices that hold keys
  if (used <= 1) return run_problem(p, Tuning{}, stream);
  if (!ws_o || !ws_lse) return ATTN_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(ws_o) & 15u) return ATTN_ERR_MISALIGNED;
  if (reinterpret_cast<uintptr_t>(ws_lse) & 3u) return ATTN_ERR_MISALIGNED;
  const uint64_t rows = static_cast<uint64_t>(B) * H * N_q;
  const uint64_t rows_k = static_cast<uint64_t>(B) * H_kv * N_k;
  const size_t qb = rows * static_cast<size_t>(d) * 2, kb = rows_k * static_cast<size_t>(d) * 2;
  const size_t wob = static_cast<size_t>(used) * rows * static_cast<size_t>(d) * 4;
  const size_t wlb = static_cast<size_t>(used) * rows * 4;
  const void* outs[4] = {o, lse, ws_o, ws_lse};
  const size_t out_bytes[4] = {qb, rows * 4, wob, wlb};
  const void* ins[3] = {q, k, v};
  const size_t in_bytes[3] = {qb, kb, kb};
  if (!outputs_disjoint(outs, out_bytes, 4, ins, in_bytes, 3)) return ATTN_ERR_INVALID_ARG;
  DeviceState* st = nullptr;
  rc = device_state(&st);
  if (rc != ATTN_OK) return rc;
  Problem part = p;
  part.o = ws_o;
  part.lse = ws_lse;
  part.o_f32 = 1;
  part.n_splits = used;
  part.split_tiles = split_tiles;
  part.split_rows = static_cast<long long>(rows);
  rc = run_problem(part, Tuning{}, stream, nullptr, st);
  if (rc != ATTN_OK) return rc;
  return run_combine(ws_o, ws_lse, used, static_cast<long long>(rows), d, o, lse, 0, stream, *st);
}

extern "C" int attn_combine(const float* o_parts, const float* lse_parts, int G, long long rows,
                            int d, void* o, float* lse, int o_fp32, attn_stream_t stream) {
  if (!o_parts || !lse_parts || !o || !lse) return ATTN_ERR_INVALID_ARG;
  if (G < 1 || G > kMaxSplits || rows < 1) return ATTN_ERR_INVALID_ARG;
  if (!head_dim_ok(d)) return ATTN_ERR_UNSUPPORTED;
  if (static_cast<uint64_t>(G) * static_cast<uint64_t>(rows) >= (1ull << 40))
    return ATTN_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(o_parts) | reinterpret_cast<uintptr_t>(o)) & 15u)
    return ATTN_ERR_MISALIGNED;
  if ((reinterpret_cast<uintptr_t>(lse_parts) | reinterpret_cast<uintptr_t>(lse)) & 3u)
    return ATTN_ERR_MISALIGNED;
  const size_t pr = static_cast<size_t>(G) * static_cast<size_t>(rows);
  const void* outs[2] = {o, lse};
  const size_t out_bytes[2] = {static_cast<size_t>(rows) * d * (o_fp32 ? 4 : 2),
                               static_cast<size_t>(rows) * 4};
  const void* ins[2] = {o_parts, lse_parts};
  const size_t in_bytes[2] = {pr * d * 4, pr * 4};
  if (!outputs_disjoint(outs, out_bytes, 2, ins, in_bytes, 2)) return ATTN_ERR_INVALID_ARG;
  DeviceState* st = nullptr;
  const int rc = device_state(&st);
  if (rc != ATTN_OK) return rc;
  return run_combine(o_parts, lse_parts, G, rows, d, o, lse, o_fp32 ? 1 : 0, stream, *st);
}

// Allocation-free entry point (include/attn_b200.h): same kernel, work
// queue in the library's fixed scratch array, cleared on every call.
extern "C" int attn_fwd_noalloc(const void* q, const void* k, const void* v, void* o, float* lse,
                                int B, int H, int N, int d, int causal, float scale,
                                attn_stream_t stream) {
  const Problem p = dense_problem(q, k, v, o, lse, B, H, N, d, causal, scale);
  int rc = check_dense(p);
  if (rc != ATTN_OK) return rc;
  DeviceState* st = nullptr;
  rc = device_state(&st);  // first call on a device: resolves the scratch address
  if (rc != ATTN_OK) return rc;
  // The queue counter is a 32-bit int that every CTA pushes once past the
  // last item: items + CTAs must stay representable.
  if (problem_items(p, st->num_sms) + st->num_sms > 0x7FFFFFFFll) return ATTN_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(st->noalloc_scratch, 0, kNoAllocQueueBytes, s) != cudaSuccess) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  return run_problem(p, Tuning{}, stream, st->noalloc_scratch, st);
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
  // Read and clear on `stream`, behind everything already queued there, and
  // synchronise once (two synchronous symbol copies on the legacy stream
  // would each wait for the whole device).
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int val = 0;
  if (cudaMemcpyAsync(&val, st->status, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaMemsetAsync(st->status, 0, sizeof(int), s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  return val;
}

extern "C" const char* attn_strerror(int status) {
  switch (status) {
    case ATTN_OK: return "ok";
    case ATTN_ERR_INVALID_ARG: return "invalid argument";
    case ATTN_ERR_UNSUPPORTED: return "unsupported shape (d must be 64, 96, 128 or 256; B*H*N below 2^31)";
    case ATTN_ERR_MISALIGNED: return "misaligned pointer (q, k, v, o need 16 bytes, lse 4)";
    case ATTN_ERR_CUDA: return "CUDA call failed";
    case ATTN_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case ATTN_ERR_DEVICE_BOUNDS: return "sequence offsets outside the buffers (device-side check)";
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

#ifdef ATTN_TEST_HOOKS
// Test builds only: the limit of every bounded wait in the attention kernels
// (nanoseconds, 0 for the default of 2 s) and the index of a K/V load that
// CTA 0's producer withholds (-1: none).  A withheld load makes a consumer's
// wait run out: the kernel then reports ATTN_ERR_DEVICE_TIMEOUT and leaves
// through its abort path (every role stops, loads and MMAs in flight drain,
// Tensor Memory is freed).  No fault, trap or endless wait is involved.
extern "C" int attn_test_set_hooks(unsigned long long wait_limit_ns, int withhold_load) {
  if (wait_limit_ns == 0) wait_limit_ns = kWaitLimitNs;
  if (cudaMemcpyToSymbol(g_test_wait_limit_ns, &wait_limit_ns, sizeof wait_limit_ns) !=
          cudaSuccess ||
      cudaMemcpyToSymbol(g_test_withhold_load, &withhold_load, sizeof withhold_load) !=
          cudaSuccess) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  return host::fp8_test_set_hooks(wait_limit_ns, withhold_load);
}
#endif

#if defined(ATTN_BOUNDS_CHECKS) && defined(ATTN_TEST_HOOKS)
// Checked test builds only: an offset added to the K/V head of CTA 0's first
// item (0 for none), which the producer's bounds check must catch before
// any load of that head is issued.
extern "C" int attn_test_set_bad_kv_head(int offset) {
  if (cudaMemcpyToSymbol(g_test_bad_kv_head, &offset, sizeof offset) != cudaSuccess) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  return ATTN_OK;
}
#endif

extern "C" int attn_release(void) {
  tmap_cache_clear();
  return ATTN_OK;
}

extern "C" int attn_version(void) { return (0 << 16) | (2 << 8) | 0; }
