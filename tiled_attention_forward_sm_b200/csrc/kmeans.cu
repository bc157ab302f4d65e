// C-ABI entry points of the k-means assignment (nearest centroid by squared
// Euclidean distance on the tensor cores): argument checks, the norm
// prologue and the assignment launch.  The contract is documented in
// include/attn_b200.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>

#include "attn_b200.h"
#include "host_common.h"
#include "kmeans_assign_kernel.cuh"

namespace attn_b200 {
namespace {

using namespace host;

template <int D>
int launch_kmeans(const void* x, const void* cent, float* ws, int32_t* assign, float* best,
                  int N, int K, cudaStream_t stream, DeviceState& st) {
  using KC = kmeans::KConfig<D>;
  CUtensorMap tx, tc;
  if (make_tmap_heads(&tx, x, 1, N, D) || make_tmap_heads(&tc, cent, 1, K, D)) return ATTN_ERR_CUDA;
  const int k_tiles = (K + kmeans::kTileN - 1) / kmeans::kTileN;
  const int64_t k_pad = static_cast<int64_t>(k_tiles) * kmeans::kTileN;
  // Centroid norms (+inf past K) for every CTA.  The point norms (needed
  // only for the distances) come from a prologue launch when the points fill
  // more than four rounds of work items over the SMs; with fewer, the
  // assignment kernel reads each point's row at the start of its item, which
  // costs a memory latency per item but saves the launch.
  float* cnorm = ws;
  float* xnorm = nullptr;
  auto norms = [&](const void* rows, int64_t n, int64_t n_pad, float* out) {
    const int64_t blocks64 = (n_pad + 7) / 8;  // 8 warps (rows) per block
    const int blocks = static_cast<int>(blocks64 < 8LL * st.num_sms ? blocks64 : 8LL * st.num_sms);
    kmeans::row_norms_kernel<<<blocks, 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(rows), n, n_pad, D, out);
    return cudaGetLastError() == cudaSuccess;
  };
  const int64_t items = (static_cast<int64_t>(N) + 2 * kBlockM - 1) / (2 * kBlockM);
  if (best != nullptr && items > 4LL * st.num_sms) xnorm = ws + k_pad;
  if (!norms(cent, K, k_pad, cnorm) || (xnorm != nullptr && !norms(x, N, N, xnorm))) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  KernelArgs args;
  std::memset(&args, 0, sizeof args);
  args.H = 1;
  args.H_kv = 1;
  args.q_per_kv = 1;
  args.N_q = N;
  args.N_k = K;
  args.n_qpairs = ((N + kBlockM - 1) / kBlockM + 1) / 2;
  args.n_splits = 1;
  args.split_tiles = k_tiles;
  args.BH = 1;
  args.n_items = args.n_qpairs;
  args.win_heads = 1;
  args.status = st.status;
  args.queue = next_queue_slot(st);
  kmeans::AssignArgs out;
  out.assign = assign;
  out.best = best;
  out.cnorm = cnorm;
  out.xnorm = xnorm;
  out.x = static_cast<const __nv_bfloat16*>(x);
  auto kern = kmeans::kmeans_assign_kernel<D>;
  static std::atomic<unsigned long long> smem_set{0};
  if (set_smem_once(reinterpret_cast<const void*>(kern), KC::kSmemBytes, st, smem_set) != ATTN_OK)
    return ATTN_ERR_CUDA;
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof cfg);
  const int grid = args.n_items < st.num_sms ? args.n_items : st.num_sms;
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(kmeans::kThreads, 1, 1);
  cfg.dynamicSmemBytes = KC::kSmemBytes;
  cfg.stream = stream;
  if (cudaLaunchKernelEx(&cfg, kern, tx, tc, args, out) != cudaSuccess) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  return ATTN_OK;
}

}  // namespace
}  // namespace attn_b200

using namespace attn_b200;
using namespace attn_b200::host;

extern "C" long long attn_kmeans_workspace_floats(int N, int K) {
  if (N <= 0 || K <= 0) return -1;
  return (static_cast<long long>(K) + kmeans::kTileN - 1) / kmeans::kTileN * kmeans::kTileN + N;
}

extern "C" int attn_kmeans_assign(const void* x, const void* centroids, float* ws,
                                  int32_t* assign, float* best, int N, int K, int d,
                                  attn_stream_t stream) {
  if (!x || !centroids || !ws || !assign) return ATTN_ERR_INVALID_ARG;
  if (N <= 0 || K <= 0) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (N >= (1 << 30) || K >= (1 << 30)) return ATTN_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(centroids) |
       reinterpret_cast<uintptr_t>(ws)) & 15u)
    return ATTN_ERR_MISALIGNED;
  if ((reinterpret_cast<uintptr_t>(assign) | reinterpret_cast<uintptr_t>(best)) & 3u)
    return ATTN_ERR_MISALIGNED;
  const size_t xb = static_cast<size_t>(N) * d * 2, cb = static_cast<size_t>(K) * d * 2;
  const size_t wb = static_cast<size_t>(attn_kmeans_workspace_floats(N, K)) * 4;
  const void* outs[3] = {ws, assign, best};
  const size_t out_bytes[3] = {wb, static_cast<size_t>(N) * 4, best ? static_cast<size_t>(N) * 4 : 0};
  const void* ins[2] = {x, centroids};
  const size_t in_bytes[2] = {xb, cb};
  if (!outputs_disjoint(outs, out_bytes, 3, ins, in_bytes, 2)) return ATTN_ERR_INVALID_ARG;
  DeviceState* st = nullptr;
  int rc = device_state(&st);
  if (rc != ATTN_OK) return rc;
  {
    const void* ptrs[5] = {x, centroids, ws, assign, best};
    rc = check_on_device(*st, ptrs, 5);
    if (rc != ATTN_OK) return rc;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return d == 128 ? launch_kmeans<128>(x, centroids, ws, assign, best, N, K, s, *st)
                  : launch_kmeans<64>(x, centroids, ws, assign, best, N, K, s, *st);
}
