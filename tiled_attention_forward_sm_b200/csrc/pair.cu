// C-ABI entry point of the CTA-pair attention forward (clusters of two CTAs
// sharing each tcgen05 product): argument checks, tensor maps and the
// cluster launch.  The contract is documented in include/attn_b200.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstring>

#include "attn_b200.h"
#include "attn_fwd_pair_kernel.cuh"
#include "host_common.h"

namespace attn_b200 {
namespace {

using namespace host;

// Clusters of two that fit on the device at once (0: not queried yet).
std::atomic<int> g_pair_clusters[kMaxDevices];

template <bool CAUSAL>
int launch_pair(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                int N, float scale, cudaStream_t stream, DeviceState& st) {
  using namespace pair;
  const int BH = B * H;
  CUtensorMap tq, tk, tv;
  if (make_tmap_heads_rows(&tq, q, BH, N, kD, 128) || make_tmap_heads_rows(&tk, k, BH, N, kD, 64) ||
      make_tmap_heads_rows(&tv, v, BH, N, kD, 128))
    return ATTN_ERR_CUDA;
  auto kern = attn_fwd_pair_kernel<CAUSAL>;
  static std::atomic<unsigned long long> smem_set{0};
  if (set_smem_once(reinterpret_cast<const void*>(kern), pair::kSmemBytes, st, smem_set) != ATTN_OK)
    return ATTN_ERR_CUDA;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof cfg);
  cfg.blockDim = dim3(pair::kThreads, 1, 1);
  cfg.dynamicSmemBytes = pair::kSmemBytes;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  int clusters = g_pair_clusters[dev].load();
  if (clusters <= 0) {
    cfg.gridDim = dim3(2 * (st.num_sms / 2), 1, 1);
    if (cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) != cudaSuccess || clusters <= 0) {
      cudaGetLastError();
      return ATTN_ERR_CUDA;
    }
    g_pair_clusters[dev].store(clusters);
  }

  const int64_t n_tiles = (static_cast<int64_t>(N) + kBlockM - 1) / kBlockM;
  const int64_t n_quads = (n_tiles + 3) / 4;
  const int64_t n_items = static_cast<int64_t>(BH) * n_quads;
  if (n_items + 2 * clusters > 0x7FFFFFFFll) return ATTN_ERR_UNSUPPORTED;
  KernelArgs args;
  std::memset(&args, 0, sizeof args);
  args.o = o;
  args.lse = lse;
  args.H = H;
  args.H_kv = H;
  args.q_per_kv = 1;
  args.N_q = N;
  args.N_k = N;
  args.n_qpairs = static_cast<int>(n_quads);
  args.n_splits = 1;
  args.split_tiles = static_cast<int>(n_tiles);
  args.BH = BH;
  args.n_items = static_cast<int>(n_items);
  {
    const int64_t want = (2 * clusters + n_quads - 1) / n_quads;
    args.win_heads = static_cast<int>(want < 1 ? 1 : (want > BH ? BH : want));
  }
  args.scale_log2 = scale * 1.4426950408889634f;
  args.rescale_tau = kRescaleTauBf16;
  args.status = st.status;
  args.queue = next_queue_slot(st);
  const int64_t grid_clusters = n_items < clusters ? n_items : clusters;
  cfg.gridDim = dim3(static_cast<unsigned>(2 * grid_clusters), 1, 1);
  if (cudaLaunchKernelEx(&cfg, kern, tq, tk, tv, args) != cudaSuccess) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  return ATTN_OK;
}

}  // namespace
}  // namespace attn_b200

using namespace attn_b200;
using namespace attn_b200::host;

extern "C" int attn_fwd_pair(const void* q, const void* k, const void* v, void* o, float* lse,
                             int B, int H, int N, int d, int causal, float scale,
                             attn_stream_t stream) {
  if (!q || !k || !v || !o || !lse) return ATTN_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || N <= 0) return ATTN_ERR_INVALID_ARG;
  if (!scale_ok(scale)) return ATTN_ERR_INVALID_ARG;
  if (d != pair::kD) return ATTN_ERR_UNSUPPORTED;
  const uint64_t rows = static_cast<uint64_t>(B) * H * N;
  if (rows >= (1ull << 31)) return ATTN_ERR_UNSUPPORTED;
  const uintptr_t al = reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
                       reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(o);
  if (al & 15u) return ATTN_ERR_MISALIGNED;
  if (reinterpret_cast<uintptr_t>(lse) & 3u) return ATTN_ERR_MISALIGNED;
  const size_t ib = rows * static_cast<size_t>(d) * 2;
  const void* outs[2] = {o, lse};
  const size_t out_bytes[2] = {ib, rows * 4};
  const void* ins[3] = {q, k, v};
  const size_t in_bytes[3] = {ib, ib, ib};
  if (!outputs_disjoint(outs, out_bytes, 2, ins, in_bytes, 3)) return ATTN_ERR_INVALID_ARG;
  DeviceState* st = nullptr;
  int rc = device_state(&st);
  if (rc != ATTN_OK) return rc;
  {
    const void* ptrs[5] = {q, k, v, o, lse};
    rc = check_on_device(*st, ptrs, 5);
    if (rc != ATTN_OK) return rc;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return causal ? launch_pair<true>(q, k, v, o, lse, B, H, N, scale, s, *st)
                : launch_pair<false>(q, k, v, o, lse, B, H, N, scale, s, *st);
}
