// C-ABI entry points of the FP8 (E4M3) attention forward and of the bf16 ->
// E4M3 conversion kernels: argument checks, 8-bit TMA tensor maps and the
// launches.  The contract is documented in include/attn_b200.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>

#include "attn_b200.h"
#include "attn_fwd_fp8_kernel.cuh"
#include "host_common.h"
#include "quantize_kernel.cuh"

namespace attn_b200 {
namespace {

using namespace host;

// 3-D view of an 8-bit tensor: dims {inner, mid, outer}, boxes of 128 x 128
// x 1 (128-byte rows, the 128-byte swizzle).
int make_tmap_u8(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t mid, uint64_t outer) {
  cuuint64_t dims[3] = {inner, mid, outer};
  cuuint64_t strides[2] = {inner, inner * mid};
  cuuint32_t box[3] = {128, 128, 1};
  return encode_tiled(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, ptr, dims, strides, box) == CUDA_SUCCESS
             ? ATTN_OK
             : ATTN_ERR_CUDA;
}

}  // namespace
}  // namespace attn_b200

using namespace attn_b200;

#ifdef ATTN_TEST_HOOKS
namespace attn_b200 {
namespace host {
int fp8_test_set_hooks(unsigned long long wait_limit_ns, int withhold_load) {
  if (cudaMemcpyToSymbol(g_test_wait_limit_ns, &wait_limit_ns, sizeof wait_limit_ns) !=
          cudaSuccess ||
      cudaMemcpyToSymbol(g_test_withhold_load, &withhold_load, sizeof withhold_load) !=
          cudaSuccess) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  return ATTN_OK;
}
}  // namespace host
}  // namespace attn_b200
#endif
using namespace attn_b200::host;

extern "C" int attn_fwd_fp8(const void* q, const void* k, const void* vt, void* o, float* lse,
                            int B, int H, int N, int d, int causal, float scale, float q_descale,
                            float k_descale, float v_descale, attn_stream_t stream) {
  if (!q || !k || !vt || !o || !lse) return ATTN_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || N <= 0) return ATTN_ERR_INVALID_ARG;
  if (!scale_ok(scale) || !scale_ok(q_descale) || !scale_ok(k_descale) || !scale_ok(v_descale))
    return ATTN_ERR_INVALID_ARG;
  if (d != fp8::kD) return ATTN_ERR_UNSUPPORTED;
  // V^T rows are N bytes long: the tensor map needs them 16-byte aligned.
  if (N % 16 != 0) return ATTN_ERR_UNSUPPORTED;
  const uint64_t rows = static_cast<uint64_t>(B) * H * N;
  if (rows >= (1ull << 31)) return ATTN_ERR_UNSUPPORTED;
  const uintptr_t al = reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
                       reinterpret_cast<uintptr_t>(vt) | reinterpret_cast<uintptr_t>(o);
  if (al & 15u) return ATTN_ERR_MISALIGNED;
  if (reinterpret_cast<uintptr_t>(lse) & 3u) return ATTN_ERR_MISALIGNED;
  const size_t ib = rows * static_cast<size_t>(d);
  const void* outs[2] = {o, lse};
  const size_t out_bytes[2] = {ib * 2, rows * 4};
  const void* ins[3] = {q, k, vt};
  const size_t in_bytes[3] = {ib, ib, ib};
  if (!outputs_disjoint(outs, out_bytes, 2, ins, in_bytes, 3)) return ATTN_ERR_INVALID_ARG;
  DeviceState* st = nullptr;
  int rc = device_state(&st);
  if (rc != ATTN_OK) return rc;
  {
    const void* ptrs[5] = {q, k, vt, o, lse};
    rc = check_on_device(*st, ptrs, 5);
    if (rc != ATTN_OK) return rc;
  }
  const uint64_t BH = static_cast<uint64_t>(B) * H;
  CUtensorMap tq, tk, tvt, to;
  if (make_tmap_u8(&tq, q, d, N, BH) || make_tmap_u8(&tk, k, d, N, BH) ||
      make_tmap_u8(&tvt, vt, N, d, BH))
    return ATTN_ERR_CUDA;
  // O (bf16), boxes of 32 rows: the epilogue's TMA stores without the mask
  to = tq;
  if (!causal && make_tmap_heads_rows(&to, o, static_cast<int>(BH), N, d, 32))
    return ATTN_ERR_CUDA;
  const int64_t n_qpairs = ((static_cast<int64_t>(N) + kBlockM - 1) / kBlockM + 1) / 2;
  const int64_t n_items = static_cast<int64_t>(BH) * n_qpairs;
  if (n_items + st->num_sms > 0x7FFFFFFFll) return ATTN_ERR_UNSUPPORTED;
  KernelArgs args;
  std::memset(&args, 0, sizeof args);
  args.o = o;
  args.lse = lse;
  args.H = H;
  args.H_kv = H;
  args.q_per_kv = 1;
  args.N_q = N;
  args.N_k = N;
  args.n_qpairs = static_cast<int>(n_qpairs);
  args.n_splits = 1;
  args.split_tiles = (N + kBlockN - 1) / kBlockN;
  args.BH = B * H;
  args.n_items = static_cast<int>(n_items);
  {
    const int want = (2 * st->num_sms + args.n_qpairs - 1) / args.n_qpairs;
    args.win_heads = want < 1 ? 1 : (want > args.BH ? args.BH : want);
  }
  args.scale_log2 = scale * q_descale * k_descale * 1.4426950408889634f;
  args.status = st->status;
  args.queue = next_queue_slot(*st);
  auto kern = causal ? fp8::attn_fwd_fp8_kernel<true> : fp8::attn_fwd_fp8_kernel<false>;
  static std::atomic<unsigned long long> smem_set[2] = {{0}, {0}};
  if (set_smem_once(reinterpret_cast<const void*>(kern), fp8::kSmemBytes, *st,
                    smem_set[causal ? 1 : 0]) != ATTN_OK)
    return ATTN_ERR_CUDA;
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof cfg);
  const int grid = args.n_items < st->num_sms ? args.n_items : st->num_sms;
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = fp8::kSmemBytes;
  cfg.stream = static_cast<cudaStream_t>(stream);
  if (cudaLaunchKernelEx(&cfg, kern, tq, tk, tvt, to, args, v_descale) != cudaSuccess) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  return ATTN_OK;
}

extern "C" int attn_quantize_e4m3(const void* src, void* dst, int BH, int N, int d,
                                  float inv_descale, int transpose, attn_stream_t stream) {
  if (!src || !dst || BH <= 0 || N <= 0) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(inv_descale) || !(inv_descale > 0.f)) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (transpose && N % 16 != 0) return ATTN_ERR_UNSUPPORTED;
  const uint64_t elems = static_cast<uint64_t>(BH) * N * d;
  if (elems >= (1ull << 40) || BH > 65535) return ATTN_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) & 15u)
    return ATTN_ERR_MISALIGNED;
  if (ranges_overlap(src, elems * 2, dst, elems)) return ATTN_ERR_INVALID_ARG;
  DeviceState* st = nullptr;
  int rc = device_state(&st);
  if (rc != ATTN_OK) return rc;
  {
    const void* ptrs[2] = {src, dst};
    rc = check_on_device(*st, ptrs, 2);
    if (rc != ATTN_OK) return rc;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (!transpose) {
    const long long n16 = static_cast<long long>(elems / 16);
    long long blocks = (n16 + 255) / 256;
    const long long cap = 8LL * st->num_sms;
    if (blocks > cap) blocks = cap;
    quant::e4m3_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(
        static_cast<const uint4*>(src), static_cast<uint4*>(dst), n16, inv_descale);
  } else {
    const dim3 grid(static_cast<unsigned>((N + 63) / 64), static_cast<unsigned>(d / 64),
                    static_cast<unsigned>(BH));
    quant::e4m3_transpose_kernel<<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(src),
                                                      static_cast<uint8_t*>(dst), N, d,
                                                      inv_descale);
  }
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  return ATTN_OK;
}

