// C-ABI entry points of the 4-bit (NVFP4) attention forward and of its bf16
// -> NVFP4 conversion: argument checks, 4-bit TMA tensor maps and the
// launches.  The contract is documented in include/attn_b200.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>

#include "attn_b200.h"
#include "attn_fwd_fp4_kernel.cuh"
#include "host_common.h"
#include "quantize_fp4_kernel.cuh"

namespace attn_b200 {
namespace {

using namespace host;

// 3-D view of packed E2M1 codes: dims {inner bytes, mid, outer}, boxes of
// 64 bytes x 128 rows x 1 with the 64-byte swizzle (one 128-value row of a
// tile per 64-byte row).
int make_tmap_e2m1(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t mid, uint64_t outer) {
  cuuint64_t dims[3] = {inner, mid, outer};
  cuuint64_t strides[2] = {inner, inner * mid};
  cuuint32_t box[3] = {64, 128, 1};
  return encode_tiled(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, ptr, dims, strides, box,
                      CU_TENSOR_MAP_SWIZZLE_64B) == CUDA_SUCCESS
             ? ATTN_OK
             : ATTN_ERR_CUDA;
}

// Scale-factor bytes of one operand: [BH, T, 2, 512].
size_t sf_bytes(uint64_t BH, int N) { return BH * static_cast<size_t>((N + 127) / 128) * 1024; }

}  // namespace
}  // namespace attn_b200

using namespace attn_b200;
using namespace attn_b200::host;

extern "C" long long attn_nvfp4_scale_bytes(int BH, int N) {
  if (BH <= 0 || N <= 0) return -1;
  return static_cast<long long>(sf_bytes(static_cast<uint64_t>(BH), N));
}

extern "C" int attn_fwd_fp4(const void* q, const void* q_sf, const void* k, const void* k_sf,
                            const void* vt, const void* vt_sf, void* o, float* lse, int B, int H,
                            int N, int d, int causal, float scale, float q_descale,
                            float k_descale, float v_descale, attn_stream_t stream) {
  if (!q || !q_sf || !k || !k_sf || !vt || !vt_sf || !o || !lse) return ATTN_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || N <= 0) return ATTN_ERR_INVALID_ARG;
  if (!scale_ok(scale) || !scale_ok(q_descale) || !scale_ok(k_descale) || !scale_ok(v_descale))
    return ATTN_ERR_INVALID_ARG;
  if (d != fp4::kD || N % 32 != 0) return ATTN_ERR_UNSUPPORTED;
  const uint64_t BH = static_cast<uint64_t>(B) * H;
  const uint64_t rows = BH * static_cast<uint64_t>(N);
  if (rows >= (1ull << 31)) return ATTN_ERR_UNSUPPORTED;
  const uintptr_t al = reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
                       reinterpret_cast<uintptr_t>(vt) | reinterpret_cast<uintptr_t>(o) |
                       reinterpret_cast<uintptr_t>(q_sf) | reinterpret_cast<uintptr_t>(k_sf) |
                       reinterpret_cast<uintptr_t>(vt_sf);
  if (al & 15u) return ATTN_ERR_MISALIGNED;
  if (reinterpret_cast<uintptr_t>(lse) & 3u) return ATTN_ERR_MISALIGNED;
  const size_t cb = rows * (fp4::kD / 2), sb = sf_bytes(BH, N);
  const void* outs[2] = {o, lse};
  const size_t out_bytes[2] = {rows * fp4::kD * 2, rows * 4};
  const void* ins[6] = {q, k, vt, q_sf, k_sf, vt_sf};
  const size_t in_bytes[6] = {cb, cb, cb, sb, sb, sb};
  if (!outputs_disjoint(outs, out_bytes, 2, ins, in_bytes, 6)) return ATTN_ERR_INVALID_ARG;
  DeviceState* st = nullptr;
  int rc = device_state(&st);
  if (rc != ATTN_OK) return rc;
  {
    const void* ptrs[8] = {q, k, vt, q_sf, k_sf, vt_sf, o, lse};
    rc = check_on_device(*st, ptrs, 8);
    if (rc != ATTN_OK) return rc;
  }
  CUtensorMap tq, tk, tvt, to;
  if (make_tmap_e2m1(&tq, q, fp4::kD / 2, N, BH) || make_tmap_e2m1(&tk, k, fp4::kD / 2, N, BH) ||
      make_tmap_e2m1(&tvt, vt, N / 2, fp4::kD, BH))
    return ATTN_ERR_CUDA;
  // O (bf16), boxes of 32 rows x 64 columns: the epilogue's TMA stores
  // without the causal mask (otherwise unused)
  to = tq;
  if (!causal && make_tmap_heads_rows(&to, o, static_cast<int>(BH), N, fp4::kD, 32))
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
  fp4::Fp4Args fa;
  fa.q_sf = static_cast<const uint8_t*>(q_sf);
  fa.k_sf = static_cast<const uint8_t*>(k_sf);
  fa.v_sf = static_cast<const uint8_t*>(vt_sf);
  fa.n_tiles = (N + 127) / 128;
  fa.v_descale = v_descale;
  auto kern = causal ? fp4::attn_fwd_fp4_kernel<true> : fp4::attn_fwd_fp4_kernel<false>;
  static std::atomic<unsigned long long> smem_set[2] = {{0}, {0}};
  if (set_smem_once(reinterpret_cast<const void*>(kern), fp4::kSmemBytes, *st,
                    smem_set[causal ? 1 : 0]) != ATTN_OK)
    return ATTN_ERR_CUDA;
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof cfg);
  const int grid = args.n_items < st->num_sms ? args.n_items : st->num_sms;
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(fp4::kThreads, 1, 1);
  cfg.dynamicSmemBytes = fp4::kSmemBytes;
  cfg.stream = static_cast<cudaStream_t>(stream);
  if (cudaLaunchKernelEx(&cfg, kern, tq, tk, tvt, to, args, fa) != cudaSuccess) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  return ATTN_OK;
}

extern "C" int attn_quantize_nvfp4(const void* src, void* codes, void* scales, int BH, int N,
                                   int d, float inv_descale, int transpose,
                                   attn_stream_t stream) {
  if (!src || !codes || !scales || BH <= 0 || N <= 0) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(inv_descale) || !(inv_descale > 0.f)) return ATTN_ERR_INVALID_ARG;
  if (d != quant4::kD) return ATTN_ERR_UNSUPPORTED;
  if (transpose && N % 32 != 0) return ATTN_ERR_UNSUPPORTED;
  const uint64_t rows = static_cast<uint64_t>(BH) * N;
  if (rows >= (1ull << 31)) return ATTN_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(codes)) & 15u)
    return ATTN_ERR_MISALIGNED;
  const size_t sb = sf_bytes(static_cast<uint64_t>(BH), N), cbytes = rows * (d / 2);
  const void* outs[2] = {codes, scales};
  const size_t out_bytes[2] = {cbytes, sb};
  const void* ins[1] = {src};
  const size_t in_bytes[1] = {rows * d * 2};
  if (!outputs_disjoint(outs, out_bytes, 2, ins, in_bytes, 1)) return ATTN_ERR_INVALID_ARG;
  DeviceState* st = nullptr;
  int rc = device_state(&st);
  if (rc != ATTN_OK) return rc;
  {
    const void* ptrs[3] = {src, codes, scales};
    rc = check_on_device(*st, ptrs, 3);
    if (rc != ATTN_OK) return rc;
  }
  const int T = (N + 127) / 128;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const __nv_bfloat16* x = static_cast<const __nv_bfloat16*>(src);
  uint8_t* c = static_cast<uint8_t*>(codes);
  uint8_t* sc = static_cast<uint8_t*>(scales);
  if (!transpose) {
    const long long threads = static_cast<long long>(BH) * T * 128 * 8;
    long long blocks = (threads + 255) / 256;
    const long long cap = 8LL * st->num_sms;
    if (blocks > cap) blocks = cap;
    quant4::rows_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(x, c, sc, BH, N, T,
                                                                       inv_descale);
  } else {
    long long blocks = static_cast<long long>(BH) * T * 8;
    const long long cap = 16LL * st->num_sms;
    if (blocks > cap) blocks = cap;
    quant4::cols_kernel<<<static_cast<unsigned>(blocks), 128, 0, s>>>(x, c, sc, BH, N, T,
                                                                       inv_descale);
  }
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  return ATTN_OK;
}
