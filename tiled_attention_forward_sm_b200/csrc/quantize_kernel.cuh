// bf16 -> FP8 E4M3 conversion for the FP8 attention path: x * inv_descale,
// rounded to nearest even and saturated at +-448 (cvt.rn.satfinite), either
// in place of layout ([rows, d] -> [rows, d]) or transposed per head
// ([BH, N, d] -> [BH, d, N], the V^T operand).  Both are bound by HBM
// bandwidth: 2 bytes read and 1 written per element.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace attn_b200 {
namespace quant {

// 16 elements per thread per step: two 16-byte loads, one 16-byte store.
__global__ void __launch_bounds__(256) e4m3_kernel(const uint4* __restrict__ src,
                                                   uint4* __restrict__ dst, long long n16,
                                                   float inv) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n16;
       i += stride) {
    const uint4 a = __ldg(src + 2 * i), b = __ldg(src + 2 * i + 1);
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[2 * q]));
      const float2 f1 =
          __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[2 * q + 1]));
      o[q] = ptx::pack_e4m3x4(f0.x * inv, f0.y * inv, f1.x * inv, f1.y * inv);
    }
    dst[i] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// Per head, a 64 x 64 tile of [N, d] converted and written as the [d, N]
// tile through shared memory (256 threads; edges of N guarded).
__global__ void __launch_bounds__(256) e4m3_transpose_kernel(const __nv_bfloat16* __restrict__ src,
                                                             uint8_t* __restrict__ dst, int N,
                                                             int d, float inv) {
  __shared__ uint8_t tile[64][64 + 16];
  const int bh = blockIdx.z;
  const int n0 = blockIdx.x * 64, c0 = blockIdx.y * 64;
  const __nv_bfloat16* s = src + static_cast<size_t>(bh) * N * d;
  uint8_t* o = dst + static_cast<size_t>(bh) * d * N;
  // load: 64 rows (keys) x 64 columns (d), 8 bf16 per thread per step
  for (int t = threadIdx.x; t < 64 * 8; t += blockDim.x) {
    const int r = t / 8, ch = t % 8;
    const int n = n0 + r;
    float f[8];
    if (n < N) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(s + static_cast<size_t>(n) * d + c0) + ch);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 p = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[q]));
        f[2 * q] = p.x * inv;
        f[2 * q + 1] = p.y * inv;
      }
    } else {
#pragma unroll
      for (int q = 0; q < 8; ++q) f[q] = 0.f;
    }
    const uint32_t lo = ptx::pack_e4m3x4(f[0], f[1], f[2], f[3]);
    const uint32_t hi = ptx::pack_e4m3x4(f[4], f[5], f[6], f[7]);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      tile[8 * ch + q][r] = static_cast<uint8_t>(lo >> (8 * q));
      tile[8 * ch + 4 + q][r] = static_cast<uint8_t>(hi >> (8 * q));
    }
  }
  __syncthreads();
  // store: 64 rows (d) x 64 keys, 16 bytes per thread
  for (int t = threadIdx.x; t < 64 * 4; t += blockDim.x) {
    const int c = t / 4, ch = t % 4;
    const int n = n0 + 16 * ch;
    if (n >= N) continue;
    uint32_t w[4];
#pragma unroll
    for (int q = 0; q < 4; ++q)
      w[q] = static_cast<uint32_t>(tile[c][16 * ch + 4 * q]) |
             (static_cast<uint32_t>(tile[c][16 * ch + 4 * q + 1]) << 8) |
             (static_cast<uint32_t>(tile[c][16 * ch + 4 * q + 2]) << 16) |
             (static_cast<uint32_t>(tile[c][16 * ch + 4 * q + 3]) << 24);
    *reinterpret_cast<uint4*>(o + static_cast<size_t>(c0 + c) * N + n) =
        make_uint4(w[0], w[1], w[2], w[3]);
  }
}

}  // namespace quant
}  // namespace attn_b200
