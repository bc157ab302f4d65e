// bf16 -> NVFP4 conversion for the 4-bit attention path: E2M1 codes (two per
// byte, the lower-indexed element in the lower nibble) and one E4M3 scale
// per 16 consecutive elements along the products' reduction axis.  The
// conversion cost is part of what page lecompute.fr/kernel-perf/
// flashattention-4-limites-calcul-matriciel, section "Le FP4 ajoute un
// compromis numerique", weighs against the faster products.
//
// Steps, in float32, per block of 16 (x = bf16 value * inv_descale):
//   amax = max |x|;  scale = E4M3(amax / 6)   (nearest even, saturating);
//   code_i = E2M1(x_i * (1 / scale))          (nearest even, saturating at
//   +-6; the reciprocal and the product correctly rounded); a block whose
//   scale is 0 stores zero codes.
//
// Scale layout, per head and 128-row tile of the MMA operand (rows are query
// or key positions for Q and K, channels for V^T), two 512-byte blocks (the
// reduction axis's first and second 64 elements of the tile); row m's four
// scales of a block are the 4 bytes at 16 (m % 32) + 4 (m / 32): the order
// in which the block-scaled MMA reads them from Tensor Memory.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace attn_b200 {
namespace quant4 {

constexpr int kD = 128;

// Byte offset of the scale of (tile row m, 16-element block kb of the tile's
// 128-long reduction axis) inside that tile's 1 KB of scales.
__device__ __forceinline__ uint32_t sf_offset(int m, int kb) {
  return static_cast<uint32_t>((kb >> 2) * 512 + 16 * (m & 31) + 4 * (m >> 5) + (kb & 3));
}

// The E4M3 scale code and 8 bytes of E2M1 codes of 16 values.
__device__ __forceinline__ uint32_t quantize16(const float* x, uint2& codes) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(x[i]));
  const uint32_t sc = ptx::f32_to_e4m3(__fdiv_rn(amax, 6.f));
  const float sv = ptx::e4m3_to_f32(sc);
  const float inv = sv > 0.f ? __frcp_rn(sv) : 0.f;
  float q[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) q[i] = __fmul_rn(x[i], inv);
  codes.x = ptx::pack_e2m1x8(q[0], q[1], q[2], q[3], q[4], q[5], q[6], q[7]);
  codes.y = ptx::pack_e2m1x8(q[8], q[9], q[10], q[11], q[12], q[13], q[14], q[15]);
  return sc;
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float inv_descale, float* x) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = __fmul_rn(__uint_as_float(w[i] << 16), inv_descale);
    x[2 * i + 1] = __fmul_rn(__uint_as_float(w[i] & 0xFFFF0000u), inv_descale);
  }
}

// Q or K: src [BH, N, 128] bf16 -> codes [BH, N, 64] bytes, scales
// [BH, T, 2, 512] (T = ceil(N / 128)); one thread per (row, block of 16),
// rows padded to whole tiles (padding rows get scale 0, no codes).
__global__ void __launch_bounds__(256) rows_kernel(const __nv_bfloat16* __restrict__ src,
                                                   uint8_t* __restrict__ codes,
                                                   uint8_t* __restrict__ scales, int BH, int N,
                                                   int T, float inv_descale) {
  const long long total = static_cast<long long>(BH) * T * 128 * 8;
  for (long long t = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; t < total;
       t += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int kb = static_cast<int>(t & 7);
    const long long prow = t >> 3;  // padded row over all heads
    const int z = static_cast<int>(prow / (static_cast<long long>(T) * 128));
    const int i = static_cast<int>(prow - static_cast<long long>(z) * T * 128);  // row in head
    uint32_t sc = 0;
    if (i < N) {
      const size_t row = static_cast<size_t>(z) * N + i;
      const uint4* p = reinterpret_cast<const uint4*>(src + row * kD + 16 * kb);
      float x[16];
      bf16x8_to_f32(p[0], inv_descale, x);
      bf16x8_to_f32(p[1], inv_descale, x + 8);
      uint2 c;
      sc = quantize16(x, c);
      *reinterpret_cast<uint2*>(codes + row * (kD / 2) + 8 * kb) = c;
    }
    scales[(static_cast<size_t>(z) * T + i / 128) * 1024 + sf_offset(i & 127, kb)] =
        static_cast<uint8_t>(sc);
  }
}

// V, transposed: src [BH, N, 128] bf16 -> codes of V^T [BH, 128, N / 2]
// bytes (N a multiple of 32), scales [BH, T, 2, 512] with rows the 128
// channels and the reduction axis the keys of each 128-key tile.  One thread
// per (channel, block of 16 keys): block x of the grid covers one head and
// 16 keys, its 128 threads the channels (reads coalesced across channels).
__global__ void __launch_bounds__(128) cols_kernel(const __nv_bfloat16* __restrict__ src,
                                                   uint8_t* __restrict__ codes,
                                                   uint8_t* __restrict__ scales, int BH, int N,
                                                   int T, float inv_descale) {
  const int c = threadIdx.x;
  const long long nkb = static_cast<long long>(T) * 8;
  for (long long bi = blockIdx.x; bi < static_cast<long long>(BH) * nkb; bi += gridDim.x) {
    const int z = static_cast<int>(bi / nkb);
    const int kb = static_cast<int>(bi - z * nkb);  // 16-key block of the head
    const int j0 = 16 * kb;
    uint32_t sc = 0;
    if (j0 < N) {
      float x[16];
      const uint16_t* col = reinterpret_cast<const uint16_t*>(src) +
                            (static_cast<size_t>(z) * N + j0) * kD + c;
#pragma unroll
      for (int i = 0; i < 16; ++i)
        x[i] = j0 + i < N ? __fmul_rn(__uint_as_float(static_cast<uint32_t>(col[i * kD]) << 16),
                                      inv_descale)
                          : 0.f;
      uint2 cc;
      sc = quantize16(x, cc);
      *reinterpret_cast<uint2*>(codes + (static_cast<size_t>(z) * kD + c) * (N / 2) + 8 * kb) = cc;
    }
    scales[(static_cast<size_t>(z) * T + kb / 8) * 1024 + sf_offset(c, kb & 7)] =
        static_cast<uint8_t>(sc);
  }
}

}  // namespace quant4
}  // namespace attn_b200
