// LSE-weighted merge of partial attention results over disjoint key sets.
//
// If O_g and lse_g are the attention output and log-sum-exp of one query
// row against key set g (the sets disjoint, their union the full key set),
// then the row's result against the union is
//   lse = log sum_g exp(lse_g),   O = sum_g exp(lse_g - lse) * O_g,
// because each O_g is its own keys' weighted sum divided by exp(lse_g).
// A part that saw no key has lse_g = -inf and weight 0; a row whose parts
// all saw no key gets O = 0 and lse = -inf.
//
// The merge reads every part once and writes the result once, so it is
// bound by HBM bandwidth: one thread per 4 columns of a row (float4 loads),
// a grid-stride loop over rows.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

namespace attn_b200 {

template <bool OUT_F32>
__global__ void __launch_bounds__(256)
    lse_combine_kernel(const float* __restrict__ o_parts, const float* __restrict__ lse_parts,
                       int G, long long rows, int d, void* __restrict__ o,
                       float* __restrict__ lse) {
  const int per_row = d / 4;
  const long long total = rows * per_row;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; t < total;
       t += stride) {
    const long long row = t / per_row;
    const int c4 = static_cast<int>(t - row * per_row);
    float mx = -INFINITY;
    for (int g = 0; g < G; ++g) mx = fmaxf(mx, __ldg(lse_parts + g * rows + row));
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float out_lse = -INFINITY;
    if (mx != -INFINITY) {
      float sum = 0.f;
      for (int g = 0; g < G; ++g) sum += expf(__ldg(lse_parts + g * rows + row) - mx);
      out_lse = mx + logf(sum);
      for (int g = 0; g < G; ++g) {
        const float w = expf(__ldg(lse_parts + g * rows + row) - out_lse);
        if (w == 0.f) continue;  // a part that saw no key (or a negligible one)
        const float4 v = __ldg(reinterpret_cast<const float4*>(o_parts + (g * rows + row) * d) + c4);
        acc.x = fmaf(w, v.x, acc.x);
        acc.y = fmaf(w, v.y, acc.y);
        acc.z = fmaf(w, v.z, acc.z);
        acc.w = fmaf(w, v.w, acc.w);
      }
    }
    if (OUT_F32) {
      reinterpret_cast<float4*>(static_cast<float*>(o) + row * d)[c4] = acc;
    } else {
      const __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
      const __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
      uint2 pk;
      pk.x = *reinterpret_cast<const uint32_t*>(&lo);
      pk.y = *reinterpret_cast<const uint32_t*>(&hi);
      reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(o) + row * d)[c4] = pk;
    }
    if (c4 == 0) lse[row] = out_lse;
  }
}

}  // namespace attn_b200
