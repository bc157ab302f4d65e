// k-means assignment on sm_100a ("FlashAssign", page lefilia.fr, Flash-
// KMeans item): every point goes to its nearest centroid, with the N x K
// distance matrix computed tile by tile on chip and never written out -- the
// same tile-and-discard structure as the attention forward, with a running
// argmin where attention keeps a running softmax.
//
// For a point x and centroids c_j,  ||x - c_j||^2 = ||x||^2 + (||c_j||^2 -
// 2 x.c_j), so the nearest centroid minimises v_j = ||c_j||^2 - 2 x.c_j.
// The products x.c_j of a 128-point tile and a 128-centroid tile are one
// tcgen05 MMA tile (M = 128 points, N = 128 centroids, K = d) into Tensor
// Memory; the centroid norms come from a short prologue kernel.
//
// Work items, queue and item ring are those of attn_fwd_kernel.cuh (an item
// is two 128-point tiles, the "keys" are the centroids).  Roles (384
// threads): warps 0-3 and 4-7 reduce the scores of point tile 0 and 1 (one
// thread per point), warp 8 loads points and centroid tiles with TMA, warp 9
// allocates Tensor Memory and issues the MMAs.
//
// Tensor Memory: point tile s owns columns [256s, 256s + 256) as two score
// buffers of 128 columns; the reducing warps read a buffer into registers
// and hand it back at once, so the MMA of the tile after next can refill it
// while they reduce.
#pragma once

#include "attn_fwd_kernel.cuh"

namespace attn_b200 {
namespace kmeans {

constexpr int kThreads = 384;
constexpr int kTileM = 128;  // points per tile
constexpr int kTileN = 128;  // centroids per tile

template <int D>
struct KConfig {
  static_assert(D == 64 || D == 128, "k-means assignment: d must be 64 or 128");
  static constexpr int kBoxes = D / 64;
  static constexpr int kBoxBytes = kTileM * 64 * 2;  // 16 KB
  static constexpr int kTileBytes = kBoxes * kBoxBytes;
  static constexpr int kStages = D == 128 ? 4 : 8;   // centroid ring depth
  static constexpr int kXOff = 0;                    // two point tiles
  static constexpr int kCOff = 2 * kTileBytes;
  static constexpr int kBarOff = kCOff + kStages * kTileBytes;
  // barriers: x_full[2], x_empty[2], c_full[S], c_empty[S], s_full[2][2],
  // s_free[2][2], drain, item_full[R], item_empty[R]
  static constexpr int kNumBars = 4 + 2 * kStages + 4 + 4 + 1 + 2 * kItemSlots;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kRingOff = kMiscOff + 16;
  static constexpr int kSmemBytes = kRingOff + 4 * kItemWords * kItemSlots + 1024;
  static constexpr uint32_t kIdesc = ptx::idesc_bf16_f32(128, kTileN, 0, 0);
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
};

struct KBars {
  uint64_t* x_full;   // [2]
  uint64_t* x_empty;  // [2] last MMA of the item on point tile s done
  uint64_t* c_full;   // [kStages]
  uint64_t* c_empty;  // [kStages]
  uint64_t* s_full;   // [2 tiles][2 buffers] scores in TMEM
  uint64_t* s_free;   // [2 tiles][2 buffers] scores read by the reducing warps
};

struct AssignArgs {
  int32_t* assign;      // [N] nearest centroid
  float* best;          // [N] squared distance to it (null: not written)
  const float* cnorm;   // [ceil(K/128)*128] ||c_j||^2, +inf past K
  const float* xnorm;   // [N] ||x_i||^2 precomputed, or null: formed here from x
  const __nv_bfloat16* x;  // [N, d] the points
};

// ||row||^2 of bf16 rows in fp32 (one warp per row); rows in [n, n_pad)
// get +inf so that padded centroids never win the argmin.
__global__ void __launch_bounds__(256) row_norms_kernel(const __nv_bfloat16* __restrict__ a,
                                                        int64_t n, int64_t n_pad, int d,
                                                        float* __restrict__ out) {
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x / 32);
  const int lane = threadIdx.x & 31;
  for (int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32;
       row < n_pad; row += warps) {
    if (row >= n) {
      if (lane == 0) out[row] = INFINITY;
      continue;
    }
    float acc = 0.f;
    for (int c = lane * 2; c < d; c += 64) {
      const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(a + row * d + c);
      const float2 f = __bfloat1622float2(v);
      acc = fmaf(f.x, f.x, acc);
      acc = fmaf(f.y, f.y, acc);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) out[row] = acc;
  }
}

template <int D>
__device__ void producer_role(const Shared& sh, const KBars& bb, const KernelArgs& a,
                              uint8_t* smem, const CUtensorMap* tx, const CUtensorMap* tc) {
  using C = KConfig<D>;
  const uint64_t pol_x = ptx::policy_evict_first();
  const uint64_t pol_c = ptx::policy_evict_last();
  auto load_tile = [&](const CUtensorMap* m, uint64_t* bar, uint8_t* dst, int row, uint64_t pol) {
    for (int b = 0; b < C::kBoxes; ++b)
      ptx::tma_load_3d(m, bar, dst + b * C::kBoxBytes, 64 * b, row, 0, pol);
  };
  int x_loads[2] = {0, 0};
  int issued = 0;
  bool ok = true;
  Item it{};
  auto claim = [&]() -> bool {
    for (;;) {
      const int idx = atomicAdd(a.queue, 1);
      if (idx >= a.n_items) return false;
      if (make_item<false>(idx, a, a.status, it)) return true;
    }
  };
  bool have = claim();
  for (int r = 0; ok; ++r) {
    if (!have) {
      post_item(sh, a, r, nullptr);
      break;
    }
    if (!post_item(sh, a, r, &it)) break;
    const int n = it.n0 > it.n1 ? it.n0 : it.n1;
    for (int s = 0; s < 2 && ok; ++s) {
      if ((s == 0 ? it.n0 : it.n1) == 0) continue;
      if (x_loads[s] > 0 &&
          !wait_one(sh, a.status, &bb.x_empty[s], static_cast<uint32_t>((x_loads[s] - 1) & 1))) {
        ok = false;
        break;
      }
      ptx::mbar_arrive_expect_tx(&bb.x_full[s], C::kTileBytes);
      load_tile(tx, &bb.x_full[s], smem + C::kXOff + s * C::kTileBytes,
                (2 * it.qpair + s) * kTileM, pol_x);
      ++x_loads[s];
    }
    for (int j = 0; j < n && ok; ++j) {
      const int st = issued % C::kStages;
      const uint32_t ph = (issued / C::kStages) & 1;
      if (!wait_one(sh, a.status, &bb.c_empty[st], ph ^ 1)) {
        ok = false;
        break;
      }
      ptx::mbar_arrive_expect_tx(&bb.c_full[st], C::kTileBytes);
      load_tile(tc, &bb.c_full[st], smem + C::kCOff + st * C::kTileBytes, j * kTileN, pol_c);
      ++issued;
    }
    if (ok) have = claim();
  }
  for (int s = 0; s < 2; ++s)
    if (x_loads[s] > 0)
      wait_one(sh, a.status, &bb.x_full[s], static_cast<uint32_t>((x_loads[s] - 1) & 1), true);
  for (int t = (issued > C::kStages ? issued - C::kStages : 0); t < issued; ++t)
    wait_one(sh, a.status, &bb.c_full[t % C::kStages], (t / C::kStages) & 1, true);
}

template <int D>
__device__ void mma_role(const Shared& sh, const KBars& bb, const KernelArgs& a, uint8_t* smem,
                         uint32_t tmem) {
  using C = KConfig<D>;
  const uint64_t x_desc = ptx::sdesc_sw128(ptx::smem_u32(smem + C::kXOff), 16, 1024);
  const uint64_t c_desc = ptx::sdesc_sw128(ptx::smem_u32(smem + C::kCOff), 16, 1024);
  constexpr uint64_t kTileUnits = C::kTileBytes >> 4;
  int consumed = 0;
  int x_uses[2] = {0, 0};
  int ts[2] = {0, 0};  // score tiles issued per point-tile slot (all items)
  Item it;
  bool ok = true;
  for (int r = 0; read_item(sh, a, r, it, ok); ++r) {
    const int n_s[2] = {it.n0, it.n1};
    const int n = it.n0 > it.n1 ? it.n0 : it.n1;
    for (int s = 0; s < 2; ++s) {
      if (n_s[s] == 0) continue;
      if (!wait_warp(sh, a.status, &bb.x_full[s], static_cast<uint32_t>(x_uses[s] & 1))) goto done;
      ++x_uses[s];
    }
    for (int j = 0; j < n; ++j) {
      const int ck = consumed++;
      const int st = ck % C::kStages;
      if (!wait_warp(sh, a.status, &bb.c_full[st], static_cast<uint32_t>((ck / C::kStages) & 1)))
        goto done;
      for (int s = 0; s < 2; ++s) {
        if (j >= n_s[s]) continue;
        const int b = ts[s] & 1;
        // the buffer's previous scores (tile ts - 2) must have been read
        if (ts[s] >= 2 && !wait_warp(sh, a.status, &bb.s_free[2 * s + b],
                                     static_cast<uint32_t>(((ts[s] >> 1) - 1) & 1)))
          goto done;
        ptx::tc_fence_after_sync();
        const uint64_t xd = x_desc + s * kTileUnits;
        const uint64_t cd = c_desc + st * kTileUnits;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off =
              static_cast<uint64_t>(((kk / 4) * C::kBoxBytes + (kk % 4) * 32) >> 4);
          ptx::mma_ss_elect(tmem + 256 * s + 128 * b, xd + off, cd + off, C::kIdesc,
                            kk > 0 ? 1u : 0u);
        }
        ptx::commit_elect(&bb.s_full[2 * s + b]);
        if (j == n_s[s] - 1) ptx::commit_elect(&bb.x_empty[s]);
        ++ts[s];
      }
      ptx::commit_elect(&bb.c_empty[st]);
    }
  }
done:
  ptx::commit_elect(sh.drain);
  wait_warp(sh, a.status, sh.drain, 0, true);
}

// ||x||^2 of one bf16 row of D values from global memory, in fp32; the D/8
// 16-byte loads are independent and issue together.
template <int D>
__device__ __forceinline__ float row_norm(const __nv_bfloat16* x, int64_t row) {
  const uint4* xr = reinterpret_cast<const uint4*>(x + row * D);
  uint4 u[D / 8];
#pragma unroll
  for (int c = 0; c < D / 8; ++c) u[c] = __ldg(xr + c);
  float xn0 = 0.f, xn1 = 0.f;
#pragma unroll
  for (int c = 0; c < D / 8; ++c) {
    const uint32_t w[4] = {u[c].x, u[c].y, u[c].z, u[c].w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float lo = __uint_as_float(w[k] << 16), hi = __uint_as_float(w[k] & 0xFFFF0000u);
      xn0 = fmaf(lo, lo, xn0);
      xn1 = fmaf(hi, hi, xn1);
    }
  }
  return xn0 + xn1;
}

// One thread per point: v_j = ||c_j||^2 - 2 x.c_j over each centroid tile,
// a running minimum and the smallest index that reaches it.
template <int D>
__device__ void reduce_role(const Shared& sh, const KBars& bb, const KernelArgs& a,
                            const AssignArgs& o, uint32_t tmem, int s, int warp_in_group) {
  const int lane = static_cast<int>(ptx::lane_id());
  const int r = warp_in_group * 32 + lane;
  const uint32_t lane_off = static_cast<uint32_t>(warp_in_group * 32) << 16;
  int ts = 0;
  Item it;
  bool ok = true;
  for (int rr = 0; read_item(sh, a, rr, it, ok); ++rr) {
    const int row = (2 * it.qpair + s) * kTileM + r;
    if ((2 * it.qpair + s) * kTileM >= it.q_len) continue;
    const int n = s == 0 ? it.n0 : it.n1;
    float best = INFINITY;
    int best_j = 0;
    // The point's ||x||^2 (only for the distance output), unless the host
    // computed all of them in a prologue: read from the point's row while
    // the first score tile is being computed.
    const float xn = (o.best != nullptr && o.xnorm == nullptr && row < it.q_len)
                         ? row_norm<D>(o.x, row)
                         : 0.f;
    for (int j = 0; j < n; ++j) {
      const int b = ts & 1;
      if (!wait_warp(sh, a.status, &bb.s_full[2 * s + b], static_cast<uint32_t>((ts >> 1) & 1)))
        return;
      ptx::tc_fence_after_sync();
      uint32_t sr[128];
      const uint32_t t_s = tmem + lane_off + 256u * s + 128u * b;
      ptx::tmem_ld32(t_s + 0, sr + 0);
      ptx::tmem_ld32(t_s + 32, sr + 32);
      ptx::tmem_ld32(t_s + 64, sr + 64);
      ptx::tmem_ld32(t_s + 96, sr + 96);
      ptx::tmem_ld_wait_tie(sr + 0);
      ptx::reg_tie32(sr + 32);
      ptx::reg_tie32(sr + 64);
      ptx::reg_tie32(sr + 96);
      // the scores are in registers: hand the buffer back
      ptx::tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&bb.s_free[2 * s + b]);
      ++ts;
      // v = ||c||^2 - 2 x.c (padded centroids have ||c||^2 = +inf)
      const float4* cn4 = reinterpret_cast<const float4*>(o.cnorm + static_cast<size_t>(j) * kTileN);
      float v[128];
#pragma unroll
      for (int q = 0; q < 32; ++q) {
        const float4 c4 = __ldg(cn4 + q);
        v[4 * q + 0] = fmaf(-2.f, __uint_as_float(sr[4 * q + 0]), c4.x);
        v[4 * q + 1] = fmaf(-2.f, __uint_as_float(sr[4 * q + 1]), c4.y);
        v[4 * q + 2] = fmaf(-2.f, __uint_as_float(sr[4 * q + 2]), c4.z);
        v[4 * q + 3] = fmaf(-2.f, __uint_as_float(sr[4 * q + 3]), c4.w);
      }
      // minimum of each 32-centroid chunk, then of the tile
      float cmin[4];
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        float m0 = v[32 * ch], m1 = v[32 * ch + 1];
#pragma unroll
        for (int c = 2; c + 4 <= 32; c += 4) {
          m0 = ptx::min3(m0, v[32 * ch + c], v[32 * ch + c + 1]);
          m1 = ptx::min3(m1, v[32 * ch + c + 2], v[32 * ch + c + 3]);
        }
        m0 = ptx::min3(m0, v[32 * ch + 30], v[32 * ch + 31]);
        cmin[ch] = fminf(m0, m1);
      }
      const float tmin = fminf(fminf(cmin[0], cmin[1]), fminf(cmin[2], cmin[3]));
      if (tmin < best) {  // strictly: an earlier tile keeps a tie
        int ch = 3;
#pragma unroll
        for (int k = 2; k >= 0; --k)
          if (cmin[k] == tmin) ch = k;
        int idx = 31;
#pragma unroll
        for (int c = 31; c >= 0; --c) {
          float vc = v[c];
#pragma unroll
          for (int k = 1; k < 4; ++k)
            if (ch == k) vc = v[32 * k + c];
          if (vc == tmin) idx = c;
        }
        best = tmin;
        best_j = j * kTileN + 32 * ch + idx;
      }
    }
    if (row < it.q_len) {
      o.assign[row] = best_j;
      if (o.best != nullptr)
        o.best[row] = fmaxf((o.xnorm != nullptr ? o.xnorm[row] : xn) + best, 0.f);
    }
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    kmeans_assign_kernel(const __grid_constant__ CUtensorMap tmap_x,
                         const __grid_constant__ CUtensorMap tmap_c, const KernelArgs args,
                         const AssignArgs out) {
  using C = KConfig<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  KBars bb;
  bb.x_full = bars;
  bb.x_empty = bars + 2;
  bb.c_full = bars + 4;
  bb.c_empty = bb.c_full + C::kStages;
  bb.s_full = bb.c_empty + C::kStages;
  bb.s_free = bb.s_full + 4;
  Shared sh = {};
  sh.drain = bb.s_free + 4;
  sh.item_full = sh.drain + 1;
  sh.item_empty = sh.item_full + kItemSlots;
  sh.tmem_base = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
  sh.abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 4);
  sh.item_ring = reinterpret_cast<volatile int*>(smem + C::kRingOff);

  const int warp = threadIdx.x / 32;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&bb.x_full[i], 1);
      ptx::mbar_init(&bb.x_empty[i], 1);
    }
    for (int i = 0; i < C::kStages; ++i) {
      ptx::mbar_init(&bb.c_full[i], 1);
      ptx::mbar_init(&bb.c_empty[i], 1);
    }
    for (int i = 0; i < 4; ++i) {
      ptx::mbar_init(&bb.s_full[i], 1);
      ptx::mbar_init(&bb.s_free[i], 4);
    }
    ptx::mbar_init(sh.drain, 1);
    for (int i = 0; i < kItemSlots; ++i) {
      ptx::mbar_init(&sh.item_full[i], 1);
      ptx::mbar_init(&sh.item_empty[i], kItemReaders);
    }
    *sh.abort_flag = 0;
    ptx::fence_barrier_init();
  }
  if (warp == 8 && ptx::lane_id() == 0) {
    ptx::prefetch_tmap(&tmap_x);
    ptx::prefetch_tmap(&tmap_c);
  }
  if (warp == 9) {
    ptx::tmem_alloc(sh.tmem_base, 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before_sync();
  __syncthreads();
  ptx::tc_fence_after_sync();
  const uint32_t tmem = *sh.tmem_base;

  if (warp < 8) {
    reduce_role<D>(sh, bb, args, out, tmem, warp / 4, warp % 4);
  } else if (warp == 8) {
    if (ptx::lane_id() == 0) producer_role<D>(sh, bb, args, smem, &tmap_x, &tmap_c);
    __syncwarp();
  } else if (warp == 9) {
    mma_role<D>(sh, bb, args, smem, tmem);
  }

  ptx::tc_fence_before_sync();
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(args.queue + 1, 1) == static_cast<int>(gridDim.x) - 1) {
      atomicExch(args.queue, 0);
      atomicExch(args.queue + 1, 0);
    }
  }
  if (warp == 9) {
    ptx::tc_fence_after_sync();
    ptx::tmem_dealloc(tmem, 512);
  }
}

}  // namespace kmeans
}  // namespace attn_b200
