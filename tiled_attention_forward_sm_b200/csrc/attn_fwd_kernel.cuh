// Dense attention forward for sm_100a: O = softmax(scale * Q K^T [+ causal
// mask]) V, plus the per-row natural-log LSE, computed tile by tile so the
// N x N score matrix never leaves the SM.
//
// Method (page lecompute.fr/kernel-perf/flashattention-4-limites-calcul-
// matriciel):
//  * section "Entre deux multiplications il faut fabriquer les poids":
//    scores from Q K^T, softmax weights, a second product with V; blocks of
//    Q/K/V are processed and O accumulated, the score matrix is not stored;
//  * section "Faire avancer plusieurs tuiles sans ecraser leurs donnees":
//    thread groups with distinct roles (data loading, softmax, MMA issue),
//    one tile in softmax while another occupies the tensor cores, several
//    result regions in Tensor Memory each with a producer/consumer lifetime;
//  * section "Deplacer une partie des exponentielles": a common scale kept
//    between old and new contributions, with some rescalings skipped under a
//    condition that keeps sums consistent and values in range.
//
// CTA work unit: two 128-row Q tiles (Q0, Q1) of one (batch, head), i.e.
// 256 query rows, against the K/V tiles they can see (128 keys per tile).
//
// Roles (12 warps, 384 threads):
//   warps 0-3   softmax group 0 (Q0): one thread per query row; also applies
//               the lazy O rescale and the epilogue for Q0
//   warps 4-7   softmax group 1 (Q1), same for Q1
//   warp  8     TMA producer: Q0/Q1 once, then K_j, V_j through a ring
//   warp  9     TMEM allocator and single-thread tcgen05 MMA issuer
//   warps 10-11 idle
//
// Tensor Memory plan (512 columns x 128 lanes x 32 bit):
//   cols [  0,128)  S0 (fp32 scores of Q0 K_j^T); P0 (bf16 pairs) in [0,64)
//   cols [128,256)  S1 / P1
//   cols [256,256+D) O0 accumulator (fp32)
//   cols [384,384+D) O1 accumulator
//
// MMA issue order per K/V step j (single thread, in-order tensor pipe):
//   PV0(j-1) ... S0(j) ... PV1(j-1) ... S1(j)
// so the commit that publishes S_s(j) also guarantees PV_s(j-1) finished:
// the softmax group may rescale O_s in place as soon as it sees S_s(j).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace attn_b200 {

// Device status word codes (mirrors attn_status in include/attn_b200.h).
constexpr int kStatusDeviceTimeout = -5;

// Bounded waits: a wait that has not completed after this long sets the
// status word and the CTA's abort flag, and every role then leaves its loop.
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

constexpr int kBlockM = 128;  // query rows per Q tile
constexpr int kBlockN = 128;  // keys per K/V tile
constexpr int kThreads = 384;

// Lazy-rescale threshold in log2 units: the running maximum is raised only
// when a tile's maximum exceeds it by more than this, so every weight stays
// at most 2^8 (fp32 row sums and bf16 weights stay far from overflow).
constexpr float kRescaleTau = 8.0f;

struct KernelArgs {
  __nv_bfloat16* o;   // [B*H*N, D]
  float* lse;         // [B*H*N]
  int N;              // keys/queries per head (multiple of 128)
  int n_qtiles;       // N / 128
  int n_qpairs;       // ceil(n_qtiles / 2)
  float scale_log2;   // scale * log2(e)
  int* status;        // device status word
};

template <int D>
struct Config {
  static_assert(D == 64 || D == 128, "head dim");
  static constexpr int kTileBytes = kBlockM * D * 2;        // one 128 x D bf16 tile
  static constexpr int kBoxes = D / 64;                      // 64-column TMA boxes per tile
  static constexpr int kBoxBytes = kBlockM * 64 * 2;         // 16 KB
  static constexpr int kStages = D == 128 ? 4 : 8;           // K/V ring depth
  static constexpr int kQOff = 0;
  static constexpr int kKVOff = 2 * kTileBytes;
  static constexpr int kBarOff = kKVOff + kStages * kTileBytes;
  // barriers: q_full, kv_full[S], kv_empty[S], s_full[2], p_ready[2],
  // o_final[2], drain
  static constexpr int kNumBars = 1 + 2 * kStages + 2 + 2 + 2 + 1;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kSmemBytes = kMiscOff + 16 + 1024;  // + alignment slack
  static constexpr uint32_t kIdescQK = ptx::idesc_bf16_f32(128, kBlockN, 0, 0);
  static constexpr uint32_t kIdescPV = ptx::idesc_bf16_f32(128, D, 0, 1);
};

struct Shared {
  uint64_t* q_full;
  uint64_t* kv_full;
  uint64_t* kv_empty;
  uint64_t* s_full;
  uint64_t* p_ready;
  uint64_t* o_final;
  uint64_t* drain;
  uint32_t* tmem_base;
  volatile int* abort_flag;
};

__device__ __forceinline__ void raise_status(const Shared& sh, int* status, int code) {
  *sh.abort_flag = 1;
  atomicCAS(status, 0, code);
}

// Single-thread bounded wait.  A drain wait (for this thread's own copies or
// MMAs in flight) ignores the abort flag but keeps the time limit.
__device__ __forceinline__ bool wait_one(const Shared& sh, int* status, uint64_t* bar,
                                         uint32_t parity, bool drain = false) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = ptx::globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0) {
      if (!drain && *sh.abort_flag) return false;
      if (ptx::globaltimer_ns() - t0 > kWaitLimitNs) {
        raise_status(sh, status, kStatusDeviceTimeout);
        return false;
      }
    }
  }
}

// Warp-uniform bounded wait (every lane returns the same answer), for roles
// whose next instructions are warp-collective tcgen05 loads/stores.
__device__ __forceinline__ bool wait_warp(const Shared& sh, int* status, uint64_t* bar,
                                          uint32_t parity) {
  uint64_t t0 = 0;
  for (uint32_t it = 0;; ++it) {
    const bool ok = ptx::mbar_try_wait(bar, parity);
    if (__all_sync(0xffffffffu, ok)) return true;
    if ((it & 63u) == 63u) {
      int stop = 0;
      if (ptx::lane_id() == 0) {
        const uint64_t now = ptx::globaltimer_ns();
        if (t0 == 0) t0 = now;
        if (*sh.abort_flag) {
          stop = 1;
        } else if (now - t0 > kWaitLimitNs) {
          raise_status(sh, status, kStatusDeviceTimeout);
          stop = 1;
        }
      }
      if (__shfl_sync(0xffffffffu, stop, 0)) return false;
    }
  }
}

// Number of K/V tiles Q tile `qt` visits.
template <bool CAUSAL>
__device__ __forceinline__ int kv_tiles_for(int qt, int n_qtiles) {
  if (qt >= n_qtiles) return 0;
  return CAUSAL ? qt + 1 : n_qtiles;
}

// ----------------------------------------------------------------- producer
template <int D, bool CAUSAL>
__device__ void producer_role(const Shared& sh, const KernelArgs& a, uint8_t* smem,
                              const CUtensorMap* tq, const CUtensorMap* tk,
                              const CUtensorMap* tv, int bh, int qpair) {
  using C = Config<D>;
  const int qt0 = 2 * qpair, qt1 = 2 * qpair + 1;
  const int n0 = kv_tiles_for<CAUSAL>(qt0, a.n_qtiles);
  const int n1 = kv_tiles_for<CAUSAL>(qt1, a.n_qtiles);
  const int n = n0 > n1 ? n0 : n1;
  const int row0 = bh * a.N;  // first row of this (b, h) in the 2-D views
  const uint64_t pol_q = ptx::policy_evict_first();
  const uint64_t pol_kv = ptx::policy_evict_last();

  // Q tiles (Q1 only if it exists)
  const int nq = (n1 > 0) ? 2 : 1;
  ptx::mbar_arrive_expect_tx(sh.q_full, nq * C::kTileBytes);
  for (int s = 0; s < nq; ++s)
    for (int b = 0; b < C::kBoxes; ++b)
      ptx::tma_load_2d(tq, sh.q_full, smem + C::kQOff + s * C::kTileBytes + b * C::kBoxBytes,
                       64 * b, row0 + (2 * qpair + s) * kBlockM, pol_q);

  int issued = 0;
  bool ok = true;
  for (int j = 0; j < n && ok; ++j) {
    for (int which = 0; which < 2; ++which) {  // 0: K_j, 1: V_j
      const int st = issued % C::kStages;
      const uint32_t ph = (issued / C::kStages) & 1;
      if (!wait_one(sh, a.status, &sh.kv_empty[st], ph ^ 1)) { ok = false; break; }
      uint8_t* dst = smem + C::kKVOff + st * C::kTileBytes;
      ptx::mbar_arrive_expect_tx(&sh.kv_full[st], C::kTileBytes);
      const CUtensorMap* m = which == 0 ? tk : tv;
      for (int b = 0; b < C::kBoxes; ++b)
        ptx::tma_load_2d(m, &sh.kv_full[st], dst + b * C::kBoxBytes, 64 * b,
                         row0 + j * kBlockN, pol_kv);
      ++issued;
    }
  }
  // Drain: every load issued must land before the CTA may exit.
  wait_one(sh, a.status, sh.q_full, 0, true);
  for (int t = (issued > C::kStages ? issued - C::kStages : 0); t < issued; ++t)
    wait_one(sh, a.status, &sh.kv_full[t % C::kStages], (t / C::kStages) & 1, true);
}

// ---------------------------------------------------------------------- MMA
template <int D, bool CAUSAL>
__device__ void mma_role(const Shared& sh, const KernelArgs& a, uint8_t* smem, uint32_t tmem,
                         int qpair) {
  using C = Config<D>;
  const int n0 = kv_tiles_for<CAUSAL>(2 * qpair, a.n_qtiles);
  const int n1 = kv_tiles_for<CAUSAL>(2 * qpair + 1, a.n_qtiles);
  const int n = n0 > n1 ? n0 : n1;
  const uint32_t q_addr = ptx::smem_u32(smem + C::kQOff);
  const uint32_t kv_addr = ptx::smem_u32(smem + C::kKVOff);
  const uint32_t t_s[2] = {tmem + 0, tmem + 128};
  const uint32_t t_o[2] = {tmem + 256, tmem + 384};

  // S_s = Q_s K^T over D (K-major operands, D/16 MMAs of K-depth 16)
  auto issue_qk = [&](int s, uint32_t k_addr) {
    const uint32_t qa = q_addr + s * C::kTileBytes;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint32_t off = (kk / 4) * C::kBoxBytes + (kk % 4) * 32;
      ptx::mma_ss(t_s[s], ptx::sdesc_sw128(qa + off, 16, 1024),
                  ptx::sdesc_sw128(k_addr + off, 16, 1024), C::kIdescQK, kk > 0 ? 1u : 0u);
    }
  };
  // O_s (+)= P_s V over the 128 keys (P from TMEM, V MN-major)
  auto issue_pv = [&](int s, uint32_t v_addr, bool accumulate) {
#pragma unroll
    for (int kk = 0; kk < kBlockN / 16; ++kk) {
      ptx::mma_ts(t_o[s], t_s[s] + 8 * kk, ptx::sdesc_sw128(v_addr + kk * 2048, C::kBoxBytes, 1024),
                  C::kIdescPV, (accumulate || kk > 0) ? 1u : 0u);
    }
  };

  int consumed = 0;
  auto stage_of = [&](int c) { return c % C::kStages; };
  auto phase_of = [&](int c) { return static_cast<uint32_t>((c / C::kStages) & 1); };

  if (!wait_one(sh, a.status, sh.q_full, 0)) goto done;
  {
    // step 0: S0(0), S1(0)
    int ck = consumed++;
    if (!wait_one(sh, a.status, &sh.kv_full[stage_of(ck)], phase_of(ck))) goto done;
    ptx::tc_fence_after_sync();
    const uint32_t k_addr0 = kv_addr + stage_of(ck) * C::kTileBytes;
    if (n0 > 0) { issue_qk(0, k_addr0); ptx::tc_commit(&sh.s_full[0]); }
    if (n1 > 0) { issue_qk(1, k_addr0); ptx::tc_commit(&sh.s_full[1]); }
    ptx::tc_commit(&sh.kv_empty[stage_of(ck)]);

    for (int j = 0; j < n; ++j) {
      const int cv = consumed++;
      if (!wait_one(sh, a.status, &sh.kv_full[stage_of(cv)], phase_of(cv))) goto done;
      const uint32_t v_addr = kv_addr + stage_of(cv) * C::kTileBytes;
      const uint32_t pj = static_cast<uint32_t>(j & 1);
      if (j < n0) {
        if (!wait_one(sh, a.status, &sh.p_ready[0], pj)) goto done;
        ptx::tc_fence_after_sync();
        issue_pv(0, v_addr, j > 0);
        if (j == n0 - 1) ptx::tc_commit(&sh.o_final[0]);
      }
      int ck2 = -1;
      uint32_t k_addr = 0;
      if (j + 1 < n) {
        ck2 = consumed++;
        if (!wait_one(sh, a.status, &sh.kv_full[stage_of(ck2)], phase_of(ck2))) goto done;
        ptx::tc_fence_after_sync();
        k_addr = kv_addr + stage_of(ck2) * C::kTileBytes;
        if (j + 1 < n0) { issue_qk(0, k_addr); ptx::tc_commit(&sh.s_full[0]); }
      }
      if (j < n1) {
        if (!wait_one(sh, a.status, &sh.p_ready[1], pj)) goto done;
        ptx::tc_fence_after_sync();
        issue_pv(1, v_addr, j > 0);
        if (j == n1 - 1) ptx::tc_commit(&sh.o_final[1]);
      }
      ptx::tc_commit(&sh.kv_empty[stage_of(cv)]);
      if (ck2 >= 0) {
        if (j + 1 < n1) { issue_qk(1, k_addr); ptx::tc_commit(&sh.s_full[1]); }
        ptx::tc_commit(&sh.kv_empty[stage_of(ck2)]);
      }
    }
  }
done:
  // Drain: every MMA this thread issued completes before TMEM is released.
  ptx::tc_commit(sh.drain);
  wait_one(sh, a.status, sh.drain, 0, true);
}

// ------------------------------------------------------------------ softmax
// One thread per query row; warp w of the group reads TMEM lanes
// [32*(w%4), 32*(w%4)+32), so row r = 32*(w%4) + lane is the tile row.
template <int D, bool CAUSAL>
__device__ void softmax_role(const Shared& sh, const KernelArgs& a, uint32_t tmem, int s, int bh,
                             int qpair, int warp_in_group) {
  const int qt = 2 * qpair + s;
  const int n_s = kv_tiles_for<CAUSAL>(qt, a.n_qtiles);
  if (n_s == 0) return;
  const int r = warp_in_group * 32 + static_cast<int>(ptx::lane_id());
  const uint32_t lane_off = static_cast<uint32_t>(warp_in_group * 32) << 16;
  const uint32_t t_s = tmem + lane_off + 128u * s;
  const uint32_t t_o = tmem + lane_off + 256u + 128u * s;
  const float sl2 = a.scale_log2;

  float m = -INFINITY;  // running max of scale*log2(e)*score (log2 units)
  float l = 0.f;        // running sum of weights, relative to 2^m

  for (int j = 0; j < n_s; ++j) {
    if (!wait_warp(sh, a.status, &sh.s_full[s], static_cast<uint32_t>(j & 1))) return;
    ptx::tc_fence_after_sync();

    uint32_t sr[128];
    ptx::tmem_ld32(t_s + 0, sr + 0);
    ptx::tmem_ld32(t_s + 32, sr + 32);
    ptx::tmem_ld32(t_s + 64, sr + 64);
    ptx::tmem_ld32(t_s + 96, sr + 96);
    ptx::tmem_ld_wait_tie(sr + 0);
    ptx::reg_tie32(sr + 32);
    ptx::reg_tie32(sr + 64);
    ptx::reg_tie32(sr + 96);

    float x[128];
#pragma unroll
    for (int c = 0; c < 128; ++c) x[c] = __uint_as_float(sr[c]);

    // Causal: the last visited tile is the diagonal one (key tile == query
    // tile); key c of it is visible to row r iff c <= r.
    if (CAUSAL && j == n_s - 1) {
#pragma unroll
      for (int c = 0; c < 128; ++c)
        if (c > r) x[c] = -INFINITY;
    }

    float mx0 = x[0], mx1 = x[1], mx2 = x[2], mx3 = x[3];
#pragma unroll
    for (int c = 4; c < 128; c += 4) {
      mx0 = fmaxf(mx0, x[c]);
      mx1 = fmaxf(mx1, x[c + 1]);
      mx2 = fmaxf(mx2, x[c + 2]);
      mx3 = fmaxf(mx3, x[c + 3]);
    }
    const float tile_max = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * sl2;

    // Lazy rescale: raise the running max only when it moves by > tau.
    float alpha = 1.f;
    bool rescale = false;
    if (tile_max - m > kRescaleTau) {  // also true on the first tile (m = -inf)
      alpha = ptx::ex2_approx(m - tile_max);  // 0 on the first tile
      m = tile_max;
      rescale = (j > 0);
    }
    const float neg_m = -m;

    float l0 = 0.f, l1 = 0.f, l2 = 0.f, l3 = 0.f;
    uint32_t pk[64];
#pragma unroll
    for (int c = 0; c < 128; c += 4) {
      const float p0 = ptx::ex2_approx(fmaf(x[c], sl2, neg_m));
      const float p1 = ptx::ex2_approx(fmaf(x[c + 1], sl2, neg_m));
      const float p2 = ptx::ex2_approx(fmaf(x[c + 2], sl2, neg_m));
      const float p3 = ptx::ex2_approx(fmaf(x[c + 3], sl2, neg_m));
      l0 += p0; l1 += p1; l2 += p2; l3 += p3;
      pk[c / 2] = ptx::pack_bf16x2(p0, p1);
      pk[c / 2 + 1] = ptx::pack_bf16x2(p2, p3);
    }
    l = l * alpha + ((l0 + l1) + (l2 + l3));

    // P_s (bf16 pairs) over the first 64 columns of the S_s region.
    ptx::tmem_st32(t_s + 0, pk + 0);
    ptx::tmem_st32(t_s + 32, pk + 32);

    // O_s *= alpha for the rows whose max moved (PV_s(j-1) is complete: its
    // commit preceded the one that published S_s(j)).
    if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t ov[32];
        ptx::tmem_ld32(t_o + c0, ov);
        ptx::tmem_ld_wait_tie(ov);
#pragma unroll
        for (int c = 0; c < 32; ++c) ov[c] = __float_as_uint(__uint_as_float(ov[c]) * alpha);
        ptx::tmem_st32(t_o + c0, ov);
      }
    }
    ptx::tmem_st_wait();
    ptx::tc_fence_before_sync();
    ptx::mbar_arrive(&sh.p_ready[s]);
  }

  // Epilogue: O_s / l -> bf16 rows; LSE = (m + log2 l) * ln 2.
  if (!wait_warp(sh, a.status, &sh.o_final[s], 0)) return;
  ptx::tc_fence_after_sync();
  const float inv_l = 1.f / l;
  const size_t row_g = static_cast<size_t>(bh) * a.N + static_cast<size_t>(qt) * kBlockM + r;
  __nv_bfloat16* orow = a.o + row_g * D;
#pragma unroll 1
  for (int c0 = 0; c0 < D; c0 += 32) {
    uint32_t ov[32];
    ptx::tmem_ld32(t_o + c0, ov);
    ptx::tmem_ld_wait_tie(ov);
    uint32_t pk[16];
#pragma unroll
    for (int c = 0; c < 16; ++c)
      pk[c] = ptx::pack_bf16x2(__uint_as_float(ov[2 * c]) * inv_l,
                               __uint_as_float(ov[2 * c + 1]) * inv_l);
    uint4* dst = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
    for (int v = 0; v < 4; ++v)
      dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
  }
  a.lse[row_g] = (m + log2f(l)) * 0.69314718055994531f;
}

// ------------------------------------------------------------------- kernel
template <int D, bool CAUSAL>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmap_q,
                    const __grid_constant__ CUtensorMap tmap_k,
                    const __grid_constant__ CUtensorMap tmap_v, const KernelArgs args) {
  using C = Config<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

  Shared sh;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  sh.q_full = bars;
  sh.kv_full = bars + 1;
  sh.kv_empty = bars + 1 + C::kStages;
  sh.s_full = bars + 1 + 2 * C::kStages;
  sh.p_ready = sh.s_full + 2;
  sh.o_final = sh.p_ready + 2;
  sh.drain = sh.o_final + 2;
  sh.tmem_base = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
  sh.abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 4);

  const int warp = threadIdx.x / 32;
  // Heaviest query tiles first under the causal mask (blockIdx.y = 0 runs
  // first and takes the last pair).
  const int bh = blockIdx.x;
  const int qpair = CAUSAL ? (args.n_qpairs - 1 - static_cast<int>(blockIdx.y))
                           : static_cast<int>(blockIdx.y);

  if (threadIdx.x == 0) {
    ptx::mbar_init(sh.q_full, 1);
    for (int i = 0; i < C::kStages; ++i) {
      ptx::mbar_init(&sh.kv_full[i], 1);
      ptx::mbar_init(&sh.kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&sh.s_full[i], 1);
      ptx::mbar_init(&sh.p_ready[i], 128);
      ptx::mbar_init(&sh.o_final[i], 1);
    }
    ptx::mbar_init(sh.drain, 1);
    *sh.abort_flag = 0;
    ptx::fence_barrier_init();
  }
  if (warp == 8 && ptx::lane_id() == 0) {
    ptx::prefetch_tmap(&tmap_q);
    ptx::prefetch_tmap(&tmap_k);
    ptx::prefetch_tmap(&tmap_v);
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
    softmax_role<D, CAUSAL>(sh, args, tmem, warp / 4, bh, qpair, warp % 4);
  } else if (warp == 8) {
    if (ptx::lane_id() == 0)
      producer_role<D, CAUSAL>(sh, args, smem, &tmap_q, &tmap_k, &tmap_v, bh, qpair);
    __syncwarp();
  } else if (warp == 9) {
    if (ptx::lane_id() == 0) mma_role<D, CAUSAL>(sh, args, smem, tmem, qpair);
    __syncwarp();
  }

  ptx::tc_fence_before_sync();
  __syncthreads();
  if (warp == 9) {
    ptx::tc_fence_after_sync();
    ptx::tmem_dealloc(tmem, 512);
  }
}

}  // namespace attn_b200
