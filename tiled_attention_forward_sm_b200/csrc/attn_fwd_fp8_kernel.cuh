// FP8 (E4M3) attention forward on sm_100a, head dim 128: the low-precision
// variant the page lecompute.fr/kernel-perf/flashattention-4-limites-calcul-
// matriciel weighs in section "Le FP4 ajoute un compromis numerique" (fewer
// bits per operand buy tensor throughput, at a numeric cost and a
// conversion cost).
//
// Same pipeline, work items and Tensor Memory plan as attn_fwd_kernel.cuh
// (two Q tiles per CTA, S and O of each in TMEM, P over its S region), with
// 8-bit operands:
//  * Q, K and V^T arrive as E4M3 with per-tensor fp32 descale factors; V is
//    taken transposed ([B, H, d, N]) so that both products read K-major
//    shared-memory operands: a 128 x 128 E4M3 tile is one 128-byte swizzle
//    row per tile row (16 KB);
//  * S = Q K^T and O += P V are tcgen05 kind::f8f6f4 MMAs (K = 32 per MMA);
//  * P is rounded to E4M3 (nearest even) in the softmax, four keys per TMEM
//    column, and read from TMEM by the second product;
//  * the row sum l is taken from the unrounded fp32 weights.
// Under the lazy rule every weight is at most 2^8, inside E4M3's range
// (448); weights below 2^-9 round to zero.
#pragma once

#include "attn_fwd_kernel.cuh"

namespace attn_b200 {
namespace fp8 {

// Of every 4 quadruples of score columns, how many take their exponentials
// from the FMA pipe (exp2_poly5) instead of the special-function unit: the
// split of the page's section "Deplacer une partie des exponentielles".
// Measured on B200 at d = 128, 1 of 4 is 2-3% faster in short runs but 3%
// slower in sustained runs, where the 1 kW power limit sets the clock: the
// polynomial costs more energy per exponential than the special-function
// unit (median clock 1790-1810 against 1840-1905 MHz).  2 of 4 is slower
// in both.  Hence 0.
constexpr int kPolyQuads = 0;

// exp2 on the FMA pipe for a pair of inputs, as exp2_poly2 in the bf16
// kernel but with a degree-5 polynomial for 2^f on [-1/2, 1/2]
// (coefficients from csrc/gen_exp2_poly.py; the fp32 sequence stays within
// 2.2e-7 relative of 2^x, about the special-function unit's error, so E4M3
// rounding of the weights flips no more often than with ex2.approx).
__device__ __forceinline__ uint64_t exp2_poly5(uint64_t x2) {
  constexpr float kE0 = 1.0000001192092896f, kE1 = 0.6931469440460205f;
  constexpr float kE2 = 0.24022120237350464f, kE3 = 0.05550713092088699f;
  constexpr float kE4 = 0.009675540961325169f, kE5 = 0.0013276472454890609f;
  constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
  float x0, x1;
  ptx::f2unpack(x2, x0, x1);
  x2 = ptx::f2pack(fmaxf(x0, -125.f), fmaxf(x1, -125.f));
  const uint64_t magic = ptx::f2pack(kMagic, kMagic);
  const uint64_t t = ptx::fadd2(x2, magic);
  const uint64_t f = ptx::fsub2(x2, ptx::fsub2(t, magic));
  uint64_t p = ptx::ffma2(f, ptx::f2pack(kE5, kE5), ptx::f2pack(kE4, kE4));
  p = ptx::ffma2(f, p, ptx::f2pack(kE3, kE3));
  p = ptx::ffma2(f, p, ptx::f2pack(kE2, kE2));
  p = ptx::ffma2(f, p, ptx::f2pack(kE1, kE1));
  p = ptx::ffma2(f, p, ptx::f2pack(kE0, kE0));
  float p0, p1, t0, t1;
  ptx::f2unpack(p, p0, p1);
  ptx::f2unpack(t, t0, t1);
  return ptx::f2pack(__uint_as_float(__float_as_uint(p0) + (__float_as_uint(t0) << 23)),
                     __uint_as_float(__float_as_uint(p1) + (__float_as_uint(t1) << 23)));
}

constexpr int kD = 128;
constexpr int kTileBytes = kBlockM * kD;  // 16 KB: 128 rows of 128 E4M3 values
constexpr int kStages = 8;                // K / V^T ring depth
constexpr int kQOff = 0;
constexpr int kKVOff = 2 * kTileBytes;
// O staging for the epilogue's TMA stores without the causal mask: one
// 64-column bf16 box of 32 rows (4 KB) per softmax warp.
constexpr int kOOff = kKVOff + kStages * kTileBytes;
constexpr int kOWarpBytes = 4096;
constexpr int kBarOff = kOOff + 8 * kOWarpBytes;
// barriers: q_full[2], q_empty[2], kv_full[S], kv_empty[S], s_full[2],
// p_ready[2 tiles][2 halves], o_final[2], drain, item_full[R], item_empty[R]
constexpr int kNumBars = 4 + 2 * kStages + 2 + 4 + 2 + 1 + 2 * kItemSlots;
constexpr int kMiscOff = kBarOff + kNumBars * 8;
constexpr int kRingOff = kMiscOff + 16;
constexpr int kSmemBytes = kRingOff + 4 * kItemWords * kItemSlots + 1024;
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
constexpr uint32_t kIdesc = ptx::idesc_e4m3_f32(128, 128, 0, 0);  // QK and PV: M = N = 128

struct Bars {
  uint64_t* q_full;
  uint64_t* q_empty;
  uint64_t* kv_full;
  uint64_t* kv_empty;
  uint64_t* s_full;
  uint64_t* p_ready;
  uint64_t* o_final;
};

template <bool CAUSAL>
__device__ void producer_role(const Shared& sh, const Bars& bb, const KernelArgs& a,
                              uint8_t* smem, const CUtensorMap* tq, const CUtensorMap* tk,
                              const CUtensorMap* tvt) {
  const uint64_t pol_q = ptx::policy_evict_first();
  const uint64_t pol_kv = ptx::policy_evict_last();
  int q_loads[2] = {0, 0};
  int issued = 0;
  bool ok = true;
  Item it{};
  auto claim = [&]() -> bool {
    for (;;) {
      const int idx = atomicAdd(a.queue, 1);
      if (idx >= a.n_items) return false;
      if (make_item<CAUSAL>(idx, a, a.status, it)) return true;
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
      if (q_loads[s] > 0 &&
          !wait_one(sh, a.status, &bb.q_empty[s], static_cast<uint32_t>((q_loads[s] - 1) & 1))) {
        ok = false;
        break;
      }
      ptx::mbar_arrive_expect_tx(&bb.q_full[s], kTileBytes);
      ptx::tma_load_3d(tq, &bb.q_full[s], smem + kQOff + s * kTileBytes, 0,
                       (2 * it.qpair + s) * kBlockM, it.qz, pol_q);
      ++q_loads[s];
    }
    for (int j = 0; j < n && ok; ++j) {
      for (int which = 0; which < 2; ++which) {  // K_j (keys x d), then V^T_j (d x keys)
        const int st = issued % kStages;
        const uint32_t ph = (issued / kStages) & 1;
        if (!wait_one(sh, a.status, &bb.kv_empty[st], ph ^ 1)) {
          ok = false;
          break;
        }
        if (withhold_load(issued)) {  // test builds only
          ++issued;
          continue;
        }
        ptx::mbar_arrive_expect_tx(&bb.kv_full[st], kTileBytes);
        if (which == 0)
          ptx::tma_load_3d(tk, &bb.kv_full[st], smem + kKVOff + st * kTileBytes, 0,
                           (it.kt0 + j) * kBlockN, it.kz, pol_kv);
        else
          ptx::tma_load_3d(tvt, &bb.kv_full[st], smem + kKVOff + st * kTileBytes,
                           (it.kt0 + j) * kBlockN, 0, it.kz, pol_kv);
        ++issued;
      }
    }
    if (ok) have = claim();
  }
  for (int s = 0; s < 2; ++s)
    if (q_loads[s] > 0)
      wait_one(sh, a.status, &bb.q_full[s], static_cast<uint32_t>((q_loads[s] - 1) & 1), true);
  for (int t = (issued > kStages ? issued - kStages : 0); t < issued; ++t)
    wait_one(sh, a.status, &bb.kv_full[t % kStages], (t / kStages) & 1, true);
}

// MMA issue order per K/V step j, as in attn_fwd_kernel.cuh:
// PV0(j), S0(j+1), PV1(j), S1(j+1).
template <bool CAUSAL>
__device__ void mma_role(const Shared& sh, const Bars& bb, const KernelArgs& a, uint8_t* smem,
                         uint32_t tmem) {
  const uint32_t t_s[2] = {tmem + 0, tmem + 128};
  const uint32_t t_o[2] = {tmem + 256, tmem + 384};
  // K-major 8-bit operands: a row is 128 B, SBO = 1024 B between 8-row
  // groups, a 32-deep K step moves 32 B inside the swizzle row.
  const uint64_t q_desc = ptx::sdesc_sw128(ptx::smem_u32(smem + kQOff), 16, 1024);
  const uint64_t kv_desc = ptx::sdesc_sw128(ptx::smem_u32(smem + kKVOff), 16, 1024);
  constexpr uint64_t kTileUnits = kTileBytes >> 4;
  auto issue_qk = [&](int s, int stage) {
    const uint64_t qd = q_desc + s * kTileUnits;
    const uint64_t kd = kv_desc + stage * kTileUnits;
#pragma unroll
    for (int kk = 0; kk < kD / 32; ++kk)
      ptx::mma_f8_ss_elect(t_s[s], qd + static_cast<uint64_t>((kk * 32) >> 4),
                           kd + static_cast<uint64_t>((kk * 32) >> 4), kIdesc, kk > 0 ? 1u : 0u);
  };
  // O_s (+)= P_s V over keys [64*half, 64*half+64): P from TMEM (four keys
  // per column, 8 columns per 32 keys), V^T K-major (32 B per 32 keys).
  auto issue_pv_half = [&](int s, int half, int stage, uint32_t accumulate) {
    const uint64_t vd = kv_desc + stage * kTileUnits;
#pragma unroll
    for (int k2 = 0; k2 < 2; ++k2) {
      const int kk = 2 * half + k2;
      ptx::mma_f8_ts_elect(t_o[s], t_s[s] + 8 * kk, vd + static_cast<uint64_t>((kk * 32) >> 4),
                           kIdesc, (accumulate | static_cast<uint32_t>(kk > 0)));
    }
  };
  int p_count[2] = {0, 0};
  auto issue_pv = [&](int s, int stage, uint32_t accumulate) -> bool {
    const uint32_t parity = static_cast<uint32_t>(p_count[s] & 1);
    ++p_count[s];
    for (int half = 0; half < 2; ++half) {
      if (!wait_warp(sh, a.status, &bb.p_ready[2 * s + half], parity)) return false;
      ptx::tc_fence_after_sync();
      issue_pv_half(s, half, stage, accumulate);
    }
    return true;
  };
  auto issue_s = [&](int s, int j, int n_s, int stage) {
    issue_qk(s, stage);
    ptx::commit_elect(&bb.s_full[s]);
    if (j == n_s - 1) ptx::commit_elect(&bb.q_empty[s]);
  };
  int consumed = 0;
  int q_uses[2] = {0, 0};
  auto stage_of = [&](int c) { return c % kStages; };
  auto phase_of = [&](int c) { return static_cast<uint32_t>((c / kStages) & 1); };
  Item it;
  bool ok = true;
  for (int r = 0; read_item(sh, a, r, it, ok); ++r) {
    const int n0 = it.n0, n1 = it.n1;
    const int n = n0 > n1 ? n0 : n1;
    if (n == 0) continue;
    for (int s = 0; s < 2; ++s) {
      if ((s == 0 ? n0 : n1) == 0) continue;
      if (!wait_warp(sh, a.status, &bb.q_full[s], static_cast<uint32_t>(q_uses[s] & 1))) goto done;
      ++q_uses[s];
    }
    {
      const int ck = consumed++;
      if (!wait_warp(sh, a.status, &bb.kv_full[stage_of(ck)], phase_of(ck))) goto done;
      ptx::tc_fence_after_sync();
      if (n0 > 0) issue_s(0, 0, n0, stage_of(ck));
      if (n1 > 0) issue_s(1, 0, n1, stage_of(ck));
      ptx::commit_elect(&bb.kv_empty[stage_of(ck)]);
      for (int j = 0; j < n; ++j) {
        const int cv = consumed++;
        if (!wait_warp(sh, a.status, &bb.kv_full[stage_of(cv)], phase_of(cv))) goto done;
        const int ck2 = (j + 1 < n) ? consumed++ : -1;
        if (ck2 >= 0 && !wait_warp(sh, a.status, &bb.kv_full[stage_of(ck2)], phase_of(ck2)))
          goto done;
        ptx::tc_fence_after_sync();
        const uint32_t acc = j > 0 ? 1u : 0u;
        if (j < n0) {
          if (!issue_pv(0, stage_of(cv), acc)) goto done;
          if (j == n0 - 1) ptx::commit_elect(&bb.o_final[0]);
        }
        if (ck2 >= 0 && j + 1 < n0) issue_s(0, j + 1, n0, stage_of(ck2));
        if (j < n1) {
          if (!issue_pv(1, stage_of(cv), acc)) goto done;
          if (j == n1 - 1) ptx::commit_elect(&bb.o_final[1]);
        }
        ptx::commit_elect(&bb.kv_empty[stage_of(cv)]);
        if (ck2 >= 0) {
          if (j + 1 < n1) issue_s(1, j + 1, n1, stage_of(ck2));
          ptx::commit_elect(&bb.kv_empty[stage_of(ck2)]);
        }
      }
    }
  }
done:
  ptx::commit_elect(sh.drain);
  wait_warp(sh, a.status, sh.drain, 0, true);
}

// The epilogue follows the bf16 kernel's: without the causal mask the two
// groups finish an item together, so O leaves through this warp's staging
// box and a TMA store per 64 columns instead of row-per-thread stores.
template <bool CAUSAL>
__device__ void softmax_role(const Shared& sh, const Bars& bb, const KernelArgs& a,
                             float v_descale, uint32_t tmem, int s, int warp_in_group,
                             uint8_t* o_stage, const CUtensorMap* tmap_o) {
  const int lane = static_cast<int>(ptx::lane_id());
  const int r = warp_in_group * 32 + lane;
  const uint32_t lane_off = static_cast<uint32_t>(warp_in_group * 32) << 16;
  const uint32_t t_s = tmem + lane_off + 128u * s;
  const uint32_t t_o = tmem + lane_off + 256u + 128u * s;
  const float sl2 = a.scale_log2;
  const uint64_t sl2x2 = ptx::f2pack(sl2, sl2);
  int s_count = 0, o_count = 0;
  Item it;
  bool ok = true;
  for (int rr = 0; read_item(sh, a, rr, it, ok); ++rr) {
    const int qt = 2 * it.qpair + s;
    const int row = qt * kBlockM + r;
    if (qt * kBlockM >= it.q_len) continue;
    const int n_s = s == 0 ? it.n0 : it.n1;
    float m = -INFINITY, l = 0.f;
    for (int j = 0; j < n_s; ++j) {
      const int key0 = (it.kt0 + j) * kBlockN;
      int key_limit = it.k_len - key0;
      if (CAUSAL) {
        const long long lim = static_cast<long long>(row) + it.delta + 1 - key0;
        if (lim < key_limit) key_limit = lim < -1 ? -1 : static_cast<int>(lim);
      }
      if (!wait_warp(sh, a.status, &bb.s_full[s], static_cast<uint32_t>(s_count & 1))) return;
      ++s_count;
      ptx::tc_fence_after_sync();
      const bool masked = __any_sync(0xffffffffu, key_limit < kBlockN);
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
      if (masked) {
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c >= key_limit) x[c] = -INFINITY;
      }
      float mx[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) mx[k] = x[k];
#pragma unroll
      for (int c = 8; c + 16 <= 128; c += 16) {
#pragma unroll
        for (int k = 0; k < 8; ++k) mx[k] = ptx::max3(mx[k], x[c + 2 * k], x[c + 2 * k + 1]);
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) mx[k] = ptx::max3(mx[k], x[120 + 2 * k], x[121 + 2 * k]);
      const float tile_max = ptx::max3(ptx::max3(mx[0], mx[1], mx[2]),
                                       ptx::max3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7])) *
                             sl2;
      float alpha = 1.f;
      bool rescale = false;
      if (tile_max - m > kRescaleTau) {
        alpha = ptx::ex2_approx(m - tile_max);
        m = tile_max;
        rescale = j > 0;
      }
      // O_s *= alpha (PV_s(j-1) complete: its commit preceded S_s(j)'s).
      if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
        for (int c0 = 0; c0 < kD; c0 += 32) {
          uint32_t ov[32];
          ptx::tmem_ld32(t_o + c0, ov);
          ptx::tmem_ld_wait_tie(ov);
#pragma unroll
          for (int c = 0; c < 32; ++c) ov[c] = __float_as_uint(__uint_as_float(ov[c]) * alpha);
          ptx::tmem_st32(t_o + c0, ov);
        }
      }
      const float negm = m == -INFINITY ? 0.f : -m;
      const uint64_t negm2 = ptx::f2pack(negm, negm);
      uint64_t sa = ptx::f2pack(0.f, 0.f), sb = sa;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t pk[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const int c = 64 * half + 4 * q;
          const uint64_t y01 = ptx::ffma2(ptx::f2pack(x[c], x[c + 1]), sl2x2, negm2);
          const uint64_t y23 = ptx::ffma2(ptx::f2pack(x[c + 2], x[c + 3]), sl2x2, negm2);
          float y0, y1, y2, y3;
          ptx::f2unpack(y01, y0, y1);
          ptx::f2unpack(y23, y2, y3);
          float p0, p1, p2, p3;
          if ((q & 3) < kPolyQuads) {
            ptx::f2unpack(exp2_poly5(y01), p0, p1);
            ptx::f2unpack(exp2_poly5(y23), p2, p3);
          } else {
            p0 = ptx::ex2_approx(y0);
            p1 = ptx::ex2_approx(y1);
            p2 = ptx::ex2_approx(y2);
            p3 = ptx::ex2_approx(y3);
          }
          sa = ptx::fadd2(sa, ptx::f2pack(p0, p1));
          sb = ptx::fadd2(sb, ptx::f2pack(p2, p3));
          pk[q] = ptx::pack_e4m3x4(p0, p1, p2, p3);
        }
        // P_s keys [64*half, 64*half+64) as E4M3 quadruples over TMEM
        // columns [16*half, 16*half+16) of the S_s region.
        ptx::tmem_st16(t_s + 16 * half, pk);
        ptx::tmem_st_wait();
        ptx::tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&bb.p_ready[2 * s + half]);
      }
      float la0, la1, lb0, lb1;
      ptx::f2unpack(sa, la0, la1);
      ptx::f2unpack(sb, lb0, lb1);
      l = l * alpha + ((la0 + la1) + (lb0 + lb1));
    }

    if (n_s > 0) {
      if (!wait_warp(sh, a.status, &bb.o_final[s], static_cast<uint32_t>(o_count & 1))) return;
      ++o_count;
      ptx::tc_fence_after_sync();
    }
    const bool row_ok = row < it.q_len;
    const bool empty = m == -INFINITY;
    const float f = empty ? 0.f : v_descale / l;
    const size_t o_row = static_cast<size_t>(it.qz) * a.N_q + row;
    __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(a.o) + o_row * kD;
    if constexpr (!CAUSAL) {
      const uint32_t row_addr = ptx::smem_u32(o_stage) + static_cast<uint32_t>(lane) * 128u;
      const uint32_t sw = static_cast<uint32_t>(lane & 7);  // 128-byte swizzle
      uint32_t ov0[32], ov1[32];
      auto load_box = [&](int b) {
        if (n_s > 0) {
          ptx::tmem_ld32(t_o + 64 * b, ov0);
          ptx::tmem_ld32(t_o + 64 * b + 32, ov1);
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) ov0[c] = ov1[c] = 0u;
        }
      };
      auto wait_box = [&]() {
        if (n_s > 0) {
          ptx::tmem_ld_wait_tie(ov0);
          ptx::reg_tie32(ov1);
        }
      };
      load_box(0);
      wait_box();
#pragma unroll 1
      for (int b = 0; b < kD / 64; ++b) {
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          pk[c] = ptx::pack_bf16x2(__uint_as_float(ov0[2 * c]) * f,
                                   __uint_as_float(ov0[2 * c + 1]) * f);
          pk[16 + c] = ptx::pack_bf16x2(__uint_as_float(ov1[2 * c]) * f,
                                        __uint_as_float(ov1[2 * c + 1]) * f);
        }
        if (b + 1 < kD / 64) load_box(b + 1);
        // the box is rewritten once the previous store has read it
        if (lane == 0) ptx::bulk_wait_read_all();
        __syncwarp();
#pragma unroll
        for (int c = 0; c < 8; ++c)
          ptx::st_shared_v4(row_addr + ((static_cast<uint32_t>(c) ^ sw) << 4), pk[4 * c],
                            pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        ptx::fence_proxy_async_smem();
        __syncwarp();
        const int row0 = qt * kBlockM + 32 * warp_in_group;
        if (lane == 0 && row0 < it.q_len) {
          ptx::tma_store_3d(tmap_o, o_stage, 64 * b, row0, it.qz);
          ptx::bulk_commit_group();
        }
        if (b + 1 < kD / 64) wait_box();
      }
    } else {
#pragma unroll 1
      for (int c0 = 0; c0 < kD; c0 += 32) {
        uint32_t ov[32];
        if (n_s > 0) {
          ptx::tmem_ld32(t_o + c0, ov);
          ptx::tmem_ld_wait_tie(ov);
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) ov[c] = 0u;
        }
        if (!row_ok) continue;
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 16; ++c)
          pk[c] = ptx::pack_bf16x2(__uint_as_float(ov[2 * c]) * f,
                                   __uint_as_float(ov[2 * c + 1]) * f);
        uint4* dst = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
        for (int v = 0; v < 4; ++v)
          dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
      }
    }
    if (row_ok) a.lse[o_row] = empty ? -INFINITY : (m + log2f(l)) * 0.69314718055994531f;
  }
}

template <bool CAUSAL>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_fp8_kernel(const __grid_constant__ CUtensorMap tmap_q,
                        const __grid_constant__ CUtensorMap tmap_k,
                        const __grid_constant__ CUtensorMap tmap_vt,
                        const __grid_constant__ CUtensorMap tmap_o, const KernelArgs args,
                        float v_descale) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBarOff);
  Bars bb;
  bb.q_full = bars;
  bb.q_empty = bars + 2;
  bb.kv_full = bars + 4;
  bb.kv_empty = bb.kv_full + kStages;
  bb.s_full = bb.kv_empty + kStages;
  bb.p_ready = bb.s_full + 2;
  bb.o_final = bb.p_ready + 4;
  Shared sh = {};
  sh.drain = bb.o_final + 2;
  sh.item_full = sh.drain + 1;
  sh.item_empty = sh.item_full + kItemSlots;
  sh.tmem_base = reinterpret_cast<uint32_t*>(smem + kMiscOff);
  sh.abort_flag = reinterpret_cast<volatile int*>(smem + kMiscOff + 4);
  sh.item_ring = reinterpret_cast<volatile int*>(smem + kRingOff);

  const int warp = threadIdx.x / 32;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&bb.q_full[i], 1);
      ptx::mbar_init(&bb.q_empty[i], 1);
      ptx::mbar_init(&bb.s_full[i], 1);
      ptx::mbar_init(&bb.p_ready[2 * i], 4);
      ptx::mbar_init(&bb.p_ready[2 * i + 1], 4);
      ptx::mbar_init(&bb.o_final[i], 1);
    }
    for (int i = 0; i < kStages; ++i) {
      ptx::mbar_init(&bb.kv_full[i], 1);
      ptx::mbar_init(&bb.kv_empty[i], 1);
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
    ptx::prefetch_tmap(&tmap_q);
    ptx::prefetch_tmap(&tmap_k);
    ptx::prefetch_tmap(&tmap_vt);
  }
  if (warp == 9) {
    ptx::tmem_alloc(sh.tmem_base, 512);
    ptx::tmem_relinquish();
  }
  if (warp >= 8) ptx::setmaxnreg_dec<kRegsOther>();
  ptx::tc_fence_before_sync();
  __syncthreads();
  ptx::tc_fence_after_sync();
  const uint32_t tmem = *sh.tmem_base;

  if (warp < 8) {
    ptx::setmaxnreg_inc<kRegsSoftmax>();
    softmax_role<CAUSAL>(sh, bb, args, v_descale, tmem, warp / 4, warp % 4,
                         smem + kOOff + warp * kOWarpBytes, &tmap_o);
    // the staging boxes are read before the CTA exits
    if constexpr (!CAUSAL) ptx::bulk_wait_read_all();
  } else if (warp == 8) {
    if (ptx::lane_id() == 0) producer_role<CAUSAL>(sh, bb, args, smem, &tmap_q, &tmap_k, &tmap_vt);
    __syncwarp();
  } else if (warp == 9) {
    mma_role<CAUSAL>(sh, bb, args, smem, tmem);
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

}  // namespace fp8
}  // namespace attn_b200
