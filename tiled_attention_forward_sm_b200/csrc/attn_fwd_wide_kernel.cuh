// Attention forward for head dim 256 on sm_100a: the same operation and
// work items as attn_fwd_kernel.cuh (whose scheduling helpers it reuses), with
// a Tensor Memory plan that fits 256-column accumulators.
//
// Two Q tiles with their own S and O (the plan of attn_fwd_kernel.cuh) would
// need 2 x (128 + 256) columns, more than the 512 of Tensor Memory.  Here a
// CTA processes the two Q tiles of a work item one after the other, with
//   cols [  0,128)  S buffer 0 (fp32 scores of even K/V tiles; P over [0,64))
//   cols [128,256)  S buffer 1 (odd tiles)
//   cols [256,512)  O (fp32, 256 columns)
// and one softmax warpgroup.  With S double-buffered the score tile
// QK(j+2) is computed while the softmax works on tile j+1, and PV(j) on the
// tensor pipe meanwhile: at d = 256 the two products of a tile take twice
// the tensor time of d = 128, which one softmax group keeps up with.
//
// MMA issue order per Q tile (one thread, in-order tensor pipe):
//   QK(0), QK(1), then per K/V tile j: PV(j) in two halves, QK(j+2).
// K and V tiles enter one two-stage ring in that consumption order:
//   K0, K1, then per tile j: V_j, K_{j+2}.
//
// Roles (6 warps, 192 threads): warps 0-3 softmax (one thread per query
// row, lazy O rescale, epilogue), warp 4 TMA producer, warp 5 TMEM
// allocator and MMA issuer.
#pragma once

#include "attn_fwd_kernel.cuh"

namespace attn_b200 {
namespace wide {

constexpr int kD = 256;
constexpr int kThreads = 192;
constexpr int kBoxes = kD / 64;                    // 64-column TMA boxes per tile
constexpr int kBoxBytes = kBlockM * 64 * 2;        // 16 KB
constexpr int kTileBytes = kBoxes * kBoxBytes;     // 64 KB: one 128 x 256 bf16 tile
constexpr int kStages = 2;                         // K/V ring depth
constexpr int kQOff = 0;                           // one Q buffer
constexpr int kKVOff = kTileBytes;
// O staging for the epilogue's TMA stores (bf16 per-head output without key
// slices): two 64-column boxes of 32 rows (2 x 4 KB) per softmax warp.  A
// warp store of row-per-thread output touches 32 rows, so one 256-column
// tile took 4 x 32 such instructions of 32 lines each through the load/store
// unit; through shared memory and TMA the same tile costs 8-row conflict-free
// 16-byte stores and 16 bulk stores.
constexpr int kOOff = kKVOff + kStages * kTileBytes;
constexpr int kOWarpBytes = 8192;
constexpr int kBarOff = kOOff + 4 * kOWarpBytes;
// barriers: q_full, q_empty, kv_full[S], kv_empty[S], s_full[2],
// p_ready[2 buffers][2 halves], pv_done, o_ready, drain, item_full[R],
// item_empty[R]
constexpr int kNumBars = 2 + 2 * kStages + 2 + 4 + 1 + 1 + 1 + 2 * kItemSlots;
constexpr int kMiscOff = kBarOff + kNumBars * 8;
constexpr int kRingOff = kMiscOff + 16;
constexpr int kSmemBytes = kRingOff + 4 * kItemWords * kItemSlots + 1024;  // + alignment slack
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
// Readers of each item-ring slot: the MMA warp and the 4 softmax warps.
constexpr int kReaders = 5;
constexpr uint32_t kIdescQK = ptx::idesc_bf16_f32(128, kBlockN, 0, 0);
constexpr uint32_t kIdescPV = ptx::idesc_bf16_f32(128, kD, 0, 1);
constexpr uint32_t kTmemO = 256;

struct Bars {
  uint64_t* q_full;
  uint64_t* q_empty;
  uint64_t* kv_full;   // [kStages]
  uint64_t* kv_empty;  // [kStages]
  uint64_t* s_full;    // [2] S buffer b holds the next tile's scores
  uint64_t* p_ready;   // [2 buffers][2 halves] half of P in S buffer b
  uint64_t* pv_done;   // PV of a K/V tile complete (one phase per tile)
  uint64_t* o_ready;   // the Q tile's last PV complete (one phase per Q tile
                       // with at least one K/V tile)
};

// The Q tiles of an item, in processing order: (tile of the pair, K/V tiles).
__device__ __forceinline__ int tile_n(const Item& it, int s) { return s == 0 ? it.n0 : it.n1; }

// --------------------------------------------------------------- producer
template <bool CAUSAL>
__device__ void producer_role(const Shared& sh, const Bars& bb, const KernelArgs& a,
                              uint8_t* smem, const CUtensorMap* tq, const CUtensorMap* tk,
                              const CUtensorMap* tv) {
  const uint64_t pol_q = ptx::policy_evict_first();
  const uint64_t pol_kv = ptx::policy_evict_last();
  const bool packed = a.cu_q != nullptr;
  auto load_tile = [&](const CUtensorMap* m, uint64_t* bar, uint8_t* dst, int row, int z,
                       uint64_t pol) {
    for (int b = 0; b < kBoxes; ++b) {
      if (packed)
        ptx::tma_load_3d(m, bar, dst + b * kBoxBytes, 64 * b, z, row, pol);
      else
        ptx::tma_load_3d(m, bar, dst + b * kBoxBytes, 64 * b, row, z, pol);
    }
  };
  Item it{};
  int q_loads = 0;
  int issued = 0;
  bool ok = true;
  auto push = [&](bool is_v, int j) -> bool {
    const int st = issued % kStages;
    const uint32_t ph = (issued / kStages) & 1;
    if (!wait_one(sh, a.status, &bb.kv_empty[st], ph ^ 1)) return false;
    if (withhold_load(issued)) {  // test builds only
      ++issued;
      return true;
    }
    const int kv_row = it.k_row0 + (it.kt0 + j) * kBlockN;
    if (!in_bounds(sh, a.status, kv_tile_ok(a, kv_row, it.kz))) return false;
    ptx::mbar_arrive_expect_tx(&bb.kv_full[st], kTileBytes);
    load_tile(is_v ? tv : tk, &bb.kv_full[st], smem + kKVOff + st * kTileBytes, kv_row, it.kz,
              pol_kv);
    ++issued;
    return true;
  };
  auto claim = [&]() -> bool {
    for (;;) {
      const int idx = atomicAdd(a.queue, 1);
      if (idx >= a.n_items) return false;
      if (make_item<CAUSAL>(idx, a, a.status, it)) return true;
    }
  };
  bool have = claim();
  if (have) it.kz += test_bad_kv_head();  // test builds only
  for (int r = 0; ok; ++r) {
    if (!have) {
      post_item(sh, a, r, nullptr);
      break;
    }
    if (!post_item(sh, a, r, &it)) break;
    for (int s = 0; s < 2 && ok; ++s) {
      const int n = tile_n(it, s);
      if (n == 0) continue;
      // Q, once the previous Q tile's last QK no longer needs the buffer.
      if (q_loads > 0 &&
          !wait_one(sh, a.status, bb.q_empty, static_cast<uint32_t>((q_loads - 1) & 1))) {
        ok = false;
        break;
      }
      const int q_row = it.q_row0 + (2 * it.qpair + s) * kBlockM;
      if (!in_bounds(sh, a.status, q_tile_ok(a, q_row, it.qz))) {
        ok = false;
        break;
      }
      ptx::mbar_arrive_expect_tx(bb.q_full, kTileBytes);
      load_tile(tq, bb.q_full, smem + kQOff, q_row, it.qz, pol_q);
      ++q_loads;
      ok = push(false, 0) && (n < 2 || push(false, 1));
      for (int j = 0; j < n && ok; ++j) ok = push(true, j) && (j + 2 >= n || push(false, j + 2));
    }
    if (ok) have = claim();
  }
  if (q_loads > 0) wait_one(sh, a.status, bb.q_full, static_cast<uint32_t>((q_loads - 1) & 1), true);
  for (int t = (issued > kStages ? issued - kStages : 0); t < issued; ++t)
    wait_one(sh, a.status, &bb.kv_full[t % kStages], (t / kStages) & 1, true);
}

// -------------------------------------------------------------------- MMA
template <bool CAUSAL>
__device__ void mma_role(const Shared& sh, const Bars& bb, const KernelArgs& a, uint8_t* smem,
                         uint32_t tmem) {
  const uint64_t q_desc = ptx::sdesc_sw128(ptx::smem_u32(smem + kQOff), 16, 1024);
  const uint64_t k_desc = ptx::sdesc_sw128(ptx::smem_u32(smem + kKVOff), 16, 1024);
  const uint64_t v_desc = ptx::sdesc_sw128(ptx::smem_u32(smem + kKVOff), kBoxBytes, 1024);
  constexpr uint64_t kTileUnits = kTileBytes >> 4;
  // S buffer b = Q K^T over 256 (16 MMAs of K-depth 16; a 16-deep step moves
  // 32 B inside the 128 B swizzle row, a 64-deep step moves one box).
  auto issue_qk = [&](int b, int stage) {
    const uint64_t kd = k_desc + stage * kTileUnits;
#pragma unroll
    for (int kk = 0; kk < kD / 16; ++kk) {
      const uint64_t off = static_cast<uint64_t>(((kk / 4) * kBoxBytes + (kk % 4) * 32) >> 4);
      ptx::mma_ss_elect(tmem + 128 * b, q_desc + off, kd + off, kIdescQK, kk > 0 ? 1u : 0u);
    }
  };
  // O (+)= P V over keys [64*half, 64*half + 64): P from TMEM (8 columns per
  // 16 keys), V MN-major (LBO one 64-column box, 2 KB per 16 keys), N = 256.
  auto issue_pv_half = [&](int b, int half, int stage, uint32_t accumulate) {
    const uint64_t vd = v_desc + stage * kTileUnits;
#pragma unroll
    for (int k4 = 0; k4 < 4; ++k4) {
      const int kk = 4 * half + k4;
      ptx::mma_ts_elect(tmem + kTmemO, tmem + 128 * b + 8 * kk,
                        vd + static_cast<uint64_t>((kk * 2048) >> 4), kIdescPV,
                        (accumulate | static_cast<uint32_t>(kk > 0)));
    }
  };
  int consumed = 0, q_uses = 0, g = 0, gp = 0;
  auto stage_of = [&](int c) { return c % kStages; };
  auto phase_of = [&](int c) { return static_cast<uint32_t>((c / kStages) & 1); };
  auto qk_next = [&](bool last) -> bool {
    const int ck = consumed++;
    if (!wait_warp(sh, a.status, &bb.kv_full[stage_of(ck)], phase_of(ck))) return false;
    ptx::tc_fence_after_sync();
    issue_qk(g & 1, stage_of(ck));
    ptx::commit_elect(&bb.s_full[g & 1]);
    ptx::commit_elect(&bb.kv_empty[stage_of(ck)]);
    if (last) ptx::commit_elect(bb.q_empty);
    ++g;
    return true;
  };

  Item it;
  bool ok = true;
  for (int r = 0; read_item(sh, a, r, it, ok); ++r) {
    for (int s = 0; s < 2; ++s) {
      const int n = tile_n(it, s);
      if (n == 0) continue;
      if (!wait_warp(sh, a.status, bb.q_full, static_cast<uint32_t>(q_uses & 1))) goto done;
      ++q_uses;
      if (!qk_next(n == 1)) goto done;
      if (n > 1 && !qk_next(n == 2)) goto done;
      for (int j = 0; j < n; ++j) {
        const int cv = consumed++;
        if (!wait_warp(sh, a.status, &bb.kv_full[stage_of(cv)], phase_of(cv))) goto done;
        const int b = gp & 1;
        const uint32_t acc = j > 0 ? 1u : 0u;
        for (int half = 0; half < 2; ++half) {
          // one barrier per (S buffer, half): the softmax may announce P for
          // the other buffer first, never twice for the same one
          if (!wait_warp(sh, a.status, &bb.p_ready[2 * b + half],
                         static_cast<uint32_t>((gp >> 1) & 1)))
            goto done;
          ptx::tc_fence_after_sync();
          issue_pv_half(b, half, stage_of(cv), acc);
        }
        ptx::commit_elect(bb.pv_done);
        ptx::commit_elect(&bb.kv_empty[stage_of(cv)]);
        if (j == n - 1) ptx::commit_elect(bb.o_ready);
        ++gp;
        if (j + 2 < n && !qk_next(j + 3 == n)) goto done;
      }
    }
  }
done:
  ptx::commit_elect(sh.drain);
  wait_warp(sh, a.status, sh.drain, 0, true);
}

// ---------------------------------------------------------------- softmax
template <bool CAUSAL, int kPolyPairs>
__device__ void softmax_role(const Shared& sh, const Bars& bb, const KernelArgs& a,
                             uint32_t tmem, int warp, uint8_t* o_stage,
                             const CUtensorMap* tmap_o) {
  const bool tma_o = !a.o_f32 && a.cu_q == nullptr && a.split_rows == 0;
  const int lane = static_cast<int>(ptx::lane_id());
  const int r = warp * 32 + lane;
  const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
  const uint32_t t_o = tmem + lane_off + kTmemO;
  const float sl2 = a.scale_log2;
  const uint64_t sl2x2 = ptx::f2pack(sl2, sl2);
  int g = 0;   // K/V tiles consumed (S buffer g % 2)
  int eo = 0;  // Q tiles with at least one K/V tile finished (o_ready phases)

  Item it;
  bool ok = true;
  for (int rr = 0; read_item(sh, a, rr, it, ok); ++rr) {
    for (int s = 0; s < 2; ++s) {
      const int qt = 2 * it.qpair + s;
      const int row = qt * kBlockM + r;
      if (qt * kBlockM >= it.q_len) continue;  // the item has no such tile
      const int n = tile_n(it, s);
      float m = -INFINITY, l = 0.f;
      for (int j = 0; j < n; ++j) {
        const int key0 = (it.kt0 + j) * kBlockN;
        int key_limit = it.k_len - key0;
        if (CAUSAL) {
          const long long lim = static_cast<long long>(row) + it.delta + 1 - key0;
          if (lim < key_limit) key_limit = lim < -1 ? -1 : static_cast<int>(lim);
        }
        const int b = g & 1;
        const uint32_t t_s = tmem + lane_off + 128u * b;
        if (!wait_warp(sh, a.status, &bb.s_full[b], static_cast<uint32_t>((g >> 1) & 1))) return;
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
        // Lazy rescale, as in attn_fwd_kernel.cuh.  O may only be touched
        // once the previous tile's PV has completed (g - 1 PVs done).
        float alpha = 1.f;
        bool rescale = false;
        if (tile_max - m > kRescaleTauBf16) {
          alpha = ptx::ex2_approx(m - tile_max);
          m = tile_max;
          rescale = j > 0;
        }
        if (__any_sync(0xffffffffu, rescale)) {
          if (!wait_warp(sh, a.status, bb.pv_done, static_cast<uint32_t>((g - 1) & 1))) return;
          ptx::tc_fence_after_sync();
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
          uint32_t pk[32];
#pragma unroll
          for (int q = 0; q < 32; ++q) {
            const int c = 64 * half + 2 * q;
            const uint64_t y2 = ptx::ffma2(ptx::f2pack(x[c], x[c + 1]), sl2x2, negm2);
            uint64_t p2;
            if ((q & 3) < kPolyPairs) {
              p2 = exp2_poly2(y2);
            } else {
              float y0, y1;
              ptx::f2unpack(y2, y0, y1);
              p2 = ptx::f2pack(ptx::ex2_approx(y0), ptx::ex2_approx(y1));
            }
            if (q & 1) sb = ptx::fadd2(sb, p2);
            else sa = ptx::fadd2(sa, p2);
            float p0, p1;
            ptx::f2unpack(p2, p0, p1);
            pk[q] = ptx::pack_bf16x2(p0, p1);
          }
          ptx::tmem_st32(t_s + 32 * half, pk);
          ptx::tmem_st_wait();
          ptx::tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(&bb.p_ready[2 * b + half]);
        }
        float la0, la1, lb0, lb1;
        ptx::f2unpack(sa, la0, la1);
        ptx::f2unpack(sb, lb0, lb1);
        l = l * alpha + ((la0 + la1) + (lb0 + lb1));
        ++g;
      }

      // Epilogue: O / l -> rows of O; LSE = (m + log2 l) ln 2; a row that
      // saw no key stores O = 0 and LSE = -inf; rows past the end of the
      // sequence are not stored.  The next Q tile's first PV (which
      // overwrites O) waits for its P, which this thread publishes only
      // after these loads.
      if (n > 0) {
        if (!wait_warp(sh, a.status, bb.o_ready, static_cast<uint32_t>(eo & 1))) return;
        ++eo;
        ptx::tc_fence_after_sync();
      }
      const bool row_ok = row < it.q_len;
      const bool empty = m == -INFINITY;
      const float inv_l = empty ? 0.f : 1.f / l;
      size_t o_row, l_row;
      if (a.cu_q != nullptr) {
        o_row = (static_cast<size_t>(it.q_row0) + row) * a.H + it.qz;
        l_row = static_cast<size_t>(it.qz) * a.T_q + it.q_row0 + row;
      } else {
        o_row = static_cast<size_t>(it.qz) * a.N_q + row;
        l_row = o_row;
      }
      o_row += static_cast<size_t>(it.split) * a.split_rows;
      l_row += static_cast<size_t>(it.split) * a.split_rows;
      const bool store = row_ok && in_bounds(sh, a.status,
                                             static_cast<long long>(o_row) < out_rows(a) &&
                                                 static_cast<long long>(l_row) < out_rows(a));
      if (tma_o) {
        // Box b (columns [64b, 64b+64)) of this warp's 32 rows goes through
        // staging box b % 2 and one TMA store; a staging box is rewritten
        // once the store two boxes back has read it.
        uint32_t ov0[32], ov1[32];
        auto load_box = [&](int b) {
          if (n > 0) {
            ptx::tmem_ld32(t_o + 64 * b, ov0);
            ptx::tmem_ld32(t_o + 64 * b + 32, ov1);
          } else {
#pragma unroll
            for (int c = 0; c < 32; ++c) ov0[c] = ov1[c] = 0u;
          }
        };
        auto wait_box = [&]() {
          if (n > 0) {
            ptx::tmem_ld_wait_tie(ov0);
            ptx::reg_tie32(ov1);
          }
        };
        const uint32_t sw = static_cast<uint32_t>(lane & 7);
        const int row0 = qt * kBlockM + 32 * warp;
        load_box(0);
        wait_box();
#pragma unroll 1
        for (int b = 0; b < kBoxes; ++b) {
          uint32_t pk[32];
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            pk[c] = ptx::pack_bf16x2(empty ? 0.f : __uint_as_float(ov0[2 * c]) * inv_l,
                                     empty ? 0.f : __uint_as_float(ov0[2 * c + 1]) * inv_l);
            pk[16 + c] = ptx::pack_bf16x2(empty ? 0.f : __uint_as_float(ov1[2 * c]) * inv_l,
                                          empty ? 0.f : __uint_as_float(ov1[2 * c + 1]) * inv_l);
          }
          if (b + 1 < kBoxes) load_box(b + 1);
          if (lane == 0) ptx::bulk_wait_read_but_one();
          __syncwarp();
          uint8_t* box = o_stage + (b & 1) * 4096;
          const uint32_t row_addr = ptx::smem_u32(box) + static_cast<uint32_t>(lane) * 128u;
#pragma unroll
          for (int c = 0; c < 8; ++c)
            ptx::st_shared_v4(row_addr + ((static_cast<uint32_t>(c) ^ sw) << 4), pk[4 * c],
                              pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
          ptx::fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && row0 < it.q_len) {
            ptx::tma_store_3d(tmap_o, box, 64 * b, row0, it.qz);
            ptx::bulk_commit_group();
          }
          if (b + 1 < kBoxes) wait_box();
        }
        if (store) a.lse[l_row] = empty ? -INFINITY : (m + log2f(l)) * 0.69314718055994531f;
        continue;
      }
#pragma unroll 1
      for (int c0 = 0; c0 < kD; c0 += 32) {
        uint32_t ov[32];
        if (n > 0) {
          ptx::tmem_ld32(t_o + c0, ov);
          ptx::tmem_ld_wait_tie(ov);
#pragma unroll
          for (int c = 0; c < 32; ++c)
            ov[c] = __float_as_uint(empty ? 0.f : __uint_as_float(ov[c]) * inv_l);
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) ov[c] = 0u;
        }
        if (!store) continue;
        if (a.o_f32) {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<float*>(a.o) + o_row * kD + c0);
#pragma unroll
          for (int v = 0; v < 8; ++v)
            dst[v] = make_uint4(ov[4 * v], ov[4 * v + 1], ov[4 * v + 2], ov[4 * v + 3]);
        } else {
          uint32_t pk[16];
#pragma unroll
          for (int c = 0; c < 16; ++c)
            pk[c] = ptx::pack_bf16x2(__uint_as_float(ov[2 * c]), __uint_as_float(ov[2 * c + 1]));
          uint4* dst =
              reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.o) + o_row * kD + c0);
#pragma unroll
          for (int v = 0; v < 4; ++v)
            dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
        }
      }
      if (store) a.lse[l_row] = empty ? -INFINITY : (m + log2f(l)) * 0.69314718055994531f;
    }
  }
}

// ----------------------------------------------------------------- kernel
template <bool CAUSAL, int kPolyPairs>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_wide_kernel(const __grid_constant__ CUtensorMap tmap_q,
                         const __grid_constant__ CUtensorMap tmap_k,
                         const __grid_constant__ CUtensorMap tmap_v,
                         const __grid_constant__ CUtensorMap tmap_o, const KernelArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBarOff);
  Bars bb;
  bb.q_full = bars;
  bb.q_empty = bars + 1;
  bb.kv_full = bars + 2;
  bb.kv_empty = bb.kv_full + kStages;
  bb.s_full = bb.kv_empty + kStages;
  bb.p_ready = bb.s_full + 2;
  bb.pv_done = bb.p_ready + 4;
  bb.o_ready = bb.pv_done + 1;
  Shared sh = {};
  sh.drain = bb.o_ready + 1;
  sh.item_full = sh.drain + 1;
  sh.item_empty = sh.item_full + kItemSlots;
  sh.tmem_base = reinterpret_cast<uint32_t*>(smem + kMiscOff);
  sh.abort_flag = reinterpret_cast<volatile int*>(smem + kMiscOff + 4);
  sh.item_ring = reinterpret_cast<volatile int*>(smem + kRingOff);

  const int warp = threadIdx.x / 32;
  if (threadIdx.x == 0) {
    ptx::mbar_init(bb.q_full, 1);
    ptx::mbar_init(bb.q_empty, 1);
    for (int i = 0; i < kStages; ++i) {
      ptx::mbar_init(&bb.kv_full[i], 1);
      ptx::mbar_init(&bb.kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) ptx::mbar_init(&bb.s_full[i], 1);
    for (int i = 0; i < 4; ++i) ptx::mbar_init(&bb.p_ready[i], 4);
    ptx::mbar_init(bb.pv_done, 1);
    ptx::mbar_init(bb.o_ready, 1);
    ptx::mbar_init(sh.drain, 1);
    for (int i = 0; i < kItemSlots; ++i) {
      ptx::mbar_init(&sh.item_full[i], 1);
      ptx::mbar_init(&sh.item_empty[i], kReaders);
    }
    *sh.abort_flag = 0;
    ptx::fence_barrier_init();
  }
  if (warp == 4 && ptx::lane_id() == 0) {
    ptx::prefetch_tmap(&tmap_q);
    ptx::prefetch_tmap(&tmap_k);
    ptx::prefetch_tmap(&tmap_v);
  }
  if (warp == 5) {
    ptx::tmem_alloc(sh.tmem_base, 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before_sync();
  __syncthreads();
  ptx::tc_fence_after_sync();
  const uint32_t tmem = *sh.tmem_base;

  if (warp < 4) {
    softmax_role<CAUSAL, kPolyPairs>(sh, bb, args, tmem, warp, smem + kOOff + warp * kOWarpBytes,
                                     &tmap_o);
    // the staging boxes are read before the CTA exits
    ptx::bulk_wait_read_all();
  } else if (warp == 4) {
    if (ptx::lane_id() == 0) producer_role<CAUSAL>(sh, bb, args, smem, &tmap_q, &tmap_k, &tmap_v);
    __syncwarp();
  } else {
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
  if (warp == 5) {
    ptx::tc_fence_after_sync();
    ptx::tmem_dealloc(tmem, 512);
  }
}

}  // namespace wide
}  // namespace attn_b200
