// Dense attention forward on CTA pairs (cluster of 2, tcgen05.mma.cta_group::2),
// head dim 128, per-head layout.  Same result as attn_fwd_kernel.  The page
// lecompute.fr/kernel-perf/flashattention-4-limites-calcul-matriciel,
// section "Blackwell déplace la limite vers les autres unités", notes that
// shared-memory reads did not keep pace with the doubled per-SM matrix rate
// of B200; the pair form of the tensor-core instructions (an M = 256
// product that reads each operand half from the shared memory of the SM
// holding it) halves each SM's K/V staging and operand reads.
//
// The pair works on 4 Q tiles of one (batch, head): softmax group s of CTA
// r (rank in the cluster) owns Q tile 4u + 2s + r, so the product for group
// s covers the 256 consecutive rows of tiles 4u + 2s and 4u + 2s + 1.
//   S_s = Q_s K_j^T : M = 256, N = 128 keys; CTA r holds its Q tile and keys
//                     [64r, 64r + 64) of K_j (16 KB instead of 32 KB);
//   O_s += P_s V_j  : M = 256, N = 128 = d; P from each CTA's TMEM, CTA r
//                     holds columns [64r, 64r + 64) of V_j.
// Per K/V step each SM thus loads and reads half of the K/V bytes of the
// one-CTA kernel.  Both tiles of a product visit the same K/V tiles (the
// later tile's count under the causal mask; the earlier tile's extra tile
// is fully masked for its rows).
//
// Roles per CTA (12 warps): 0-7 softmax groups (as in the one-CTA kernel,
// on the CTA's own TMEM), 8 TMA producer (own halves), 9 on rank 0 the MMA
// issuer, on rank 1 only the TMEM allocation.
//
// Barriers: loads of both CTAs complete on rank 0's full barriers (rank 0
// announces the byte count of both halves); rank 0's commits arrive on the
// barrier at the same address in both CTAs; P is announced to rank 0 by the
// 8 softmax warps of both CTAs.  Work items come from the launch's queue,
// claimed by rank 0's producer and written into both CTAs' item rings.
#pragma once

#include "attn_fwd_kernel.cuh"

namespace attn_b200 {
namespace pair {

constexpr int kD = 128;
constexpr int kThreads = 384;
constexpr int kQBoxBytes = kBlockM * 64 * 2;        // 128 rows x 64 columns
constexpr int kQTileBytes = 2 * kQBoxBytes;         // one Q tile
constexpr int kKBoxBytes = (kBlockN / 2) * 64 * 2;  // 64 keys x 64 columns
constexpr int kStageBytes = 16384;                  // a K half (2 boxes) or a V half (1 box)
constexpr int kStages = 8;
constexpr int kQOff = 0;
constexpr int kKVOff = 2 * kQTileBytes;
constexpr int kBarOff = kKVOff + kStages * kStageBytes;
// q_full[2], q_empty[2], kv_full[S], kv_empty[S], s_full[2], p_ready[4],
// o_final[2], drain, item_full[R], item_empty[R]
constexpr int kNumBars = 4 + 2 * kStages + 2 + 4 + 2 + 1 + 2 * kItemSlots;
constexpr int kMiscOff = kBarOff + kNumBars * 8;
constexpr int kRingOff = kMiscOff + 16;
constexpr int kSmemBytes = kRingOff + 4 * kItemWords * kItemSlots + 1024;
// TMEM columns of S_s / P_s and of O_s (the one-CTA kernel's plan).
constexpr uint32_t kTmemS = 0;
constexpr uint32_t kTmemO = 256;
constexpr uint32_t kIdescQK = ptx::idesc_bf16_f32(256, kBlockN, 0, 0);
constexpr uint32_t kIdescPV = ptx::idesc_bf16_f32(256, kD, 0, 1);
// Readers of an item slot: rank 0's MMA warp and 8 softmax warps, rank 1's
// producer and 8 softmax warps; all arrive on rank 0's item_empty.
constexpr int kPairReaders = 18;
static_assert(kSmemBytes <= 227 * 1024, "shared memory");

__device__ __forceinline__ uint32_t leader_addr(const void* p) {
  return ptx::mapa(ptx::smem_u32(p), 0);
}

// Warp-uniform bounded wait with cluster-scope acquire.
__device__ __forceinline__ bool wait_warp_cl(const Shared& sh, int* status, uint64_t* bar,
                                             uint32_t parity, bool drain = false) {
  uint64_t t0 = 0;
  for (uint32_t it = 0;; ++it) {
    const bool ok = ptx::mbar_try_wait_cluster(bar, parity);
    if (__all_sync(0xffffffffu, ok)) return true;
    if ((it & 63u) == 63u) {
      int stop = 0;
      if (ptx::lane_id() == 0) {
        const uint64_t now = ptx::globaltimer_ns();
        if (t0 == 0) t0 = now;
        if (!drain && *sh.abort_flag) {
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

// Single-thread form of wait_warp_cl.
__device__ __forceinline__ bool wait_one_cl(const Shared& sh, int* status, uint64_t* bar,
                                            uint32_t parity) {
  if (ptx::mbar_try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = ptx::globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (ptx::mbar_try_wait_cluster(bar, parity)) return true;
    if ((it & 63u) == 0) {
      if (*sh.abort_flag) return false;
      if (ptx::globaltimer_ns() - t0 > kWaitLimitNs) {
        raise_status(sh, status, kStatusDeviceTimeout);
        return false;
      }
    }
  }
}

// Item numbering as in the one-CTA kernel, with groups of 4 Q tiles
// ("quads", a.n_qpairs of them per head) in place of pairs.  n0 / n1 are
// the K/V tiles of the products for tiles (4u, 4u+1) and (4u+2, 4u+3).
template <bool CAUSAL>
__device__ __forceinline__ bool make_item_pair(int idx, const KernelArgs& a, Item& it) {
  int h0, wh;
  item_window(idx, a.BH, a.win_heads, a.n_qpairs, h0, wh);
  const int k = idx - h0 * a.n_qpairs;
  const int qd_idx = k / wh;
  const int bh = h0 + (k - qd_idx * wh);
  const int b = bh / a.H, h = bh - b * a.H;
  it.qpair = CAUSAL ? (a.n_qpairs - 1 - qd_idx) : qd_idx;
  it.q_row0 = 0;
  it.q_len = a.N_q;
  it.k_row0 = 0;
  it.k_len = a.N_k;
  it.qz = bh;
  it.kz = b * a.H_kv + h / a.q_per_kv;
  it.delta = a.delta;
  if (4 * it.qpair * kBlockM >= it.q_len) return false;
  it.split = 0;
  it.kt0 = 0;
  const int t = 4 * it.qpair;
  const int a0 = tiles_for<CAUSAL>(t, it, a.split_tiles), a1 = tiles_for<CAUSAL>(t + 1, it, a.split_tiles);
  const int b0 = tiles_for<CAUSAL>(t + 2, it, a.split_tiles), b1 = tiles_for<CAUSAL>(t + 3, it, a.split_tiles);
  it.n0 = a0 > a1 ? a0 : a1;
  it.n1 = b0 > b1 ? b0 : b1;
  return true;
}

// Rank 0's producer: item r (or the end) into slot r % R of both CTAs' rings.
__device__ __forceinline__ bool post_item_pair(const Shared& sh, const KernelArgs& a, int r,
                                               const Item* it) {
  const int slot = r % kItemSlots;
  const uint32_t ph = static_cast<uint32_t>((r / kItemSlots) & 1);
  if (!wait_one_cl(sh, a.status, &sh.item_empty[slot], ph ^ 1)) return false;
  int v[13];
  v[0] = it != nullptr ? 1 : 0;
  if (it != nullptr) {
    v[1] = it->qpair; v[2] = it->n0; v[3] = it->n1; v[4] = it->kt0; v[5] = it->q_len;
    v[6] = it->k_len; v[7] = it->delta; v[8] = it->qz; v[9] = it->kz; v[10] = it->q_row0;
    v[11] = it->k_row0; v[12] = it->split;
  }
  volatile int* w = sh.item_ring + slot * kItemWords;
  const uint32_t peer = ptx::mapa(ptx::smem_u32(const_cast<int*>(w)), 1);
  const int n = it != nullptr ? 13 : 1;
  for (int i = 0; i < n; ++i) {
    w[i] = v[i];
    ptx::st_cluster_u32(peer + 4 * i, static_cast<uint32_t>(v[i]));
  }
  ptx::mbar_arrive(&sh.item_full[slot]);
  ptx::mbar_arrive_cluster(ptx::mapa(ptx::smem_u32(&sh.item_full[slot]), 1));
  return true;
}

// Reader warp of either CTA: its r-th item from the local ring.
__device__ __forceinline__ bool read_item_pair(const Shared& sh, const KernelArgs& a, int r,
                                               Item& it, bool& ok) {
  const int slot = r % kItemSlots;
  if (!wait_warp_cl(sh, a.status, &sh.item_full[slot],
                    static_cast<uint32_t>((r / kItemSlots) & 1))) {
    ok = false;
    return false;
  }
  const volatile int* w = sh.item_ring + slot * kItemWords;
  const bool valid = w[0] != 0;
  if (valid) {
    it.qpair = w[1]; it.n0 = w[2]; it.n1 = w[3]; it.kt0 = w[4]; it.q_len = w[5];
    it.k_len = w[6]; it.delta = w[7]; it.qz = w[8]; it.kz = w[9]; it.q_row0 = w[10];
    it.k_row0 = w[11]; it.split = w[12];
  }
  __syncwarp();
  if (ptx::lane_id() == 0) ptx::mbar_arrive_cluster(leader_addr(&sh.item_empty[slot]));
  return valid;
}

// ----------------------------------------------------------------- producer
// One thread.  Both ranks load their own halves; rank 0 also claims the
// items and announces each full barrier's bytes (its half and the peer's).
template <bool CAUSAL>
__device__ void producer_role(const Shared& sh, const KernelArgs& a, uint8_t* smem, uint32_t rank,
                              const CUtensorMap* tq, const CUtensorMap* tk,
                              const CUtensorMap* tv) {
  const uint64_t pol_q = ptx::policy_evict_first();
  const uint64_t pol_kv = ptx::policy_evict_last();
  const bool lead = rank == 0;
  int q_loads[2] = {0, 0};
  int issued = 0;
  bool ok = true;
  Item it;
  auto claim = [&]() -> bool {
    for (;;) {
      const int idx = atomicAdd(a.queue, 1);
      if (idx >= a.n_items) return false;
      if (make_item_pair<CAUSAL>(idx, a, it)) return true;
    }
  };
  // Rank 1 reads its items like the other readers (one lane: a whole-warp
  // read is not needed, so the ring read is done by this thread alone).
  auto next = [&](int r) -> bool {
    if (lead) {
      const bool have = claim();
      if (!post_item_pair(sh, a, r, have ? &it : nullptr)) {
        ok = false;
        return false;
      }
      return have;
    }
    const int slot = r % kItemSlots;
    if (!wait_one_cl(sh, a.status, &sh.item_full[slot], static_cast<uint32_t>((r / kItemSlots) & 1))) {
      ok = false;
      return false;
    }
    const volatile int* w = sh.item_ring + slot * kItemWords;
    const bool valid = w[0] != 0;
    if (valid) {
      it.qpair = w[1]; it.n0 = w[2]; it.n1 = w[3]; it.kt0 = w[4]; it.q_len = w[5];
      it.k_len = w[6]; it.delta = w[7]; it.qz = w[8]; it.kz = w[9]; it.q_row0 = w[10];
      it.k_row0 = w[11]; it.split = w[12];
    }
    ptx::mbar_arrive_cluster(leader_addr(&sh.item_empty[slot]));
    return valid;
  };
  for (int r = 0; ok && next(r); ++r) {
    const int n = it.n0 > it.n1 ? it.n0 : it.n1;
    for (int s = 0; s < 2 && ok; ++s) {
      if ((s == 0 ? it.n0 : it.n1) == 0) continue;
      if (q_loads[s] > 0 &&
          !wait_one(sh, a.status, &sh.q_empty[s], static_cast<uint32_t>((q_loads[s] - 1) & 1))) {
        ok = false;
        break;
      }
      if (lead) ptx::mbar_arrive_expect_tx(&sh.q_full[s], 2 * kQTileBytes);
      const uint32_t bar = leader_addr(&sh.q_full[s]);
      const int row = (4 * it.qpair + 2 * s + static_cast<int>(rank)) * kBlockM;
      uint8_t* dst = smem + kQOff + s * kQTileBytes;
      ptx::tma_load_3d_pair(tq, bar, dst, 0, row, it.qz, pol_q);
      ptx::tma_load_3d_pair(tq, bar, dst + kQBoxBytes, 64, row, it.qz, pol_q);
      ++q_loads[s];
    }
    for (int j = 0; j < n && ok; ++j) {
      const int key0 = (it.kt0 + j) * kBlockN;
      for (int which = 0; which < 2; ++which) {  // 0: K_j half, 1: V_j half
        const int st = issued % kStages;
        const uint32_t ph = (issued / kStages) & 1;
        if (!wait_one(sh, a.status, &sh.kv_empty[st], ph ^ 1)) { ok = false; break; }
        uint8_t* dst = smem + kKVOff + st * kStageBytes;
        if (lead) ptx::mbar_arrive_expect_tx(&sh.kv_full[st], 2 * kStageBytes);
        const uint32_t bar = leader_addr(&sh.kv_full[st]);
        if (which == 0) {
          // keys [64 rank, 64 rank + 64) of the tile, both 64-column halves
          const int row = key0 + (kBlockN / 2) * static_cast<int>(rank);
          ptx::tma_load_3d_pair(tk, bar, dst, 0, row, it.kz, pol_kv);
          ptx::tma_load_3d_pair(tk, bar, dst + kKBoxBytes, 64, row, it.kz, pol_kv);
        } else {
          // columns [64 rank, 64 rank + 64) of all 128 keys
          ptx::tma_load_3d_pair(tv, bar, dst, 64 * static_cast<int>(rank), key0, it.kz, pol_kv);
        }
        ++issued;
      }
    }
  }
  // Rank 0 drains its full barriers (they complete once both halves have
  // landed).  Rank 1's loads are covered by them too: rank 0's MMA warp
  // waits on every phase it consumes, and the CTAs leave together.
  if (lead) {
    for (int s = 0; s < 2; ++s)
      if (q_loads[s] > 0)
        wait_one(sh, a.status, &sh.q_full[s], static_cast<uint32_t>((q_loads[s] - 1) & 1), true);
    for (int t = (issued > kStages ? issued - kStages : 0); t < issued; ++t)
      wait_one(sh, a.status, &sh.kv_full[t % kStages], (t / kStages) & 1, true);
  }
}

// ---------------------------------------------------------------------- MMA
// Rank 0's warp 9 only.  Same issue order as the one-CTA kernel:
// PV0(j), S0(j+1), PV1(j), S1(j+1).
template <bool CAUSAL>
__device__ void mma_role(const Shared& sh, const KernelArgs& a, uint8_t* smem, uint32_t tmem) {
  const uint32_t t_s[2] = {tmem + kTmemS, tmem + kTmemS + 128};
  const uint32_t t_o[2] = {tmem + kTmemO, tmem + kTmemO + 128};
  const uint64_t q_desc = ptx::sdesc_sw128(ptx::smem_u32(smem + kQOff), 16, 1024);
  const uint64_t k_desc = ptx::sdesc_sw128(ptx::smem_u32(smem + kKVOff), 16, 1024);
  // V half: 128 keys x 64 columns (one swizzle atom wide), MN-major.
  const uint64_t v_desc = ptx::sdesc_sw128(ptx::smem_u32(smem + kKVOff), kStageBytes, 1024);
  constexpr uint64_t kStageUnits = kStageBytes >> 4;
  constexpr uint64_t kQTileUnits = kQTileBytes >> 4;

  auto issue_qk = [&](int s, int stage) {
    const uint64_t qd = q_desc + s * kQTileUnits;
    const uint64_t kd = k_desc + stage * kStageUnits;
#pragma unroll
    for (int kk = 0; kk < kD / 16; ++kk) {
      const uint64_t qo = static_cast<uint64_t>(((kk / 4) * kQBoxBytes + (kk % 4) * 32) >> 4);
      const uint64_t ko = static_cast<uint64_t>(((kk / 4) * kKBoxBytes + (kk % 4) * 32) >> 4);
      ptx::mma_pair_ss_elect(t_s[s], qd + qo, kd + ko, kIdescQK, kk > 0 ? 1u : 0u);
    }
  };
  // (the parts of P that the shared softmax step publishes: keys
  // [0, kPFirstKeys) and the rest)
  auto issue_pv_half = [&](int s, int half, int stage, uint32_t accumulate) {
    const uint64_t vd = v_desc + stage * kStageUnits;
    constexpr int kKa = kPFirstKeys / 16;
#pragma unroll
    for (int kk = half ? kKa : 0; kk < (half ? 8 : kKa); ++kk) {
      ptx::mma_pair_ts_elect(t_o[s], t_s[s] + 8 * kk, vd + static_cast<uint64_t>((kk * 2048) >> 4),
                             kIdescPV, (accumulate | static_cast<uint32_t>(kk > 0)));
    }
  };
  int p_count[2] = {0, 0};
  auto issue_pv = [&](int s, int stage, uint32_t accumulate) -> bool {
    const uint32_t parity = static_cast<uint32_t>(p_count[s] & 1);
    ++p_count[s];
    if (!wait_warp_cl(sh, a.status, &sh.p_ready[2 * s], parity)) return false;
    ptx::tc_fence_after_sync();
    issue_pv_half(s, 0, stage, accumulate);
    if (!wait_warp_cl(sh, a.status, &sh.p_ready[2 * s + 1], parity)) return false;
    ptx::tc_fence_after_sync();
    issue_pv_half(s, 1, stage, accumulate);
    return true;
  };
  auto issue_s = [&](int s, int j, int n_s, int stage) {
    issue_qk(s, stage);
    ptx::commit_pair_elect(&sh.s_full[s]);
    if (j == n_s - 1) ptx::commit_pair_elect(&sh.q_empty[s]);
  };

  int consumed = 0;
  int q_uses[2] = {0, 0};
  auto stage_of = [&](int c) { return c % kStages; };
  auto phase_of = [&](int c) { return static_cast<uint32_t>((c / kStages) & 1); };

  Item it;
  bool ok = true;
  for (int r = 0; read_item_pair(sh, a, r, it, ok); ++r) {
    const int n0 = it.n0, n1 = it.n1;
    const int n = n0 > n1 ? n0 : n1;
    if (n == 0) continue;
    for (int s = 0; s < 2; ++s) {
      if ((s == 0 ? n0 : n1) == 0) continue;
      if (!wait_warp(sh, a.status, &sh.q_full[s], static_cast<uint32_t>(q_uses[s] & 1)))
        goto done;
      ++q_uses[s];
    }
    {
      const int ck = consumed++;
      if (!wait_warp(sh, a.status, &sh.kv_full[stage_of(ck)], phase_of(ck))) goto done;
      ptx::tc_fence_after_sync();
      if (n0 > 0) issue_s(0, 0, n0, stage_of(ck));
      if (n1 > 0) issue_s(1, 0, n1, stage_of(ck));
      ptx::commit_pair_elect(&sh.kv_empty[stage_of(ck)]);
      for (int j = 0; j < n; ++j) {
        const int cv = consumed++;
        if (!wait_warp(sh, a.status, &sh.kv_full[stage_of(cv)], phase_of(cv))) goto done;
        const int ck2 = (j + 1 < n) ? consumed++ : -1;
        if (ck2 >= 0 && !wait_warp(sh, a.status, &sh.kv_full[stage_of(ck2)], phase_of(ck2)))
          goto done;
        ptx::tc_fence_after_sync();
        const uint32_t acc = j > 0 ? 1u : 0u;
        if (j < n0) {
          if (!issue_pv(0, stage_of(cv), acc)) goto done;
          if (j == n0 - 1) ptx::commit_pair_elect(&sh.o_final[0]);
        }
        if (ck2 >= 0 && j + 1 < n0) issue_s(0, j + 1, n0, stage_of(ck2));
        if (j < n1) {
          if (!issue_pv(1, stage_of(cv), acc)) goto done;
          if (j == n1 - 1) ptx::commit_pair_elect(&sh.o_final[1]);
        }
        ptx::commit_pair_elect(&sh.kv_empty[stage_of(cv)]);
        if (ck2 >= 0) {
          if (j + 1 < n1) issue_s(1, j + 1, n1, stage_of(ck2));
          ptx::commit_pair_elect(&sh.kv_empty[stage_of(ck2)]);
        }
      }
    }
  }
done:
  ptx::commit_pair_elect(sh.drain);
  wait_warp(sh, a.status, sh.drain, 0, true);
}

// ------------------------------------------------------------------ softmax
// One thread per row of the CTA's own Q tile 4u + 2s + rank.  Both CTAs
// run every step of the product (their rows past the sequence end are
// computed on zeros and not stored).
template <bool CAUSAL>
__device__ void softmax_role(const Shared& sh, const KernelArgs& a, uint32_t tmem, uint32_t rank,
                             int s, int warp_in_group) {
  const int lane = static_cast<int>(ptx::lane_id());
  const int r = warp_in_group * 32 + lane;
  const uint32_t lane_off = static_cast<uint32_t>(warp_in_group * 32) << 16;
  const uint32_t t_s = tmem + lane_off + kTmemS + 128u * s;
  const uint32_t t_o = tmem + lane_off + kTmemO + 128u * s;
  int s_count = 0;
  int o_count = 0;
  Item it;
  bool ok = true;
  for (int rr = 0; read_item_pair(sh, a, rr, it, ok); ++rr) {
    const int qt = 4 * it.qpair + 2 * s + static_cast<int>(rank);
    const int row = qt * kBlockM + r;
    const int n_s = s == 0 ? it.n0 : it.n1;
    if (n_s == 0 && qt * kBlockM >= it.q_len) continue;
    float m = -INFINITY;
    float l = 0.f;
    for (int j = 0; j < n_s; ++j) {
      const int key0 = (it.kt0 + j) * kBlockN;
      int key_limit = it.k_len - key0;
      if (CAUSAL) {
        const long long lim = static_cast<long long>(row) + it.delta + 1 - key0;
        if (lim < key_limit) key_limit = lim < -1 ? -1 : static_cast<int>(lim);
      }
      if (!softmax_step<kD, CAUSAL, 0, true>(sh, a, s, t_s, t_o, r, lane, key_limit, j == 0,
                                             static_cast<uint32_t>(s_count & 1), -1, m, l))
        return;
      ++s_count;
    }
    if (n_s > 0) {
      if (!wait_warp(sh, a.status, &sh.o_final[s], static_cast<uint32_t>(o_count & 1))) return;
      ++o_count;
      ptx::tc_fence_after_sync();
    }
    const bool row_ok = row < it.q_len;
    const bool empty = m == -INFINITY;
    const float inv_l = empty ? 0.f : 1.f / l;
    const size_t o_row = static_cast<size_t>(it.qz) * a.N_q + row;
#pragma unroll 1
    for (int c0 = 0; c0 < kD; c0 += 32) {
      uint32_t ov[32];
      if (n_s > 0) {
        ptx::tmem_ld32(t_o + c0, ov);
        ptx::tmem_ld_wait_tie(ov);
#pragma unroll
        for (int c = 0; c < 32; ++c)
          ov[c] = __float_as_uint(empty ? 0.f : __uint_as_float(ov[c]) * inv_l);
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) ov[c] = 0u;
      }
      if (!row_ok) continue;
      uint32_t pk[16];
#pragma unroll
      for (int c = 0; c < 16; ++c)
        pk[c] = ptx::pack_bf16x2(__uint_as_float(ov[2 * c]), __uint_as_float(ov[2 * c + 1]));
      uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.o) + o_row * kD + c0);
#pragma unroll
      for (int v = 0; v < 4; ++v)
        dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
    }
    if (row_ok) a.lse[o_row] = empty ? -INFINITY : (m + log2f(l)) * 0.69314718055994531f;
  }
}

// ------------------------------------------------------------------- kernel
// Launched with clusters of 2 CTAs (x dimension); tmap_k has boxes of 64
// keys x 64 columns, tmap_q and tmap_v boxes of 128 rows x 64 columns.
template <bool CAUSAL>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_pair_kernel(const __grid_constant__ CUtensorMap tmap_q,
                         const __grid_constant__ CUtensorMap tmap_k,
                         const __grid_constant__ CUtensorMap tmap_v, const KernelArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t rank = ptx::cluster_ctarank();

  Shared sh;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBarOff);
  sh.q_full = bars;
  sh.q_empty = bars + 2;
  sh.kv_full = bars + 4;
  sh.kv_empty = sh.kv_full + kStages;
  sh.s_full = sh.kv_empty + kStages;
  sh.p_ready = sh.s_full + 2;
  sh.o_final = sh.p_ready + 4;
  sh.drain = sh.o_final + 2;
  sh.item_full = sh.drain + 1;
  sh.item_empty = sh.item_full + kItemSlots;
  sh.tmem_base = reinterpret_cast<uint32_t*>(smem + kMiscOff);
  sh.abort_flag = reinterpret_cast<volatile int*>(smem + kMiscOff + 4);
  sh.item_ring = reinterpret_cast<volatile int*>(smem + kRingOff);

  const int warp = threadIdx.x / 32;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&sh.q_full[i], 1);
      ptx::mbar_init(&sh.q_empty[i], 1);
      ptx::mbar_init(&sh.s_full[i], 1);
      ptx::mbar_init(&sh.p_ready[2 * i], 8);
      ptx::mbar_init(&sh.p_ready[2 * i + 1], 8);
      ptx::mbar_init(&sh.o_final[i], 1);
    }
    for (int i = 0; i < kStages; ++i) {
      ptx::mbar_init(&sh.kv_full[i], 1);
      ptx::mbar_init(&sh.kv_empty[i], 1);
    }
    ptx::mbar_init(sh.drain, 1);
    for (int i = 0; i < kItemSlots; ++i) {
      ptx::mbar_init(&sh.item_full[i], 1);
      ptx::mbar_init(&sh.item_empty[i], kPairReaders);
    }
    *sh.abort_flag = 0;
    ptx::fence_barrier_init();
  }
  if (warp == 8 && ptx::lane_id() == 0) {
    ptx::prefetch_tmap(&tmap_q);
    ptx::prefetch_tmap(&tmap_k);
    ptx::prefetch_tmap(&tmap_v);
  }
  if (warp == 9) {
    ptx::tmem_alloc_pair(sh.tmem_base, 512);
    ptx::tmem_relinquish_pair();
  }
  if (warp >= 8) ptx::setmaxnreg_dec<kRegsOther>();
  ptx::tc_fence_before_sync();
  // Both CTAs' barriers are initialised before any arrival crosses over.
  ptx::cluster_sync();
  ptx::tc_fence_after_sync();
  const uint32_t tmem = *sh.tmem_base;

  if (warp < 8) {
    ptx::setmaxnreg_inc<kRegsSoftmax>();
    softmax_role<CAUSAL>(sh, args, tmem, rank, warp / 4, warp % 4);
  } else if (warp == 8) {
    if (ptx::lane_id() == 0) producer_role<CAUSAL>(sh, args, smem, rank, &tmap_q, &tmap_k, &tmap_v);
    __syncwarp();
  } else if (warp == 9) {
    if (rank == 0) {
      mma_role<CAUSAL>(sh, args, smem, tmem);
    } else {
      // Rank 0's last commit reaches this CTA too: no product reads or
      // writes this CTA's memory after it.
      wait_warp(sh, args.status, sh.drain, 0, true);
    }
  }

  // After an abort, loads already issued may still be in flight: give them
  // time to land (bounded) before the CTAs leave.
  if (*sh.abort_flag) {
    const uint64_t t0 = ptx::globaltimer_ns();
    while (ptx::globaltimer_ns() - t0 < 100000ull) {
    }
  }
  __syncwarp();
  ptx::tc_fence_before_sync();
  ptx::cluster_sync();
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(args.queue + 1, 1) == static_cast<int>(gridDim.x) - 1) {
      atomicExch(args.queue, 0);
      atomicExch(args.queue + 1, 0);
    }
  }
  if (warp == 9) {
    ptx::tc_fence_after_sync();
    ptx::tmem_dealloc_pair(tmem, 512);
  }
}

}  // namespace pair
}  // namespace attn_b200
