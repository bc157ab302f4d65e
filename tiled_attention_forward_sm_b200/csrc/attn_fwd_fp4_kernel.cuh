// 4-bit (NVFP4) attention forward on sm_100a, head dim 128: the four-bit
// variant of page lecompute.fr/kernel-perf/flashattention-4-limites-calcul-
// matriciel, section "Le FP4 ajoute un compromis numerique" (fewer bits per
// operand buy tensor throughput, at a numeric cost, and preparing the data
// eats into the gain).
//
// Operands.  Q, K and V^T arrive as E2M1 codes (two per byte, the lower
// nibble first) with one E4M3 scale per 16 consecutive elements along the
// products' reduction axis (d for Q and K, the keys for V^T), and a
// per-tensor fp32 descale each; attn_quantize_nvfp4 produces them from
// bf16.  Both products are block-scaled tcgen05 MMAs (kind::mxf4nvf4,
// K = 64 per MMA, fp32 accumulators).  The softmax rounds P to NVFP4 too:
// per row and 16 keys, scale = E4M3(max / 6), codes = E2M1(p / scale).
//
// Scale factors.  The MMA reads them from Tensor Memory: for 128 rows and
// one MMA (4 scales per row) a block of 4 columns in which row m's four
// scales form the 32-bit word of column m / 32, lane m % 32 (the same word
// in all four lane quarters).  Each 128-row tile's scales are stored in
// global memory as two 512-byte blocks in exactly that order (byte
// 16 (m % 32) + 4 (m / 32) + s), loaded with the tile, and copied into TMEM
// with tcgen05.cp 32x128b.warpx4 by the MMA thread just before the MMAs
// that read them.
//
// Work and roles follow the head-dim-256 kernel (attn_fwd_wide_kernel.cuh):
// a CTA processes the two Q tiles of a work item one after the other, with
// S double-buffered, so QK(j+2) runs while the softmax works on tile j+1.
// Two Q tiles with their own S and O (the bf16 plan) would leave no Tensor
// Memory for the scale factors.  Tensor Memory plan (512 columns):
//   [  0,128)  S buffer 0: fp32 scores; then P codes in [0,16) and P's
//              scale factors in [16,24)
//   [128,256)  S buffer 1
//   [256,384)  O (fp32)
//   [384,400)  Q scale factors, two slots of 8 columns (Q tiles alternate)
//   [400,464)  K or V scale factors, one slot of 8 columns per ring stage
// Roles (10 warps): warps 0-7 softmax, two threads per query row: warp w
// reads TMEM lanes 32 (w % 4) .. + 31 and keys 64 (w / 4) .. + 63 of every
// score tile (the two halves of a row exchange their maxima through shared
// memory, so both take the same lazy decision; each rescales, quantises and
// stores its half of P and of O), warp 8 TMA producer, warp 9 TMEM
// allocator and MMA issuer.
#pragma once

#include "attn_fwd_kernel.cuh"

namespace attn_b200 {
namespace fp4 {

constexpr int kD = 128;
constexpr int kThreads = 320;
constexpr int kRowBytes = kD / 2;                    // 64 B: one row of 128 E2M1 codes
constexpr int kCodeBytes = kBlockM * kRowBytes;      // 8 KB per 128-row tile
constexpr int kScaleBytes = 1024;                    // 2 blocks of 512 B per tile
constexpr int kSlotBytes = 10240;                    // codes + scales, 1024-aligned
constexpr int kStages = 8;                           // K / V^T ring depth
constexpr int kQOff = 0;                             // one Q buffer (codes + scales)
constexpr int kKVOff = kSlotBytes;
constexpr int kPScaleOff = kKVOff + kStages * kSlotBytes;  // P scales, 2 buffers x 1 KB
// exchange of the two half-rows' values (row maxima, then row sums): 2
// parities x 2 halves x 128 rows, fp32
constexpr int kXchOff = kPScaleOff + 2 * kScaleBytes;
// O staging for the epilogue's TMA stores without the causal mask: each
// softmax warp's 32 rows x 64 columns of a tile (one 4 KB box, 128-byte
// swizzle).
constexpr int kOOff = kXchOff + 4 * 128 * 4;
constexpr int kOWarpBytes = 4096;
constexpr int kBarOff = kOOff + 8 * kOWarpBytes;
// barriers: q_full, q_empty, kv_full[S], kv_empty[S], s_full[2],
// p_ready[2 buffers][2 halves], pv_done, o_ready, drain, item_full[R],
// item_empty[R], xch[4 lane quarters]
constexpr int kNumBars = 2 + 2 * kStages + 2 + 4 + 1 + 1 + 1 + 2 * kItemSlots + 4;
constexpr int kMiscOff = kBarOff + kNumBars * 8;
constexpr int kRingOff = kMiscOff + 16;
constexpr int kSmemBytes = kRingOff + 4 * kItemWords * kItemSlots + 1024;  // + alignment slack
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
constexpr int kReaders = 9;  // item-ring readers: the MMA warp and 8 softmax warps
constexpr uint32_t kIdesc = ptx::idesc_nvfp4_f32(128, 128);  // QK and PV: M = N = 128
constexpr uint32_t kTmemO = 256;
constexpr uint32_t kTmemQsf = 384;   // + 8 * (Q tile parity)
constexpr uint32_t kTmemKVsf = 400;  // + 8 * ring stage
constexpr uint32_t kTmemPsf = 16;    // inside each S buffer

// The arguments beyond KernelArgs: scale-factor arrays ([BH, T, 2, 512]
// bytes, T = ceil(N / 128)) and the V descale.
struct Fp4Args {
  const uint8_t* q_sf;
  const uint8_t* k_sf;
  const uint8_t* v_sf;
  int n_tiles;  // T
  float v_descale;
};

struct Bars {
  uint64_t* q_full;
  uint64_t* q_empty;
  uint64_t* kv_full;   // [kStages]
  uint64_t* kv_empty;  // [kStages]
  uint64_t* s_full;    // [2]
  uint64_t* p_ready;   // [2 buffers][2 halves]
  uint64_t* pv_done;   // PV of a K/V tile complete (one phase per tile)
  uint64_t* o_ready;   // the Q tile's last PV complete
  uint64_t* xch;       // [4] the two warps of a lane quarter have posted their half-rows
};

__device__ __forceinline__ int tile_n(const Item& it, int s) { return s == 0 ? it.n0 : it.n1; }

// --------------------------------------------------------------- producer
// K and V^T tiles (codes, then their scale factors) enter one ring in the
// MMA's consumption order: K0, K1, then per tile j: V_j, K_{j+2}.
template <bool CAUSAL>
__device__ void producer_role(const Shared& sh, const Bars& bb, const KernelArgs& a,
                              const Fp4Args& f, uint8_t* smem, const CUtensorMap* tq,
                              const CUtensorMap* tk, const CUtensorMap* tvt) {
  const uint64_t pol_q = ptx::policy_evict_first();
  const uint64_t pol_kv = ptx::policy_evict_last();
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
    uint8_t* dst = smem + kKVOff + st * kSlotBytes;
    const int kt = it.kt0 + j;
    ptx::mbar_arrive_expect_tx(&bb.kv_full[st], kCodeBytes + kScaleBytes);
    if (is_v)
      ptx::tma_load_3d(tvt, &bb.kv_full[st], dst, kt * kRowBytes, 0, it.kz, pol_kv);
    else
      ptx::tma_load_3d(tk, &bb.kv_full[st], dst, 0, kt * kBlockN, it.kz, pol_kv);
    const uint8_t* sf = (is_v ? f.v_sf : f.k_sf) +
                        (static_cast<size_t>(it.kz) * f.n_tiles + kt) * kScaleBytes;
    ptx::bulk_load(dst + kCodeBytes, sf, kScaleBytes, &bb.kv_full[st], pol_kv);
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
  for (int r = 0; ok; ++r) {
    if (!have) {
      post_item(sh, a, r, nullptr);
      break;
    }
    if (!post_item(sh, a, r, &it)) break;
    for (int s = 0; s < 2 && ok; ++s) {
      const int n = tile_n(it, s);
      if (n == 0) continue;
      if (q_loads > 0 &&
          !wait_one(sh, a.status, bb.q_empty, static_cast<uint32_t>((q_loads - 1) & 1))) {
        ok = false;
        break;
      }
      const int qt = 2 * it.qpair + s;
      ptx::mbar_arrive_expect_tx(bb.q_full, kCodeBytes + kScaleBytes);
      ptx::tma_load_3d(tq, bb.q_full, smem + kQOff, 0, qt * kBlockM, it.qz, pol_q);
      ptx::bulk_load(smem + kQOff + kCodeBytes,
                     f.q_sf + (static_cast<size_t>(it.qz) * f.n_tiles + qt) * kScaleBytes,
                     kScaleBytes, bb.q_full, pol_q);
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
  // K-major E2M1 tiles: 64-byte rows with the 64-byte swizzle, 8-row groups
  // 512 B apart; a 64-deep K step moves 32 B inside the row.
  const uint32_t q_base = ptx::smem_u32(smem + kQOff);
  const uint32_t kv_base = ptx::smem_u32(smem + kKVOff);
  const uint32_t ps_base = ptx::smem_u32(smem + kPScaleOff);
  // Copy a tile's two 512-byte scale blocks into TMEM columns [col, col+8).
  auto copy_sf = [&](uint32_t src, uint32_t col) {
    ptx::tmem_cp_32x128b_x4_elect(tmem + col, ptx::sdesc_rows16(src));
    ptx::tmem_cp_32x128b_x4_elect(tmem + col + 4, ptx::sdesc_rows16(src + 512));
  };
  int consumed = 0, q_uses = 0, g = 0, gp = 0;
  uint32_t q_sf_col = kTmemQsf;
  auto stage_of = [&](int c) { return c % kStages; };
  auto phase_of = [&](int c) { return static_cast<uint32_t>((c / kStages) & 1); };
  auto qk_next = [&](bool last) -> bool {
    const int ck = consumed++;
    const int st = stage_of(ck);
    if (!wait_warp(sh, a.status, &bb.kv_full[st], phase_of(ck))) return false;
    ptx::tc_fence_after_sync();
    const uint32_t kv_sf_col = kTmemKVsf + 8u * st;
    copy_sf(kv_base + st * kSlotBytes + kCodeBytes, kv_sf_col);
    const uint64_t qd = ptx::sdesc_sw64(q_base, 512);
    const uint64_t kd = ptx::sdesc_sw64(kv_base + st * kSlotBytes, 512);
#pragma unroll
    for (int kk = 0; kk < 2; ++kk)
      ptx::mma_fp4_ss_elect(tmem + 128 * (g & 1), qd + static_cast<uint64_t>(2 * kk),
                            kd + static_cast<uint64_t>(2 * kk), kIdesc, tmem + q_sf_col + 4 * kk,
                            tmem + kv_sf_col + 4 * kk, kk > 0 ? 1u : 0u);
    ptx::commit_elect(&bb.s_full[g & 1]);
    ptx::commit_elect(&bb.kv_empty[st]);
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
      ptx::tc_fence_after_sync();
      q_sf_col = kTmemQsf + 8u * (q_uses & 1);
      ++q_uses;
      copy_sf(q_base + kCodeBytes, q_sf_col);
      if (!qk_next(n == 1)) goto done;
      if (n > 1 && !qk_next(n == 2)) goto done;
      for (int j = 0; j < n; ++j) {
        const int cv = consumed++;
        const int st = stage_of(cv);
        if (!wait_warp(sh, a.status, &bb.kv_full[st], phase_of(cv))) goto done;
        ptx::tc_fence_after_sync();
        const uint32_t v_sf_col = kTmemKVsf + 8u * st;
        copy_sf(kv_base + st * kSlotBytes + kCodeBytes, v_sf_col);
        const uint64_t vd = ptx::sdesc_sw64(kv_base + st * kSlotBytes, 512);
        const int b = gp & 1;
        const uint32_t acc = j > 0 ? 1u : 0u;
        for (int half = 0; half < 2; ++half) {
          if (!wait_warp(sh, a.status, &bb.p_ready[2 * b + half],
                         static_cast<uint32_t>((gp >> 1) & 1)))
            goto done;
          ptx::tc_fence_after_sync();
          // P's scale factors for keys [64 half, 64 half + 64): one 512-byte
          // block written by the softmax, into 4 columns of its S buffer.
          const uint32_t p_sf_col = 128u * b + kTmemPsf + 4u * half;
          ptx::tmem_cp_32x128b_x4_elect(tmem + p_sf_col,
                                        ptx::sdesc_rows16(ps_base + b * kScaleBytes + 512 * half));
          // O (+)= P V^T over those keys: P from TMEM (8 columns per 64
          // keys), V^T K-major.
          ptx::mma_fp4_ts_elect(tmem + kTmemO, tmem + 128 * b + 8 * half,
                                vd + static_cast<uint64_t>(2 * half), kIdesc, tmem + p_sf_col,
                                tmem + v_sf_col + 4 * half, acc | static_cast<uint32_t>(half));
        }
        ptx::commit_elect(bb.pv_done);
        ptx::commit_elect(&bb.kv_empty[st]);
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
// NVFP4 codes of 16 weights p (fp32, >= 0): the block scale E4M3(max / 6)
// (max times the fp32 reciprocal of 6) and E2M1(p / scale) (p times the
// approximate reciprocal of the scale), two words of 8 codes, the first
// weight in the lowest nibble.  A block whose scale rounds to 0 stores zero
// codes.
__device__ __forceinline__ uint32_t quantize_block16(const float* p, uint32_t& w0, uint32_t& w1) {
  float mx = fmaxf(ptx::max3(p[0], p[1], p[2]), ptx::max3(p[3], p[4], p[5]));
  mx = fmaxf(mx, ptx::max3(p[6], p[7], p[8]));
  mx = fmaxf(mx, ptx::max3(p[9], p[10], p[11]));
  mx = fmaxf(mx, ptx::max3(p[12], p[13], p[14]));
  mx = fmaxf(mx, p[15]);
  const uint32_t sc = ptx::f32_to_e4m3(mx * 0.16666667163372040f);
  const float sv = ptx::e4m3_to_f32(sc);
  const float inv = sv > 0.f ? ptx::rcp_approx(sv) : 0.f;
  w0 = ptx::pack_e2m1x8(p[0] * inv, p[1] * inv, p[2] * inv, p[3] * inv, p[4] * inv, p[5] * inv,
                        p[6] * inv, p[7] * inv);
  w1 = ptx::pack_e2m1x8(p[8] * inv, p[9] * inv, p[10] * inv, p[11] * inv, p[12] * inv,
                        p[13] * inv, p[14] * inv, p[15] * inv);
  return sc;
}

template <bool CAUSAL>
__device__ void softmax_role(const Shared& sh, const Bars& bb, const KernelArgs& a,
                             const Fp4Args& f, uint8_t* smem, uint32_t tmem, int warp,
                             const CUtensorMap* tmap_o) {
  uint8_t* o_stage = smem + kOOff + warp * kOWarpBytes;
  const int lane = static_cast<int>(ptx::lane_id());
  const int quarter = warp & 3;  // TMEM lanes of this warp
  const int h = warp >> 2;       // key half of every tile (and column half of O)
  const int r = quarter * 32 + lane;
  const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
  const uint32_t t_o = tmem + lane_off + kTmemO + 64u * h;
  // this row's word in its half's 512-byte scale block: byte 16 (r % 32) + 4 (r / 32)
  uint32_t* ps_word = reinterpret_cast<uint32_t*>(smem + kPScaleOff + 512 * h + 16 * lane +
                                                  4 * quarter);
  float* xbuf = reinterpret_cast<float*>(smem + kXchOff);  // [parity][half][row]
  uint64_t* xbar = &bb.xch[quarter];
  const float sl2 = a.scale_log2;
  const uint64_t sl2x2 = ptx::f2pack(sl2, sl2);
  int g = 0;   // K/V tiles consumed (S buffer g % 2)
  int eo = 0;  // Q tiles with at least one K/V tile finished
  int xc = 0;  // exchanges with the other half of the row
  // Post this half-row's value and take the other half's (both warps of the
  // lane quarter arrive on xbar; bounded wait).  A partner is at most one
  // exchange behind, so slots alternate by the exchange's parity.
  auto exchange = [&](float v, float& other) -> bool {
    float* slots = xbuf + (xc & 1) * 256;
    slots[h * 128 + r] = v;
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(xbar);
    if (!wait_warp(sh, a.status, xbar, static_cast<uint32_t>(xc & 1))) return false;
    ++xc;
    other = slots[(1 - h) * 128 + r];
    return true;
  };

  Item it;
  bool ok = true;
  for (int rr = 0; read_item(sh, a, rr, it, ok); ++rr) {
    for (int s = 0; s < 2; ++s) {
      const int qt = 2 * it.qpair + s;
      const int row = qt * kBlockM + r;
      if (qt * kBlockM >= it.q_len) continue;
      const int n = tile_n(it, s);
      float m = -INFINITY, l = 0.f;
      for (int j = 0; j < n; ++j) {
        const int key0 = (it.kt0 + j) * kBlockN + 64 * h;
        int key_limit = it.k_len - key0;  // keys of this half visible to the row
        if (CAUSAL) {
          const long long lim = static_cast<long long>(row) + it.delta + 1 - key0;
          if (lim < key_limit) key_limit = lim < -1 ? -1 : static_cast<int>(lim);
        }
        const int b = g & 1;
        const uint32_t t_s = tmem + lane_off + 128u * b + 64u * h;
        if (!wait_warp(sh, a.status, &bb.s_full[b], static_cast<uint32_t>((g >> 1) & 1))) return;
        ptx::tc_fence_after_sync();
        const bool masked = __any_sync(0xffffffffu, key_limit < 64);
        uint32_t sr[64];
        ptx::tmem_ld32(t_s + 0, sr + 0);
        ptx::tmem_ld32(t_s + 32, sr + 32);
        ptx::tmem_ld_wait_tie(sr + 0);
        ptx::reg_tie32(sr + 32);
        float x[64];
#pragma unroll
        for (int c = 0; c < 64; ++c) x[c] = __uint_as_float(sr[c]);
        if (masked) {
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (c >= key_limit) x[c] = -INFINITY;
        }
        float mx[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) mx[k] = x[k];
#pragma unroll
        for (int c = 8; c + 16 <= 64; c += 16) {
#pragma unroll
          for (int k = 0; k < 8; ++k) mx[k] = ptx::max3(mx[k], x[c + 2 * k], x[c + 2 * k + 1]);
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) mx[k] = ptx::max3(mx[k], x[56 + 2 * k], x[57 + 2 * k]);
        const float half_max = ptx::max3(ptx::max3(mx[0], mx[1], mx[2]),
                                         ptx::max3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
        float other_max;
        if (!exchange(half_max, other_max)) return;
        const float tile_max = fmaxf(half_max, other_max) * sl2;
        // Lazy rescale, the same decision in both halves of the row; O may
        // be touched only once the previous tile's PV has completed.
        float alpha = 1.f;
        bool rescale = false;
        if (tile_max - m > kRescaleTau) {
          alpha = ptx::ex2_approx(m - tile_max);
          m = tile_max;
          rescale = j > 0;
        }
        if (__any_sync(0xffffffffu, rescale)) {
          if (!wait_warp(sh, a.status, bb.pv_done, static_cast<uint32_t>((g - 1) & 1))) return;
          ptx::tc_fence_after_sync();
#pragma unroll 1
          for (int c0 = 0; c0 < 64; c0 += 32) {
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
        for (int q = 0; q < 32; ++q) {
          const int c = 2 * q;
          const uint64_t y2 = ptx::ffma2(ptx::f2pack(x[c], x[c + 1]), sl2x2, negm2);
          float y0, y1;
          ptx::f2unpack(y2, y0, y1);
          const uint64_t p2 = ptx::f2pack(ptx::ex2_approx(y0), ptx::ex2_approx(y1));
          if (q & 1) sb = ptx::fadd2(sb, p2);
          else sa = ptx::fadd2(sa, p2);
          ptx::f2unpack(p2, x[c], x[c + 1]);
        }
        // four 16-key blocks: 8 words of codes, 4 scale bytes
        uint32_t pk[8];
        uint32_t sw = 0;
#pragma unroll
        for (int blk = 0; blk < 4; ++blk) {
          const uint32_t sc = quantize_block16(x + 16 * blk, pk[2 * blk], pk[2 * blk + 1]);
          sw |= sc << (8 * blk);
        }
        // codes -> TMEM columns [8 h, 8 h + 8) of the S buffer, scales ->
        // this row's word of the buffer's scale block h
        ptx::tmem_st8(tmem + lane_off + 128u * b + 8u * h, pk);
        ps_word[(b * kScaleBytes) / 4] = sw;
        ptx::tmem_st_wait();
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&bb.p_ready[2 * b + h]);
        float la0, la1, lb0, lb1;
        ptx::f2unpack(sa, la0, la1);
        ptx::f2unpack(sb, lb0, lb1);
        l = l * alpha + ((la0 + la1) + (lb0 + lb1));
        ++g;
      }

      // Epilogue: the row sum of both halves; this half's 64 columns of
      // O v_descale / l -> bf16; LSE = (m + log2 l) ln 2 (written by half 0).
      float l_other = 0.f;
      if (!exchange(l, l_other)) return;
      l += l_other;
      if (n > 0) {
        if (!wait_warp(sh, a.status, bb.o_ready, static_cast<uint32_t>(eo & 1))) return;
        ++eo;
        ptx::tc_fence_after_sync();
      }
      const bool row_ok = row < it.q_len;
      const bool empty = m == -INFINITY;
      const float fo = empty ? 0.f : f.v_descale / l;
      const size_t o_row = static_cast<size_t>(it.qz) * a.N_q + row;
      // All eight warps reach the epilogue together.  Without the causal
      // mask (every tile of an item as long as the next) row-per-thread
      // stores, 32 rows per warp instruction, fill the load/store queue
      // there: this warp's 32 rows x 64 columns go through its staging box
      // and one TMA store instead (rows past the end of the head are
      // outside the map).  Under the mask that path measured 4% faster on
      // short items but 2% slower at N = 32768, so rows are stored
      // directly.
      if constexpr (!CAUSAL) {
        uint32_t ov0[32], ov1[32];
        if (n > 0) {
          ptx::tmem_ld32(t_o, ov0);
          ptx::tmem_ld32(t_o + 32, ov1);
          ptx::tmem_ld_wait_tie(ov0);
          ptx::reg_tie32(ov1);
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) ov0[c] = ov1[c] = 0u;
        }
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          pk[c] = ptx::pack_bf16x2(__uint_as_float(ov0[2 * c]) * fo,
                                   __uint_as_float(ov0[2 * c + 1]) * fo);
          pk[16 + c] = ptx::pack_bf16x2(__uint_as_float(ov1[2 * c]) * fo,
                                        __uint_as_float(ov1[2 * c + 1]) * fo);
        }
        // the box is rewritten once the previous tile's store has read it
        if (lane == 0) ptx::bulk_wait_read_all();
        __syncwarp();
        const uint32_t row_addr = ptx::smem_u32(o_stage) + static_cast<uint32_t>(lane) * 128u;
        const uint32_t sw = static_cast<uint32_t>(lane & 7);  // 128-byte swizzle
#pragma unroll
        for (int c = 0; c < 8; ++c)
          ptx::st_shared_v4(row_addr + ((static_cast<uint32_t>(c) ^ sw) << 4), pk[4 * c],
                            pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        ptx::fence_proxy_async_smem();
        __syncwarp();
        const int row0 = qt * kBlockM + 32 * quarter;
        if (lane == 0 && row0 < it.q_len) {
          ptx::tma_store_3d(tmap_o, o_stage, 64 * h, row0, it.qz);
          ptx::bulk_commit_group();
        }
      } else {
        __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(a.o) + o_row * kD + 64 * h;
#pragma unroll 1
        for (int c0 = 0; c0 < 64; c0 += 32) {
          uint32_t ov[32];
          if (n > 0) {
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
            pk[c] = ptx::pack_bf16x2(__uint_as_float(ov[2 * c]) * fo,
                                     __uint_as_float(ov[2 * c + 1]) * fo);
          uint4* dst = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
          for (int v = 0; v < 4; ++v)
            dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
        }
      }
      if (row_ok && h == 0) a.lse[o_row] = empty ? -INFINITY : (m + log2f(l)) * 0.69314718055994531f;
    }
  }
}

// ----------------------------------------------------------------- kernel
template <bool CAUSAL>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_fp4_kernel(const __grid_constant__ CUtensorMap tmap_q,
                        const __grid_constant__ CUtensorMap tmap_k,
                        const __grid_constant__ CUtensorMap tmap_vt,
                        const __grid_constant__ CUtensorMap tmap_o, const KernelArgs args,
                        const Fp4Args fargs) {
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
  bb.xch = bb.o_ready + 1;
  Shared sh = {};
  sh.drain = bb.xch + 4;
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
    for (int i = 0; i < 4; ++i) ptx::mbar_init(&bb.xch[i], 2);
    ptx::mbar_init(sh.drain, 1);
    for (int i = 0; i < kItemSlots; ++i) {
      ptx::mbar_init(&sh.item_full[i], 1);
      ptx::mbar_init(&sh.item_empty[i], kReaders);
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
  ptx::tc_fence_before_sync();
  __syncthreads();
  ptx::tc_fence_after_sync();
  const uint32_t tmem = *sh.tmem_base;

  if (warp < 8) {
    softmax_role<CAUSAL>(sh, bb, args, fargs, smem, tmem, warp, &tmap_o);
    // the staging boxes are read before the CTA exits
    if constexpr (!CAUSAL) ptx::bulk_wait_read_all();
  } else if (warp == 8) {
    if (ptx::lane_id() == 0)
      producer_role<CAUSAL>(sh, bb, args, fargs, smem, &tmap_q, &tmap_k, &tmap_vt);
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
  if (warp == 9) {
    ptx::tc_fence_after_sync();
    ptx::tmem_dealloc(tmem, 512);
  }
}

}  // namespace fp4
}  // namespace attn_b200
