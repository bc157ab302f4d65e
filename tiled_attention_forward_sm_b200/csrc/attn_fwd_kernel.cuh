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
//    result regions in Tensor Memory each with a producer/consumer lifetime,
//    and the first part of the weights announced before the rest;
//  * section "Deplacer une partie des exponentielles": a common scale kept
//    between old and new contributions, with some rescalings skipped under a
//    condition that keeps sums consistent and values in range; part of the
//    exponentials can be computed with ordinary multiply-adds.
//
// Work item: two 128-row Q tiles (Q0, Q1) of one (batch, head), i.e. 256
// query rows, against the K/V tiles they can see (128 keys per tile), or
// against one slice of those tiles when the keys are split.  The
// kernel is persistent: one CTA per SM takes work items from a shared queue
// (page lecompute.fr/en/kernel-perf/flapping-airplanes-thunderkittens-
// megakernels, section "Choose between predetermined work and a shared work
// queue": a queue rebalances, at the cost of one atomic per item), in an
// order that keeps the running CTAs on a few heads, and all barrier phases
// run on across items.
//
// Roles (12 warps, 384 threads):
//   warps 0-3   softmax group 0 (Q0): one thread per query row; also applies
//               the lazy O rescale and the epilogue for Q0
//   warps 4-7   softmax group 1 (Q1), same for Q1
//   warp  8     TMA producer: Q0/Q1 per item, then K_j, V_j through a ring
//   warp  9     TMEM allocator and tcgen05 MMA issuer (warp-uniform control,
//               one elected lane issues)
//   warps 10-11 idle
//
// Tensor Memory plan (512 columns x 128 lanes x 32 bit):
//   cols [  0,128)  S0 (fp32 scores of Q0 K_j^T); P0 (bf16 pairs) in [0,64)
//   cols [128,256)  S1 / P1
//   cols [256,256+D) O0 accumulator (fp32)
//   cols [384,384+D) O1 accumulator
//
// MMA issue order per K/V step j (one thread, in-order tensor pipe):
//   PV0(j-1) ... S0(j) ... PV1(j-1) ... S1(j)
// so the commit that publishes S_s(j) also guarantees PV_s(j-1) finished:
// the softmax group may rescale O_s in place as soon as it sees S_s(j).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>
#include <type_traits>

#include "ptx.cuh"

namespace attn_b200 {

// Device status word codes (mirrors attn_status in include/attn_b200.h).
constexpr int kStatusDeviceTimeout = -5;
constexpr int kStatusDeviceBounds = -6;

// Bounded waits: a wait that has not completed after this long sets the
// status word and the CTA's abort flag, and every role then leaves its loop.
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

#ifdef ATTN_TEST_HOOKS
// Test builds only (the product library never defines ATTN_TEST_HOOKS): the
// limit of every bounded wait, and one K/V tile load that the producer of
// CTA 0 skips (its index among that CTA's K/V loads; -1 for none), so that
// a consumer's wait runs out and the kernel's abort path runs, with no
// fault anywhere.  Every translation unit has its own copy; the test
// library's attn_test_set_hooks sets all of them.
static __device__ unsigned long long g_test_wait_limit_ns = kWaitLimitNs;
static __device__ int g_test_withhold_load = -1;
__device__ __forceinline__ uint64_t wait_limit_ns() { return g_test_wait_limit_ns; }
__device__ __forceinline__ bool withhold_load(int issued) {
  return blockIdx.x == 0 && issued == g_test_withhold_load;
}
#else
__device__ __forceinline__ constexpr uint64_t wait_limit_ns() { return kWaitLimitNs; }
__device__ __forceinline__ constexpr bool withhold_load(int) { return false; }
#endif

// Checked builds (ATTN_BOUNDS_CHECKS, libattn_b200_checked.so only) test
// every tensor-map coordinate and every O / LSE store index against the
// extents of the launch's tensors before the access is issued.  A failed
// check writes the bounds status, raises the CTA's abort flag and skips the
// access; nothing traps.  With the test hooks as well, the producer of CTA 0
// can be told to add an offset to its first item's K/V head, which a
// checked build must catch before any load of that head is issued.
#if defined(ATTN_BOUNDS_CHECKS) && defined(ATTN_TEST_HOOKS)
static __device__ int g_test_bad_kv_head = 0;
__device__ __forceinline__ int test_bad_kv_head() {
  return blockIdx.x == 0 ? g_test_bad_kv_head : 0;
}
#else
__device__ __forceinline__ constexpr int test_bad_kv_head() { return 0; }
#endif

// Softmax arithmetic form: packed f32x2 FMA/ADD (1) or scalar FMA/ADD (0).
// Measured on B200 the packed form is faster.
#ifndef ATTN_PACKED_SOFTMAX
#define ATTN_PACKED_SOFTMAX 1
#endif

// Default K/V ring depth for d = 96 and 128 (each stage holds one 128-row
// tile, 32 KB); d = 64 tiles are half as large and take 8 stages.
constexpr int kDefaultStagesD128 = 4;

// Work items announced by the producer to the MMA and softmax warps through
// a small ring in shared memory (kItemWords ints per slot).
constexpr int kItemSlots = 4;
constexpr int kItemWords = 16;
// Readers of each ring slot: the MMA warp and the 8 softmax warps.
constexpr int kItemReaders = 9;

constexpr int kBlockM = 128;  // query rows per Q tile
constexpr int kBlockN = 128;  // keys per K/V tile
constexpr int kThreads = 384;
// Register split: softmax warpgroups (256 threads) grow to kRegsSoftmax,
// the producer/MMA warpgroup (128 threads) shrinks to kRegsOther.  The sum
// must not exceed what the CTA was launched with (384 threads x 168).
constexpr int kRegsSoftmax = 200;
constexpr int kRegsOther = 104;
constexpr int kRegSplitTotal = 256 * kRegsSoftmax + 128 * kRegsOther;
static_assert(kRegSplitTotal <= kThreads * 168, "register split exceeds the launch budget");

// Keys of a score tile in the first published part of P (a multiple of 16,
// one PV MMA per 16 keys); the second part holds the remaining 48.  The
// uneven split leaves three PV MMAs, not four, between the last part's
// announcement and the next S of the same Q tile, while the first part's
// five MMAs run during the second part's exponentials (+1.1-1.5% with
// peaky scores, unchanged elsewhere; 96 + 32 is slower).
constexpr int kPFirstKeys = 80;
static_assert(kPFirstKeys % 16 == 0 && kPFirstKeys > 0 && kPFirstKeys < 128, "P split");

// Lazy-rescale thresholds in log2 units: the running maximum is raised only
// when a tile's maximum exceeds it by more than this, so every weight stays
// below 2^tau.  The limit is the format P is rounded to.  bf16 P (the same
// exponent range as fp32, 8-bit significand at any magnitude) with fp32 row
// sums and O accumulators is far from overflow at 2^12; a larger threshold
// means fewer rescales, which matters for peaky scores (2.2% faster than 8
// with q_std 3, unchanged on the others).  The narrow formats must stay near
// their largest value: E4M3 P tops out at 448 (2^8.8) and an NVFP4 block at
// 6 x 448, so the FP8 and 4-bit kernels keep 8.  The two-tile kernel takes
// its threshold from KernelArgs::rescale_tau (attn_fwd_ex can change it, 0
// meaning an eager rescale whenever the maximum grows); the other bf16
// kernels use kRescaleTauBf16.
constexpr float kRescaleTauBf16 = 12.0f;
constexpr float kRescaleTau = 8.0f;  // FP8 and NVFP4 P

// Optional timeline tracing (compiled in only with ATTN_TRACE_ENABLED; the
// library build leaves it out): clock64 stamps at each role's hand-off for
// the first work item of the first kTraceCtas CTAs and kTraceSteps K/V
// steps, written to a device buffer registered by the tracing build.
enum TraceEvent : int {
  kTrMmaS0 = 0, kTrMmaPV0a, kTrMmaPV0b, kTrMmaS1, kTrMmaPV1a, kTrMmaPV1b, kTrMmaV,
  kTrSm0Full, kTrSm0Ld, kTrSm0Max, kTrSm0Pa, kTrSm0Pb,
  kTrSm1Full, kTrSm1Ld, kTrSm1Max, kTrSm1Pa, kTrSm1Pb,
  kTrProdK, kTrProdV, kTrStart, kTrEnd, kTrMmaS0end, kTrMmaS1end, kTrMmaPV0end, kTrNumEvents
};
constexpr int kTraceCtas = 64;
constexpr int kTraceSteps = 72;
#ifdef ATTN_TRACE_ENABLED
__device__ unsigned long long* g_trace_buf = nullptr;
__device__ __forceinline__ void trace_stamp(int ev, int j) {
  const int cta = blockIdx.x;
  if (g_trace_buf != nullptr && cta < kTraceCtas && j >= 0 && j < kTraceSteps)
    g_trace_buf[(static_cast<size_t>(cta) * kTrNumEvents + ev) * kTraceSteps + j] = clock64();
}
#define ATTN_TRACE(ev, j) ::attn_b200::trace_stamp((ev), (j))
#else
#define ATTN_TRACE(ev, j) ((void)0)
#endif

// One launch's problem.  Two layouts:
//  * per-head ("dense"): Q is [B, H, N_q, D], K and V are [B, H_kv, N_k, D],
//    O is laid out like Q, LSE is [B, H, N_q];
//  * packed token-major (cu_q != null): Q is [T_q, H, D], K and V are
//    [T_k, H_kv, D]; sequence b owns query tokens [cu_q[b], cu_q[b+1]) and
//    key tokens [cu_k[b], cu_k[b+1]); O is laid out like Q, LSE is [H, T_q].
// Query head h reads K/V head h / (H / H_kv).  Under the causal mask key j
// of a sequence is visible to its query i iff j <= i + delta, with delta
// given (dense) or k_len - q_len of the sequence (packed: the last query
// sees the last key).  A row that sees no key gets O = 0 and LSE = -inf.
// With n_splits > 1 the K/V tiles of a head are cut into slices of
// split_tiles tiles; slice s writes its normalised partial O and LSE at
// row offset s * split_rows, for a later LSE-weighted merge.
struct KernelArgs {
  void* o;            // bf16 O, or fp32 (o_f32) O; rows of D values
  float* lse;
  const int* cu_q;    // packed layout: B+1 query token offsets (else null)
  const int* cu_k;    // packed layout: B+1 key token offsets
  int H, H_kv, q_per_kv;  // query heads, K/V heads, H / H_kv
  int N_q, N_k;       // dense: rows per head; packed: the longest sequence
  int T_q, T_k;       // packed: total query and key tokens
  int delta;          // dense causal offset
  int n_qpairs;       // ceil(ceil(N_q / 128) / 2)
  int n_splits;       // key slices per (head, Q tile pair)
  int split_tiles;    // K/V tiles per slice
  long long split_rows;  // rows of one slice of the outputs (0 without slices)
  int o_f32;          // store O as fp32 instead of bf16
  int BH;             // B * H (B * H_kv when two query heads share an item)
  int B;              // batch (sequences in the packed layout)
  int n_items;        // BH * n_qpairs * n_splits work items (some may be empty)
  int win_heads;      // heads per scheduling window (item order, see make_item)
  float scale_log2;   // scale * log2(e)
  float rescale_tau;  // lazy-rescale threshold (log2 units) of softmax_step
  int* status;        // device status word
  int* queue;         // {next item, CTAs finished}: this launch's queue slot
  int head_pack;      // dense, N_q <= 128: an item pairs two query heads of
                      // one K/V head (n_qpairs = head pairs per K/V head)
};

// STAGES: K/V ring depth, 0 for the default of the head dim.  TMA_O: the
// epilogue stores O through shared memory and TMA where there is room (the
// kernel asks for it without the causal mask, see softmax_role).
template <int D, int STAGES = 0, bool TMA_O = false>
struct Config {
  static_assert(D == 64 || D == 96 || D == 128, "head dim");
  static_assert(STAGES == 0 || (STAGES >= 2 && STAGES <= 5 && D > 64), "ring depth");
  // A tile is kBoxes 64-column TMA boxes of 128 rows; at D = 96 the second
  // box's columns 96..127 lie outside the tensor and arrive as zeros (the
  // products below never read them: QK stops at K = D, PV's N is D).
  static constexpr int kBoxes = (D + 63) / 64;
  static constexpr int kBoxBytes = kBlockM * 64 * 2;         // 16 KB
  static constexpr int kTileBytes = kBoxes * kBoxBytes;      // one 128 x 64*kBoxes tile
  static constexpr int kStages = STAGES > 0 ? STAGES : (D > 64 ? kDefaultStagesD128 : 8);
  static constexpr int kQOff = 0;
  static constexpr int kKVOff = 2 * kTileBytes;
  // barriers: q_full[2], q_empty[2], kv_full[S], kv_empty[S], s_full[2],
  // p_ready[2 tiles][2 halves], o_final[2], drain, item_full[R], item_empty[R]
  static constexpr int kNumBars = 4 + 2 * kStages + 2 + 4 + 2 + 1 + 2 * kItemSlots;
  // barriers, misc (tmem base, abort flag), the item ring, alignment slack
  static constexpr int kTailBytes = kNumBars * 8 + 16 + 4 * kItemWords * kItemSlots + 1024;
  // O staging for the epilogue's TMA stores: one 64-column box of 32 rows
  // (4 KB) per softmax warp, 32 KB in all, where it fits beside the K/V ring
  // (not beside a 5-stage ring at d > 64; the epilogue then stores rows
  // directly).
  static constexpr int kOOff = kKVOff + kStages * kTileBytes;
  static constexpr int kOWarpBytes = kBoxBytes / 4;
  static constexpr bool kOStage = TMA_O && kOOff + 8 * kOWarpBytes + kTailBytes <= 227 * 1024;
  static constexpr int kBarOff = kOOff + (kOStage ? 8 * kOWarpBytes : 0);
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kRingOff = kMiscOff + 16;
  static constexpr int kSmemBytes = kRingOff + 4 * kItemWords * kItemSlots + 1024;  // + alignment slack
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
  static constexpr uint32_t kIdescQK = ptx::idesc_bf16_f32(128, kBlockN, 0, 0);
  static constexpr uint32_t kIdescPV = ptx::idesc_bf16_f32(128, D, 0, 1);
};

struct Shared {
  uint64_t* q_full;    // [2] Q_s landed in shared memory
  uint64_t* q_empty;   // [2] last S_s of the item done: Q_s buffer reusable
  uint64_t* kv_full;   // [kStages]
  uint64_t* kv_empty;  // [kStages]
  uint64_t* s_full;    // [2] S_s(j) in TMEM
  uint64_t* p_ready;   // [2*s + half] half of P_s(j) in TMEM
  uint64_t* o_final;   // [2] last PV_s of the item done
  uint64_t* drain;
  uint64_t* item_full;   // [kItemSlots] item index written
  uint64_t* item_empty;  // [kItemSlots] every reader has taken it
  volatile int* item_ring;
  uint32_t* tmem_base;
  volatile int* abort_flag;
};

__device__ __forceinline__ void raise_status(const Shared& sh, int* status, int code) {
  *sh.abort_flag = 1;
  atomicCAS(status, 0, code);
}

// In checked builds: ok, or the bounds status written and the abort flag
// raised (the caller then skips the access).  Elsewhere: true.
__device__ __forceinline__ bool in_bounds(const Shared& sh, int* status, bool ok) {
#ifdef ATTN_BOUNDS_CHECKS
  if (!ok) raise_status(sh, status, kStatusDeviceBounds);
  return ok;
#else
  (void)sh;
  (void)status;
  (void)ok;
  return true;
#endif
}

// Tile coordinates inside the tensor maps: the first row (token) of a tile
// lies inside the tensor and the head exists.  Rows of a tile past the end
// of a ragged sequence are the maps' zero fill, not an error.
__device__ __forceinline__ bool q_tile_ok(const KernelArgs& a, long long row, int z) {
  if (a.cu_q != nullptr) return row >= 0 && row < a.T_q && z >= 0 && z < a.H;
  return row >= 0 && row < a.N_q && z >= 0 && z < a.B * a.H;
}
__device__ __forceinline__ bool kv_tile_ok(const KernelArgs& a, long long row, int z) {
  if (a.cu_q != nullptr) return row >= 0 && row < a.T_k && z >= 0 && z < a.H_kv;
  return row >= 0 && row < a.N_k && z >= 0 && z < a.B * a.H_kv;
}
// O rows (of D values) and LSE entries of the launch's outputs.
__device__ __forceinline__ long long out_rows(const KernelArgs& a) {
  const long long one = a.cu_q != nullptr ? static_cast<long long>(a.T_q) * a.H
                                          : static_cast<long long>(a.B) * a.H * a.N_q;
  return a.n_splits > 1 ? a.n_splits * a.split_rows : one;
}

// Single-thread bounded wait.  A drain wait (for this thread's own copies or
// MMAs in flight) ignores the abort flag but keeps the time limit (0: the
// kernel's limit).
__device__ __forceinline__ bool wait_one(const Shared& sh, int* status, uint64_t* bar,
                                         uint32_t parity, bool drain = false,
                                         uint64_t limit_ns = 0) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  if (limit_ns == 0) limit_ns = wait_limit_ns();
  const uint64_t t0 = ptx::globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0) {
      if (!drain && *sh.abort_flag) return false;
      if (ptx::globaltimer_ns() - t0 > limit_ns) {
        raise_status(sh, status, kStatusDeviceTimeout);
        return false;
      }
    }
  }
}

// Warp-uniform bounded wait (every lane returns the same answer), for roles
// whose next instructions are warp-collective tcgen05 loads/stores.
__device__ __forceinline__ bool wait_warp(const Shared& sh, int* status, uint64_t* bar,
                                          uint32_t parity, bool drain = false,
                                          uint64_t limit_ns = 0) {
  if (limit_ns == 0) limit_ns = wait_limit_ns();
  uint64_t t0 = 0;
  for (uint32_t it = 0;; ++it) {
    const bool ok = ptx::mbar_try_wait(bar, parity);
    if (__all_sync(0xffffffffu, ok)) return true;
    if ((it & 63u) == 63u) {
      int stop = 0;
      if (ptx::lane_id() == 0) {
        const uint64_t now = ptx::globaltimer_ns();
        if (t0 == 0) t0 = now;
        if (!drain && *sh.abort_flag) {
          stop = 1;
        } else if (now - t0 > limit_ns) {
          raise_status(sh, status, kStatusDeviceTimeout);
          stop = 1;
        }
      }
      if (__shfl_sync(0xffffffffu, stop, 0)) return false;
    }
  }
}

// ------------------------------------------------------------ work schedule
struct Item {
  int qpair;         // Q tiles 2*qpair and 2*qpair + 1 of the sequence
  int n0, n1;        // K/V tiles Q0 and Q1 visit in this item (0: none)
  int kt0;           // the item's first K/V tile
  int q_len, k_len;  // query rows and keys of the sequence
  int delta;         // causal: key j visible to query i iff j <= i + delta
  int qz, kz;        // map coordinate of the (batch, head) of Q and of K/V
  int q_row0, k_row0;  // row coordinate of query 0 and key 0 in the maps
  int split;         // key slice (offset of the partial outputs)
  int pack;          // 1: Q0 and Q1 are tile 0 of query heads qz and qz1
  int qz1;           // pack: map coordinate of Q1's head (-1: no second head)
};

// Q tile index and query-head map coordinate of softmax group s's tile.
__device__ __forceinline__ int item_qtile(const Item& it, int s) {
  return it.pack ? 0 : 2 * it.qpair + s;
}
__device__ __forceinline__ int item_qz(const Item& it, int s) {
  return (it.pack && s == 1) ? it.qz1 : it.qz;
}

// K/V tiles that Q tile `qt` of `it` visits inside the slice starting at
// tile it.kt0 (at most split_tiles of them).
template <bool CAUSAL>
__device__ __forceinline__ int tiles_for(int qt, const Item& it, int split_tiles) {
  const long long row_lo = static_cast<long long>(qt) * kBlockM;
  if (row_lo >= it.q_len) return 0;
  long long hi = it.k_len;  // keys [0, hi) can be seen by some row of the tile
  if (CAUSAL) {
    const long long q_hi = row_lo + kBlockM < it.q_len ? row_lo + kBlockM : it.q_len;
    if (q_hi + it.delta < hi) hi = q_hi + it.delta;
  }
  if (hi <= 0) return 0;
  const long long n = (hi + kBlockN - 1) / kBlockN - it.kt0;
  return n <= 0 ? 0 : (n > split_tiles ? split_tiles : static_cast<int>(n));
}

// Scheduling window of the item with head-major index `base` (units of
// n_per_head items per head): heads are cut into ceil(BH / win_heads)
// windows of equal size to within one head (the first ones one head
// larger), so the last window is as large as the others and its heaviest
// items do not start after every other CTA has run dry.  Returns the
// window's first head h0 and head count wh; base - h0 * n_per_head indexes
// the item inside it.
__device__ __forceinline__ void item_window(int base, int BH, int win_heads, int n_per_head,
                                            int& h0, int& wh) {
  const int n_win = (BH + win_heads - 1) / win_heads;
  const int wsz = BH / n_win, wrem = BH - wsz * n_win;  // wrem windows of wsz + 1 heads
  const int hpos = base / n_per_head;
  const int big = wrem * (wsz + 1);
  const int w = hpos < big ? hpos / (wsz + 1) : wrem + (hpos - big) / wsz;
  h0 = w * wsz + (w < wrem ? w : wrem);
  wh = wsz + (w < wrem ? 1 : 0);
}

// Item numbering: items are (head, Q tile pair, key slice) with the slice
// innermost.  Heads are taken in windows of at most win_heads (item_window);
// inside a window the pairs are numbered heaviest first under the causal
// mask (pair-major over the window's heads).  Items handed out in this
// order keep the CTAs that run together on a few heads, whose K/V then
// stays in L2, while the light pairs at the end of each window even out the
// CTAs' finishing times.
// Returns false for an item with no query rows (a pair past the end of a
// shorter sequence) or, after raising the bounds status, for a sequence
// whose offsets do not fit the buffers.
template <bool CAUSAL>
__device__ __forceinline__ bool make_item(int idx, const KernelArgs& a, int* status,
                                          Item& it) {
  int base = idx, split = 0;
  if (a.n_splits > 1) {
    base = idx / a.n_splits;
    split = idx - base * a.n_splits;
  }
  if (a.head_pack) {
    // One Q tile per head (per sequence in the packed layout): item
    // (b, K/V head hk, pair p) takes query heads hk*q_per_kv + 2p and
    // + 2p + 1, which read the same K/V head, so one K/V stream feeds both
    // softmax groups.
    const int b = base / (a.H_kv * a.n_qpairs);
    const int rem = base - b * (a.H_kv * a.n_qpairs);
    const int hk = rem / a.n_qpairs;
    const int pp = rem - hk * a.n_qpairs;
    const int h0 = hk * a.q_per_kv + 2 * pp;
    const bool two = 2 * pp + 1 < a.q_per_kv;
    it.pack = 1;
    it.qpair = 0;
    if (a.cu_q != nullptr) {
      const int q0 = a.cu_q[b], q1 = a.cu_q[b + 1], k0 = a.cu_k[b], k1 = a.cu_k[b + 1];
      if (q0 < 0 || q1 < q0 || q1 > a.T_q || q1 - q0 > a.N_q || k0 < 0 || k1 < k0 ||
          k1 > a.T_k || k1 - k0 > a.N_k) {
        atomicCAS(status, 0, kStatusDeviceBounds);
        return false;
      }
      if (q1 == q0) return false;  // a sequence without queries
      it.q_row0 = q0;
      it.q_len = q1 - q0;
      it.k_row0 = k0;
      it.k_len = k1 - k0;
      it.qz = h0;
      it.kz = hk;
      it.delta = it.k_len - it.q_len;
    } else {
      it.q_row0 = 0;
      it.q_len = a.N_q;
      it.k_row0 = 0;
      it.k_len = a.N_k;
      it.qz = b * a.H + h0;
      it.kz = b * a.H_kv + hk;
      it.delta = a.delta;
    }
    it.qz1 = two ? it.qz + 1 : -1;
    it.split = split;
    it.kt0 = split * a.split_tiles;
    it.n0 = tiles_for<CAUSAL>(0, it, a.split_tiles);
    it.n1 = it.qz1 >= 0 ? it.n0 : 0;
    return true;
  }
  it.pack = 0;
  it.qz1 = -1;
  int h0, wh;
  item_window(base, a.BH, a.win_heads, a.n_qpairs, h0, wh);
  const int k = base - h0 * a.n_qpairs;
  const int qp_idx = k / wh;
  const int bh = h0 + (k - qp_idx * wh);
  const int b = bh / a.H, h = bh - b * a.H;
  const int hk = h / a.q_per_kv;
  it.qpair = CAUSAL ? (a.n_qpairs - 1 - qp_idx) : qp_idx;
  if (a.cu_q != nullptr) {
    const int q0 = a.cu_q[b], q1 = a.cu_q[b + 1], k0 = a.cu_k[b], k1 = a.cu_k[b + 1];
    if (q0 < 0 || q1 < q0 || q1 > a.T_q || q1 - q0 > a.N_q || k0 < 0 || k1 < k0 ||
        k1 > a.T_k || k1 - k0 > a.N_k) {
      atomicCAS(status, 0, kStatusDeviceBounds);
      return false;
    }
    it.q_row0 = q0;
    it.q_len = q1 - q0;
    it.k_row0 = k0;
    it.k_len = k1 - k0;
    it.qz = h;
    it.kz = hk;
    it.delta = it.k_len - it.q_len;
  } else {
    it.q_row0 = 0;
    it.q_len = a.N_q;
    it.k_row0 = 0;
    it.k_len = a.N_k;
    it.qz = bh;
    it.kz = b * a.H_kv + hk;
    it.delta = a.delta;
  }
  if (2 * it.qpair * kBlockM >= it.q_len) return false;
  it.split = split;
  it.kt0 = split * a.split_tiles;
  it.n0 = tiles_for<CAUSAL>(2 * it.qpair, it, a.split_tiles);
  it.n1 = tiles_for<CAUSAL>(2 * it.qpair + 1, it, a.split_tiles);
  return true;
}

// Producer: announce its r-th item (or the end, it == nullptr) in ring slot
// r % R.
__device__ __forceinline__ bool post_item(const Shared& sh, const KernelArgs& a, int r,
                                          const Item* it) {
  const int slot = r % kItemSlots;
  const uint32_t ph = static_cast<uint32_t>((r / kItemSlots) & 1);
  if (!wait_one(sh, a.status, &sh.item_empty[slot], ph ^ 1)) return false;
  volatile int* w = sh.item_ring + slot * kItemWords;
  if (it == nullptr) {
    w[0] = 0;
  } else {
    w[0] = 1;
    w[1] = it->qpair;
    w[2] = it->n0;
    w[3] = it->n1;
    w[4] = it->kt0;
    w[5] = it->q_len;
    w[6] = it->k_len;
    w[7] = it->delta;
    w[8] = it->qz;
    w[9] = it->kz;
    w[10] = it->q_row0;
    w[11] = it->k_row0;
    w[12] = it->split;
    w[13] = it->pack;
    w[14] = it->qz1;
  }
  ptx::mbar_arrive(&sh.item_full[slot]);  // release: the writes are seen by waiters
  return true;
}

// Reader warp: its r-th item.  Returns false at the end of the work (or on
// abort, with ok cleared).
__device__ __forceinline__ bool read_item(const Shared& sh, const KernelArgs& a, int r, Item& it,
                                          bool& ok) {
  const int slot = r % kItemSlots;
  if (!wait_warp(sh, a.status, &sh.item_full[slot], static_cast<uint32_t>((r / kItemSlots) & 1))) {
    ok = false;
    return false;
  }
  const volatile int* w = sh.item_ring + slot * kItemWords;
  const bool valid = w[0] != 0;
  if (valid) {
    it.qpair = w[1];
    it.n0 = w[2];
    it.n1 = w[3];
    it.kt0 = w[4];
    it.q_len = w[5];
    it.k_len = w[6];
    it.delta = w[7];
    it.qz = w[8];
    it.kz = w[9];
    it.q_row0 = w[10];
    it.k_row0 = w[11];
    it.split = w[12];
    it.pack = w[13];
    it.qz1 = w[14];
  }
  __syncwarp();
  if (ptx::lane_id() == 0) ptx::mbar_arrive(&sh.item_empty[slot]);
  return valid;
}

// ----------------------------------------------------------------- producer
template <int D, bool CAUSAL, int STAGES = 0>
__device__ void producer_role(const Shared& sh, const KernelArgs& a, uint8_t* smem,
                              const CUtensorMap* tq, const CUtensorMap* tk,
                              const CUtensorMap* tv) {
  using C = Config<D, STAGES, !CAUSAL>;
  const uint64_t pol_q = ptx::policy_evict_first();
  const uint64_t pol_kv = ptx::policy_evict_last();
  const bool packed = a.cu_q != nullptr;
  // Tile load: per-head maps are indexed (column, row, head), packed maps
  // (column, head, token).
  auto load_tile = [&](const CUtensorMap* m, uint64_t* bar, uint8_t* dst, int row, int z,
                       uint64_t pol) {
    for (int b = 0; b < C::kBoxes; ++b) {
      if (packed)
        ptx::tma_load_3d(m, bar, dst + b * C::kBoxBytes, 64 * b, z, row, pol);
      else
        ptx::tma_load_3d(m, bar, dst + b * C::kBoxBytes, 64 * b, row, z, pol);
    }
  };
  int q_loads[2] = {0, 0};  // loads into Q buffer s so far
  int issued = 0;           // K/V tiles issued into the ring so far
  bool ok = true;
  // The next non-empty item from the launch's queue (one atomic per claim;
  // an index >= n_items means the work is done).
  Item it;
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
    const int n = it.n0 > it.n1 ? it.n0 : it.n1;
    // Q_s, once the previous item's last S_s no longer needs the buffer.
    for (int s = 0; s < 2 && ok; ++s) {
      if ((s == 0 ? it.n0 : it.n1) == 0) continue;
      if (q_loads[s] > 0 &&
          !wait_one(sh, a.status, &sh.q_empty[s], static_cast<uint32_t>((q_loads[s] - 1) & 1))) {
        ok = false;
        break;
      }
      const int q_row = it.q_row0 + item_qtile(it, s) * kBlockM;
      if (!in_bounds(sh, a.status, q_tile_ok(a, q_row, item_qz(it, s)))) {
        ok = false;
        break;
      }
      ptx::mbar_arrive_expect_tx(&sh.q_full[s], C::kTileBytes);
      load_tile(tq, &sh.q_full[s], smem + C::kQOff + s * C::kTileBytes, q_row, item_qz(it, s),
                pol_q);
      ++q_loads[s];
    }
    for (int j = 0; j < n && ok; ++j) {
      for (int which = 0; which < 2; ++which) {  // 0: K_j, 1: V_j
        const int st = issued % C::kStages;
        const uint32_t ph = (issued / C::kStages) & 1;
        if (!wait_one(sh, a.status, &sh.kv_empty[st], ph ^ 1)) { ok = false; break; }
        if (withhold_load(issued)) {  // test builds only
          ++issued;
          continue;
        }
        uint8_t* dst = smem + C::kKVOff + st * C::kTileBytes;
        const int kv_row = it.k_row0 + (it.kt0 + j) * kBlockN;
        if (!in_bounds(sh, a.status, kv_tile_ok(a, kv_row, it.kz))) { ok = false; break; }
        ATTN_TRACE(which == 0 ? kTrProdK : kTrProdV, r == 0 ? j : -1);
        ptx::mbar_arrive_expect_tx(&sh.kv_full[st], C::kTileBytes);
        load_tile(which == 0 ? tk : tv, &sh.kv_full[st], dst, kv_row, it.kz, pol_kv);
        ++issued;
      }
    }
    // Claim the next item only now: the ring holds the last K/V steps of
    // this one, so the claim's latency overlaps them, and a CTA never holds
    // an item it cannot start soon (which would lengthen the tail).
    if (ok) have = claim();
  }
  // Drain: every load issued must land before the CTA may exit.
  for (int s = 0; s < 2; ++s)
    if (q_loads[s] > 0)
      wait_one(sh, a.status, &sh.q_full[s], static_cast<uint32_t>((q_loads[s] - 1) & 1), true);
  for (int t = (issued > C::kStages ? issued - C::kStages : 0); t < issued; ++t)
    wait_one(sh, a.status, &sh.kv_full[t % C::kStages], (t / C::kStages) & 1, true);
}

// ---------------------------------------------------------------------- MMA
// Executed by the whole MMA warp so descriptors stay warp-uniform; each
// tcgen05.mma / tcgen05.commit is issued by one elected lane.  Descriptors
// are built once and advanced by constant offsets (the start-address field
// is the low 14 bits, in 16-byte units; no carry can leave it because
// shared memory is below 256 KB).
template <int D, bool CAUSAL, int STAGES = 0>
__device__ void mma_role(const Shared& sh, const KernelArgs& a, uint8_t* smem, uint32_t tmem) {
  using C = Config<D, STAGES, !CAUSAL>;
  const uint32_t t_s[2] = {tmem + 0, tmem + 128};
  const uint32_t t_o[2] = {tmem + 256, tmem + 384};
  // K-major (Q, K): SBO = 1024 B between 8-row groups; MN-major (V):
  // LBO = one 64-column box (16 KB), SBO = 1024 B between 8-key groups.
  const uint64_t q_desc = ptx::sdesc_sw128(ptx::smem_u32(smem + C::kQOff), 16, 1024);
  const uint64_t k_desc = ptx::sdesc_sw128(ptx::smem_u32(smem + C::kKVOff), 16, 1024);
  const uint64_t v_desc = ptx::sdesc_sw128(ptx::smem_u32(smem + C::kKVOff), C::kBoxBytes, 1024);
  constexpr uint64_t kTileUnits = C::kTileBytes >> 4;

  // S_s = Q_s K^T over D (D/16 MMAs of K-depth 16; a 16-deep step moves 32 B
  // inside the 128 B swizzle row, a 64-deep step moves one box)
  auto issue_qk = [&](int s, int stage) {
    const uint64_t qd = q_desc + s * kTileUnits;
    const uint64_t kd = k_desc + stage * kTileUnits;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint64_t off = static_cast<uint64_t>(((kk / 4) * C::kBoxBytes + (kk % 4) * 32) >> 4);
      ptx::mma_ss_elect(t_s[s], qd + off, kd + off, C::kIdescQK, kk > 0 ? 1u : 0u);
    }
  };
  // O_s (+)= P_s V over the keys of one published part of P (half 0: keys
  // [0, kPFirstKeys), half 1: the rest): P from TMEM (8 columns per 16
  // keys), V MN-major (2 KB per 16 keys)
  auto issue_pv_half = [&](int s, int half, int stage, uint32_t accumulate) {
    const uint64_t vd = v_desc + stage * kTileUnits;
    constexpr int kKa = kPFirstKeys / 16;  // MMAs of the first part
#pragma unroll
    for (int kk = half ? kKa : 0; kk < (half ? 8 : kKa); ++kk) {
      ptx::mma_ts_elect(t_o[s], t_s[s] + 8 * kk, vd + static_cast<uint64_t>((kk * 2048) >> 4),
                        C::kIdescPV, (accumulate | static_cast<uint32_t>(kk > 0)));
    }
  };
  int trace_j = -1;
  (void)trace_j;
  int p_count[2] = {0, 0};  // P_s publications consumed so far (all items)
  // Both halves of PV_s(j); the first half is issued as soon as the softmax
  // has published keys 0-63 of P, before keys 64-127 are ready.
  auto issue_pv = [&](int s, int stage, uint32_t accumulate) -> bool {
    const uint32_t parity = static_cast<uint32_t>(p_count[s] & 1);
    ++p_count[s];
    if (!wait_warp(sh, a.status, &sh.p_ready[2 * s], parity)) return false;
    ptx::tc_fence_after_sync();
    ATTN_TRACE(s == 0 ? kTrMmaPV0a : kTrMmaPV1a, trace_j);
    issue_pv_half(s, 0, stage, accumulate);
    if (!wait_warp(sh, a.status, &sh.p_ready[2 * s + 1], parity)) return false;
    ptx::tc_fence_after_sync();
    ATTN_TRACE(s == 0 ? kTrMmaPV0b : kTrMmaPV1b, trace_j);
    issue_pv_half(s, 1, stage, accumulate);
    return true;
  };
  // S_s(j) of an item visiting n_s K/V tiles; after its last S the Q_s
  // buffer is handed back to the producer.
  auto issue_s = [&](int s, int j, int n_s, int stage) {
    issue_qk(s, stage);
    ptx::commit_elect(&sh.s_full[s]);
    if (j == n_s - 1) ptx::commit_elect(&sh.q_empty[s]);
  };

  int consumed = 0;
  int q_uses[2] = {0, 0};
  auto stage_of = [&](int c) { return c % C::kStages; };
  auto phase_of = [&](int c) { return static_cast<uint32_t>((c / C::kStages) & 1); };

  Item it;
  bool ok = true;
  for (int r = 0; read_item(sh, a, r, it, ok); ++r) {
    const int n0 = it.n0, n1 = it.n1;
    const int n = n0 > n1 ? n0 : n1;
    if (n == 0) continue;  // rows that see no key: the softmax groups write them
    for (int s = 0; s < 2; ++s) {
      if ((s == 0 ? n0 : n1) == 0) continue;
      if (!wait_warp(sh, a.status, &sh.q_full[s], static_cast<uint32_t>(q_uses[s] & 1)))
        goto done;
      ++q_uses[s];
    }
    {
      // step 0: S0(0), S1(0)
      const int ck = consumed++;
      if (!wait_warp(sh, a.status, &sh.kv_full[stage_of(ck)], phase_of(ck))) goto done;
      ptx::tc_fence_after_sync();
      ATTN_TRACE(kTrMmaS0, r == 0 ? 0 : -1);
      if (n0 > 0) issue_s(0, 0, n0, stage_of(ck));
      ATTN_TRACE(kTrMmaS1, r == 0 ? 0 : -1);
      if (n1 > 0) issue_s(1, 0, n1, stage_of(ck));
      ptx::commit_elect(&sh.kv_empty[stage_of(ck)]);

      // Per step j: both K/V waits come first (the tiles are normally
      // resident long before), so that PV_s(j) and S_s(j+1) issue back to
      // back and no barrier round trip sits on a tile's S -> softmax -> PV
      // -> S chain.
      for (int j = 0; j < n; ++j) {
        const int cv = consumed++;
        trace_j = r == 0 ? j : -1;
        if (!wait_warp(sh, a.status, &sh.kv_full[stage_of(cv)], phase_of(cv))) goto done;
        const int ck2 = (j + 1 < n) ? consumed++ : -1;
        if (ck2 >= 0 &&
            !wait_warp(sh, a.status, &sh.kv_full[stage_of(ck2)], phase_of(ck2)))
          goto done;
        ptx::tc_fence_after_sync();
        ATTN_TRACE(kTrMmaV, trace_j);
        const uint32_t acc = j > 0 ? 1u : 0u;
        if (j < n0) {
          if (!issue_pv(0, stage_of(cv), acc)) goto done;
          ATTN_TRACE(kTrMmaPV0end, trace_j);
          if (j == n0 - 1) ptx::commit_elect(&sh.o_final[0]);
        }
        if (ck2 >= 0) {
          ATTN_TRACE(kTrMmaS0, r == 0 ? j + 1 : -1);
          if (j + 1 < n0) issue_s(0, j + 1, n0, stage_of(ck2));
          ATTN_TRACE(kTrMmaS0end, r == 0 ? j + 1 : -1);
        }
        if (j < n1) {
          if (!issue_pv(1, stage_of(cv), acc)) goto done;
          if (j == n1 - 1) ptx::commit_elect(&sh.o_final[1]);
        }
        ptx::commit_elect(&sh.kv_empty[stage_of(cv)]);
        if (ck2 >= 0) {
          ATTN_TRACE(kTrMmaS1, r == 0 ? j + 1 : -1);
          if (j + 1 < n1) issue_s(1, j + 1, n1, stage_of(ck2));
          ATTN_TRACE(kTrMmaS1end, r == 0 ? j + 1 : -1);
          ptx::commit_elect(&sh.kv_empty[stage_of(ck2)]);
        }
      }
    }
  }
done:
  // Drain: every MMA this warp issued completes before TMEM is released.
  ptx::commit_elect(sh.drain);
  wait_warp(sh, a.status, sh.drain, 0, true);
}

// ------------------------------------------------------------------ softmax
// exp2 on the FMA pipe for a pair of inputs: 2^x = 2^j * 2^f with j the
// nearest integer (1.5*2^23 rounding trick) and f in [-1/2, 1/2]; 2^f by a
// degree-3 polynomial minimising relative error (coefficients from
// csrc/gen_exp2_poly.py, max relative error 7.5e-5); 2^j added to the
// exponent field.  Inputs are clamped at -125 so the exponent stays normal.
__device__ __forceinline__ uint64_t exp2_poly2(uint64_t x2) {
  constexpr float kC0 = 0.9999280571937561f, kC1 = 0.6932609677314758f;
  constexpr float kC2 = 0.2426111251115799f, kC3 = 0.0551716685295105f;
  constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
  float x0, x1;
  ptx::f2unpack(x2, x0, x1);
  x2 = ptx::f2pack(fmaxf(x0, -125.f), fmaxf(x1, -125.f));
  const uint64_t magic = ptx::f2pack(kMagic, kMagic);
  const uint64_t t = ptx::fadd2(x2, magic);
  const uint64_t f = ptx::fsub2(x2, ptx::fsub2(t, magic));
  uint64_t p = ptx::ffma2(f, ptx::f2pack(kC3, kC3), ptx::f2pack(kC2, kC2));
  p = ptx::ffma2(f, p, ptx::f2pack(kC1, kC1));
  p = ptx::ffma2(f, p, ptx::f2pack(kC0, kC0));
  float p0, p1, t0, t1;
  ptx::f2unpack(p, p0, p1);
  ptx::f2unpack(t, t0, t1);
  return ptx::f2pack(__uint_as_float(__float_as_uint(p0) + (__float_as_uint(t0) << 23)),
                     __uint_as_float(__float_as_uint(p1) + (__float_as_uint(t1) << 23)));
}

// Scalar form of exp2_poly2 (same steps, one input).
__device__ __forceinline__ float exp2_poly1(float x) {
  constexpr float kC0 = 0.9999280571937561f, kC1 = 0.6932609677314758f;
  constexpr float kC2 = 0.2426111251115799f, kC3 = 0.0551716685295105f;
  constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
  x = fmaxf(x, -125.f);
  const float t = x + kMagic;
  const float f = x - (t - kMagic);
  float p = fmaf(f, kC3, kC2);
  p = fmaf(f, p, kC1);
  p = fmaf(f, p, kC0);
  return __uint_as_float(__float_as_uint(p) + (__float_as_uint(t) << 23));
}

// N consecutive TMEM columns of this thread's lane from pk, in stores of 32,
// 16 and 8 columns (N a multiple of 8).
template <int N>
__device__ __forceinline__ void store_cols(uint32_t taddr, const uint32_t* pk) {
  if constexpr (N >= 32) {
    ptx::tmem_st32(taddr, pk);
    store_cols<N - 32>(taddr + 32, pk + 32);
  } else if constexpr (N >= 16) {
    ptx::tmem_st16(taddr, pk);
    store_cols<N - 16>(taddr + 16, pk + 16);
  } else if constexpr (N >= 8) {
    ptx::tmem_st8(taddr, pk);
    store_cols<N - 8>(taddr + 8, pk + 8);
  }
}

// One K/V step of the online softmax for one query row (one thread):
// S_s(j) from TMEM -> running max (lazy rule) -> weights -> P_s(j) back to
// TMEM in two published parts (keys [0, kPFirstKeys) and the rest); m and
// l are the row's running max (log2 units) and sum.  PAIR: the CTA is one
// of a cluster pair whose rank-0 CTA
// issues the MMAs, so P is announced on that CTA's barrier.
template <int D, bool CAUSAL, int kPolyPairs, bool PAIR = false>
__device__ __forceinline__ bool softmax_step(const Shared& sh, const KernelArgs& a, int s,
                                             uint32_t t_s, uint32_t t_o, int r, int lane,
                                             int key_limit, bool first, uint32_t s_parity,
                                             int tj, float& m, float& l) {
  const float sl2 = a.scale_log2;
  if (!wait_warp(sh, a.status, &sh.s_full[s], s_parity)) return false;
  ptx::tc_fence_after_sync();
  if (r == 0) ATTN_TRACE(s == 0 ? kTrSm0Full : kTrSm1Full, tj);

  // Keys c >= key_limit of this tile are invisible to row r: under the
  // causal mask on the tiles the diagonal crosses, and on the last tile of a
  // key sequence whose length is not a multiple of 128.  Elsewhere key_limit
  // is at least 128 and nothing is masked.
  const bool masked = __any_sync(0xffffffffu, key_limit < 128);
  uint32_t sr[128];
  float x[128];
  // Row max: eight independent chains of three-input maxima.
  float mx[8];
  ptx::tmem_ld32(t_s + 0, sr + 0);
  ptx::tmem_ld32(t_s + 32, sr + 32);
  ptx::tmem_ld32(t_s + 64, sr + 64);
  ptx::tmem_ld32(t_s + 96, sr + 96);
  ptx::tmem_ld_wait_tie(sr + 0);
  ptx::reg_tie32(sr + 32);
  ptx::reg_tie32(sr + 64);
  ptx::reg_tie32(sr + 96);
#pragma unroll
  for (int c = 0; c < 128; ++c) x[c] = __uint_as_float(sr[c]);
  if (r == 0) ATTN_TRACE(s == 0 ? kTrSm0Ld : kTrSm1Ld, tj);
  if (masked) {
#pragma unroll
    for (int c = 0; c < 128; ++c)
      if (c >= key_limit) x[c] = -INFINITY;
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) mx[k] = x[k];
#pragma unroll
  for (int c = 8; c + 16 <= 128; c += 16) {
#pragma unroll
    for (int k = 0; k < 8; ++k) mx[k] = ptx::max3(mx[k], x[c + 2 * k], x[c + 2 * k + 1]);
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) mx[k] = ptx::max3(mx[k], x[120 + 2 * k], x[121 + 2 * k]);
  const float tile_max =
      ptx::max3(ptx::max3(mx[0], mx[1], mx[2]), ptx::max3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7])) *
      sl2;
  if (r == 0) ATTN_TRACE(s == 0 ? kTrSm0Max : kTrSm1Max, tj);

  // Lazy rescale: raise the running max only when it moves by > tau.
  float alpha = 1.f;
  bool rescale = false;
  if (tile_max - m > a.rescale_tau) {  // also true on the first tile (m = -inf)
    alpha = ptx::ex2_approx(m - tile_max);  // 0 on the first tile
    m = tile_max;
    rescale = !first;
  }
  // O_s *= alpha for the rows whose max moved (PV_s(j-1) is complete: its
  // commit preceded the one that published S_s(j)), before any P is
  // published, so the first half of PV_s(j) sees the rescaled O.  Where:
  // under the causal mask after the first half's weights, which the
  // warp-wide vote then overlaps (1.7% faster on B2 H32 N8192, 5% at
  // N 32768, 0.6% slower with peaky scores); without the mask before them
  // (the late form is 0.3-0.7% faster there with ordinary scores but 1.5%
  // slower with peaky ones, whose frequent rescales it leaves exposed).
  constexpr bool kLateRescale = CAUSAL;
  const bool any_rescale = __any_sync(0xffffffffu, rescale);
  if (!kLateRescale && any_rescale) {
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
  // (the late form in 16-column pieces: half of P and the second half's
  // scores still hold registers)
  auto rescale_o_late = [&]() {
#pragma unroll 1
    for (int c0 = 0; c0 < D; c0 += 16) {
      uint32_t ov[16];
      ptx::tmem_ld16(t_o + c0, ov);
      ptx::tmem_ld_wait_tie16(ov);
#pragma unroll
      for (int c = 0; c < 16; ++c) ov[c] = __float_as_uint(__uint_as_float(ov[c]) * alpha);
      ptx::tmem_st16(t_o + c0, ov);
    }
  };
  const uint64_t sl2x2 = ptx::f2pack(sl2, sl2);
  // A row that has seen no visible key yet keeps m = -inf; its weights are
  // then computed against 0 (all masked scores give 0, never NaN).
  const float negm = m == -INFINITY ? 0.f : -m;
  const uint64_t negm2 = ptx::f2pack(negm, negm);
  (void)sl2x2;
  (void)negm2;

#if ATTN_PACKED_SOFTMAX
  uint64_t lsum2a = ptx::f2pack(0.f, 0.f), lsum2b = lsum2a;
#else
  float ls0 = 0.f, ls1 = 0.f, ls2 = 0.f, ls3 = 0.f;
#endif
  // the two published parts of P: pairs [0, kPa) and [kPa, 64)
  auto part = [&](auto half_c) {
    constexpr int half = decltype(half_c)::value;
    constexpr int kPa = kPFirstKeys / 2;
    constexpr int q0 = half ? kPa : 0, q1 = half ? 64 : kPa;
    uint32_t pk[q1 - q0];
#pragma unroll
    for (int q = q0; q < q1; ++q) {
      const int c = 2 * q;
#if ATTN_PACKED_SOFTMAX
      const uint64_t y2 = ptx::ffma2(ptx::f2pack(x[c], x[c + 1]), sl2x2, negm2);
      uint64_t p2;
      if ((q & 3) < kPolyPairs) {
        // A masked key (-inf) comes out as 2^-125 rather than 0: against a
        // row sum l >= 1 and O entries summed in fp32 that weight is far
        // below one unit in the last place, so it cannot change O or LSE.
        p2 = exp2_poly2(y2);
      } else {
        float y0, y1;
        ptx::f2unpack(y2, y0, y1);
        p2 = ptx::f2pack(ptx::ex2_approx(y0), ptx::ex2_approx(y1));
      }
      if (q & 1) lsum2b = ptx::fadd2(lsum2b, p2);
      else lsum2a = ptx::fadd2(lsum2a, p2);
      float p0, p1;
      ptx::f2unpack(p2, p0, p1);
#else
      const float y0 = fmaf(x[c], sl2, negm), y1 = fmaf(x[c + 1], sl2, negm);
      float p0, p1;
      if ((q & 3) < kPolyPairs) {
        p0 = exp2_poly1(y0);
        p1 = exp2_poly1(y1);
      } else {
        p0 = ptx::ex2_approx(y0);
        p1 = ptx::ex2_approx(y1);
      }
      if (q & 1) { ls2 += p0; ls3 += p1; } else { ls0 += p0; ls1 += p1; }
#endif
      pk[q - q0] = ptx::pack_bf16x2(p0, p1);
    }
    if constexpr (half == 0) {
      if (kLateRescale && any_rescale) rescale_o_late();
    }
    // P_s keys [2 q0, 2 q1) as bf16 pairs over TMEM columns [q0, q1) of the
    // S_s region, in stores of 32, 16 and 8 columns; publish this part.
    store_cols<q1 - q0>(t_s + q0, pk);
    ptx::tmem_st_wait();
    ptx::tc_fence_before_sync();
    __syncwarp();
    if (lane == 0) {
      if constexpr (PAIR)
        ptx::mbar_arrive_cluster(ptx::mapa(ptx::smem_u32(&sh.p_ready[2 * s + half]), 0));
      else
        ptx::mbar_arrive(&sh.p_ready[2 * s + half]);
    }
    if (r == 0) ATTN_TRACE(s == 0 ? (half ? kTrSm0Pb : kTrSm0Pa) : (half ? kTrSm1Pb : kTrSm1Pa), tj);
  };
  part(std::integral_constant<int, 0>{});
  part(std::integral_constant<int, 1>{});
#if ATTN_PACKED_SOFTMAX
  float la0, la1, lb0, lb1;
  ptx::f2unpack(lsum2a, la0, la1);
  ptx::f2unpack(lsum2b, lb0, lb1);
  l = l * alpha + ((la0 + la1) + (lb0 + lb1));
#else
  l = l * alpha + ((ls0 + ls1) + (ls2 + ls3));
#endif
  return true;
}

// One thread per query row; warp w of the group reads TMEM lanes
// [32*(w%4), 32*(w%4)+32), so row r = 32*(w%4) + lane is the tile row.
//
// Without the causal mask both Q tiles of an item visit the same K/V tiles,
// so the two groups reach their epilogues together.  Row-per-thread stores
// from both (each warp store touching 32 rows) then fill the SM's
// load/store queue for microseconds, and the MMA warp's next barrier
// operations wait behind them.  There (bf16 per-head output, no key slices,
// staging room) the epilogue hands O to TMA stores instead: each warp writes
// its 32 rows of a 64-column box into its own 128-byte-swizzled staging box,
// and lane 0 stores the box.  Rows past the end of the sequence fall outside
// the tensor map and are not written.  Otherwise each thread stores its row.
template <int D, bool CAUSAL, int kPolyPairs, int STAGES>
__device__ void softmax_role(const Shared& sh, const KernelArgs& a, uint32_t tmem, int s,
                             int warp_in_group, uint8_t* o_stage, const CUtensorMap* tmap_o) {
  using C = Config<D, STAGES, !CAUSAL>;
  const bool tma_o = C::kOStage && !a.o_f32 && a.cu_q == nullptr && a.split_rows == 0;
  const int lane = static_cast<int>(ptx::lane_id());
  const int r = warp_in_group * 32 + lane;
  const uint32_t lane_off = static_cast<uint32_t>(warp_in_group * 32) << 16;
  const uint32_t t_s = tmem + lane_off + 128u * s;
  const uint32_t t_o = tmem + lane_off + 256u + 128u * s;
  int s_count = 0;  // S_s tiles consumed so far (all items)
  int o_count = 0;  // items finished by this group

  Item it;
  bool ok = true;
  for (int rr = 0; read_item(sh, a, rr, it, ok); ++rr) {
    const int qt = item_qtile(it, s);
    const int qz = item_qz(it, s);
    const int row = qt * kBlockM + r;  // query row in the sequence
    if (qt * kBlockM >= it.q_len || qz < 0) continue;  // the item has no such tile
    const int n_s = s == 0 ? it.n0 : it.n1;
    float m = -INFINITY;  // running max of scale*log2(e)*score (log2 units)
    float l = 0.f;        // running sum of weights, relative to 2^m
    for (int j = 0; j < n_s; ++j) {
      // Keys of tile kt0 + j visible to this row: those that exist and,
      // under the causal mask, those at or before row + delta.
      const int key0 = (it.kt0 + j) * kBlockN;
      int key_limit = it.k_len - key0;
      if (CAUSAL) {
        const long long lim = static_cast<long long>(row) + it.delta + 1 - key0;
        if (lim < key_limit) key_limit = lim < -1 ? -1 : static_cast<int>(lim);
      }
      if (!softmax_step<D, CAUSAL, kPolyPairs>(sh, a, s, t_s, t_o, r, lane, key_limit, j == 0,
                                               static_cast<uint32_t>(s_count & 1),
                                               rr == 0 ? j : -1, m, l))
        return;
      ++s_count;
    }

    // Epilogue: O_s / l -> rows of O; LSE = (m + log2 l) * ln 2.  The next
    // item's first PV_s (which overwrites O_s) is only issued after this
    // thread publishes that item's P, i.e. after these loads completed.
    // Rows past the end of the sequence (last tile of a ragged length) are
    // computed on whatever the tile holds and not stored; a row that saw no
    // key (m = -inf) stores O = 0 and LSE = -inf.
    if (n_s > 0) {
      if (!wait_warp(sh, a.status, &sh.o_final[s], static_cast<uint32_t>(o_count & 1))) return;
      ++o_count;
      ptx::tc_fence_after_sync();
    }
    const bool row_ok = row < it.q_len;
    const bool empty = m == -INFINITY;
    const float inv_l = empty ? 0.f : 1.f / l;
    size_t o_row, l_row;
    if (a.cu_q != nullptr) {
      o_row = (static_cast<size_t>(it.q_row0) + row) * a.H + qz;
      l_row = static_cast<size_t>(qz) * a.T_q + it.q_row0 + row;
    } else {
      o_row = static_cast<size_t>(qz) * a.N_q + row;
      l_row = o_row;
    }
    o_row += static_cast<size_t>(it.split) * a.split_rows;
    l_row += static_cast<size_t>(it.split) * a.split_rows;
    const bool store = row_ok && in_bounds(sh, a.status,
                                           static_cast<long long>(o_row) < out_rows(a) &&
                                               static_cast<long long>(l_row) < out_rows(a));
    if (tma_o) {
      // Box b holds columns [64b, 64b+64) of this warp's 32 rows.  The next
      // box's TMEM loads are in flight while this one is staged and stored;
      // the staging box is rewritten only after the previous store has read
      // it.
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
      for (int b = 0; b < C::kBoxes; ++b) {
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          pk[c] = ptx::pack_bf16x2(empty ? 0.f : __uint_as_float(ov0[2 * c]) * inv_l,
                                   empty ? 0.f : __uint_as_float(ov0[2 * c + 1]) * inv_l);
          pk[16 + c] = ptx::pack_bf16x2(empty ? 0.f : __uint_as_float(ov1[2 * c]) * inv_l,
                                        empty ? 0.f : __uint_as_float(ov1[2 * c + 1]) * inv_l);
        }
        if (b + 1 < C::kBoxes) load_box(b + 1);
        // (returns at once when no store is outstanding)
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
          ptx::tma_store_3d(tmap_o, o_stage, 64 * b, row0, qz);
          ptx::bulk_commit_group();
        }
        if (b + 1 < C::kBoxes) wait_box();
      }
    } else {
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
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
        if (!store) continue;
        if (a.o_f32) {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<float*>(a.o) + o_row * D + c0);
#pragma unroll
          for (int v = 0; v < 8; ++v)
            dst[v] = make_uint4(ov[4 * v], ov[4 * v + 1], ov[4 * v + 2], ov[4 * v + 3]);
        } else {
          uint32_t pk[16];
#pragma unroll
          for (int c = 0; c < 16; ++c)
            pk[c] =
                ptx::pack_bf16x2(__uint_as_float(ov[2 * c]), __uint_as_float(ov[2 * c + 1]));
          uint4* dst =
              reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.o) + o_row * D + c0);
#pragma unroll
          for (int v = 0; v < 4; ++v)
            dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
        }
      }
    }
    if (store) a.lse[l_row] = empty ? -INFINITY : (m + log2f(l)) * 0.69314718055994531f;
  }
}

// ------------------------------------------------------------------- kernel
template <int D, bool CAUSAL, int kPolyPairs, int STAGES = 0>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmap_q,
                    const __grid_constant__ CUtensorMap tmap_k,
                    const __grid_constant__ CUtensorMap tmap_v,
                    const __grid_constant__ CUtensorMap tmap_o, const KernelArgs args) {
  using C = Config<D, STAGES, !CAUSAL>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

  Shared sh;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  sh.q_full = bars;
  sh.q_empty = bars + 2;
  sh.kv_full = bars + 4;
  sh.kv_empty = sh.kv_full + C::kStages;
  sh.s_full = sh.kv_empty + C::kStages;
  sh.p_ready = sh.s_full + 2;
  sh.o_final = sh.p_ready + 4;
  sh.drain = sh.o_final + 2;
  sh.item_full = sh.drain + 1;
  sh.item_empty = sh.item_full + kItemSlots;
  sh.tmem_base = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
  sh.abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 4);
  sh.item_ring = reinterpret_cast<volatile int*>(smem + C::kRingOff);

  const int warp = threadIdx.x / 32;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&sh.q_full[i], 1);
      ptx::mbar_init(&sh.q_empty[i], 1);
      ptx::mbar_init(&sh.s_full[i], 1);
      ptx::mbar_init(&sh.p_ready[2 * i], 4);
      ptx::mbar_init(&sh.p_ready[2 * i + 1], 4);
      ptx::mbar_init(&sh.o_final[i], 1);
    }
    for (int i = 0; i < C::kStages; ++i) {
      ptx::mbar_init(&sh.kv_full[i], 1);
      ptx::mbar_init(&sh.kv_empty[i], 1);
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
    ptx::prefetch_tmap(&tmap_v);
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
  if (threadIdx.x == 0) ATTN_TRACE(kTrStart, 0);

  // Register split (see kRegsSoftmax): the producer/MMA warpgroup released
  // its share before the CTA-wide barrier above.
  if (warp < 8) {
    ptx::setmaxnreg_inc<kRegsSoftmax>();
    softmax_role<D, CAUSAL, kPolyPairs, STAGES>(
        sh, args, tmem, warp / 4, warp % 4,
        C::kOStage ? smem + C::kOOff + warp * C::kOWarpBytes : nullptr,
        C::kOStage ? &tmap_o : nullptr);
    // the staging boxes are read before the CTA exits
    if constexpr (C::kOStage) ptx::bulk_wait_read_all();
  } else if (warp == 8) {
    if (ptx::lane_id() == 0)
      producer_role<D, CAUSAL, STAGES>(sh, args, smem, &tmap_q, &tmap_k, &tmap_v);
    __syncwarp();
  } else if (warp == 9) {
    mma_role<D, CAUSAL, STAGES>(sh, args, smem, tmem);
  }

  ptx::tc_fence_before_sync();
  __syncthreads();
  if (threadIdx.x == 0) {
    ATTN_TRACE(kTrEnd, 0);
    // The last CTA to finish resets this launch's queue slot for its next
    // user (every CTA's claims precede its arrival here).
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

// ------------------------------------------------------- wait self-test
// Failure detection without a fault: one warp waits, through the same
// bounded wait the attention kernel uses, on an mbarrier that nothing ever
// arrives on.  After limit_ns the wait gives up, writes the timeout code to
// the status word and returns; the CTA exits normally and the context stays
// usable.
static __global__ void __launch_bounds__(32, 1) wait_timeout_selftest_kernel(int* status,
                                                                           uint64_t limit_ns) {
  __shared__ uint64_t never;
  __shared__ int abort_flag;
  Shared sh = {};
  sh.abort_flag = &abort_flag;
  if (threadIdx.x == 0) {
    ptx::mbar_init(&never, 1);
    abort_flag = 0;
    ptx::fence_barrier_init();
  }
  __syncwarp();
  wait_warp(sh, status, &never, 0, false, limit_ns);
}

}  // namespace attn_b200
