/*
 * attn_b200.h -- C ABI of the B200 (sm_100a) dense attention forward pass.
 *
 * The operation (page lecompute.fr/kernel-perf/flashattention-4-limites-
 * calcul-matriciel, section "Entre deux multiplications il faut fabriquer
 * les poids"): queries Q are compared with keys K by a first matrix product
 * (the scores); a softmax turns each row of scores into positive weights
 * summing to one; a second product mixes the values V with those weights.
 * The work is done tile by tile with a running maximum and running sum (same
 * page, section "Deplacer une partie des exponentielles"), so the N x N score
 * matrix never reaches device memory.  Under the causal mask (section "Le FP4
 * ajoute un compromis numerique") key j is visible to query i iff j <= i.
 *
 *   O[b,h,i,:] = sum_j w_ij V[b,h,j,:],   w_ij = exp(s_ij - LSE[b,h,i])
 *   s_ij       = scale * <Q[b,h,i,:], K[b,h,j,:]>   (j visible to i)
 *   LSE[b,h,i] = log sum_j exp(s_ij)                 (natural log)
 *
 * Numerics: bf16 inputs, fp32 scores and accumulation, weights rounded to
 * bf16 before the second product, O rounded to bf16 (nearest even), LSE fp32.
 *
 * All entry points return an attn_status (0 = ATTN_OK); none of them throws,
 * aborts or prints.
 */
#ifndef ATTN_B200_H
#define ATTN_B200_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ATTN_OK = 0,
  ATTN_ERR_INVALID_ARG = -1,   /* null pointer, non-positive size, bad scale,
                                  or a buffer that is not device memory of the
                                  current device */
  ATTN_ERR_UNSUPPORTED = -2,   /* d not in {64,96,128,256}, or B*H*N >= 2^31 */
  ATTN_ERR_MISALIGNED = -3,    /* a device pointer is not 16-byte aligned */
  ATTN_ERR_CUDA = -4,          /* a CUDA runtime/driver call failed */
  ATTN_ERR_DEVICE_TIMEOUT = -5,/* a bounded wait inside the kernel ran out */
  ATTN_ERR_DEVICE_BOUNDS = -6, /* device-side check: sequence offsets do not
                                  fit the buffers (attn_fwd_varlen); in the
                                  bounds-checked debug build also a tile
                                  coordinate or output index outside the
                                  launch's tensors */
  ATTN_ERR_NO_DEVICE = -7      /* no usable sm_100 device is current */
} attn_status;

/* Opaque CUDA stream (cudaStream_t); 0 is the legacy default stream. */
typedef void* attn_stream_t;

/*
 * attn_fwd -- O = softmax(scale * Q K^T [causal]) V and LSE, on the device.
 *
 *   q, k, v  device, bf16 [B, H, N, d], contiguous (d fastest).  Read only.
 *            May alias one another.
 *   o        device, bf16 [B, H, N, d], contiguous.  Written.
 *   lse      device, fp32 [B, H, N].  Written (natural log of the softmax
 *            denominator of the scaled, masked scores).
 *   o and lse must not overlap q, k, v or each other.
 *   B, H, N  > 0 (any N; tiles past N are masked); B*H*N < 2^31.
 *   d        64, 96, 128 or 256.
 *   causal   0: every key visible; non-zero: key j visible to query i iff j <= i.
 *   scale    finite and > 0 (typically 1/sqrt(d)).
 *   stream   CUDA stream the kernel is enqueued on.
 *
 * Device: every buffer must be device memory (cudaMalloc or a pool over it)
 * of the device current on the calling thread, which the stream must belong
 * to; host, managed or another GPU's memory returns ATTN_ERR_INVALID_ARG
 * (checked with cudaPointerGetAttributes; this holds for every entry point
 * below that takes device buffers).
 *
 * Ownership: the caller owns every buffer; the call allocates no device
 * memory.  Asynchrony: returns once the kernel is enqueued; results are valid
 * after the stream reaches that point.  Errors: argument and precondition
 * failures return a negative status before anything is enqueued; a failed
 * launch returns ATTN_ERR_CUDA.  A device-side timeout is reported later by
 * attn_last_device_error().  Stream capture: once a first call with the same
 * head dim, mask and options has run on the device (it sets up the device
 * state and the kernel's shared-memory attribute), the call can be captured
 * into a CUDA graph.  The captured launch keeps the work-queue slot it took
 * at capture time and its last CTA resets it, so replays in stream order are
 * correct; replays that may overlap on the GPU need separate captures.
 */
int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
             int B, int H, int N, int d, int causal, float scale,
             attn_stream_t stream);

/*
 * Tuning options for attn_fwd_ex.  Every option only changes how the same
 * result is computed (rounding differs within the documented tolerance).
 * Start from attn_opts_default() and set the fields you need.
 *   exp2_poly_pairs  of every 4 pairs of score columns, how many take their
 *                    exponential from an FMA-pipe polynomial instead of the
 *                    special-function unit (the split described on the page's
 *                    section "Deplacer une partie des exponentielles");
 *                    0, 1 or 2, or -1 for the library default.
 *   kv_stages        depth of the shared-memory ring that K and V tiles flow
 *                    through (page lecompute.fr/en/kernel-perf/flapping-
 *                    airplanes-thunderkittens-megakernels, section "Prepare
 *                    the next operation without overwriting the current
 *                    one"): 0 for the default (4 at d = 96 and 128, 8 at
 *                    d = 64), or 2, 3, 4 or 5 at d = 128 with the default
 *                    exponential split (other head dims or splits return
 *                    ATTN_ERR_UNSUPPORTED; 1 or more than 5 return
 *                    ATTN_ERR_INVALID_ARG).
 *   rescale_tau      the lazy-rescale threshold, in log2 units of the
 *                    scores (section "Deplacer une partie des
 *                    exponentielles": some rescalings are skipped under a
 *                    condition): the running maximum moves only when a
 *                    tile's maximum exceeds it by more than rescale_tau, so
 *                    weights stay below 2^rescale_tau.  -1 for the default
 *                    (12: bf16 weights up to 2^12 with fp32 sums are far
 *                    from overflow), or 0 .. 16 (0: rescale whenever the
 *                    maximum grows); d <= 128 only (ATTN_ERR_UNSUPPORTED at
 *                    d = 256, whose kernel also uses 12).
 *                    Note 0 is a valid threshold, not the default.
 */
typedef struct {
  int exp2_poly_pairs;
  int kv_stages;
  float rescale_tau;
} attn_opts;

/* Every option at its default: {-1, 0, -1.f}. */
attn_opts attn_opts_default(void);

/*
 * attn_fwd_ex -- attn_fwd with tuning options (opts may be NULL: defaults).
 * Same contract as attn_fwd; an out-of-range option returns
 * ATTN_ERR_INVALID_ARG before anything is enqueued.
 */
int attn_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse,
                int B, int H, int N, int d, int causal, float scale,
                const attn_opts* opts, attn_stream_t stream);

/*
 * attn_fwd_pair -- attn_fwd computed by pairs of CTAs on neighbouring SMs
 * (thread-block clusters of 2) that share each tensor-core product
 * (tcgen05.mma.cta_group::2, M = 256 query rows): each SM stages and reads
 * half of every K and V tile instead of all of it.  Motivation: page
 * lecompute.fr/kernel-perf/flashattention-4-limites-calcul-matriciel,
 * section "Blackwell deplace la limite vers les autres unites" (shared-memory
 * reads did not keep pace with the doubled per-SM matrix rate).  Measured on
 * B200 it is slower than attn_fwd: the P hand-off then crosses SMs.
 *
 * Same arguments, results (to rounding: the same arithmetic in another
 * order of products) and errors as attn_fwd, except that d must be 128
 * (other head dims return ATTN_ERR_UNSUPPORTED).  Allocates nothing.
 */
int attn_fwd_pair(const void* q, const void* k, const void* v, void* o, float* lse,
                  int B, int H, int N, int d, int causal, float scale,
                  attn_stream_t stream);

/*
 * attn_fwd_noalloc -- attn_fwd for callers that cannot allocate device
 * memory: a framework whose caching allocator has already reserved the
 * GPU's memory (a cudaMalloc would fail, or force it to give its cache
 * back), or a serving loop that fixed its memory budget at start-up and
 * must keep cudaMalloc, with its implicit device synchronisation, out of
 * its hot path.  There is no counterpart on the source pages: it is a
 * property of this library, not of the method.
 *
 * Same arguments, results and errors as attn_fwd; nothing is allocated.
 * The kernel's only scratch, its work-queue counter (8 bytes), lives in a
 * fixed 256-byte array the library holds in device memory on every GPU that
 * loads it, until the process exits.  The call clears that counter on
 * `stream` before its kernel, so each call starts clean, but every call
 * shares the same array: calls that overlap on the GPU (other streams, or
 * other threads' streams) race and must be serialised by the caller.
 * Problems whose work-item count plus the number of SMs would overflow the
 * 32-bit counter return ATTN_ERR_UNSUPPORTED.
 *
 * The first call of any entry point on a device (this one included) looks
 * up the scratch array's device address for that device; make that first
 * call before beginning any stream capture.
 */
int attn_fwd_noalloc(const void* q, const void* k, const void* v, void* o, float* lse,
                     int B, int H, int N, int d, int causal, float scale,
                     attn_stream_t stream);

/*
 * attn_fwd_chunk -- attention of N_q queries per head against N_k keys per
 * head, with an explicit causal offset and shared K/V heads.  This is the
 * building block for key/value caches (queries are the last N_q positions:
 * causal_delta = N_k - N_q), for splitting the keys into slices, and for
 * sharding them over GPUs: a chunk's O and LSE are the exact inputs of
 * attn_combine.
 *
 *   q        device, bf16 [B, H, N_q, d].          k, v  bf16 [B, H_kv, N_k, d].
 *   o        device, [B, H, N_q, d]: bf16, or fp32 when o_fp32 != 0.  Written.
 *   lse      device, fp32 [B, H, N_q].  Written.
 *   H_kv     K/V heads; H % H_kv == 0, query head h reads K/V head h/(H/H_kv).
 *   N_q, N_k > 0; B*H*N_q < 2^31 and B*H_kv*N_k < 2^31.
 *   causal   non-zero: key j visible to query i iff j <= i + causal_delta
 *            (|causal_delta| <= 2^30).  A query that sees no key gets O = 0
 *            and LSE = -inf.  causal = 0 ignores causal_delta.
 *   d, scale, stream, alignment, overlap, ownership, errors: as attn_fwd
 *   (o must be 16-byte aligned in both formats).
 */
int attn_fwd_chunk(const void* q, const void* k, const void* v, void* o, float* lse,
                   int B, int H, int H_kv, int N_q, int N_k, int d, int causal,
                   int causal_delta, float scale, int o_fp32, attn_stream_t stream);

/*
 * attn_fwd_varlen -- a batch of sequences of different lengths, packed
 * token-major without padding.
 *
 *   q        device, bf16 [total_q, H, d]: the query tokens of sequence b are
 *            rows cu_seqlens_q[b] .. cu_seqlens_q[b+1]-1.
 *   k, v     device, bf16 [total_k, H_kv, d], split by cu_seqlens_k.
 *   o        device, bf16 [total_q, H, d].  Written for every token of every
 *            sequence.
 *   lse      device, fp32 [H, total_q].  Written likewise.
 *   cu_seqlens_q, cu_seqlens_k  device, int32 [B+1], non-decreasing, from 0
 *            to total_q / total_k; a sequence may be empty.  Read only.
 *   max_seqlen_q, max_seqlen_k  upper bounds of the sequence lengths (> 0).
 *   causal   non-zero: inside sequence b, key j visible to query i iff
 *            j <= i + (len_k(b) - len_q(b)) (the last query sees the last
 *            key); a query that sees no key gets O = 0 and LSE = -inf.
 *   H % H_kv == 0; total_q*H and total_k*H_kv < 2^31.
 *   d, scale, stream, alignment (q, k, v, o: 16 bytes; lse and the offset
 *   arrays: 4), overlap, ownership and errors: as attn_fwd.  The offsets are
 *   device data, so they are checked on the device: a sequence whose offsets
 *   fall outside [0, total] or whose length exceeds its max_seqlen is skipped
 *   and attn_last_device_error() reports ATTN_ERR_DEVICE_BOUNDS.
 */
int attn_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                    const int* cu_seqlens_q, const int* cu_seqlens_k,
                    int B, int H, int H_kv, int max_seqlen_q, int max_seqlen_k,
                    int total_q, int total_k, int d, int causal, float scale,
                    attn_stream_t stream);

/*
 * attn_fwd_splitkv -- attn_fwd_chunk with each head's keys cut into
 * n_splits slices that run as separate work items, merged by attn_combine.
 * Same result as attn_fwd_chunk with a bf16 O (within its tolerance); it
 * pays when B*H*ceil(N_q/256) work items are too few to fill the GPU, e.g.
 * a short block of queries against a long key/value cache.
 *
 *   q, k, v, o, lse, B, H, H_kv, N_q, N_k, d, causal, causal_delta, scale,
 *   stream: as attn_fwd_chunk, with a bf16 O.
 *   n_splits  1 .. 256; it is reduced so that every slice holds keys
 *             (at most ceil(N_k/128) slices).  With one slice this is
 *             attn_fwd_chunk.
 *   ws_o      device, fp32, n_splits * B*H*N_q*d values, 16-byte aligned.
 *   ws_lse    device, fp32, n_splits * B*H*N_q values.
 *             Caller-owned scratch (the call allocates nothing); it must not
 *             overlap the other buffers.  Unused (may be NULL) with one slice.
 */
int attn_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse,
                     int B, int H, int H_kv, int N_q, int N_k, int d, int causal,
                     int causal_delta, float scale, int n_splits, float* ws_o,
                     float* ws_lse, attn_stream_t stream);

/*
 * attn_combine -- merge G partial results of the same query rows against
 * disjoint key sets (slices of one sequence, or shards on other GPUs) into
 * the result against their union:
 *   LSE = log sum_g exp(LSE_g),   O = sum_g exp(LSE_g - LSE) O_g.
 * This is the online softmax's common-scale rule (page lecompute.fr/kernel-
 * perf/flashattention-4-limites-calcul-matriciel, section "Deplacer une
 * partie des exponentielles") applied across slices instead of tiles.
 *
 *   o_parts    device, fp32 [G, rows, d], 16-byte aligned.  Read only.
 *   lse_parts  device, fp32 [G, rows] (-inf: the part saw no key).
 *   o          device, [rows, d]: bf16, or fp32 when o_fp32 != 0.  Written.
 *   lse        device, fp32 [rows].  Written (-inf if no part saw a key,
 *              with O = 0).
 *   G          1 .. 256;  rows >= 1;  d 64, 96, 128 or 256.
 *   Outputs must not overlap the inputs.  Errors and asynchrony as attn_fwd.
 */
int attn_combine(const float* o_parts, const float* lse_parts, int G, long long rows, int d,
                 void* o, float* lse, int o_fp32, attn_stream_t stream);

/*
 * attn_fwd_fp8 -- attention forward with FP8 (OCP E4M3) operands, head dim
 * 128: the low-precision variant weighed on page lecompute.fr/kernel-perf/
 * flashattention-4-limites-calcul-matriciel, section "Le FP4 ajoute un
 * compromis numerique".  Scores are (scale * q_descale * k_descale) Q K^T;
 * the weights are rounded to E4M3 before the second product (their row sum
 * is kept in fp32); O = v_descale * P V / l in bf16; LSE as attn_fwd.
 *
 *   q, k     device, E4M3 bytes [B, H, N, 128].  Read only.
 *   vt       device, E4M3 bytes [B, H, 128, N]: V transposed, so that both
 *            products read K-major operands.  Read only.
 *   o        device, bf16 [B, H, N, 128].  Written.   lse  fp32 [B, H, N].
 *   N        > 0 and a multiple of 16 (the V^T rows must be 16-byte
 *            aligned); B*H*N < 2^31.
 *   scale, q_descale, k_descale, v_descale  finite and > 0.
 * The weights' rounding (3 mantissa bits; below 2^-9 they flush to zero)
 * is the numeric cost of the format.  Errors and asynchrony as attn_fwd.
 */
int attn_fwd_fp8(const void* q, const void* k, const void* vt, void* o, float* lse,
                 int B, int H, int N, int d, int causal, float scale, float q_descale,
                 float k_descale, float v_descale, attn_stream_t stream);

/*
 * attn_quantize_e4m3 -- the conversion the FP8 path's inputs go through:
 * dst = E4M3(src * inv_descale), rounded to nearest even, saturated at
 * +-448.  src is device bf16 [BH, N, d]; dst device bytes, [BH, N, d]
 * (transpose = 0, for Q and K) or [BH, d, N] (transpose != 0, the V^T
 * operand; N must be a multiple of 16).  d 64 or 128; BH <= 65535; both
 * pointers 16-byte aligned, not overlapping.  Errors and asynchrony as
 * attn_fwd.
 */
int attn_quantize_e4m3(const void* src, void* dst, int BH, int N, int d, float inv_descale,
                       int transpose, attn_stream_t stream);

/*
 * attn_fwd_fp4 -- 4-bit (NVFP4) attention forward, d = 128 (page
 * lecompute.fr/kernel-perf/flashattention-4-limites-calcul-matriciel,
 * section "Le FP4 ajoute un compromis numerique": four-bit products, whose
 * data preparation eats into the gain).  Both products are block-scaled
 * 4-bit tensor-core MMAs: E2M1 elements with one E4M3 scale per 16
 * elements of the reduction axis, fp32 accumulation.  The softmax weights
 * are rounded to the same format (per row and 16 keys: scale =
 * E4M3(max / 6), codes = E2M1(p / scale)); the row sum uses the unrounded
 * fp32 weights.  O is bf16 and LSE fp32 as in attn_fwd, of the scores
 * scale * q_descale * k_descale * (Q K^T), with O scaled by v_descale.
 *
 *   q, k      device, E2M1 codes [B, H, N, 64] bytes (two per byte, the
 *             lower-indexed element in the lower nibble), from
 *             attn_quantize_nvfp4(transpose = 0).
 *   q_sf, k_sf  device, their E4M3 scales, attn_nvfp4_scale_bytes(B*H, N)
 *             bytes, from the same call.
 *   vt        device, E2M1 codes of V transposed per head, [B, H, 128, N/2]
 *             bytes; vt_sf its scales; from attn_quantize_nvfp4(transpose).
 *   o, lse    as attn_fwd (bf16 [B, H, N, 128]; fp32 [B, H, N]).  Written.
 *   N         > 0 and a multiple of 32 (V^T rows of N/2 bytes must be
 *             16-byte aligned); d must be 128: otherwise ATTN_ERR_UNSUPPORTED.
 *   descales  finite and > 0.
 * Every pointer 16-byte aligned (lse 4); outputs must not overlap inputs.
 * Causal mask, errors, asynchrony and ownership as attn_fwd.
 */
int attn_fwd_fp4(const void* q, const void* q_sf, const void* k, const void* k_sf,
                 const void* vt, const void* vt_sf, void* o, float* lse, int B, int H, int N,
                 int d, int causal, float scale, float q_descale, float k_descale,
                 float v_descale, attn_stream_t stream);

/*
 * attn_quantize_nvfp4 -- the conversion the 4-bit path's inputs go through.
 * x = src * inv_descale (float32); per 16 consecutive elements along d
 * (transpose = 0: Q and K, codes [BH, N, 64] bytes) or along the keys
 * (transpose != 0: V, codes of V^T [BH, 128, N/2] bytes, N a multiple of
 * 32): scale = E4M3(amax / 6) (nearest even, saturating at 448),
 * code = E2M1(x * (1 / scale)) (nearest even, saturating at +-6; zero codes
 * where the scale is 0).  The scales go to `scales`
 * (attn_nvfp4_scale_bytes(BH, N) bytes), per head and 128-row tile of the
 * product's operand in the order the block-scaled MMA reads them: two
 * 512-byte blocks (the first and second 64 elements of the reduction axis),
 * row m's four scales at byte 16 (m % 32) + 4 (m / 32) of a block.
 * src device bf16 [BH, N, 128]; d must be 128; src and codes 16-byte
 * aligned; no overlaps.  Errors and asynchrony as attn_fwd.
 */
int attn_quantize_nvfp4(const void* src, void* codes, void* scales, int BH, int N, int d,
                        float inv_descale, int transpose, attn_stream_t stream);

/* Bytes of one NVFP4 scale array for BH heads of N rows (or keys): -1 for
 * non-positive sizes. */
long long attn_nvfp4_scale_bytes(int BH, int N);

/*
 * attn_kmeans_assign -- the assignment step of k-means (page lefilia.fr,
 * Flash-KMeans item, "FlashAssign"): every point goes to its nearest
 * centroid, computed tile by tile without writing the N x K distance
 * matrix.  Same tile machinery as the attention forward, with a running
 * argmin where attention keeps a running softmax.
 *
 *   x          device, bf16 [N, d] points, contiguous.  Read only.
 *   centroids  device, bf16 [K, d], contiguous.  Read only.
 *   ws         device, fp32 scratch of attn_kmeans_workspace_floats(N, K)
 *              values (centroid norms, and point norms for large N),
 *              16-byte aligned, caller-owned; overwritten.
 *   assign     device, int32 [N].  Written: the index of the nearest
 *              centroid (among distances equal in fp32, the smallest index).
 *   best       device, fp32 [N] or NULL.  Written when given: the squared
 *              distance to that centroid, ||x||^2 + ||c||^2 - 2 x.c in fp32.
 *   N, K       > 0 and < 2^30;  d  64 or 128.
 * Distances are formed in fp32 from the bf16 inputs (products exact, sums
 * rounded), so points whose two nearest centroids are within that rounding
 * may pick either.  Errors and asynchrony as attn_fwd.
 */
int attn_kmeans_assign(const void* x, const void* centroids, float* ws, int32_t* assign,
                       float* best, int N, int K, int d, attn_stream_t stream);

/* Scratch size (fp32 values) attn_kmeans_assign needs: K rounded up to a
 * multiple of 128, plus N; or -1 for bad sizes. */
long long attn_kmeans_workspace_floats(int N, int K);

/*
 * attn_fwd_host -- the same operation on HOST buffers: copies q, k, v from
 * host to the caller's device buffers, runs attn_fwd, and copies o and lse
 * back.  Problems of 64 MiB of inputs or more run as a pipeline over up to 8
 * groups of heads: each group's host-to-device copies, its kernel and its
 * device-to-host copies go to three streams the library owns (one set per
 * device), so transfers in both directions overlap the kernels.  The work
 * starts after everything enqueued on `stream` before the call, and `stream`
 * continues after the last copy.  With pageable host memory the copies do
 * not overlap.  The call returns once everything has completed, so the host
 * results are valid on return; calls on the same device are serialised.
 *
 *   q_h, k_h, v_h   host bf16 [B,H,N,d];   o_h host bf16 [B,H,N,d];
 *   lse_h           host fp32 [B,H,N];
 *   q_d, k_d, v_d, o_d, lse_d   device buffers of the same sizes (caller
 *                   owned; the same rules as attn_fwd).
 * Returns ATTN_OK, an argument error (nothing enqueued), ATTN_ERR_CUDA, or
 * the device status word's error if the kernel reported one.
 */
int attn_fwd_host(const void* q_h, const void* k_h, const void* v_h, void* o_h, float* lse_h,
                  void* q_d, void* k_d, void* v_d, void* o_d, float* lse_d,
                  int B, int H, int N, int d, int causal, float scale,
                  attn_stream_t stream);

/*
 * attn_last_device_error -- reads and clears the device status word written
 * by kernels on the current device, behind the work already enqueued on
 * `stream`, and synchronises `stream` once (ATTN_OK if no kernel reported an
 * error).  Work on other streams is not waited for: join it into `stream`
 * first.  Returns ATTN_ERR_CUDA if the read or the synchronisation fails.
 */
int attn_last_device_error(attn_stream_t stream);

/*
 * attn_selftest_wait_timeout -- exercises the kernels' failure detection
 * without a fault: enqueues on `stream` one warp that waits, through the
 * same bounded wait the attention kernel uses, on a barrier nothing ever
 * completes.  After limit_us microseconds (1 .. 10^7) the wait gives up and
 * records ATTN_ERR_DEVICE_TIMEOUT in the device status word, which the next
 * attn_last_device_error(stream) returns (and clears); the context stays
 * usable.  Returns ATTN_OK once enqueued, ATTN_ERR_INVALID_ARG for an
 * out-of-range limit.
 */
int attn_selftest_wait_timeout(int limit_us, attn_stream_t stream);

/* Static string for a status code (never NULL). */
const char* attn_strerror(int status);

/*
 * attn_check_args -- the precondition check attn_fwd performs, without any
 * CUDA call: returns ATTN_OK or the status attn_fwd would return.
 */
int attn_check_args(const void* q, const void* k, const void* v, const void* o,
                    const float* lse, int B, int H, int N, int d, float scale);

/*
 * attn_release -- drop the library's host-side cache of encoded TMA tensor
 * maps.  Every launch needs three maps (Q, K, V views); they are cached,
 * keyed by every argument of the encode (buffer address, extents, strides,
 * box), so a repeated call on the same buffers skips the host work of
 * encoding them.  A cached map is bit for bit the one a fresh encode would
 * give, so a buffer that is freed and reallocated at the same address needs
 * no call here; the cache only holds host memory (a few KB), which this
 * call returns to its empty state.  Thread-safe.  Always ATTN_OK.
 */
int attn_release(void);

/* Library version, (major << 16) | (minor << 8) | patch. */
int attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_B200_H */
