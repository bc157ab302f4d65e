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
  ATTN_ERR_INVALID_ARG = -1,   /* null pointer, non-positive size, bad scale */
  ATTN_ERR_UNSUPPORTED = -2,   /* d not in {64,128}, or B*H*N >= 2^31 */
  ATTN_ERR_MISALIGNED = -3,    /* a device pointer is not 16-byte aligned */
  ATTN_ERR_CUDA = -4,          /* a CUDA runtime/driver call failed */
  ATTN_ERR_DEVICE_TIMEOUT = -5,/* a bounded wait inside the kernel ran out */
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
 *   d        64 or 128.
 *   causal   0: every key visible; non-zero: key j visible to query i iff j <= i.
 *   scale    finite and > 0 (typically 1/sqrt(d)).
 *   stream   CUDA stream the kernel is enqueued on.
 *
 * Ownership: the caller owns every buffer; the call allocates no device
 * memory.  Asynchrony: returns once the kernel is enqueued; results are valid
 * after the stream reaches that point.  Errors: argument and precondition
 * failures return a negative status before anything is enqueued; a failed
 * launch returns ATTN_ERR_CUDA.  A device-side timeout is reported later by
 * attn_last_device_error().
 */
int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
             int B, int H, int N, int d, int causal, float scale,
             attn_stream_t stream);

/*
 * Tuning options for attn_fwd_ex.  Every option only changes how the same
 * result is computed (rounding differs within the documented tolerance).
 *   exp2_poly_pairs  of every 4 pairs of score columns, how many take their
 *                    exponential from an FMA-pipe polynomial instead of the
 *                    special-function unit (the split described on the page's
 *                    section "Deplacer une partie des exponentielles");
 *                    0, 1 or 2, or -1 for the library default.
 */
typedef struct {
  int exp2_poly_pairs;
} attn_opts;

/*
 * attn_fwd_ex -- attn_fwd with tuning options (opts may be NULL: defaults).
 * Same contract as attn_fwd; an out-of-range option returns
 * ATTN_ERR_INVALID_ARG before anything is enqueued.
 */
int attn_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse,
                int B, int H, int N, int d, int causal, float scale,
                const attn_opts* opts, attn_stream_t stream);

/*
 * attn_fwd_noalloc -- attn_fwd for callers that cannot allocate device
 * memory, e.g. code running under global-mode CUDA stream capture (where
 * cudaMalloc is refused) or inside a framework whose allocator owns all
 * device memory.  There is no counterpart on the source pages: it is a
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
 * attn_fwd_host -- the same operation on HOST buffers: copies q, k, v from
 * host to the caller's device buffers, runs attn_fwd, and copies o and lse
 * back, all enqueued on `stream` (pinned host memory makes the copies
 * asynchronous).  Synchronises `stream` before returning, so the host
 * results are valid on return.
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
 * attn_last_device_error -- synchronises `stream`, then reads and clears the
 * device status word written by kernels on the current device (ATTN_OK if no
 * kernel reported an error).  Returns ATTN_ERR_CUDA if synchronisation or
 * the read fails.
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

/* Library version, (major << 16) | (minor << 8) | patch. */
int attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_B200_H */
