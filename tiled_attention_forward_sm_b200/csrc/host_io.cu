// C-ABI host-buffer entry point attn_fwd_host: copies in, the attention
// kernel, copies out, pipelined over groups of heads on streams the library
// owns.  The contract is documented in include/attn_b200.h.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "attn_b200.h"
#include "host_common.h"

using namespace attn_b200::host;

namespace attn_b200 {
namespace {

using namespace host;

// Streams and events of attn_fwd_host's pipeline, one set per device,
// created on first use.  The call holds `mu` until it has synchronised, so
// the events are never shared by two calls in flight.
constexpr int kHostChunksMax = 8;
struct HostPipe {
  std::mutex mu;
  bool ready = false;
  cudaStream_t h2d = nullptr, comp = nullptr, d2h = nullptr;
  cudaEvent_t start = nullptr, done = nullptr;
  cudaEvent_t in[kHostChunksMax] = {}, out[kHostChunksMax] = {};
};
HostPipe g_pipe[kMaxDevices];

int host_pipe(HostPipe& hp) {
  if (hp.ready) return ATTN_OK;
  const unsigned ef = cudaEventDisableTiming;
  bool ok = cudaStreamCreateWithFlags(&hp.h2d, cudaStreamNonBlocking) == cudaSuccess &&
            cudaStreamCreateWithFlags(&hp.comp, cudaStreamNonBlocking) == cudaSuccess &&
            cudaStreamCreateWithFlags(&hp.d2h, cudaStreamNonBlocking) == cudaSuccess &&
            cudaEventCreateWithFlags(&hp.start, ef) == cudaSuccess &&
            cudaEventCreateWithFlags(&hp.done, ef) == cudaSuccess;
  for (int c = 0; ok && c < kHostChunksMax; ++c)
    ok = cudaEventCreateWithFlags(&hp.in[c], ef) == cudaSuccess &&
         cudaEventCreateWithFlags(&hp.out[c], ef) == cudaSuccess;
  if (!ok) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  hp.ready = true;
  return ATTN_OK;
}

}  // namespace
}  // namespace attn_b200

using namespace attn_b200;

extern "C" int attn_fwd_host(const void* q_h, const void* k_h, const void* v_h, void* o_h,
                             float* lse_h, void* q_d, void* k_d, void* v_d, void* o_d,
                             float* lse_d, int B, int H, int N, int d, int causal, float scale,
                             attn_stream_t stream) {
  if (!q_h || !k_h || !v_h || !o_h || !lse_h) return ATTN_ERR_INVALID_ARG;
  int rc = attn_check_args(q_d, k_d, v_d, o_d, lse_d, B, H, N, d, scale);
  if (rc != ATTN_OK) return rc;
  DeviceState* st = nullptr;
  rc = device_state(&st);
  if (rc != ATTN_OK) return rc;
  {
    const void* ptrs[5] = {q_d, k_d, v_d, o_d, lse_d};
    rc = check_on_device(*st, ptrs, 5);
    if (rc != ATTN_OK) return rc;
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  HostPipe& hp = g_pipe[dev];
  std::lock_guard<std::mutex> lock(hp.mu);
  rc = host_pipe(hp);
  if (rc != ATTN_OK) return rc;

  // Heads are independent and contiguous ([B*H] blocks of N rows), so the
  // call runs as a pipeline over groups of heads: group c's host-to-device
  // copies, its kernel and its device-to-host copies go to three streams,
  // and the copies of one group overlap the kernel and the copies of the
  // others.  Small problems run as one group.
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int BH = B * H;
  const size_t head_rows = static_cast<size_t>(N);
  const size_t head_bytes = head_rows * static_cast<size_t>(d) * 2;
  const size_t total = static_cast<size_t>(BH) * head_bytes * 3;
  int n_chunks = total >= (64ull << 20) ? kHostChunksMax : 1;
  if (n_chunks > BH) n_chunks = BH;
  if (n_chunks == 1) {
    // One group: copies in, the kernel and copies out in order on the
    // caller's stream, with no cross-stream events.
    const size_t bytes = static_cast<size_t>(BH) * head_bytes;
    const size_t rows = static_cast<size_t>(BH) * head_rows;
    if (cudaMemcpyAsync(q_d, q_h, bytes, cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaMemcpyAsync(k_d, k_h, bytes, cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaMemcpyAsync(v_d, v_h, bytes, cudaMemcpyHostToDevice, s) != cudaSuccess) {
      cudaGetLastError();
      return ATTN_ERR_CUDA;
    }
    rc = attn_fwd(q_d, k_d, v_d, o_d, lse_d, B, H, N, d, causal, scale, stream);
    if (rc != ATTN_OK) return rc;
    if (cudaMemcpyAsync(o_h, o_d, bytes, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaMemcpyAsync(lse_h, lse_d, rows * 4, cudaMemcpyDeviceToHost, s) != cudaSuccess) {
      cudaGetLastError();
      return ATTN_ERR_CUDA;
    }
    return attn_last_device_error(stream);
  }
  const uint8_t* qh = static_cast<const uint8_t*>(q_h);
  const uint8_t* kh = static_cast<const uint8_t*>(k_h);
  const uint8_t* vh = static_cast<const uint8_t*>(v_h);
  uint8_t* oh = static_cast<uint8_t*>(o_h);
  uint8_t* qd = static_cast<uint8_t*>(q_d);
  uint8_t* kd = static_cast<uint8_t*>(k_d);
  uint8_t* vd = static_cast<uint8_t*>(v_d);
  uint8_t* od = static_cast<uint8_t*>(o_d);
  bool ok = cudaEventRecord(hp.start, s) == cudaSuccess &&
            cudaStreamWaitEvent(hp.h2d, hp.start, 0) == cudaSuccess &&
            cudaStreamWaitEvent(hp.comp, hp.start, 0) == cudaSuccess &&
            cudaStreamWaitEvent(hp.d2h, hp.start, 0) == cudaSuccess;
  int launch_rc = ATTN_OK;
  for (int c = 0; ok && c < n_chunks; ++c) {
    const int h0 = static_cast<int>(static_cast<int64_t>(BH) * c / n_chunks);
    const int h1 = static_cast<int>(static_cast<int64_t>(BH) * (c + 1) / n_chunks);
    const size_t off = static_cast<size_t>(h0) * head_bytes;
    const size_t bytes = static_cast<size_t>(h1 - h0) * head_bytes;
    const size_t loff = static_cast<size_t>(h0) * head_rows;
    const size_t lrows = static_cast<size_t>(h1 - h0) * head_rows;
    ok = cudaMemcpyAsync(qd + off, qh + off, bytes, cudaMemcpyHostToDevice, hp.h2d) == cudaSuccess &&
         cudaMemcpyAsync(kd + off, kh + off, bytes, cudaMemcpyHostToDevice, hp.h2d) == cudaSuccess &&
         cudaMemcpyAsync(vd + off, vh + off, bytes, cudaMemcpyHostToDevice, hp.h2d) == cudaSuccess &&
         cudaEventRecord(hp.in[c], hp.h2d) == cudaSuccess &&
         cudaStreamWaitEvent(hp.comp, hp.in[c], 0) == cudaSuccess;
    if (!ok) break;
    launch_rc = attn_fwd(qd + off, kd + off, vd + off, od + off, lse_d + loff, 1, h1 - h0, N, d,
                         causal, scale, hp.comp);
    if (launch_rc != ATTN_OK) break;
    ok = cudaEventRecord(hp.out[c], hp.comp) == cudaSuccess &&
         cudaStreamWaitEvent(hp.d2h, hp.out[c], 0) == cudaSuccess &&
         cudaMemcpyAsync(oh + off, od + off, bytes, cudaMemcpyDeviceToHost, hp.d2h) == cudaSuccess &&
         cudaMemcpyAsync(lse_h + loff, lse_d + loff, lrows * 4, cudaMemcpyDeviceToHost, hp.d2h) ==
             cudaSuccess;
  }
  // Whatever was enqueued completes before the call returns; the caller's
  // stream then continues after the last copy.
  const bool joined = cudaEventRecord(hp.done, hp.d2h) == cudaSuccess &&
                      cudaStreamWaitEvent(s, hp.done, 0) == cudaSuccess;
  cudaStreamSynchronize(hp.h2d);
  cudaStreamSynchronize(hp.comp);
  cudaStreamSynchronize(hp.d2h);
  if (!ok || !joined) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  if (launch_rc != ATTN_OK) return launch_rc;
  return attn_last_device_error(stream);
}
