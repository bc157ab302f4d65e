// Host-side pieces shared by the library's translation units: the per-device
// state (capability check, device addresses of the status word and of the
// work-queue slots), TMA tensor-map encoding and buffer checks.  Internal to
// the library; the public contract is include/attn_b200.h.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstddef>
#include <cstdint>

namespace attn_b200 {
namespace host {

// Devices the library keeps state for (device ordinals below this).
constexpr int kMaxDevices = 64;

// Work-queue slots of the device array g_attn_queue ({next item, CTAs
// finished} each); a launch takes the next slot round-robin.
constexpr int kQueueSlots = 256;

struct DeviceState {
  bool checked = false;
  bool usable = false;
  int* status = nullptr;           // device address of g_attn_status
  int* queue = nullptr;            // device address of g_attn_queue
  int* noalloc_scratch = nullptr;  // device address of g_attn_noalloc_scratch
  int num_sms = 0;
  int ordinal = -1;                // the device's ordinal
  std::atomic<unsigned> launches{0};
};

// State of the current device, set up on first use: ATTN_OK, or
// ATTN_ERR_NO_DEVICE when there is none or it is not sm_100, or
// ATTN_ERR_CUDA when a runtime call failed.
int device_state(DeviceState** out);

// Device address of the next work-queue slot for one launch.
int* next_queue_slot(DeviceState& st);

// cuTensorMapEncodeTiled for a 3-D tensor with the 128-byte swizzle (or the
// one given), no
// interleave, zero fill out of bounds; dims/strides/box as the driver call
// takes them (strides: the two outer ones, in bytes).  device_state() must
// have succeeded first.  Encoded maps are cached host-side, keyed by every
// argument of the encode (a map holds nothing else, so a cached map is the
// one a fresh encode would give).
CUresult encode_tiled(CUtensorMap* m, CUtensorMapDataType type, const void* ptr,
                      const cuuint64_t* dims, const cuuint64_t* strides, const cuuint32_t* box,
                      CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B);

#ifdef ATTN_TEST_HOOKS
// Test builds only: set the bounded-wait limit and the withheld K/V load
// (see g_test_withhold_load) of the FP8 translation unit's kernels.
int fp8_test_set_hooks(unsigned long long wait_limit_ns, int withhold_load);
#endif

// Drop every cached tensor map (attn_release); later calls encode again.
void tmap_cache_clear();

// cudaFuncSetAttribute(kern, MaxDynamicSharedMemorySize, bytes) on the
// current device, once per device: `done` is the kernel's bit mask of the
// devices already set (one static per kernel at the call site).
int set_smem_once(const void* kern, int bytes, const DeviceState& st,
                  std::atomic<unsigned long long>& done);

// Per-head bf16 view [Z][N][d], boxes of 128 rows x 64 columns.
int make_tmap_heads(CUtensorMap* m, const void* ptr, int Z, int N, int d);

// The same view with boxes of box_rows rows x 64 columns.
int make_tmap_heads_rows(CUtensorMap* m, const void* ptr, int Z, int N, int d, int box_rows);

// Token-major bf16 view [T][Hx][d], boxes of 64 columns x 1 head x 128 tokens.
int make_tmap_tokens(CUtensorMap* m, const void* ptr, int T, int Hx, int d);

// ATTN_OK when every non-null pointer is device memory of the device `st`
// describes (the current device at set-up); ATTN_ERR_INVALID_ARG when one
// is host memory, managed memory, another GPU's memory or unknown to CUDA:
// the kernel would otherwise read it through a tensor map on the wrong GPU.
int check_on_device(const DeviceState& st, const void* const* ptrs, int n);

bool ranges_overlap(const void* a, size_t na, const void* b, size_t nb);

bool scale_ok(float scale);

// True when no output range overlaps an input range or another output.
bool outputs_disjoint(const void* const* outs, const size_t* out_bytes, int n_out,
                      const void* const* ins, const size_t* in_bytes, int n_in);

}  // namespace host
}  // namespace attn_b200
