// Shared helpers of libtr: status reporting, per-device state, bf16 conversion.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <stdio.h>
#include <string>

#include "../../include/tr.h"

namespace tr {

// ---------------------------------------------------------------- error reporting
void set_error(const char* fmt, ...);
tr_status fail(tr_status code, const char* fmt, ...);

#define TR_CUDA_TRY(expr)                                                                 \
  do {                                                                                    \
    cudaError_t _e = (expr);                                                              \
    if (_e != cudaSuccess)                                                                \
      return ::tr::fail(TR_ERR_CUDA, "%s failed: %s (%s:%d)", #expr, cudaGetErrorString(_e), \
                        __FILE__, __LINE__);                                              \
  } while (0)

void count_launch();

#define TR_LAUNCH_CHECK(what)                                                             \
  do {                                                                                    \
    ::tr::count_launch();                                                                 \
    cudaError_t _e = cudaGetLastError();                                                  \
    if (_e != cudaSuccess)                                                                \
      return ::tr::fail(TR_ERR_CUDA, "launch of %s failed: %s", what, cudaGetErrorString(_e)); \
  } while (0)

#define TR_TRY(expr)               \
  do {                             \
    tr_status _s = (expr);         \
    if (_s != TR_OK) return _s;    \
  } while (0)

// ---------------------------------------------------------------- device status word
// Bits set by kernels that meet input only the device can check.
enum : int { STATUS_KEY_RANGE = 1, STATUS_KERNEL_TIMEOUT = 2 };

// Per-device state: the status word.
struct DeviceState {
  int* status = nullptr;       // device int
};
tr_status device_state(DeviceState** out);                 // of the current device
// Scratch of the multi-kernel (CUDA-core) calls: one grow-only buffer per (device, stream),
// so that calls on different streams never share scratch.  Growing it synchronises the
// stream and reallocates.
tr_status workspace(size_t bytes, cudaStream_t st, void** out);
// A few zero-initialised device ints per (device, stream), for kernels that claim work at
// run time (a launch zeroes what it uses on its stream first).  Allocated on first use.
tr_status stream_counters(cudaStream_t st, int** out);
// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) once per (device, kernel), under a lock.
tr_status ensure_smem_attr(const void* kernel, int bytes);

// ---------------------------------------------------------------- numeric helpers
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

inline int ceil_div(int64_t a, int64_t b) { return (int)((a + b - 1) / b); }
inline int round_up16(int x) { return (x + 15) & ~15; }

constexpr int kDHead = 16;     // head width every kernel assumes
constexpr float kLnEps = 1e-5f;

}  // namespace tr
