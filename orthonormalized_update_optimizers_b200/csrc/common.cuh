// Shared helpers of liborthoupd: error reporting, element conversions,
// bounded waits, batch descriptors.  Internal to the library.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cstdio>
#include <string>

#include "../../include/orthoupd.h"

namespace ouo {

// ---------------------------------------------------------------- host side

// Records a message for ouo_last_error() and returns `code`.
int set_error(int code, const char* fmt, ...);
void clear_error();

#define OUO_CHECK_CUDA(expr)                                                   \
  do {                                                                         \
    cudaError_t err__ = (expr);                                                \
    if (err__ != cudaSuccess)                                                  \
      return ::ouo::set_error(OUO_ERR_CUDA, "%s failed: %s (%s:%d)", #expr,    \
                              cudaGetErrorString(err__), __FILE__, __LINE__);  \
  } while (0)

// Counts every kernel this library enqueues (read by ouo_launch_count()).
void count_launch();

#define OUO_CHECK_LAUNCH()                                                     \
  do {                                                                         \
    ::ouo::count_launch();                                                     \
    cudaError_t err__ = cudaGetLastError();                                    \
    if (err__ != cudaSuccess)                                                  \
      return ::ouo::set_error(OUO_ERR_CUDA, "kernel launch failed: %s (%s:%d)",\
                              cudaGetErrorString(err__), __FILE__, __LINE__);  \
  } while (0)

#define OUO_TRY(expr)                                                          \
  do {                                                                         \
    int rc__ = (expr);                                                         \
    if (rc__ != OUO_OK) return rc__;                                           \
  } while (0)

inline size_t elem_size(int dtype) { return dtype == OUO_BF16 ? 2 : 4; }

// Number of SMs of the current device (cached per device).
int num_sms();
// Returns OUO_OK when the current device is an sm_100 part.
int require_sm100();

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// -------------------------------------------------------------- device side

__device__ __forceinline__ float bf16_to_f32(uint16_t h) {
  return __uint_as_float(((uint32_t)h) << 16);
}

__device__ __forceinline__ uint16_t f32_to_bf16(float f) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  return (uint32_t)f32_to_bf16(lo) | ((uint32_t)f32_to_bf16(hi) << 16);
}

// Round an fp32 value to the nearest tf32 value (ties away from zero), kept
// in an fp32 container, so that the tensor core's tf32 read of it is exact.
__device__ __forceinline__ float round_tf32(float f) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(f));
  return __uint_as_float(r);
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Upper bound of every device-side spin wait (nanoseconds).  A wait that
// runs out ORs OUO_STATUS_TIMEOUT into the status word and gives up.
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

__device__ __forceinline__ void report_status(int* status, int bits) {
  if (status) atomicOr(status, bits);
}

}  // namespace ouo
