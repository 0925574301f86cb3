// Shared device helpers of the H-BitLinear library: the device error flag, bounded waits,
// and small bit utilities. Everything here is sm_100a device code or plain host code.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace hbl {

// Error bits raised by kernels instead of trapping; read and cleared by hbl_device_status().
enum : int {
  kErrTimeout = 1,       // a bounded wait on an mbarrier or flag ran out
  kErrBadTernary = 2,    // hbl_pack_ternary saw a code outside {-1, 0, 1}
};

// One flag per device (the library's module is loaded once per device context).
__device__ int g_error_flags;

__device__ __forceinline__ void raise_error(int bits) { atomicOr(&g_error_flags, bits); }

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Wall-clock limit of every device-side wait. Legitimate waits last microseconds.
constexpr uint64_t kWaitLimitNs = 1000ull * 1000ull * 1000ull;  // 1 s

__host__ __device__ constexpr int ilog2_c(int v) { return v <= 1 ? 0 : 1 + ilog2_c(v >> 1); }

__host__ __device__ constexpr size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

}  // namespace hbl
