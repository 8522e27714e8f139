// Internal helpers shared by the libtps kernels (not part of the public ABI).
#pragma once

#include <cuda_runtime.h>
#include <atomic>
#include <stdint.h>
#include <stddef.h>

#include "../../include/tps.h"

namespace tps {

// ---- host-side error handling ------------------------------------------------
// Records a message for tps_last_error() and returns `code`.
int fail(int code, const char* fmt, ...);
// Clears the thread's message and returns TPS_OK.
int ok();
// Returns TPS_ERR_CUDA (with the runtime's message) if `e` is an error.
int cuda_status(cudaError_t e, const char* what);
// Checks the launch that was just issued.
int launch_status(const char* what);

// Device address of this device's status word (resolved once per device).
unsigned int* device_status(int* err);

// Number of SMs of the current device (cached per device).
int sm_count();

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ---- device-side helpers -------------------------------------------------------
enum : unsigned int { STATUS_BOUNDS = 1u, STATUS_TIMEOUT = 2u };

__device__ __forceinline__ void raise_status(unsigned int* st, unsigned int bit) {
  if (st) atomicOr(st, bit);
}

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Two fp32 values -> packed bf16x2 (lo in bits 0-15), round to nearest even,
// with the hardware conversion instruction.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ uint4 ld16(const void* p) {
  return *reinterpret_cast<const uint4*>(p);
}
__device__ __forceinline__ void st16(void* p, uint4 v) { *reinterpret_cast<uint4*>(p) = v; }

// Clamped active count: min(*count, cap), never negative.
__device__ __forceinline__ int64_t active_count(const int32_t* count, int64_t cap) {
  int64_t c = *count;
  c = c < 0 ? 0 : c;
  return c < cap ? c : cap;
}

}  // namespace tps
