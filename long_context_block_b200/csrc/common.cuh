// Shared device helpers for the MISA indexer kernels (sm_100a).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "misa.h"

namespace misa {

constexpr int kHeadDim = MISA_HEAD_DIM;     // d

// bf16 bit pattern -> fp32 (exact).
__device__ __forceinline__ float bf16_to_f32(uint32_t bits16) {
  return __uint_as_float(bits16 << 16);
}
// Two bf16 values packed in a 32-bit word -> (low, high) fp32.
__device__ __forceinline__ float bf16lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

// Order-preserving map of an fp32 score to uint32: a > b  <=>  key(a) > key(b).
// -0.0 is folded onto +0.0 first so that equal scores get equal keys.
__device__ __forceinline__ uint32_t score_key(float x) {
  uint32_t u = __float_as_uint(x + 0.0f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_score(uint32_t key) {
  uint32_t u = (key & 0x80000000u) ? (key & 0x7fffffffu) : ~key;
  return __uint_as_float(u);
}

// First statements of a kernel started by launch_pdl: let the next kernel in the stream
// begin launching, then wait until the previous kernel has completed and its writes are
// visible (both are no-ops for a kernel launched without the attribute).
__device__ __forceinline__ void pdl_prologue() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Record a device-side condition in the workspace status word (first one wins).
__device__ __forceinline__ void set_status(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

// Prefix length of a query, clamped to [1, L]; out-of-range positions are reported.
__device__ __forceinline__ int prefix_len(const int32_t* pos, int64_t row, int64_t L, int* status) {
  int p = pos[row];
  if (p < 0 || (int64_t)p >= L) {
    set_status(status, MISA_ERR_BAD_DEVICE_INPUT);
    p = p < 0 ? 0 : (int)(L - 1);
  }
  return p + 1;
}

}  // namespace misa
