// Shared device helpers of the MLA library (one translation unit: api.cu
// includes every kernel header, so file-scope device state is unique).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace mla {

// Device-side error word set by bounded waits that gave up (see
// mla_check_device_status). Bit values:
enum : uint32_t {
  kDevErrTimeout = 1u,      // an mbarrier / flag wait exceeded its limit
  kDevErrBadInput = 2u,     // a device-resident argument was out of range
  kDevErrRange = 4u,        // a value exceeded the fp16 range of an internal buffer
};

__device__ uint32_t g_device_error;

__device__ __forceinline__ void raise_device_error(uint32_t bits) {
  atomicOr(&g_device_error, bits);
}

// ---- element access in either run dtype (fp32 math throughout) ----------
template <typename T> __device__ __forceinline__ float to_f32(T v);
template <> __device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}
template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Rotary table row of a device-resident position; an out-of-range position
// sets the error word and falls back to row 0 (the identity rotation at the
// table's scale) so that no access leaves the table.
__device__ __forceinline__ int64_t checked_pos(int64_t pos, int max_pos) {
  if (pos < 0 || pos >= max_pos) {
    raise_device_error(kDevErrBadInput);
    return 0;
  }
  return pos;
}

// Index of the partner slots of rotary pair i inside a head's rotary part of
// width P: half-split pairs (i, i + P/2) or interleaved pairs (2i, 2i + 1).
__device__ __forceinline__ void rope_pair_slots(int i, int P, int interleaved, int& a, int& b) {
  if (interleaved) { a = 2 * i; b = 2 * i + 1; }
  else { a = i; b = i + P / 2; }
}

// Counter-clockwise turn of one rotary pair: (x, y) -> (x c - y s, y c + x s).
__device__ __forceinline__ void rope_turn(float x, float y, float c, float s, float& ox, float& oy) {
  ox = x * c - y * s;
  oy = y * c + x * s;
}

}  // namespace mla
