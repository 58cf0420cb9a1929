// common.cuh -- shared constants of the device code.
#pragma once

#include <cstdint>

namespace afd {

// bits of the device error word (afd_ffn_get_error maps them to status codes)
constexpr int kErrBadExpert = 1;   // an expert index outside [0, E): pair skipped
constexpr int kErrBadPos = 2;      // a dispatched position outside the dispatched rows: skipped
constexpr int kErrBadOffsets = 4;  // group offsets not monotone / out of range: group skipped
constexpr int kErrTimeout = 8;     // a bounded on-device wait gave up

constexpr float kE4m3Max = 448.0f;

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ int warp_incl_scan(int v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  return v;
}

}  // namespace afd
