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

// Sum over the CTA (blockDim.x a multiple of 32, at most 1024); red: 32 floats of shared memory.
// Every thread receives the total.
__device__ __forceinline__ float block_sum(float v, float* red) {
  const int tid = threadIdx.x;
  v = warp_sum(v);
  __syncthreads();  // red may still be read by a previous call
  if ((tid & 31) == 0) red[tid >> 5] = v;
  __syncthreads();
  if (tid < 32) {
    float t = tid < static_cast<int>(blockDim.x >> 5) ? red[tid] : 0.f;
    t = warp_sum(t);
    if (tid == 0) red[0] = t;
  }
  __syncthreads();
  return red[0];
}

// f16 storage of the SwiGLU output of a token row x (large bf16 micro-batches).  Every act
// value of the row is bounded by ||x||^2 C (C: the handle's bound over the expert weights), so
// the row is stored as act / s with the power of two s >= 1 that keeps that bound times two
// below 32768: the f16 range (65504) cannot be exceeded and the scaling itself is exact.
// ss = ||x||^2; f16_bound = 2 C / 32768.
__device__ __forceinline__ float f16_row_scale(float ss, float f16_bound) {
  const float b = ss * f16_bound;
  if (!(b > 1.0f)) return 1.0f;
  if (!(b < 0x1p100f)) return 0x1p100f;
  int e;
  frexpf(b, &e);  // b = m 2^e, m in [0.5, 1): 2^e >= b
  return ldexpf(1.0f, e);
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
