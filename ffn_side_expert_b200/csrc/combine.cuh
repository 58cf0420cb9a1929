// combine.cuh -- weighted combine of the expert outputs back into token order.
//
// Combine returns the experts' outputs to their tokens (A/F 分离, 机制; an all-to-all
// across GPUs, a gather here).  Reading taken: out[t] = sum_j w[t,j] * Y[pos[t,j]] + Ys[t],
// summed in fp32 in j order with the shared expert last, rounded once to bf16.  No atomics:
// one CTA per token, so the result does not depend on scheduling.
#pragma once

#include <cuda_bf16.h>

#include "common.cuh"

namespace afd {

__global__ void __launch_bounds__(256)
combine_kernel(const float* __restrict__ Y, const float* __restrict__ w, const int32_t* __restrict__ pos,
               int T, int k, int H, int n_rows, int with_shared, __nv_bfloat16* __restrict__ out, int* err) {
  __shared__ int sp[32];
  __shared__ float sw[32];
  const int t = blockIdx.x;
  if (threadIdx.x < k) {
    int p = pos[static_cast<size_t>(t) * k + threadIdx.x];
    if (p >= n_rows) { atomicOr(err, kErrBadPos); p = -1; }
    sp[threadIdx.x] = p;
    sw[threadIdx.x] = w[static_cast<size_t>(t) * k + threadIdx.x];
  }
  __syncthreads();
  const float* ys = Y + (static_cast<size_t>(T) * k + t) * H;  // shared-expert row
  for (int v = threadIdx.x; v < H / 4; v += blockDim.x) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < k; ++j) {
      const int p = sp[j];
      if (p < 0) continue;
      const float wj = sw[j];
      const float4 y = reinterpret_cast<const float4*>(Y + static_cast<size_t>(p) * H)[v];
      acc.x = fmaf(wj, y.x, acc.x);
      acc.y = fmaf(wj, y.y, acc.y);
      acc.z = fmaf(wj, y.z, acc.z);
      acc.w = fmaf(wj, y.w, acc.w);
    }
    if (with_shared) {
      const float4 s = reinterpret_cast<const float4*>(ys)[v];
      acc.x += s.x; acc.y += s.y; acc.z += s.z; acc.w += s.w;
    }
    __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
    __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
    uint2 packed;
    packed.x = *reinterpret_cast<uint32_t*>(&lo);
    packed.y = *reinterpret_cast<uint32_t*>(&hi);
    reinterpret_cast<uint2*>(out + static_cast<size_t>(t) * H)[v] = packed;
  }
}

}  // namespace afd
