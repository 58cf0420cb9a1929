// combine.cuh -- weighted combine of the expert outputs back into token order.
//
// Combine returns the experts' outputs to their tokens (A/F 分离, 机制; an all-to-all
// across GPUs, a gather here).  Reading taken: out[t] = sum_j w[t,j] * Y[pos[t,j]] + Ys[t],
// summed in fp32 in j order with the shared expert last, rounded once to bf16.  No atomics:
// one CTA per token, so the result does not depend on scheduling.  Y is fp32 on the bf16 path
// and bf16 on the W8A8 path (its 6e-2 error budget leaves room; it halves the bytes read).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>

#include "common.cuh"

namespace afd {

__device__ __forceinline__ float4 load4(const float* p, size_t i) { return reinterpret_cast<const float4*>(p)[i]; }
__device__ __forceinline__ float4 load4(const __nv_bfloat16* p, size_t i) {
  const uint2 u = reinterpret_cast<const uint2*>(p)[i];
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
  return make_float4(a.x, a.y, b.x, b.y);
}

// Ys: the shared expert's rows [T][H], or nullptr when they follow the routed rows in Y.
// Grid: (T, slices); the slices of a token split its H.
inline int combine_slices(int T, int H) {
  const int vec_per_cta = 256;                     // one float4 per thread per pass
  const int most = (H / 4 + vec_per_cta - 1) / vec_per_cta;
  // (eight slices at T=256 measured slower than four: 16.7 vs 15.6 us)
  return T >= 1024 ? 1 : (T >= 512 ? std::min(2, most) : std::min(4, most));
}
template <typename YT>
__global__ void __launch_bounds__(256)
combine_kernel(const YT* __restrict__ Y, const YT* __restrict__ Ys, const float* __restrict__ w,
               const int32_t* __restrict__ pos, int T, int k, int H, int n_rows, int with_shared,
               __nv_bfloat16* __restrict__ out, int* err) {
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
  const YT* ys = Ys ? Ys + static_cast<size_t>(t) * H : Y + (static_cast<size_t>(T) * k + t) * H;  // shared-expert row
  // gridDim.y CTAs share the token's row (small micro-batches: more loads in flight); every
  // element is still summed by one thread in j order, so the result does not depend on it
  for (int v = blockIdx.y * blockDim.x + threadIdx.x; v < H / 4; v += gridDim.y * blockDim.x) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if constexpr (sizeof(YT) == 4) {
      // fp32 rows: four rows' loads in flight at once, accumulated in j order (measured 15 %
      // faster at T=256; the bf16 rows of the W8A8 path run faster with the plain loop)
      for (int j0 = 0; j0 < k; j0 += 4) {
        float4 y[4];
#pragma unroll
        for (int d = 0; d < 4; ++d) {
          const int j = j0 + d;
          const int p = j < k ? sp[j] : -1;
          y[d] = p >= 0 ? load4(Y + static_cast<size_t>(p) * H, v) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int d = 0; d < 4; ++d) {
          const int j = j0 + d;
          if (j >= k || sp[j] < 0) continue;
          const float wj = sw[j];
          acc.x = fmaf(wj, y[d].x, acc.x);
          acc.y = fmaf(wj, y[d].y, acc.y);
          acc.z = fmaf(wj, y[d].z, acc.z);
          acc.w = fmaf(wj, y[d].w, acc.w);
        }
      }
    } else {
      for (int j = 0; j < k; ++j) {
        const int p = sp[j];
        if (p < 0) continue;
        const float wj = sw[j];
        const float4 y = load4(Y + static_cast<size_t>(p) * H, v);
        acc.x = fmaf(wj, y.x, acc.x);
        acc.y = fmaf(wj, y.y, acc.y);
        acc.z = fmaf(wj, y.z, acc.z);
        acc.w = fmaf(wj, y.w, acc.w);
      }
    }
    if (with_shared) {
      const float4 s = load4(ys, v);
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

// The same combine for bf16 expert rows with H a multiple of 8: eight columns per thread
// (16-byte loads), the loads of up to eight rows in flight before they are summed in j order,
// so the sums are those of combine_kernel<__nv_bfloat16> bit for bit.
constexpr int kCombine8Threads = 128;
inline int combine8_slices(int T, int H) {
  const int most = (H / 8 + kCombine8Threads - 1) / kCombine8Threads;
  return T >= 1024 ? 1 : (T >= 512 ? std::min(2, most) : std::min(4, most));
}
__global__ void __launch_bounds__(kCombine8Threads)
combine8_kernel(const __nv_bfloat16* __restrict__ Y, const __nv_bfloat16* __restrict__ Ys, const float* __restrict__ w,
                const int32_t* __restrict__ pos, int T, int k, int H, int n_rows, int with_shared,
                __nv_bfloat16* __restrict__ out, int* err) {
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
  const __nv_bfloat16* ys = Ys ? Ys + static_cast<size_t>(t) * H : Y + (static_cast<size_t>(T) * k + t) * H;
  for (int v = blockIdx.y * blockDim.x + threadIdx.x; v < H / 8; v += gridDim.y * blockDim.x) {
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    for (int j0 = 0; j0 < k; j0 += 8) {
      uint4 y[8];
#pragma unroll
      for (int d = 0; d < 8; ++d) {
        const int j = j0 + d;
        const int p = j < k ? sp[j] : -1;
        y[d] = p >= 0 ? reinterpret_cast<const uint4*>(Y + static_cast<size_t>(p) * H)[v] : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int d = 0; d < 8; ++d) {
        const int j = j0 + d;
        if (j >= k || sp[j] < 0) continue;
        const float wj = sw[j];
        const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&y[d]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(b[e]);
          acc[2 * e] = fmaf(wj, f.x, acc[2 * e]);
          acc[2 * e + 1] = fmaf(wj, f.y, acc[2 * e + 1]);
        }
      }
    }
    if (with_shared) {
      const uint4 u = reinterpret_cast<const uint4*>(ys)[v];
      const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(b[e]);
        acc[2 * e] += f.x;
        acc[2 * e + 1] += f.y;
      }
    }
    uint4 packed;
    uint32_t* pk = reinterpret_cast<uint32_t*>(&packed);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      __nv_bfloat162 q = __floats2bfloat162_rn(acc[2 * e], acc[2 * e + 1]);
      pk[e] = *reinterpret_cast<uint32_t*>(&q);
    }
    reinterpret_cast<uint4*>(out + static_cast<size_t>(t) * H)[v] = packed;
  }
}

// Copy blocks of rows: block b moves blocks[3b+2] rows of row_bytes from row blocks[3b] of src
// to row blocks[3b+1] of dst.  blockIdx.x = block, blockIdx.y splits its rows; moves of V
// (16 bytes, or 4 for rows that are not a multiple of 16 bytes, such as per-row scales).
template <typename V>
__global__ void __launch_bounds__(256)
copy_row_blocks_kernel(const V* __restrict__ src, V* __restrict__ dst, const int32_t* __restrict__ blocks,
                       int row_vecs) {
  const int b = blockIdx.x;
  const size_t s0 = static_cast<size_t>(blocks[3 * b]), d0 = static_cast<size_t>(blocks[3 * b + 1]);
  const int rows = blocks[3 * b + 2];
  for (int r = blockIdx.y; r < rows; r += gridDim.y) {
    const V* sr = src + (s0 + r) * row_vecs;
    V* dr = dst + (d0 + r) * row_vecs;
    for (int v = threadIdx.x; v < row_vecs; v += blockDim.x) dr[v] = sr[v];
  }
}

// f16 copy of bf16 weights (the down projection of large bf16 micro-batches).  Every bf16 value
// of magnitude in [2^-14, 65504] is exact in f16; smaller ones become f16 subnormals (absolute
// error <= 2^-25); a magnitude above 65504 sets *overflow and the handle keeps the bf16 path.
__global__ void bf16_to_f16_kernel(const __nv_bfloat16* __restrict__ src, __half* __restrict__ dst, size_t n,
                                   int* overflow) {
  bool big = false;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const float f = __bfloat162float(src[i]);
    big |= !(fabsf(f) <= 65504.0f);  // also catches NaN
    dst[i] = __float2half_rn(f);
  }
  if (big) atomicOr(overflow, 1);
}

// Weight side of the f16 row scale: for every expert g and intermediate column i,
// |silu(x.wg_i) (x.wu_i)| <= |x.wg_i| |x.wu_i| <= ||x||^2 ||wg_i|| ||wu_i||  (|silu(z)| <= |z|;
// Cauchy-Schwarz), so C = max over g, i of ||wg_i|| ||wu_i|| bounds every act value of a token
// row by ||x||^2 C.  Warps stride over the (g, i) pairs of w13 [G][2I][H] bf16; *c_bits receives
// C as the bits of a non-negative float (atomicMax on the bits orders non-negative floats).
__global__ void __launch_bounds__(256)
w13_norm_bound_kernel(const __nv_bfloat16* __restrict__ w13, int G, int I, int H, unsigned* c_bits) {
  const int lane = threadIdx.x & 31;
  const long long nwarps = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  float c = 0.f;
  for (long long p = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
       p < static_cast<long long>(G) * I; p += nwarps) {
    const long long g = p / I, i = p - g * I;
    const uint4* rg = reinterpret_cast<const uint4*>(w13 + (g * 2 * I + i) * H);
    const uint4* ru = reinterpret_cast<const uint4*>(w13 + (g * 2 * I + I + i) * H);
    float sg = 0.f, su = 0.f;
    for (int v = lane; v < H / 8; v += 32) {
      const uint4 a = rg[v], b = ru[v];
      const __nv_bfloat162* pa = reinterpret_cast<const __nv_bfloat162*>(&a);
      const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 fa = __bfloat1622float2(pa[j]), fb = __bfloat1622float2(pb[j]);
        sg = fmaf(fa.x, fa.x, fmaf(fa.y, fa.y, sg));
        su = fmaf(fb.x, fb.x, fmaf(fb.y, fb.y, su));
      }
    }
    sg = warp_sum(sg);
    su = warp_sum(su);
    c = fmaxf(c, sqrtf(sg) * sqrtf(su));
  }
  if (lane == 0) atomicMax(c_bits, __float_as_uint(c));
}

// f16 row scales of rows that arrive already dispatched (one CTA of 256 threads per row).
__global__ void __launch_bounds__(256)
f16_row_scale_kernel(const __nv_bfloat16* __restrict__ rows, int H, float f16_bound, float* __restrict__ xscale) {
  __shared__ float red[32];
  const uint4* r4 = reinterpret_cast<const uint4*>(rows + static_cast<size_t>(blockIdx.x) * H);
  float ss = 0.f;
  for (int v = threadIdx.x; v < H / 8; v += blockDim.x) {
    const uint4 x = r4[v];
    const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&x);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __bfloat1622float2(b[j]);
      ss = fmaf(f.x, f.x, fmaf(f.y, f.y, ss));
    }
  }
  ss = block_sum(ss, red);
  if (threadIdx.x == 0) xscale[blockIdx.x] = f16_row_scale(ss, f16_bound);
}

// Widen bf16 rows to fp32 (copy-out of the W8A8 expert outputs by afd_ffn_expert_gemm).
__global__ void bf16_to_f32_kernel(const __nv_bfloat16* __restrict__ src, float* __restrict__ dst, size_t n) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x)
    dst[i] = __bfloat162float(src[i]);
}

}  // namespace afd
