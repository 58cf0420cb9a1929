// dispatch.cuh -- dispatch order, dispatched-row gather, W8A8 row quantisation and the
// device-side GEMM schedule.
//
// Dispatch sends each token's hidden state to its selected experts (A/F 分离, 机制; across
// GPUs it is an all-to-all, here a local permutation).  Order taken: expert-major, and inside
// an expert ascending token index, so every expert's rows are one contiguous block:
//   counts[e], offsets = exclusive prefix sum, pos[t,j] = offsets[e] + #{t' < t chose e}.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "common.cuh"

namespace afd {

constexpr int kDispatchThreads = 1024;
constexpr int kMaxExperts = 256;

// One CTA of 1024 threads.  Each warp takes one contiguous segment of the flat (t, j) array
// (flat order = token order for any one expert, since a token selects an expert at most once),
// ranks its pairs per expert 32 at a time with a warp match (stable inside the segment) and
// counts them per expert; the per-warp counts are then prefix-summed across warps and experts
// and a second pass turns local ranks into global positions.  No atomics on the data path.
__global__ void __launch_bounds__(kDispatchThreads)
dispatch_order_kernel(const int32_t* __restrict__ idx, int T, int k, int E,
                      int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                      int32_t* __restrict__ pos, int32_t* __restrict__ src, int* err) {
  __shared__ int cnt[32][kMaxExperts];
  __shared__ int ebase[kMaxExperts];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int i = tid; i < 32 * kMaxExperts; i += kDispatchThreads) (&cnt[0][0])[i] = 0;
  __syncthreads();

  const int n = T * k;
  const int seg = ((n + 31) / 32 + 31) & ~31;
  const int begin = min(n, warp * seg), end = min(n, begin + seg);
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int b = begin; b < end; b += 32) {
    const int i = b + lane;
    const bool in = i < end;
    const int e = in ? idx[i] : -1;
    const bool valid = in && e >= 0 && e < E;
    if (in && !valid) atomicOr(err, kErrBadExpert);
    const int key = valid ? e : -1 - lane;  // invalid lanes stay alone
    const unsigned grp = __match_any_sync(0xffffffffu, key);
    const int rank = __popc(grp & lt_mask);
    const int before = valid ? cnt[warp][e] : 0;
    __syncwarp();
    if (valid) {
      pos[i] = before + rank;                       // local rank, finished below
      if (rank == 0) cnt[warp][e] = before + __popc(grp);
    } else if (in) {
      pos[i] = -1;
    }
    __syncwarp();
  }
  __syncthreads();
  if (tid < E) {  // exclusive prefix over warps, per expert
    int run = 0;
    for (int w = 0; w < 32; ++w) {
      const int c = cnt[w][tid];
      cnt[w][tid] = run;
      run += c;
    }
    ebase[tid] = run;
    counts[tid] = run;
  }
  __syncthreads();
  if (warp == 0) {  // exclusive prefix over experts, 8 per lane
    int v[8], s = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane * 8 + i;
      v[i] = e < E ? ebase[e] : 0;
      s += v[i];
    }
    const int incl = warp_incl_scan(s, lane);
    int run = incl - s;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane * 8 + i;
      if (e < E) { ebase[e] = run; offsets[e] = run; }
      run += v[i];
    }
    if (lane == 31) offsets[E] = incl;
  }
  __syncthreads();
  for (int b = begin; b < end; b += 32) {
    const int i = b + lane;
    if (i >= end) continue;
    const int e = idx[i];
    if (e < 0 || e >= E) continue;
    const int p = ebase[e] + cnt[warp][e] + pos[i];
    pos[i] = p;
    src[p] = i / k;
  }
}

// Row gather: dispatched row pos[t,j] <- hidden row t, and (shared expert) row shared_base + t
// <- hidden row t.  bf16 rows are copied with 16-byte vectors.  W8A8: the row is quantised
// first -- scale = amax / 448 (1 for a zero row), e4m3 = round-to-nearest-even, saturating,
// of the fp32 quotient x / scale -- and the scale travels with every copy.
template <bool FP8>
__global__ void __launch_bounds__(256)
gather_rows_kernel(const __nv_bfloat16* __restrict__ hidden, const int32_t* __restrict__ pos,
                   int T, int k, int H, int shared_base, int with_shared, int n_rows,
                   uint8_t* __restrict__ xp, float* __restrict__ xscale, int* err) {
  __shared__ int dst[34];  // up to 32 routed + 1 shared destinations; count in [33]
  __shared__ float red[8];
  const int t = blockIdx.x;
  const int tid = threadIdx.x;
  if (tid == 0) {
    int nd = 0;
    for (int j = 0; j < k; ++j) {
      const int p = pos[static_cast<size_t>(t) * k + j];
      if (p < 0) continue;
      if (p >= n_rows) { atomicOr(err, kErrBadPos); continue; }
      dst[nd++] = p;
    }
    if (with_shared) dst[nd++] = shared_base + t;
    dst[33] = nd;
  }
  __syncthreads();
  const int nd = dst[33];
  const __nv_bfloat16* row = hidden + static_cast<size_t>(t) * H;
  if constexpr (!FP8) {
    const uint4* s4 = reinterpret_cast<const uint4*>(row);
    for (int v = tid; v < H / 8; v += blockDim.x) {
      const uint4 x = s4[v];
      for (int d = 0; d < nd; ++d)
        reinterpret_cast<uint4*>(xp + static_cast<size_t>(dst[d]) * H * 2)[v] = x;
    }
  } else {
    float amax = 0.f;
    for (int i = tid; i < H; i += blockDim.x) amax = fmaxf(amax, fabsf(__bfloat162float(row[i])));
    amax = warp_max(amax);
    if ((tid & 31) == 0) red[tid >> 5] = amax;
    __syncthreads();
    if (tid < 32) {
      float m = tid < (blockDim.x >> 5) ? red[tid] : 0.f;
      m = warp_max(m);
      if (tid == 0) red[0] = m;
    }
    __syncthreads();
    amax = red[0];
    const float scale = amax > 0.f ? __fdiv_rn(amax, kE4m3Max) : 1.0f;
    for (int v = tid; v < H / 4; v += blockDim.x) {
      uint32_t packed = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float x = __fdiv_rn(__bfloat162float(row[v * 4 + i]), scale);
        packed |= static_cast<uint32_t>(__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3)) << (8 * i);
      }
      for (int d = 0; d < nd; ++d)
        reinterpret_cast<uint32_t*>(xp + static_cast<size_t>(dst[d]) * H)[v] = packed;
    }
    if (tid < nd) xscale[dst[tid]] = scale;
  }
}

// W8A8: quantise each row of the fp32 SwiGLU output act32 [R][I] to e4m3 with its own
// scale, the same rule as the hidden rows.  One CTA per row.
__global__ void __launch_bounds__(256)
quantize_act_kernel(const float* __restrict__ act32, int I, uint8_t* __restrict__ actq,
                    float* __restrict__ ascale) {
  __shared__ float red[8];
  const size_t r = blockIdx.x;
  const float* row = act32 + r * I;
  const int tid = threadIdx.x;
  float amax = 0.f;
  for (int i = tid; i < I; i += blockDim.x) amax = fmaxf(amax, fabsf(row[i]));
  amax = warp_max(amax);
  if ((tid & 31) == 0) red[tid >> 5] = amax;
  __syncthreads();
  if (tid < 32) {
    float m = tid < (blockDim.x >> 5) ? red[tid] : 0.f;
    m = warp_max(m);
    if (tid == 0) red[0] = m;
  }
  __syncthreads();
  amax = red[0];
  const float scale = amax > 0.f ? __fdiv_rn(amax, kE4m3Max) : 1.0f;
  for (int v = tid; v < I / 4; v += blockDim.x) {
    const float4 x = reinterpret_cast<const float4*>(row)[v];
    const float xv[4] = {x.x, x.y, x.z, x.w};
    uint32_t packed = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      packed |= static_cast<uint32_t>(__nv_cvt_float_to_fp8(__fdiv_rn(xv[i], scale), __NV_SATFINITE, __NV_E4M3))
                << (8 * i);
    reinterpret_cast<uint32_t*>(actq + r * I)[v] = packed;
  }
  if (tid == 0) ascale[r] = scale;
}

// GEMM schedule from the group offsets: group g < E is expert g (rows offsets[g]..offsets[g+1]),
// group E is the shared expert (rows T*k .. T*k + T).  Each group contributes
// ceil(rows / bn1) * mt1 tile units to the gate/up GEMM and ceil(rows / bn2) * mt2 to the
// down GEMM; unit bases are exclusive prefix sums.  One CTA of 512 threads (G <= 257).
__global__ void __launch_bounds__(512)
build_schedule_kernel(const int32_t* __restrict__ offsets, int E, int n_shared, int T, int k, int bn1, int bn2,
                      int mt1, int mt2, int32_t* __restrict__ grp_rows, int32_t* __restrict__ grp_base,
                      int32_t* __restrict__ ub1, int32_t* __restrict__ ub2, int* err) {
  __shared__ int wsum1[16], wsum2[16];
  const int g = threadIdx.x, lane = g & 31, warp = g >> 5;
  const int G = E + n_shared;
  int rows = 0, rbase = 0;
  if (g < E) {
    const int a = offsets[g], b = offsets[g + 1];
    if (a < 0 || b < a || b > T * k || (g == 0 && a != 0)) {
      atomicOr(err, kErrBadOffsets);
    } else {
      rows = b - a;
      rbase = a;
    }
  } else if (g < G) {
    rows = T;
    rbase = T * k;  // shared-expert rows follow the routed rows
  }
  const int u1 = (rows + bn1 - 1) / bn1 * mt1, u2 = (rows + bn2 - 1) / bn2 * mt2;
  const int i1 = warp_incl_scan(u1, lane), i2 = warp_incl_scan(u2, lane);
  if (lane == 31) { wsum1[warp] = i1; wsum2[warp] = i2; }
  __syncthreads();
  if (warp == 0) {
    const int a = lane < 16 ? wsum1[lane] : 0, b = lane < 16 ? wsum2[lane] : 0;
    const int ia = warp_incl_scan(a, lane), ib = warp_incl_scan(b, lane);
    if (lane < 16) { wsum1[lane] = ia - a; wsum2[lane] = ib - b; }
  }
  __syncthreads();
  const int e1 = wsum1[warp] + i1 - u1, e2 = wsum2[warp] + i2 - u2;
  if (g < G) {
    grp_rows[g] = rows;
    grp_base[g] = rbase;
    ub1[g] = e1;
    ub2[g] = e2;
  }
  if (g == G - 1) {
    ub1[G] = e1 + u1;
    ub2[G] = e2 + u2;
  }
}

}  // namespace afd
