// router.cuh -- router logits, top-k selection and gate weights.
//
// The FFN path is dominated by the routing computation and the exchange of hidden states
// (vLLM AFD Plugin, Attention-FFN 解耦的原理); the router picks a few of the layer's many
// experts per token (LLM 推理提速: Attention与FFN分离AFD方, 一个在啃带宽，一个在吃算力).
// Reading taken: l = hidden . Wr^T (+ bias) in fp32, the k largest logits in descending
// order (ties to the lower expert), w = softmax over the selected logits.
//
// The handle's router (afd_ffn_route / afd_ffn_forward) is MODE 2 of the grouped GEMM in
// gemm.cuh (tensor cores, Wr as three bf16 planes whose sum represents it to ~2^-27, split-K
// partial logits over stretches of at most 1024 elements of H) followed by router_topk_kernel,
// which adds the partials in split order in fp32 and selects and normalises from those logits.
// The allocation-free afd_ffn_route_static uses router_logits_kernel (fp32 FMA GEMM, 64 tokens
// x 64 experts per CTA, 4x4 outputs per thread, K tiles of 32 in shared memory, optionally split
// over K) and router_topk_kernel (one warp per token; 8 logits per lane, k rounds of warp
// arg-max, a warp sum normalises the weights).
#pragma once

#include <cuda_bf16.h>

#include "common.cuh"

namespace afd {

constexpr int kRtTok = 64, kRtExp = 64, kRtK = 32;

__global__ void __launch_bounds__(256)
router_logits_kernel(const __nv_bfloat16* __restrict__ hidden, const float* __restrict__ wr,
                     float* __restrict__ part, int T, int H, int E, int ktiles_per_split) {
  __shared__ float xs[kRtK][kRtTok + 4];
  __shared__ float ws[kRtK][kRtExp + 4];
  const int t0 = blockIdx.y * kRtTok;
  const int e0 = blockIdx.x * kRtExp;
  const int kt0 = blockIdx.z * ktiles_per_split;
  const int kt1 = min(H / kRtK, kt0 + ktiles_per_split);
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int lr = threadIdx.x >> 2, lc = (threadIdx.x & 3) * 8;

  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

  for (int kt = kt0; kt < kt1; ++kt) {
    const int kb = kt * kRtK;
    {  // 64 tokens x 32 hidden values, one 16-byte load per thread
      const int t = t0 + lr;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (t < T) v = *reinterpret_cast<const uint4*>(hidden + static_cast<size_t>(t) * H + kb + lc);
      const __nv_bfloat16* hv = reinterpret_cast<const __nv_bfloat16*>(&v);
#pragma unroll
      for (int i = 0; i < 8; ++i) xs[lc + i][lr] = __bfloat162float(hv[i]);
    }
    {  // 64 experts x 32 hidden values of the fp32 router, two 16-byte loads per thread
      const int e = e0 + lr;
      float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
      if (e < E) {
        const float4* p = reinterpret_cast<const float4*>(wr + static_cast<size_t>(e) * H + kb + lc);
        a = p[0];
        b = p[1];
      }
      ws[lc + 0][lr] = a.x; ws[lc + 1][lr] = a.y; ws[lc + 2][lr] = a.z; ws[lc + 3][lr] = a.w;
      ws[lc + 4][lr] = b.x; ws[lc + 5][lr] = b.y; ws[lc + 6][lr] = b.z; ws[lc + 7][lr] = b.w;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < kRtK; ++kk) {
      const float4 a = *reinterpret_cast<const float4*>(&xs[kk][ty * 4]);
      const float4 b = *reinterpret_cast<const float4*>(&ws[kk][tx * 4]);
      const float av[4] = {a.x, a.y, a.z, a.w};
      const float bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int t = t0 + ty * 4 + i;
    if (t >= T) continue;
    float* dst = part + (static_cast<size_t>(blockIdx.z) * T + t) * E;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e = e0 + tx * 4 + j;
      if (e < E) dst[e] = acc[i][j];
    }
  }
}

// WPT warps per token (one, or four when the partial logits come in many splits: a small
// micro-batch's router GEMM splits H widely to fill the SMs).  part: [nsplit][T][E] partial
// logits; warp g of a token adds splits g*per .. (g+1)*per - 1 in order, then warp 0 adds the
// WPT sums in order (a fixed order, independent of scheduling); bias: [E] or nullptr.  Writes
// the k selected experts (descending logit, ties to the lower index) and the softmax of their
// logits.  blockDim = 256: 8 / WPT tokens per CTA.
template <int WPT>
__global__ void __launch_bounds__(256)
router_topk_kernel(const float* __restrict__ part, int nsplit, const float* __restrict__ bias,
                   int T, int E, int k, int32_t* __restrict__ idx, float* __restrict__ w) {
  __shared__ float red[WPT > 1 ? 8 * 8 * 32 : 1];  // [token in CTA][warp of the token][i][lane]
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int tl = warp / WPT, g = warp % WPT;
  const int t = blockIdx.x * (8 / WPT) + tl;
  float v[8];
  unsigned taken = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = 0.f;
  if (t < T) {
    // WPT = 4 (small micro-batches): the loads of four splits (eight values each) are issued
    // together, then added in split order, so a lane waits for one memory round trip per four
    // splits (T=256: 14.5 -> 12.4 us).  WPT = 1 takes one split per round trip: with many tokens
    // the warps overlap each other, and the batched form measured slower there (its registers
    // cost occupancy).
    const int per = (nsplit + WPT - 1) / WPT;
    const int s1 = min(nsplit, (g + 1) * per);
    constexpr int kB = WPT > 1 ? 4 : 1;  // splits per round trip
    for (int sp0 = g * per; sp0 < s1; sp0 += kB) {
      float pv[kB][8];
#pragma unroll
      for (int d = 0; d < kB; ++d) {
        const int sp = sp0 + d;
        const float* ps = part + (static_cast<size_t>(sp) * T + t) * E;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int e = lane + 32 * i;
          pv[d][i] = (sp < s1 && e < E) ? ps[e] : 0.f;
        }
      }
#pragma unroll
      for (int d = 0; d < kB; ++d) {
        if (sp0 + d < s1) {
#pragma unroll
          for (int i = 0; i < 8; ++i) v[i] += pv[d][i];
        }
      }
    }
  }
  if constexpr (WPT > 1) {
#pragma unroll
    for (int i = 0; i < 8; ++i) red[((tl * WPT + g) * 8 + i) * 32 + lane] = v[i];
    __syncthreads();
    if (g != 0) return;
    for (int gg = 1; gg < WPT; ++gg) {
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] += red[((tl * WPT + gg) * 8 + i) * 32 + lane];
    }
  }
  if (t >= T) return;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int e = lane + 32 * i;
    if (e < E) {
      if (bias) v[i] += bias[e];
    } else {
      v[i] = -INFINITY;
    }
  }
  int my_e = -1;
  float my_v = -INFINITY;
  for (int j = 0; j < k; ++j) {
    float bv = -INFINITY;
    int be = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < 8; ++i) {  // expert index grows with i: the first best is the lowest
      const int e = lane + 32 * i;
      if (e < E && !(taken >> i & 1u) && (v[i] > bv || (be == 0x7fffffff && v[i] == bv))) {
        bv = v[i];
        be = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oe = __shfl_xor_sync(0xffffffffu, be, o);
      if (ov > bv || (ov == bv && oe < be)) { bv = ov; be = oe; }
    }
    if (be != 0x7fffffff && (be & 31) == lane) taken |= 1u << (be >> 5);
    if (lane == j) { my_e = (be == 0x7fffffff) ? -1 : be; my_v = bv; }
  }
  const float vmax = __shfl_sync(0xffffffffu, my_v, 0);
  const float z = (lane < k) ? expf(my_v - vmax) : 0.f;
  const float sum = warp_sum(z);
  if (lane < k) {
    idx[static_cast<size_t>(t) * k + lane] = my_e;
    w[static_cast<size_t>(t) * k + lane] = z / sum;
  }
}

// Selection and gate weights from nsplit partial logits: four warps per token when the partials
// come in eight or more splits (a small micro-batch), else one.
inline void launch_router_topk(const float* part, int nsplit, const float* bias, int T, int E, int k, int32_t* idx,
                               float* w, cudaStream_t s) {
  if (nsplit >= 8)
    router_topk_kernel<4><<<(T + 1) / 2, 256, 0, s>>>(part, nsplit, bias, T, E, k, idx, w);
  else
    router_topk_kernel<1><<<(T + 7) / 8, 256, 0, s>>>(part, nsplit, bias, T, E, k, idx, w);
}

// Router weights for the tensor-core router: Wr (fp32) -> three bf16 planes [3][n] with
// hi = bf16(Wr), mid = bf16(Wr - hi), lo = bf16(Wr - hi - mid).  Both subtractions are exact in
// fp32 (each plane holds the leading bits of what is left), so Wr = hi + mid + lo to ~2^-27.
__global__ void router_split_planes_kernel(const float* __restrict__ wr, size_t n,
                                           __nv_bfloat16* __restrict__ planes) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const float w = wr[i];
    const __nv_bfloat16 hi = __float2bfloat16_rn(w);
    const float r1 = w - __bfloat162float(hi);
    const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
    const float r2 = r1 - __bfloat162float(mid);
    planes[i] = hi;
    planes[n + i] = mid;
    planes[2 * n + i] = __float2bfloat16_rn(r2);
  }
}

}  // namespace afd
