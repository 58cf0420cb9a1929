// dispatch.cuh -- dispatch order, dispatched-row gather, W8A8 row quantisation and the
// device-side GEMM schedule.
//
// Dispatch sends each token's hidden state to its selected experts (A/F 分离, 机制; across
// GPUs it is an all-to-all, here a local permutation).  Order taken: expert-major, and inside
// an expert ascending token index, so every expert's rows are one contiguous block:
//   counts[e], offsets = exclusive prefix sum, pos[t,j] = offsets[e] + #{t' < t chose e}.
// Three launches: per-chunk ranks and counts (many CTAs), a scan over chunks and experts
// (one CTA), and the final positions fused with the row gather (one CTA per token).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "common.cuh"

namespace afd {

constexpr int kMaxExperts = 256;
constexpr int kChunkTokens = 128;   // tokens per CTA of dispatch_count_kernel
constexpr int kCountThreads = 256;  // 8 warps

// Dispatch order, step 1 of 3 (many CTAs).  CTA c takes the tokens [c*128, (c+1)*128) and ranks
// their (t, j) pairs per expert in flat order (flat order = token order for any one expert,
// since a token selects an expert at most once): each warp ranks a contiguous part 32 pairs at
// a time with a warp match, then the warps' counts are prefix-summed per expert.  Writes the
// rank inside the chunk to pos[t, j] (-1 for an expert outside [0, E): flagged, skipped) and
// the chunk's per-expert counts to chunk_counts[c][E].  No atomics on the data path.
__global__ void __launch_bounds__(kCountThreads)
dispatch_count_kernel(const int32_t* __restrict__ idx, int T, int k, int E, int32_t* __restrict__ pos,
                      int32_t* __restrict__ chunk_counts, int* err) {
  __shared__ int cnt[kCountThreads / 32][kMaxExperts];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int i = tid; i < (kCountThreads / 32) * kMaxExperts; i += kCountThreads) (&cnt[0][0])[i] = 0;
  __syncthreads();
  const int p0 = blockIdx.x * kChunkTokens * k;
  const int p1 = min(T, (blockIdx.x + 1) * kChunkTokens) * k;
  const int seg = (((p1 - p0) + 7) / 8 + 31) & ~31;
  const int begin = min(p1, p0 + warp * seg), end = min(p1, begin + seg);
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
      pos[i] = before + rank;
      if (rank == 0) cnt[warp][e] = before + __popc(grp);
    } else if (in) {
      pos[i] = -1;
    }
    __syncwarp();
  }
  __syncthreads();
  if (tid < E) {  // exclusive prefix over the warps, per expert; the total is the chunk's count
    int run = 0;
#pragma unroll
    for (int w = 0; w < kCountThreads / 32; ++w) {
      const int c = cnt[w][tid];
      cnt[w][tid] = run;
      run += c;
    }
    chunk_counts[static_cast<size_t>(blockIdx.x) * E + tid] = run;
  }
  __syncthreads();
  for (int b = begin; b < end; b += 32) {
    const int i = b + lane;
    if (i >= end) continue;
    const int e = idx[i];
    if (e >= 0 && e < E) pos[i] += cnt[warp][e];
  }
}

// Dispatch order, step 2 of 3 (one CTA, thread e = expert e): counts[e] = sum over chunks,
// offsets = exclusive prefix sum over experts (offsets[E] = valid pairs), and
// chunk_base[c][e] = offsets[e] + rows of expert e in the chunks before c.
__global__ void __launch_bounds__(kMaxExperts)
dispatch_scan_kernel(const int32_t* __restrict__ chunk_counts, int nchunks, int E, int32_t* __restrict__ counts,
                     int32_t* __restrict__ offsets, int32_t* __restrict__ chunk_base) {
  __shared__ int wsum[kMaxExperts / 32];
  const int e = threadIdx.x, lane = e & 31, warp = e >> 5;
  int run = 0;
  if (e < E) {
    for (int c = 0; c < nchunks; ++c) {
      const int v = chunk_counts[static_cast<size_t>(c) * E + e];
      chunk_base[static_cast<size_t>(c) * E + e] = run;
      run += v;
    }
    counts[e] = run;
  }
  const int incl = warp_incl_scan(run, lane);
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int v = lane < kMaxExperts / 32 ? wsum[lane] : 0;
    const int iv = warp_incl_scan(v, lane);
    if (lane < kMaxExperts / 32) wsum[lane] = iv - v;
  }
  __syncthreads();
  const int excl = wsum[warp] + incl - run;
  if (e < E) {
    offsets[e] = excl;
    for (int c = 0; c < nchunks; ++c) chunk_base[static_cast<size_t>(c) * E + e] += excl;
  }
  if (e == E - 1) offsets[E] = excl + run;
}

// Dispatch order, step 3 of 3, fused with the row gather (one CTA per token t): the final
// position of pair (t, j) is chunk_base[t / 128][e] + its rank inside the chunk; pos and src
// are written, and hidden row t is copied to every dispatched row and (shared expert) to row
// T*k + t.  bf16 rows move as 16-byte vectors.  W8A8: the row is quantised first --
// scale = amax / 448 (1 for a zero row), e4m3 = round-to-nearest-even, saturating, of the fp32
// quotient x / scale -- and the scale travels with every copy.  bf16 with f16_bound > 0 (the
// f16 activations of large micro-batches): the row's power-of-two act scale (f16_row_scale of
// ||x||^2) is written for every copy instead.
template <bool FP8>
__global__ void __launch_bounds__(256)
gather_rows_kernel(const __nv_bfloat16* __restrict__ hidden, const int32_t* __restrict__ idx,
                   const int32_t* __restrict__ chunk_base, int32_t* __restrict__ pos,
                   int32_t* __restrict__ src, int T, int k, int E, int H, int with_shared,
                   uint8_t* __restrict__ xp, float* __restrict__ xscale, float f16_bound = 0.f) {
  __shared__ int dst[34];  // up to 32 routed + 1 shared destinations; count in [33]
  __shared__ float red[32];
  const int t = blockIdx.x;
  const int tid = threadIdx.x;
  if (tid < 32) {
    int p = -1;
    if (tid < k) {
      const size_t ij = static_cast<size_t>(t) * k + tid;
      const int e = idx[ij];
      if (e >= 0 && e < E) {
        p = chunk_base[static_cast<size_t>(t / kChunkTokens) * E + e] + pos[ij];
        pos[ij] = p;
        src[p] = t;
      }
    }
    const unsigned m = __ballot_sync(0xffffffffu, p >= 0);
    if (p >= 0) dst[__popc(m & ((1u << tid) - 1u))] = p;
    if (tid == 0) {
      int nd = __popc(m);
      if (with_shared) dst[nd++] = T * k + t;
      dst[33] = nd;
    }
  }
  __syncthreads();
  const int nd = dst[33];
  const __nv_bfloat16* row = hidden + static_cast<size_t>(t) * H;
  const uint4* s4 = reinterpret_cast<const uint4*>(row);
  if constexpr (!FP8) {
    const bool scaled = f16_bound > 0.f && xscale != nullptr;  // uniform over the CTA
    float ss = 0.f;
    for (int v = tid; v < H / 8; v += blockDim.x) {
      const uint4 x = s4[v];
      for (int d = 0; d < nd; ++d)
        reinterpret_cast<uint4*>(xp + static_cast<size_t>(dst[d]) * H * 2)[v] = x;
      if (scaled) {
        const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&x);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = __bfloat1622float2(b[i]);
          ss = fmaf(f.x, f.x, fmaf(f.y, f.y, ss));
        }
      }
    }
    if (scaled) {
      ss = block_sum(ss, red);
      if (tid < nd) xscale[dst[tid]] = f16_row_scale(ss, f16_bound);
    }
  } else {
    float amax = 0.f;
    for (int v = tid; v < H / 8; v += blockDim.x) {
      const uint4 x = s4[v];
      const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&x);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(b[i]);
        amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
      }
    }
    amax = warp_max(amax);
    if ((tid & 31) == 0) red[tid >> 5] = amax;
    __syncthreads();
    if (tid < 32) {
      float mx = tid < (blockDim.x >> 5) ? red[tid] : 0.f;
      mx = warp_max(mx);
      if (tid == 0) red[0] = mx;
    }
    __syncthreads();
    amax = red[0];
    const float scale = amax > 0.f ? __fdiv_rn(amax, kE4m3Max) : 1.0f;
    for (int v = tid; v < H / 8; v += blockDim.x) {  // the row is L1-resident by now
      const uint4 x = s4[v];
      const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&x);
      uint32_t q[2] = {0u, 0u};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(b[i]);
        const uint32_t lo = __nv_cvt_float_to_fp8(__fdiv_rn(f.x, scale), __NV_SATFINITE, __NV_E4M3);
        const uint32_t hi = __nv_cvt_float_to_fp8(__fdiv_rn(f.y, scale), __NV_SATFINITE, __NV_E4M3);
        q[i >> 1] |= (lo | (hi << 8)) << (16 * (i & 1));
      }
      const uint2 packed = make_uint2(q[0], q[1]);
      for (int d = 0; d < nd; ++d)
        reinterpret_cast<uint2*>(xp + static_cast<size_t>(dst[d]) * H)[v] = packed;
    }
    if (tid < nd) xscale[dst[tid]] = scale;
  }
}

// W8A8: quantise each row of the fp32 SwiGLU output act32 [R][I] to e4m3 with its own scale,
// the same rule as the hidden rows.  128 threads per row, two rows per CTA of 256: each thread
// keeps up to kActRegVecs float4 of its row in registers between the amax and the quantisation
// (one pass over memory for I <= 2048; longer rows read their second pass back through the
// cache), and the small per-thread footprint lets eight CTAs share an SM, so the loads of many
// rows are in flight while others quantise.  (One warp per row with all 2048 values in its
// registers measured 0.17 ms at T=8192.)
constexpr int kActThreadsPerRow = 128;
constexpr int kActRegVecs = 4;  // float4 per thread: I <= 4 * 4 * 128 = 2048 stays in registers
__global__ void __launch_bounds__(256)
quantize_act_kernel(const float* __restrict__ act32, int R, int I, uint8_t* __restrict__ actq,
                    float* __restrict__ ascale) {
  __shared__ float wmax[8];
  const int tid = threadIdx.x, half = tid / kActThreadsPerRow, lt = tid % kActThreadsPerRow;
  const int warp = tid >> 5, lane = tid & 31;
  const size_t r = static_cast<size_t>(blockIdx.x) * 2 + half;
  const bool valid = r < static_cast<size_t>(R);
  const float4* row = reinterpret_cast<const float4*>(act32 + r * I);
  uint32_t* out = reinterpret_cast<uint32_t*>(actq + r * I);
  const int nv = I / 4;  // float4 per row
  const bool in_regs = nv <= kActRegVecs * kActThreadsPerRow;
  auto quant4 = [](const float4 x, float scale) {
    const float xv[4] = {x.x, x.y, x.z, x.w};
    uint32_t packed = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      packed |= static_cast<uint32_t>(__nv_cvt_float_to_fp8(__fdiv_rn(xv[i], scale), __NV_SATFINITE, __NV_E4M3))
                << (8 * i);
    return packed;
  };
  auto amax4 = [](const float4 x) { return fmaxf(fmaxf(fabsf(x.x), fabsf(x.y)), fmaxf(fabsf(x.z), fabsf(x.w))); };
  float4 x[kActRegVecs];
  float amax = 0.f;
  if (valid) {
    if (in_regs) {
#pragma unroll
      for (int i = 0; i < kActRegVecs; ++i) {
        const int v = lt + kActThreadsPerRow * i;
        if (v < nv) {
          x[i] = row[v];
          amax = fmaxf(amax, amax4(x[i]));
        }
      }
    } else {
      for (int v = lt; v < nv; v += kActThreadsPerRow) amax = fmaxf(amax, amax4(row[v]));
    }
  }
  amax = warp_max(amax);
  if (lane == 0) wmax[warp] = amax;
  __syncthreads();
  const float* wm = wmax + 4 * half;  // the row's four warps
  amax = fmaxf(fmaxf(wm[0], wm[1]), fmaxf(wm[2], wm[3]));
  if (!valid) return;
  const float scale = amax > 0.f ? __fdiv_rn(amax, kE4m3Max) : 1.0f;
  if (in_regs) {
#pragma unroll
    for (int i = 0; i < kActRegVecs; ++i) {
      const int v = lt + kActThreadsPerRow * i;
      if (v < nv) out[v] = quant4(x[i], scale);
    }
  } else {
    for (int v = lt; v < nv; v += kActThreadsPerRow) out[v] = quant4(row[v], scale);
  }
  if (lt == 0) ascale[r] = scale;
}

// GEMM schedule from the group offsets: group g < E is expert g (rows offsets[g]..offsets[g+1]),
// group E is the shared expert (rows T*k .. T*k + T).  Each group contributes
// ceil(rows / bn1) * mt1 tile units to the gate/up GEMM and ceil(rows / bn2) * mt2 to the
// down GEMM; unit bases are exclusive prefix sums.  One CTA of 512 threads (G <= 257).
// Also: tile_base[g] = first N tile (of bn1 rows) of group g, and the per-tile counters of the
// fused kernel's act dependencies are zeroed.
__global__ void __launch_bounds__(512)
build_schedule_kernel(const int32_t* __restrict__ offsets, int E, int n_shared, int T, int k, int bn1, int bn2,
                      int mt1, int mt2, int32_t* __restrict__ grp_rows, int32_t* __restrict__ grp_base,
                      int32_t* __restrict__ ub1, int32_t* __restrict__ ub2, int32_t* __restrict__ tile_base,
                      int* __restrict__ tile_done, int* err) {
  __shared__ int wsum1[16], wsum2[16], wsum3[16];
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
  const int nt = (rows + bn1 - 1) / bn1;
  const int u1 = nt * mt1, u2 = (rows + bn2 - 1) / bn2 * mt2;
  const int i1 = warp_incl_scan(u1, lane), i2 = warp_incl_scan(u2, lane), i3 = warp_incl_scan(nt, lane);
  if (lane == 31) { wsum1[warp] = i1; wsum2[warp] = i2; wsum3[warp] = i3; }
  __syncthreads();
  if (warp == 0) {
    const int a = lane < 16 ? wsum1[lane] : 0, b = lane < 16 ? wsum2[lane] : 0, c = lane < 16 ? wsum3[lane] : 0;
    const int ia = warp_incl_scan(a, lane), ib = warp_incl_scan(b, lane), ic = warp_incl_scan(c, lane);
    if (lane < 16) { wsum1[lane] = ia - a; wsum2[lane] = ib - b; wsum3[lane] = ic - c; }
  }
  __syncthreads();
  const int e1 = wsum1[warp] + i1 - u1, e2 = wsum2[warp] + i2 - u2, e3 = wsum3[warp] + i3 - nt;
  if (g < G) {
    grp_rows[g] = rows;
    grp_base[g] = rbase;
    ub1[g] = e1;
    ub2[g] = e2;
    tile_base[g] = e3;
    for (int i = 0; i < nt; ++i) tile_done[e3 + i] = 0;
  }
  if (g == G - 1) {
    ub1[G] = e1 + u1;
    ub2[G] = e2 + u2;
  }
}

}  // namespace afd
