// gemm.cuh -- grouped expert GEMMs on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// One persistent kernel serves both expert projections of the layer (each expert is a large
// matrix product: A/F 分离, section 为什么要拆):
//   MODE 0 (gate/up):  for expert g and its token rows X_g:  act = silu(X_g Wg^T) * (X_g Wu^T)
//   MODE 1 (down):     Y_g = act_g W2^T
// "Swap-AB" form: the weight rows fill the 128-row M side of each MMA and the expert's token
// rows are the N side (16..BN rows, rounded up to 16), so a decode micro-batch with ~8 rows
// per expert still streams full 128-row weight tiles.  Every work unit is one pair of
// 128-row weight tiles (gate rows j.., up rows I+j.. for MODE 0; down rows h.., h+128.. for
// MODE 1) against one tile of up to BN token rows, accumulated over the whole K dimension
// into two fp32 TMEM accumulators; the SwiGLU (MODE 0) and the scales of the W8A8 path are
// applied in the epilogue straight from TMEM.
//
// bf16 path, two-term activations: the gate/up epilogue stores the fp32 SwiGLU output as
// hi = bf16(act) and lo = bf16(act - hi) in two planes, and the down GEMM (SPLIT_B) multiplies
// each weight tile by both and accumulates into one TMEM accumulator, so the activation enters
// the down projection with ~2^-17 relative error instead of bf16's 2^-9 (the two-term bfloat16
// split of Henry, Tang and Heinecke, "Leveraging the bfloat16 AI datatype for higher-precision
// computations", 2019).  The only bf16 rounding left on the output path is the layer output.
//
// Warp roles (192 threads): warp 0 lane 0 issues TMA loads into a STAGES-deep shared-memory
// ring; warp 1 owns the TMEM allocation and its lane 0 issues tcgen05.mma; warps 2..5 are
// the epilogue (warp w reads TMEM lanes 32*(w%4)..+31).  Units are assigned round-robin over
// the persistent grid from a per-group schedule built on the device, so the host never needs
// the per-expert row counts.  Every wait is bounded (ptx.cuh: mbar_wait); a CTA that gives
// up records AFD timeout in the error word, drains its own copies and MMAs, frees TMEM and
// returns.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "ptx.cuh"

namespace afd {

struct GemmArgs {
  const int32_t* grp_rows;   // [G]   token rows of each group (expert)
  const int32_t* grp_base;   // [G]   first dispatched row of each group
  const int32_t* unit_base;  // [G+1] first unit of each group; unit_base[G] = total units
  int G;                     // groups: routed experts, then the shared expert
  int K;                     // reduction length in elements (H for gate/up, I for down)
  int a_rows;                // weight rows per group (2I for gate/up, H for down)
  int mt_stride;             // weight rows between consecutive tile pairs (128 / 256)
  int second_off;            // row offset of a pair's second tile (I / 128)
  void* out;                 // MODE 0: act (bf16, or fp32 for W8A8) [R][I]; MODE 1: Y fp32 [R][H]
  int out_ld;                // elements per output row
  int lo_rows;               // bf16 two-term activations: row offset of the lo plane (R_max)
  const float* a_scale;      // W8A8: per weight row [G * a_rows]
  const float* b_scale;      // W8A8: per token row [R]
  int* err;                  // device error word
};

template <int BN, bool SPLIT_B = false>
struct GemmShape {
  static constexpr int kATile = 128 * 128;              // one 128-row x 128-byte weight tile
  static constexpr int kBTile = BN * 128;               // up to BN token rows x 128 bytes
  static constexpr int kStageBytes = 2 * kATile + (SPLIT_B ? 2 : 1) * kBTile;
  static constexpr int kNacc = (4 * BN <= 512) ? 2 : 1;  // accumulator sets in TMEM
  static constexpr int kColsUsed = kNacc * 2 * BN;
  static constexpr int kTmemCols = kColsUsed <= 32 ? 32 : kColsUsed <= 64 ? 64 : kColsUsed <= 128 ? 128
                                   : kColsUsed <= 256 ? 256 : 512;
  static_assert(kColsUsed <= 512, "TMEM has 512 columns");
  static_assert(BN % 16 == 0 && BN <= 256, "N tile");
};

template <int BN, int STAGES, bool SPLIT_B>
constexpr int gemm_smem_bytes() {
  return STAGES * GemmShape<BN, SPLIT_B>::kStageBytes + 1024 /*alignment slack*/ + 256 /*barriers*/;
}

__device__ __forceinline__ int find_group(const int32_t* __restrict__ unit_base, int G, int u) {
  int lo = 0, hi = G - 1;  // largest g with unit_base[g] <= u
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(unit_base + mid) <= u) lo = mid; else hi = mid - 1;
  }
  return lo;
}

struct Unit {
  int g, mt, rows, row0, n16;  // group, tile pair, valid token rows, first row, MMA N
};

template <int BN>
__device__ __forceinline__ Unit decode_unit(const GemmArgs& a, int u) {
  Unit w;
  w.g = find_group(a.unit_base, a.G, u);
  const int local = u - __ldg(a.unit_base + w.g);
  const int grows = __ldg(a.grp_rows + w.g);
  const int ntiles = (grows + BN - 1) / BN;
  w.mt = local / ntiles;
  const int nt = local - w.mt * ntiles;
  w.rows = min(BN, grows - nt * BN);
  w.row0 = __ldg(a.grp_base + w.g) + nt * BN;
  w.n16 = (w.rows + 15) & ~15;
  return w;
}

__device__ __forceinline__ float silu_f(float z) { return z / (1.0f + expf(-z)); }

template <int BN, int STAGES, bool FP8, int MODE, bool SPLIT_B>
__global__ void __launch_bounds__(192, 1)
grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const GemmArgs args) {
  static_assert(!(SPLIT_B && (FP8 || MODE != 1)), "two-term B only for the bf16 down GEMM");
  using S = GemmShape<BN, SPLIT_B>;
  constexpr int kNacc = S::kNacc;
  constexpr int kKChunk = FP8 ? 128 : 64;  // elements per 128-byte row slice

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t bars = base + STAGES * S::kStageBytes;
  // barrier block: full[STAGES], empty[STAGES], tfull[kNacc], tempty[kNacc], done
  auto full_bar = [&](int s) { return bars + 8u * s; };
  auto empty_bar = [&](int s) { return bars + 8u * (STAGES + s); };
  auto tfull_bar = [&](int i) { return bars + 8u * (2 * STAGES + i); };
  auto tempty_bar = [&](int i) { return bars + 8u * (2 * STAGES + kNacc + i); };
  const uint32_t done_bar = bars + 8u * (2 * STAGES + 2 * kNacc);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + STAGES * S::kStageBytes + 8 * (2 * STAGES + 2 * kNacc + 1));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int i = 0; i < kNacc; ++i) {
      mbar_init(tfull_bar(i), 1);
      mbar_init(tempty_bar(i), 4);
    }
    mbar_init(done_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), S::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int total = __ldg(args.unit_base + args.G);
  const int kchunks = args.K / kKChunk;

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------------- TMA producer
    int s = 0;
    uint32_t ph = 0;
    int issued = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
      const Unit w = decode_unit<BN>(args, u);
      const int ya = w.g * args.a_rows + w.mt * args.mt_stride;
      const uint32_t tx = 2u * S::kATile + (SPLIT_B ? 2u : 1u) * static_cast<uint32_t>(w.n16) * 128u;
      for (int kc = 0; kc < kchunks; ++kc) {
        if (!mbar_wait(empty_bar(s), ph ^ 1u, abort_flag)) { ok = false; break; }
        const uint32_t st = base + s * S::kStageBytes;
        const int x = kc * kKChunk;
        mbar_arrive_expect_tx(full_bar(s), tx);
        tma_load_2d(st, &tmA, full_bar(s), x, ya, kEvictFirst);
        tma_load_2d(st + S::kATile, &tmA, full_bar(s), x, ya + args.second_off, kEvictFirst);
        for (int r = 0; r < w.n16; r += 16)
          tma_load_2d(st + 2 * S::kATile + r * 128, &tmB, full_bar(s), x, w.row0 + r, kEvictLast);
        if constexpr (SPLIT_B) {
          for (int r = 0; r < w.n16; r += 16)
            tma_load_2d(st + 2 * S::kATile + S::kBTile + r * 128, &tmB, full_bar(s), x,
                        args.lo_rows + w.row0 + r, kEvictLast);
        }
        ++issued;
        if (++s == STAGES) { s = 0; ph ^= 1u; }
      }
    }
    if (!ok) { *abort_flag = 1; atomicOr(args.err, kErrTimeout); }
    // drain: the last min(issued, STAGES) stages may still be landing in shared memory
    for (int i = 0; i < min(issued, STAGES); ++i) {
      if (--s < 0) { s = STAGES - 1; ph ^= 1u; }
      volatile int never = 0;
      mbar_wait(full_bar(s), ph, &never);
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------------- MMA issuer
    int s = 0;
    uint32_t ph = 0;
    int acc = 0;
    uint32_t acc_ph = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
      const Unit w = decode_unit<BN>(args, u);
      const uint32_t idesc = idesc_m128(w.n16, FP8);
      if (!mbar_wait(tempty_bar(acc), acc_ph ^ 1u, abort_flag)) { ok = false; break; }
      tc_fence_after();
      const uint32_t d0 = tmem + static_cast<uint32_t>(acc * 2 * BN);
      const uint32_t d1 = d0 + BN;
      for (int kc = 0; kc < kchunks; ++kc) {
        if (!mbar_wait(full_bar(s), ph, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t st = base + s * S::kStageBytes;
        const uint64_t da0 = sw128_desc(st);
        const uint64_t da1 = sw128_desc(st + S::kATile);
        const uint64_t db = sw128_desc(st + 2 * S::kATile);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {  // four 32-byte K slices of the 128-byte rows
          const uint32_t accum = (kc > 0 || kk > 0) ? 1u : 0u;
          tc_mma<FP8>(d0, da0 + 2 * kk, db + 2 * kk, idesc, accum);
          tc_mma<FP8>(d1, da1 + 2 * kk, db + 2 * kk, idesc, accum);
          if constexpr (SPLIT_B) {  // the lo plane of the activations, same accumulators
            const uint64_t dl = sw128_desc(st + 2 * S::kATile + S::kBTile);
            tc_mma<FP8>(d0, da0 + 2 * kk, dl + 2 * kk, idesc, 1u);
            tc_mma<FP8>(d1, da1 + 2 * kk, dl + 2 * kk, idesc, 1u);
          }
        }
        tc_commit(empty_bar(s));  // frees the stage once these MMAs have read it
        if (++s == STAGES) { s = 0; ph ^= 1u; }
      }
      if (!ok) break;
      tc_commit(tfull_bar(acc));
      if (++acc == kNacc) { acc = 0; acc_ph ^= 1u; }
    }
    if (!ok) { *abort_flag = 1; atomicOr(args.err, kErrTimeout); }
    // every MMA issued above has completed once this commit arrives
    tc_commit(done_bar);
    volatile int never = 0;
    mbar_wait(done_bar, 0, &never);
  } else if (warp >= 2) {
    // ---------------------------------------------------------------- epilogue
    const int q = warp & 3;               // TMEM lane quarter of this warp
    const int m = q * 32 + lane;          // row within the 128-row weight tile
    int acc = 0;
    uint32_t acc_ph = 0;
    for (int u = blockIdx.x; u < total; u += gridDim.x) {
      const Unit w = decode_unit<BN>(args, u);
      if (!mbar_wait(tfull_bar(acc), acc_ph, abort_flag)) {
        *abort_flag = 1;
        atomicOr(args.err, kErrTimeout);
        break;
      }
      tc_fence_after();
      const uint32_t t0 = tmem + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * 2 * BN);
      const uint32_t t1 = t0 + BN;
      // weight rows of this thread in the two tiles
      const int wrow0 = w.mt * args.mt_stride + m;
      const int wrow1 = wrow0 + args.second_off;
      float sa0 = 1.f, sa1 = 1.f;
      if constexpr (FP8) {
        sa0 = __ldg(args.a_scale + static_cast<size_t>(w.g) * args.a_rows + wrow0);
        sa1 = __ldg(args.a_scale + static_cast<size_t>(w.g) * args.a_rows + wrow1);
      }
      for (int c = 0; c < w.n16; c += 16) {
        uint32_t r0[16], r1[16];
        tmem_ld16(t0 + c, r0);
        tmem_ld16(t1 + c, r1);
        tmem_ld_wait(r0, r1);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int n = c + i;
          if (n < w.rows) {
            const size_t row = static_cast<size_t>(w.row0 + n);
            float v0 = __uint_as_float(r0[i]);
            float v1 = __uint_as_float(r1[i]);
            if constexpr (FP8) {
              const float sb = __ldg(args.b_scale + row);
              v0 = v0 * sa0 * sb;
              v1 = v1 * sa1 * sb;
            }
            if constexpr (MODE == 0) {
              const float act = silu_f(v0) * v1;  // gate tile first, up tile second
              if constexpr (FP8) {
                static_cast<float*>(args.out)[row * args.out_ld + wrow0] = act;
              } else {
                const __nv_bfloat16 hi = __float2bfloat16_rn(act);
                const __nv_bfloat16 lo = __float2bfloat16_rn(act - __bfloat162float(hi));
                __nv_bfloat16* o = static_cast<__nv_bfloat16*>(args.out);
                o[row * args.out_ld + wrow0] = hi;
                o[(static_cast<size_t>(args.lo_rows) + row) * args.out_ld + wrow0] = lo;
              }
            } else {
              float* y = static_cast<float*>(args.out) + row * args.out_ld;
              y[wrow0] = v0;
              y[wrow1] = v1;
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty_bar(acc));
      if (++acc == kNacc) { acc = 0; acc_ph ^= 1u; }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, S::kTmemCols);
  }
}

}  // namespace afd
