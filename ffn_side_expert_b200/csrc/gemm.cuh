// gemm.cuh -- grouped expert GEMMs (and the router) on the 5th-generation tensor cores
// (tcgen05 + TMEM + TMA).
//
// One persistent kernel serves both expert projections of the layer (each expert is a large
// matrix product: A/F 分离, section 为什么要拆) and the router:
//   MODE 0 (gate/up):  for expert g and its token rows X_g:  act = silu(X_g Wg^T) * (X_g Wu^T)
//   MODE 1 (down):     Y_g = act_g W2^T
//   MODE 2 (router):   logits[t][e] = sum_h hidden[t][h] * Wr[e][h]
// "Swap-AB" form: weight rows fill the 128-row M side of each MMA and the token rows are the
// N side (16..BN rows, rounded up to 16), so a decode micro-batch with ~8 rows per expert still
// streams full 128-row weight tiles.  A work unit is two 128-row weight tiles (gate rows j..,
// up rows I+j.. for MODE 0; down rows h.., h+128.. for MODE 1) against one tile of up to BN
// token rows, accumulated over K into two fp32 TMEM accumulators; SwiGLU (MODE 0) and the
// scales of the W8A8 path are applied in the epilogue straight from TMEM.  W8A8 large
// micro-batches use one-accumulator units instead (GemmShape ONE: one interleaved gate/up tile
// against up to 256 token rows).
//
// bf16 path, two-term activations: the gate/up epilogue stores the fp32 SwiGLU output as
// hi = bf16(act) and lo = bf16(act - hi) in two planes, and the down GEMM (SPLIT_B) multiplies
// each weight tile by both and accumulates into one TMEM accumulator, so the activation enters
// the down projection with ~2^-17 relative error instead of bf16's 2^-9 (the two-term bfloat16
// split of Henry, Tang and Heinecke, "Leveraging the bfloat16 AI datatype for higher-precision
// computations", 2019).  The only bf16 rounding left on the output path is the layer output.
//
// MODE 3 (fused, bf16): gate/up units and down units in ONE persistent launch.  Every CTA takes
// its gate/up units first, then its down units.  A gate/up epilogue publishes each finished act
// tile with a release increment of its (expert, N tile) counter; the producer of a down unit
// waits (acquire, bounded) until all I/128 act tiles of its rows are in, then issues its loads.
// Every dependency lies earlier in each CTA's unit order and the launch is cooperative (every
// CTA resident at once), so the waits always end; the HBM-bound weight stream of late gate/up
// units overlaps the tensor-heavier down units.
//
// MODE 2 (router): the fp32 router weights are stored once as three bf16 planes hi + mid + lo
// (each the bf16 rounding of what the previous planes leave), so Wr is represented to ~2^-27
// relative; bf16 x bf16 products are exact in fp32 and the three planes accumulate into one
// TMEM accumulator.  The reduction over H is split across units (partial logits, summed in
// order in fp32 by the top-k kernel): into stretches of at most 1024 elements, which keeps the
// tensor core's accumulation error far below the gate-weight tolerance, and further to spread a
// small micro-batch over more SMs.
//
// Pipeline: one ring of STAGES shared-memory stages, each holding the weight tiles and the
// token tile of one 128-byte K chunk.  Warp roles (64 + 32 x kEpiWarps threads): warp 0 lane 0
// issues the TMA loads, warp 1 owns the TMEM allocation and its lane 0 issues tcgen05.mma (one
// commit per stage), warps 2.. are the epilogue.  An epilogue warp w reads TMEM lanes
// 32*(w%4)..+31 (the lane quarter the hardware lets it access); with 8 epilogue warps two warps
// share each quarter and take alternate 16-column chunks, so every scheduler runs two epilogue
// warps and the SwiGLU / scaling math of one unit overlaps the next unit's MMAs.
// Decode shape of the bf16 down GEMM: the hi and lo activation rows of a stage sit back to
// back, so one MMA of N = 2 x rows covers both planes and the epilogue adds the two halves --
// half the MMA instructions of issuing each plane separately, which matters when every MMA is
// only 16 tokens wide.  Units are assigned round-robin over the persistent grid from a per-group
// schedule built on the device, so the host never needs the per-expert row counts.  Every wait
// is bounded (ptx.cuh: mbar_wait); a CTA that gives up records a timeout in the error word,
// drains its own copies and MMAs, frees TMEM and returns.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "ptx.cuh"

namespace afd {

struct GemmArgs {
  const int32_t* grp_rows;   // [G]   token rows of each group (expert)
  const int32_t* grp_base;   // [G]   first dispatched row of each group
  const int32_t* unit_base;  // [G+1] first unit of each group; unit_base[G] = total units
  int G;                     // groups: routed experts, then the shared expert
  int K;                     // reduction length in elements (H for gate/up and router, I for down)
  int a_rows;                // weight rows per group (2I gate/up, H down); router: valid rows E
  int mt_stride;             // weight rows between consecutive units' tile pairs (128 gate/up, 256 down)
  int second_off;            // offset of a pair's second tile (I / 128); router: plane stride E
  void* out;                 // MODE 0: act (bf16 planes, or fp32 for W8A8); MODE 1: Y fp32 (bf16 for W8A8);
                             // MODE 2: partial logits fp32 [ksplit][rows][E]
  int out_ld;                // elements per output row
  int lo_rows;               // bf16 two-term activations: row offset of the lo plane (R_max)
  int single_rows;           // >= 0: one group of that many rows starting at row 0 (router);
                             // -1: groups from grp_rows / grp_base / unit_base
  int single_mt;             // router: weight tiles (ceil(E / 128))
  int single_total;          // router: units = N tiles x weight tiles x K splits
  int kc_per;                // router: 128-byte K chunks per split (all splits non-empty)
  uint64_t a_policy;         // L2 policy of the weight-tile loads (MODE 0 / 1)
  const float* a_scale;      // W8A8: per weight row [G * a_rows]
  const float* b_scale;      // W8A8: per token row [R]
  int* err;                  // device error word
  // MODE 3 (fused): the down GEMM's side and the act-tile dependency counters
  const int32_t* unit_base2; // [G+1] units of the down GEMM
  const int32_t* tile_base;  // [G] first N tile of each group
  int* tile_done;            // [N tiles] gate/up units finished per (group, N tile)
  int K2, a_rows2, mt_stride2, second_off2, out_ld2;
  void* out2;                // Y
  int mt1;                   // gate/up units per N tile (I / 128)
};

// ONE (W8A8 large micro-batches): one 128-row weight tile and one accumulator per unit, with up
// to BN = 256 token rows -- so a unit still fits twice in TMEM.  Gate/up (MODE 0) then loads the
// tile interleaved (for each lane quarter 16 gate rows and their 16 up rows, from a 5-D tensor
// map), and a unit covers 64 act columns; down (MODE 1) covers 128 output rows.  Fewer, wider
// units: a tail of a few rows rides in a balanced tile instead of costing a unit of its own.
template <int BN, bool SPLIT_B = false, int MODE = 0, bool ONE = false>
struct GemmShape {
  static constexpr bool kFused = MODE == 3;
  static constexpr int kNA = MODE == 2 ? 3 : (ONE ? 1 : 2);     // weight tiles per stage
  static constexpr int kNDU = (MODE == 2 || ONE) ? 1 : 2;       // accumulators per unit
  static constexpr int kATile = 128 * 128;              // one 128-row x 128-byte weight tile
  static constexpr int kAStage = kNA * kATile;
  static constexpr int kBRows = BN;                     // token rows of a tile
  static constexpr int kBTile = kBRows * 128;           // up to kBRows token rows x 128 bytes
  static constexpr int kBStage = (SPLIT_B ? 2 : 1) * kBTile;
  static constexpr int kStageBytes = kAStage + kBStage;
  // two-term activations in one MMA (hi rows, then lo rows): the N of an MMA doubles
#ifndef AFD_CONCAT_MAX_BN
#define AFD_CONCAT_MAX_BN 64
#endif
  static constexpr bool kConcat = SPLIT_B && BN <= AFD_CONCAT_MAX_BN;
  // rows per TMA box of a token tile: few large boxes keep the single producer thread from
  // becoming the bottleneck; a box may overrun the unit's rows (the MMA reads only n16 rows)
  // except in the concatenated layout, where the lo rows follow the hi rows directly.
  // kBoxRowsX: single-plane token tiles (the gate/up side of the fused kernel)
  static constexpr int kBoxRowsX = kBRows < 64 ? kBRows : 64;
  static constexpr int kBoxRows = kConcat ? (BN <= 32 ? 16 : 32) : kBoxRowsX;
  // concatenated layout: hi rows padded to whole boxes, then the lo rows
  __device__ static int npad(int n16) { return kConcat ? (n16 + kBoxRows - 1) / kBoxRows * kBoxRows : n16; }
  static constexpr int kUnitCols = kNDU * BN * (kConcat ? 2 : 1);  // TMEM columns of one unit
  static constexpr int kNacc = (2 * kUnitCols <= 512) ? 2 : 1;  // unit buffers in TMEM
  static constexpr int kColsUsed = kNacc * kUnitCols;
  static constexpr int kTmemCols = kColsUsed <= 32 ? 32 : kColsUsed <= 64 ? 64 : kColsUsed <= 128 ? 128
                                   : kColsUsed <= 256 ? 256 : 512;
  static_assert(kColsUsed <= 512, "TMEM has 512 columns");
  static_assert(BN % 16 == 0 && BN <= 256, "N tile");
  static_assert(kStageBytes % 1024 == 0, "stages keep 1024-byte alignment");
  static_assert(!ONE || ((MODE == 0 || MODE == 1) && !SPLIT_B), "one-accumulator units: wide gate/up or down");
};

// Shared memory: the group schedule (one int4 per group: first unit, rows, first row), then
// the 1024-byte aligned rings, then the barriers.
constexpr int kMaxGroups = 257;
constexpr int kSchedBytes = (kMaxGroups + 1) * 16;

template <int BN, int STAGES, bool SPLIT_B, int MODE = 0, bool ONE = false>
constexpr int gemm_smem_bytes() {
  return (MODE == 3 ? 2 : 1) * kSchedBytes + 1024 /*alignment slack*/ +
         STAGES * GemmShape<BN, SPLIT_B, MODE, ONE>::kStageBytes + 256 /*barriers*/;
}

// Largest g with tab[g].x (first unit of group g) <= u; the table sits in shared memory.
__device__ __forceinline__ int find_group(const int4* tab, int G, int u) {
  int lo = 0, hi = G - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (tab[mid].x <= u) lo = mid; else hi = mid - 1;
  }
  return lo;
}

struct Unit {
  int g, mt, rows, row0, n16;  // group, tile pair, valid token rows, first row, MMA N
  int kc0, kc1, split;         // K chunks [kc0, kc1) and their split index
  int mode, tile;              // 0 gate/up, 1 down, 2 router; (group, N tile) id for MODE 3
};

template <int BN, int MODE>
__device__ __forceinline__ Unit decode_unit(const GemmArgs& a, const int4* tab, const int4* tab2, int u,
                                           int kchunks, int kchunks2) {
  Unit w;
  w.mode = MODE == 3 ? 0 : MODE;
  if constexpr (MODE == 3) {
    const int u1 = tab[a.G].x;
    if (u >= u1) {  // a down unit
      u -= u1;
      tab = tab2;
      kchunks = kchunks2;
      w.mode = 1;
    }
  }
  if (a.single_rows >= 0) {
    const int ntiles = (a.single_rows + BN - 1) / BN;
    const int per_split = ntiles * a.single_mt;
    w.split = u / per_split;
    const int local = u - w.split * per_split;
    w.g = 0;
    w.mt = local / ntiles;
    const int nt = local - w.mt * ntiles;
    w.rows = min(BN, a.single_rows - nt * BN);
    w.row0 = nt * BN;
    w.kc0 = w.split * a.kc_per;
    w.kc1 = min(kchunks, w.kc0 + a.kc_per);
    w.tile = 0;
  } else {
    w.g = find_group(tab, a.G, u);
    const int4 gs = tab[w.g];
    const int local = u - gs.x;
    const int grows = gs.y;
    const int ntiles = (grows + BN - 1) / BN;
    w.mt = local / ntiles;
    const int nt = local - w.mt * ntiles;
    // wide tiles: a group's rows are spread evenly over its ntiles tiles (sizes rounded up to 16)
    // instead of full tiles and a ragged last one -- an expert with 270 rows runs 96 + 96 + 78
    // rather than 128 + 128 + 14, and a small-N MMA costs nearly as much as a 128-row one.
    // (ntiles - 1) * sz < grows, since sz <= BN, so the last tile is never empty.
    const int sz = BN >= 128 ? min(BN, ((grows + ntiles - 1) / ntiles + 15) & ~15) : BN;
    w.rows = min(sz, grows - nt * sz);
    w.row0 = gs.z + nt * sz;
    w.split = 0;
    w.kc0 = 0;
    w.kc1 = kchunks;
    w.tile = gs.w + nt;
  }
  w.n16 = (w.rows + 15) & ~15;
  return w;
}

// silu(z) = z / (1 + e^-z) with the fast exponential and division intrinsics (relative error of
// a few 1e-7 over the range that matters; the limit z -> -inf gives -0).
__device__ __forceinline__ float silu_f(float z) { return __fdividef(z, 1.0f + __expf(-z)); }

#ifndef AFD_EPI_WARPS
#define AFD_EPI_WARPS 8
#endif
constexpr int kEpiWarps = AFD_EPI_WARPS;          // 4 or 8
static_assert(kEpiWarps == 4 || kEpiWarps == 8, "epilogue warps");
constexpr int kGemmThreads = 64 + 32 * kEpiWarps;

__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Wait until the gate/up units of a down unit's rows are all published (bounded like mbar_wait),
// then order the async-proxy (TMA) reads that follow after them.
__device__ __forceinline__ bool wait_tile(const int* cnt, int need, volatile int* abort) {
  const long long t0 = clock64();
  while (ld_acquire_gpu(cnt) < need) {
    if (*abort || clock64() - t0 > kWaitLimitCycles) return false;
    __nanosleep(64);
  }
  asm volatile("fence.proxy.async.global;" ::: "memory");
  return true;
}

// ACT16 (bf16 large micro-batches): the gate/up epilogue stores the SwiGLU output as one f16
// plane (MODE 0), and the down GEMM multiplies it by an f16 copy of W2 (MODE 1, kind::f16 with
// f16 operands) -- f16 keeps 10 mantissa bits where bf16 keeps 7, so one term suffices.  Each
// token row is stored divided by its power-of-two scale b_scale[row] (f16_row_scale: the row's
// bound on |act| stays inside the f16 range), and the down epilogue multiplies it back.
template <int BN, int STAGES, bool FP8, int MODE, bool SPLIT_B, bool ACT16 = false, bool ONE = false>
__global__ void __launch_bounds__(kGemmThreads, 1)
grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmB2,
                    const GemmArgs args) {
  static_assert(!(SPLIT_B && (FP8 || (MODE != 1 && MODE != 3))), "two-term B only for the bf16 down GEMM");
  static_assert(!((MODE == 2 || MODE == 3) && FP8), "router and fused modes run on bf16");
  static_assert(!ACT16 || (!FP8 && !SPLIT_B && (MODE == 0 || MODE == 1)), "f16 activations: wide bf16 GEMMs");
  static_assert(!ONE || (FP8 && !ACT16), "one-accumulator units serve the W8A8 wide GEMMs");
  using S = GemmShape<BN, SPLIT_B, MODE, ONE>;
  constexpr int kNacc = S::kNacc;
  constexpr bool kWarpMma = MODE != 3;  // MMA issue by an elected lane of the whole warp
  constexpr int kKChunk = FP8 ? 128 : 64;  // elements per 128-byte row slice

  extern __shared__ uint8_t smem_raw[];
  int4* sched = reinterpret_cast<int4*>(smem_raw);  // group schedule copy
  int4* sched2 = sched + (kMaxGroups + 1);          // MODE 3: the down GEMM's schedule
  constexpr int kSchedAll = (MODE == 3 ? 2 : 1) * kSchedBytes;
  const uint32_t raw = smem_u32(smem_raw) + kSchedAll;
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + kSchedAll + (base - raw);
  const uint32_t bars = base + STAGES * S::kStageBytes;
  // barrier block: full[STAGES], empty[STAGES], tfull[kNacc], tempty[kNacc], done
  const uint32_t full = bars, empty = bars + 8u * STAGES;
  const uint32_t tfull = bars + 16u * STAGES, tempty = tfull + 8u * kNacc;
  const uint32_t done_bar = tempty + 8u * kNacc;
  // MODE 3: per accumulator buffer, the four epilogue warps finished an act tile.  A warp arrives
  // here before it releases the buffer, so the next unit on the same buffer cannot arrive early.
  const uint32_t epi_bar = done_bar + 8u;
  constexpr int kBars = 2 * STAGES + 3 * kNacc + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + STAGES * S::kStageBytes + 8 * kBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int unit0 = static_cast<int>(blockIdx.x);
  const int unit_step = static_cast<int>(gridDim.x);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full + 8u * s, 1);
      mbar_init(empty + 8u * s, 1);
    }
    for (int i = 0; i < kNacc; ++i) {
      mbar_init(tfull + 8u * i, 1);
      mbar_init(tempty + 8u * i, kEpiWarps);
    }
    mbar_init(done_bar, 1);
    for (int i = 0; i < kNacc; ++i) mbar_init(epi_bar + 8u * i, kEpiWarps);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if constexpr (MODE == 3) {
      tma_prefetch_desc(&tmA2);
      tma_prefetch_desc(&tmB2);
    }
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), S::kTmemCols);
    tmem_relinquish();
  }
  if (args.single_rows < 0) {
    for (int g = threadIdx.x; g <= args.G; g += blockDim.x) {
      const int tb = (MODE == 3 && g < args.G) ? __ldg(args.tile_base + g) : 0;
      sched[g] = g < args.G ? make_int4(__ldg(args.unit_base + g), __ldg(args.grp_rows + g), __ldg(args.grp_base + g), tb)
                            : make_int4(__ldg(args.unit_base + g), 0, 0, 0);
      if constexpr (MODE == 3)
        sched2[g] = g < args.G ? make_int4(__ldg(args.unit_base2 + g), __ldg(args.grp_rows + g),
                                           __ldg(args.grp_base + g), tb)
                               : make_int4(__ldg(args.unit_base2 + g), 0, 0, 0);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int total = args.single_rows >= 0 ? args.single_total
                                          : sched[args.G].x + (MODE == 3 ? sched2[args.G].x : 0);
  const int kchunks = args.K / kKChunk;
  const int kchunks2 = MODE == 3 ? args.K2 / kKChunk : kchunks;

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------------- TMA producer
    int s = 0;
    uint32_t ph = 0;
    int issued = 0;
    bool ok = true;
    for (int u = unit0; u < total && ok; u += unit_step) {
      const Unit w = decode_unit<BN, MODE>(args, sched, sched2, u, kchunks, kchunks2);
      // the down side of the fused kernel uses the second set of maps and coordinates
      const bool down = MODE == 3 && w.mode == 1;
      const CUtensorMap* mA = down ? &tmA2 : &tmA;
      const CUtensorMap* mB = down ? &tmB2 : &tmB;
      const int ya = down ? w.g * args.a_rows2 + w.mt * args.mt_stride2 : w.g * args.a_rows + w.mt * args.mt_stride;
      const int soff = down ? args.second_off2 : args.second_off;
      const bool two = SPLIT_B && (MODE != 3 || down);           // hi and lo planes
      const int boxr = (MODE == 3 && !down) ? S::kBoxRowsX : S::kBoxRows;
      const int brows = w.n16;  // token rows loaded (the MMA reads n16 of them)
      const int brow0 = w.row0;
      const int nbox = (brows + boxr - 1) / boxr;                  // token-tile boxes per plane
      const uint32_t tx = S::kAStage + (two ? 2u : 1u) * static_cast<uint32_t>(nbox * boxr) * 128u;
      // the lo activation rows follow the (padded) hi rows or sit one tile further
      const uint32_t lo_off = S::kConcat ? static_cast<uint32_t>(S::npad(w.n16)) * 128u : S::kBTile;
      const uint64_t apol = MODE == 2 ? kEvictLast : args.a_policy;
      if (down && !wait_tile(args.tile_done + w.tile, args.mt1, abort_flag)) { ok = false; break; }
      for (int kc = w.kc0; kc < w.kc1; ++kc) {
        if (!mbar_wait(empty + 8u * s, ph ^ 1u, abort_flag)) { ok = false; break; }
        const uint32_t st = base + s * S::kStageBytes;
        const uint32_t fb = full + 8u * s;
        const int x = kc * kKChunk;
        mbar_arrive_expect_tx(full + 8u * s, tx);
        if constexpr (ONE && MODE == 0) {
          // 64 act columns: blocks 4 mt .. 4 mt + 3 of 16 gate rows, each with its up rows
          tma_load_5d(st, mA, fb, x, 0, 0, 4 * w.mt, w.g, apol);
        } else {
          // the tile pair (MODE 0/1), one tile (ONE down) or the three router planes (MODE 2)
#pragma unroll
          for (int i = 0; i < S::kNA; ++i) tma_load_2d(st + i * S::kATile, mA, fb, x, ya + i * soff, apol);
        }
        const uint32_t sb = st + S::kAStage;
        for (int b = 0; b < nbox; ++b) tma_load_2d(sb + b * boxr * 128, mB, fb, x, brow0 + b * boxr, kEvictLast);
        if (two) {
          for (int b = 0; b < nbox; ++b)
            tma_load_2d(sb + lo_off + b * boxr * 128, mB, fb, x, args.lo_rows + brow0 + b * boxr, kEvictLast);
        }
        ++issued;
        if (++s == STAGES) { s = 0; ph ^= 1u; }
      }
    }
    if (!ok) { *abort_flag = 1; atomicOr(args.err, kErrTimeout); }
    // drain: the last min(issued, STAGES) stages may still be landing in shared memory (bounded)
    for (int i = 0; i < min(issued, STAGES); ++i) {
      if (--s < 0) { s = STAGES - 1; ph ^= 1u; }
      volatile int never = 0;
      mbar_wait(full + 8u * s, ph, &never);
    }
  } else if (warp == 1 && (kWarpMma || lane == 0)) {
    // ---------------------------------------------------------------- MMA issuer
    // Wide units: the whole warp runs this loop, so its barrier waits and descriptor arithmetic
    // stay warp-uniform, and one elected lane issues the tcgen05 instructions.  Measured on B200
    // with data always ready: one MMA of N <= 144 every ~81 cycles this way, ~113 from a lone
    // thread; the large micro-batches ran 2-3 % faster.  The fused decode kernel (HBM-bound)
    // measured 0.5 % slower this way and keeps a lone issuing thread.
    const bool leader = kWarpMma ? elect_one() : true;
    auto all = [](bool v) {
      if constexpr (kWarpMma) return __all_sync(0xffffffffu, v) != 0;
      return v;
    };
    auto sync = [] {
      if constexpr (kWarpMma) __syncwarp();
    };
    int s = 0;
    uint32_t ph = 0;
    int acc = 0;
    uint32_t acc_ph = 0;
    bool ok = true;
    for (int u = unit0; u < total && ok; u += unit_step) {
      const Unit w = decode_unit<BN, MODE>(args, sched, sched2, u, kchunks, kchunks2);
      const bool down = MODE == 1 || (MODE == 3 && w.mode == 1);
      const bool cat = S::kConcat && down;
      const uint32_t idesc = idesc_mn(128, cat ? 2 * S::npad(w.n16) : w.n16, FP8, ACT16 && MODE == 1);
      if (!all(mbar_wait(tempty + 8u * acc, acc_ph ^ 1u, abort_flag))) { ok = false; break; }
      tc_fence_after();
      const uint32_t d0 = tmem + static_cast<uint32_t>(acc * S::kUnitCols);
      const uint32_t d1 = d0 + S::kUnitCols / 2;
      for (int kc = w.kc0; kc < w.kc1; ++kc) {
        if (!all(mbar_wait(full + 8u * s, ph, abort_flag))) { ok = false; break; }
        tc_fence_after();
        const uint32_t st = base + s * S::kStageBytes;
        const uint64_t da0 = sw128_desc(st);
        const uint64_t da1 = sw128_desc(st + S::kATile);
        const uint64_t db = sw128_desc(st + S::kAStage);
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {  // four 32-byte K slices of the 128-byte rows
            const uint32_t accum = (kc > w.kc0 || kk > 0) ? 1u : 0u;
            if constexpr (MODE == 2) {  // hi, mid, lo planes into one accumulator
              const uint64_t da2 = sw128_desc(st + 2 * S::kATile);
              tc_mma<false>(d0, da0 + 2 * kk, db + 2 * kk, idesc, accum);
              tc_mma<false>(d0, da1 + 2 * kk, db + 2 * kk, idesc, 1u);
              tc_mma<false>(d0, da2 + 2 * kk, db + 2 * kk, idesc, 1u);
            } else {
              tc_mma<FP8>(d0, da0 + 2 * kk, db + 2 * kk, idesc, accum);
              if constexpr (S::kNDU == 2) tc_mma<FP8>(d1, da1 + 2 * kk, db + 2 * kk, idesc, accum);
              if constexpr (SPLIT_B && !S::kConcat) {  // the lo plane as separate MMAs
                if (down) {
                  const uint64_t dl = sw128_desc(st + S::kAStage + S::kBTile);
                  tc_mma<FP8>(d0, da0 + 2 * kk, dl + 2 * kk, idesc, 1u);
                  tc_mma<FP8>(d1, da1 + 2 * kk, dl + 2 * kk, idesc, 1u);
                }
              }
            }
          }
          tc_commit(empty + 8u * s);  // frees the stage once these MMAs have read it
        }
        sync();
        if (++s == STAGES) { s = 0; ph ^= 1u; }
      }
      if (!ok) break;
      if (leader) tc_commit(tfull + 8u * acc);
      sync();
      if (++acc == kNacc) { acc = 0; acc_ph ^= 1u; }
    }
    if (!ok && leader) { *abort_flag = 1; atomicOr(args.err, kErrTimeout); }
    // every MMA issued above has completed once this commit arrives
    if (leader) tc_commit(done_bar);
    sync();
    volatile int never = 0;
    mbar_wait(done_bar, 0, &never);
  } else if (warp >= 2 && warp < 2 + kEpiWarps) {
    // ---------------------------------------------------------------- epilogue
    const int q = warp & 3;               // TMEM lane quarter of this warp
    const int m = q * 32 + lane;          // row within the 128-row weight tile
    constexpr int kCStep = 16 * (kEpiWarps / 4);  // the column chunks of the warps sharing q
    const int c_first = 16 * ((warp - 2) / 4);
    int acc = 0;
    uint32_t acc_ph = 0;
    uint32_t epi_ph = 0;  // parity bit per accumulator buffer
    for (int u = unit0; u < total; u += unit_step) {
      const Unit w = decode_unit<BN, MODE>(args, sched, sched2, u, kchunks, kchunks2);
      if (!mbar_wait(tfull + 8u * acc, acc_ph, abort_flag)) {
        *abort_flag = 1;
        atomicOr(args.err, kErrTimeout);
        break;
      }
      tc_fence_after();
      const uint32_t t0 = tmem + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * S::kUnitCols);
      const uint32_t t1 = t0 + S::kUnitCols / 2;
      // weight rows of this thread in the two tiles
      const bool down = MODE == 1 || (MODE == 3 && w.mode == 1);
      const int wrow0 = w.mt * (MODE == 3 && down ? args.mt_stride2 : args.mt_stride) +
                        m;
      const int wrow1 = wrow0 + (MODE == 3 && down ? args.second_off2 : args.second_off);
      if constexpr (MODE == 2) {  // partial logits [split][t][e]; rows past E are padding
        const int e = wrow0;
        float* lg = static_cast<float*>(args.out) + static_cast<size_t>(w.split) * args.single_rows * args.out_ld;
        for (int c = c_first; c < w.n16; c += kCStep) {
          uint32_t r0[16];
          tmem_ld16(t0 + c, r0);
          tmem_ld_wait(r0);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int n = c + i;
            if (n < w.rows && e < args.a_rows)
              lg[static_cast<size_t>(w.row0 + n) * args.out_ld + e] = __uint_as_float(r0[i]);
          }
        }
      } else if constexpr (ONE && MODE == 0) {
        // interleaved gate/up: this warp's lane quarter q holds act columns jc0 .. jc0 + 15, with
        // jc0 = 64 mt + 16 q; lane l reads the gate row of column jc0 + l (l < 16) or the up row of
        // column jc0 + l - 16.
        // For each 16-token chunk the gate lane takes tokens 0..7 and the up lane tokens 8..15,
        // trading the other half with its partner lane (l xor 16).
        const int up = lane >> 4;
        const int jc = w.mt * args.mt_stride + 16 * q + (lane & 15);  // act column
        const float sa = __ldg(args.a_scale + static_cast<size_t>(w.g) * args.a_rows + up * args.second_off + jc);
        for (int c = c_first; c < w.n16; c += kCStep) {
          float sb_lane = 0.f;  // token scales, lane i < 16 holding token c + i
          if (lane < 16 && c + lane < w.rows) sb_lane = __ldg(args.b_scale + w.row0 + c + lane);
          uint32_t r0[16];
          tmem_ld16(t0 + c, r0);
          tmem_ld_wait(r0);
          float v[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r0[i]) * sa * __shfl_sync(0xffffffffu, sb_lane, i);
#pragma unroll
          for (int n = 0; n < 8; ++n) {
            const float other = __shfl_xor_sync(0xffffffffu, up ? v[n] : v[n + 8], 16);
            const float g = up ? other : v[n];
            const float uv = up ? v[n + 8] : other;
            const int tok = c + n + 8 * up;
            if (tok < w.rows)  // fp32 SwiGLU row, quantised per row before the down GEMM
              static_cast<float*>(args.out)[static_cast<size_t>(w.row0 + tok) * args.out_ld + jc] = silu_f(g) * uv;
          }
        }
      } else {
        float sa0 = 1.f, sa1 = 1.f;
        if constexpr (FP8) {
          sa0 = __ldg(args.a_scale + static_cast<size_t>(w.g) * args.a_rows + wrow0);
          sa1 = __ldg(args.a_scale + static_cast<size_t>(w.g) * args.a_rows + wrow1);
        }
        for (int c = c_first; c < w.n16; c += kCStep) {
          // W8A8 (and the f16 activations): lane i < 16 fetches the scale of token row c + i once;
          // shuffled to all lanes below
          float sb_lane = 0.f;
          if constexpr (FP8 || ACT16) {
            if (lane < 16 && c + lane < w.rows) sb_lane = __ldg(args.b_scale + w.row0 + c + lane);
          }
          uint32_t r0[16], r1[16];
          tmem_ld16(t0 + c, r0);
          if constexpr (S::kNDU == 2) {
            tmem_ld16(t1 + c, r1);
            tmem_ld_wait(r0, r1);
          } else {
            tmem_ld_wait(r0);
#pragma unroll
            for (int i = 0; i < 16; ++i) r1[i] = 0u;
          }
          if (S::kConcat && down) {  // add the lo-plane half (columns npad..) of each tile
            uint32_t l0[16], l1[16];
            tmem_ld16(t0 + S::npad(w.n16) + c, l0);
            tmem_ld16(t1 + S::npad(w.n16) + c, l1);
            tmem_ld_wait(l0, l1);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              r0[i] = __float_as_uint(__uint_as_float(r0[i]) + __uint_as_float(l0[i]));
              r1[i] = __float_as_uint(__uint_as_float(r1[i]) + __uint_as_float(l1[i]));
            }
          }
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int n = c + i;
            float sb = 1.f;
            if constexpr (FP8 || ACT16) sb = __shfl_sync(0xffffffffu, sb_lane, i);
            if (n < w.rows) {
              const size_t row = static_cast<size_t>(w.row0 + n);
              float v0 = __uint_as_float(r0[i]);
              float v1 = __uint_as_float(r1[i]);
              if constexpr (FP8) {
                v0 = v0 * sa0 * sb;
                v1 = v1 * sa1 * sb;
              }
              if (!down) {
                const float act = silu_f(v0) * v1;  // gate tile first, up tile second
                if constexpr (FP8) {
                  static_cast<float*>(args.out)[row * args.out_ld + wrow0] = act;
                } else if constexpr (ACT16) {  // act / s, s the row's power-of-two f16 scale (exact)
                  static_cast<__half*>(args.out)[row * args.out_ld + wrow0] = __float2half_rn(act * __frcp_rn(sb));
                } else {
                  const __nv_bfloat16 hi = __float2bfloat16_rn(act);
                  const __nv_bfloat16 lo = __float2bfloat16_rn(act - __bfloat162float(hi));
                  __nv_bfloat16* o = static_cast<__nv_bfloat16*>(args.out);
                  o[row * args.out_ld + wrow0] = hi;
                  o[(static_cast<size_t>(args.lo_rows) + row) * args.out_ld + wrow0] = lo;
                }
              } else if constexpr (FP8) {  // W8A8: expert outputs kept as bf16 (combine input)
                __nv_bfloat16* y = static_cast<__nv_bfloat16*>(args.out) + row * args.out_ld;
                y[wrow0] = __float2bfloat16_rn(v0);
                if constexpr (S::kNDU == 2) y[wrow1] = __float2bfloat16_rn(v1);
              } else {
                float* y = static_cast<float*>(MODE == 3 ? args.out2 : args.out) +
                           row * (MODE == 3 ? args.out_ld2 : args.out_ld);
                if constexpr (ACT16) {  // undo the row's f16 scale of the activations
                  v0 *= sb;
                  v1 *= sb;
                }
                y[wrow0] = v0;
                if constexpr (S::kNDU == 2) y[wrow1] = v1;
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if constexpr (MODE == 3) {
        if (!down) {  // publish this act tile once all four epilogue warps have stored their rows
          const uint32_t eb = epi_bar + 8u * acc;
          asm volatile("fence.proxy.async.global;" ::: "memory");  // stores above -> later TMA reads
          __syncwarp();
          if (lane == 0) mbar_arrive(eb);
          if (warp == 2 && lane == 0) {
            if (mbar_wait(eb, (epi_ph >> acc) & 1u, abort_flag)) {
              __threadfence();
              atomicAdd(args.tile_done + w.tile, 1);
            } else {
              *abort_flag = 1;
              atomicOr(args.err, kErrTimeout);
            }
          }
          epi_ph ^= 1u << acc;
        }
      }
      if (lane == 0) {
        mbar_arrive(tempty + 8u * acc);
      }
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
