// afd_ffn.cu -- host side of libafd_ffn.so: argument checks, workspace, TMA descriptors and
// the launch sequence of the FFN-service MoE layer.  The declarations, conventions and
// readings are documented in include/afd_ffn.h.
//
// Launch sequence of afd_ffn_forward (one stream, no host synchronisation):
//   router_logits -> router_topk -> dispatch_order -> gather_rows (W8A8: + quantise) ->
//   build_schedule -> grouped_gemm<gate/up> -> (W8A8: quantize_act) -> grouped_gemm<down>
//   -> combine
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>

#include "afd_ffn.h"
#include "combine.cuh"
#include "dispatch.cuh"
#include "gemm.cuh"
#include "router.cuh"

using namespace afd;

namespace {

// Tile shapes of the grouped GEMMs (N tile and ring stages; GemmPair below): "narrow" for decode micro-batches (a few rows per expert, N <= 32) and "wide" for
// large micro-batches (N <= 128).  The bf16 down GEMM reads two activation planes (hi, lo) per
// token stage.  Both keep two accumulator sets in TMEM so the epilogue of one unit overlaps the
// next unit's MMAs.
// tensor-core router: N tile of 64 tokens, three weight planes per stage
// Router GEMM tiles: 64 tokens per unit for small micro-batches (more units to spread over the
// SMs), 128 from kRouterWideT tokens up (an N = 128 MMA costs 64 cycles where an N = 64 one
// still costs ~50, so the wide tile halves the issue time per token).  Both load the hidden
// rows in 64-row boxes, so they share one tensor map.
constexpr int kRouterBN = 64, kRouterStages = 3;
constexpr int kRouterBNWide = 128, kRouterWideT = 1024;
// Longest stretch of H (in 64-element chunks) one tensor-core accumulation of the router covers:
// the partial logits of consecutive stretches are then added in fp32, in order, by the top-k
// kernel.  Measured on B200 at the DeepSeek-V3 router shape, the gate weights from the summed
// logits stay within 7e-7 of the fp64 ones with 384-element stretches but drift to 9e-6 with a
// single 3584-element one; 1024 elements keeps the accumulations short at every micro-batch size.
constexpr int kRouterMaxSplitChunks = 16;

thread_local int g_create_cuda_error = 0;

}  // namespace

struct afd_ffn_handle {
  afd_ffn_cfg cfg;
  afd_ffn_weights w;
  int device = 0;
  int num_sms = 0;
  int fused_grid = 0; // CTAs of the fused decode launch (cooperative: all resident at once)
  bool fp8 = false;
  int G = 0;       // E + n_shared
  int R_max = 0;   // rows of the dispatched-row buffers: T_max * (k + 1)
  size_t part_floats = 0;

  void* ws = nullptr;
  float* part = nullptr;
  int32_t* idx = nullptr;
  float* wts = nullptr;
  void* wr_planes = nullptr; // [3][E][H] bf16: router weights hi, mid, lo
  int32_t* counts = nullptr;
  int32_t* offsets = nullptr;
  int32_t* pos = nullptr;
  int32_t* src = nullptr;
  int32_t* chunk_counts = nullptr;  // [ceil(T_max/128)][E] per-chunk expert counts
  int32_t* chunk_base = nullptr;    // [ceil(T_max/128)][E] first row of each (chunk, expert)
  int32_t* grp_rows = nullptr;
  int32_t* grp_base = nullptr;
  int32_t* ub1 = nullptr;
  int32_t* ub2 = nullptr;
  int32_t* tile_base = nullptr;  // [G] first N tile of each group
  int* tile_done = nullptr;      // [N tiles] act-tile counters of the fused expert kernel
  int max_tiles = 0;
  uint8_t* xp = nullptr;     // dispatched rows [R_max][H] bf16 / e4m3
  float* xscale = nullptr;   // [R_max]
  void* act = nullptr;       // [2][R_max][I] bf16 hi/lo planes (or [R_max][I] fp32 in W8A8)
  uint8_t* actq = nullptr;   // W8A8: [R_max][I] e4m3
  float* ascale = nullptr;   // W8A8: [R_max]
  float* Y = nullptr;        // [R_max][H] fp32 (bf16 on the W8A8 path)
  int* err = nullptr;        // device error word
  void* hin = nullptr;       // [T_max][H] bf16 staging for afd_ffn_forward_host
  void* hout = nullptr;
  void* hin2 = nullptr;      // second staging pair of afd_ffn_forward_host_batches
  void* hout2 = nullptr;
  cudaStream_t copy_in = nullptr, copy_out = nullptr;   // copy streams of the batch loop
  cudaEvent_t ev_in[2] = {}, ev_done[2] = {}, ev_out[2] = {};

  CUtensorMap tm_w13, tm_w2, tm_wr;
  CUtensorMap tm_w13i;       // W13 as interleaved gate/up blocks (5-D view) for one-accumulator units
  bool one = false;          // large W8A8 micro-batches run the one-accumulator GEMMs
  // bf16 large micro-batches: f16 copy of W2 and the f16 activation plane (single-term down GEMM)
  void* w2h = nullptr;       // [E+S][H][I] f16, owned; NULL when unused
  bool act16 = false;
  float f16_bound = 0.f;     // 2 C / 32768 (w13_norm_bound_kernel): the f16 act row scales' input
  CUtensorMap tm_w2h, tm_act16;
  CUtensorMap tm_xp[2], tm_act[2];  // token rows for the [narrow, wide] shapes (box heights differ)
  cudaStream_t last_stream = nullptr;
  int last_cuda_error = 0;
  cudaEvent_t events[AFD_FFN_NUM_STAGES + 1];
  int n_events = 0;
};

namespace {

int cuda_fail(afd_ffn_handle* h, cudaError_t e) {
  if (h) h->last_cuda_error = static_cast<int>(e); else g_create_cuda_error = static_cast<int>(e);
  return AFD_ERR_CUDA;
}

#define AFD_CUDA(h, call)                                  \
  do {                                                     \
    cudaError_t e_ = (call);                               \
    if (e_ != cudaSuccess) return cuda_fail((h), e_);      \
  } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

void router_split(int T, int H, int E, int sms, int* nsplit, int* per) {
  const int tiles = ((T + kRtTok - 1) / kRtTok) * ((E + kRtExp - 1) / kRtExp);
  const int kt = H / kRtK;
  int want = std::max(1, (2 * sms + tiles - 1) / std::max(tiles, 1));
  want = std::min(want, std::min(32, kt));
  *per = (kt + want - 1) / want;
  *nsplit = (kt + *per - 1) / *per;
}

bool use_narrow(const afd_ffn_handle* h, int T) {
  return static_cast<long long>(T) * h->cfg.k <= 32LL * h->cfg.E;
}

int check_device(afd_ffn_handle* h) {
  int dev = -1;
  AFD_CUDA(h, cudaGetDevice(&dev));
  if (dev != h->device) return AFD_ERR_INVALID_ARG;
  return AFD_OK;
}

int check_T(const afd_ffn_handle* h, int32_t T) {
  if (T < 0) return AFD_ERR_INVALID_ARG;
  if (T > h->cfg.T_max) return AFD_ERR_T_TOO_LARGE;
  return AFD_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess && q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 2-D K-major tensor [rows][inner] of 1- or 2-byte elements; box = (128 bytes) x box_rows,
// 128-byte swizzle, zero fill outside the tensor.
bool encode_2d(CUtensorMap* m, const void* base, bool byte_elems, uint64_t inner, uint64_t rows,
               uint32_t box_rows) {
  auto enc = get_encode();
  if (!enc) return false;
  const uint32_t esz = byte_elems ? 1 : 2;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner * esz};
  cuuint32_t box[2] = {128u / esz, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, byte_elems ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                   const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// W13 [G][2I][H] (1- or 2-byte elements) viewed as 5-D {H, 16 rows, gate|up, I/16 blocks, G}, so
// that one box {128 bytes, 16, 2, 4, 1} holds 64 consecutive gate rows interleaved with their up
// rows: 16 gate rows, their 16 up rows, the next 16 gate rows, ... (128 rows of 128 bytes, the
// 128-byte swizzle applied to each row as in a 2-D box).
bool encode_w13_interleaved(CUtensorMap* m, const void* base, bool byte_elems, uint64_t H, uint64_t I,
                            uint64_t G) {
  auto enc = get_encode();
  if (!enc || I % 64 != 0) return false;
  const uint64_t esz = byte_elems ? 1 : 2;
  cuuint64_t dims[5] = {H, 16, 2, I / 16, G};
  cuuint64_t strides[4] = {H * esz, I * H * esz, 16 * H * esz, 2 * I * H * esz};
  cuuint32_t box[5] = {static_cast<cuuint32_t>(128 / esz), 16, 2, 4, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = enc(m, byte_elems ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5,
                   const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int BN, int ST, bool FP8, int MODE, bool SPLIT, bool ACT16 = false, bool ONE = false>
cudaError_t set_gemm_attr() {
  return cudaFuncSetAttribute(grouped_gemm_kernel<BN, ST, FP8, MODE, SPLIT, ACT16, ONE>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              gemm_smem_bytes<BN, ST, SPLIT, MODE, ONE>());
}

// bf16 large micro-batches with f16 activations: gate/up (f16 act plane) and down (f16 operands)
#ifndef AFD_ACT16
#define AFD_ACT16 1
#endif
#ifndef AFD_ACT16_G1_ST
#define AFD_ACT16_G1_ST 4
#endif
#ifndef AFD_ACT16_G2_ST
#define AFD_ACT16_G2_ST 4
#endif
constexpr int kAct16BN = 128;

// W8A8 large micro-batches: one-accumulator units of up to kOneBN token rows (GemmShape ONE),
// kOneST ring stages of 48 KB.  Gate/up units cover 64 act columns, down units 128 output rows.
// Measured on one B200 machine against the two-accumulator 128-row tiles, A/B in the same call:
// W8A8 T=8192 4.49-4.54 vs 4.59-4.74 ms per step.  bf16 with f16 activations measured slower
// this way (T=4096 Zipf: 5.61-5.65 vs 5.16-5.33 ms): its 2-byte token rows, re-read by twice as
// many units, cost more than the weight re-streams saved, so it keeps the 128-row tiles.
#ifndef AFD_ONE
#define AFD_ONE 1
#endif
constexpr int kOneBN = 256, kOneST = 4;

// (gate/up, down) kernel pairs of each path and tile shape: N tile and ring stages of each
// GEMM.  Compile-time tunable for tile sweeps: -DAFD_<path>_BN=.. -DAFD_<path>_ST=..
// bf16 decode, gate/up
#ifndef AFD_NB_G1_BN
#define AFD_NB_G1_BN 32
#endif
#ifndef AFD_NB_G1_ST
#define AFD_NB_G1_ST 6
#endif
// bf16 decode, down (hi and lo activation rows in one MMA)
#ifndef AFD_NB_G2_BN
#define AFD_NB_G2_BN 32
#endif
#ifndef AFD_NB_G2_ST
#define AFD_NB_G2_ST 5
#endif
// bf16 large micro-batch, gate/up
#ifndef AFD_WB_G1_BN
#define AFD_WB_G1_BN 128
#endif
#ifndef AFD_WB_G1_ST
#define AFD_WB_G1_ST 4
#endif
// bf16 large micro-batch, down (two activation planes per stage)
#ifndef AFD_WB_G2_BN
#define AFD_WB_G2_BN 128
#endif
#ifndef AFD_WB_G2_ST
#define AFD_WB_G2_ST 3
#endif
// W8A8 decode, gate/up
#ifndef AFD_NF_G1_BN
#define AFD_NF_G1_BN 32
#endif
#ifndef AFD_NF_G1_ST
#define AFD_NF_G1_ST 6
#endif
// W8A8 decode, down
#ifndef AFD_NF_G2_BN
#define AFD_NF_G2_BN 32
#endif
#ifndef AFD_NF_G2_ST
#define AFD_NF_G2_ST 6
#endif
// W8A8 large micro-batch, gate/up
#ifndef AFD_WF_G1_BN
#define AFD_WF_G1_BN 128
#endif
#ifndef AFD_WF_G1_ST
#define AFD_WF_G1_ST 4
#endif
// W8A8 large micro-batch, down
#ifndef AFD_WF_G2_BN
#define AFD_WF_G2_BN 128
#endif
#ifndef AFD_WF_G2_ST
#define AFD_WF_G2_ST 4
#endif

// bf16 decode shape: the gate/up and down GEMMs run fused in one launch (MODE 3) with stf ring
// stages (measured on B200 at T=256: 3.45 ms fused vs 3.49 ms as two launches).  The large
// micro-batch shape stays two launches: sharing one ring with the down GEMM's 64 KB stages
// leaves the gate/up side three stages instead of four, which cost 0.95 ms at T=4096.
#ifndef AFD_FUSED
#define AFD_FUSED 1
#endif
#ifndef AFD_NB_F_ST
#define AFD_NB_F_ST 5
#endif
#ifndef AFD_WB_F_ST
#define AFD_WB_F_ST 0
#endif

template <int BN1, int ST1, int BN2, int ST2, bool SPLIT, int STF = 0>
struct GemmPairT {
  static constexpr int bn1 = BN1, st1 = ST1, bn2 = BN2, st2 = ST2;
  static constexpr int stf = STF;
  static constexpr bool split = SPLIT;
  static constexpr bool fused = STF > 0 && BN1 == BN2 && AFD_FUSED;
  static constexpr int gate_rows_per_unit = 128;  // gate/up units: 128 gate rows + 128 up rows
};
// Tile shapes: kNarrow (decode micro-batches) and kWide (large micro-batches).
constexpr int kNarrow = 0, kWide = 1;
template <bool FP8, int SHAPE>
struct GemmPair;
template <>
struct GemmPair<false, kNarrow>
    : GemmPairT<AFD_NB_G1_BN, AFD_NB_G1_ST, AFD_NB_G2_BN, AFD_NB_G2_ST, true, AFD_NB_F_ST> {};
template <>
struct GemmPair<false, kWide> : GemmPairT<AFD_WB_G1_BN, AFD_WB_G1_ST, AFD_WB_G2_BN, AFD_WB_G2_ST, true, AFD_WB_F_ST> {};
template <>
struct GemmPair<true, kNarrow> : GemmPairT<AFD_NF_G1_BN, AFD_NF_G1_ST, AFD_NF_G2_BN, AFD_NF_G2_ST, false> {};
template <>
struct GemmPair<true, kWide> : GemmPairT<AFD_WF_G1_BN, AFD_WF_G1_ST, AFD_WF_G2_BN, AFD_WF_G2_ST, false> {};

// Token-tile TMA box height of the gate/up (gemm = 1) or down (gemm = 2) kernel of a shape.
template <int SHAPE>
uint32_t box_rows(bool fp8, int gemm) {
  if (fp8) {
    using P = GemmPair<true, SHAPE>;
    return gemm == 1 ? GemmShape<P::bn1, false, 0>::kBoxRows : GemmShape<P::bn2, false, 1>::kBoxRows;
  }
  using P = GemmPair<false, SHAPE>;
  return gemm == 1 ? GemmShape<P::bn1, false, 0>::kBoxRows : GemmShape<P::bn2, P::split, 1>::kBoxRows;
}

template <bool FP8, int SHAPE>
cudaError_t set_pair_attrs() {
  using P = GemmPair<FP8, SHAPE>;
  if constexpr (P::fused) {
    return set_gemm_attr<P::bn1, (P::fused ? P::stf : 1), FP8, 3, true>();
  } else {
    cudaError_t e = set_gemm_attr<P::bn1, P::st1, FP8, 0, false>();
    if (e != cudaSuccess) return e;
    return set_gemm_attr<P::bn2, P::st2, FP8, 1, P::split>();
  }
}

template <bool FP8>
cudaError_t set_all_gemm_attrs() {
  cudaError_t e = set_pair_attrs<FP8, kNarrow>();
  if (e != cudaSuccess) return e;
  e = set_gemm_attr<kRouterBN, kRouterStages, false, 2, false>();
  if (e != cudaSuccess) return e;
  e = set_gemm_attr<kRouterBNWide, kRouterStages, false, 2, false>();
  if (e != cudaSuccess) return e;
  e = set_pair_attrs<FP8, kWide>();
  if (e != cudaSuccess) return e;
  if constexpr (!FP8) {
    e = set_gemm_attr<kAct16BN, AFD_ACT16_G1_ST, false, 0, false, true>();
    if (e != cudaSuccess) return e;
    e = set_gemm_attr<kAct16BN, AFD_ACT16_G2_ST, false, 1, false, true>();
    if (e != cudaSuccess) return e;
  }
  if constexpr (FP8) {
    e = set_gemm_attr<kOneBN, kOneST, true, 0, false, false, true>();
    if (e != cudaSuccess) return e;
    e = set_gemm_attr<kOneBN, kOneST, true, 1, false, false, true>();
  }
  return e;
}

template <int BN, int ST, bool FP8, int MODE, bool SPLIT, bool ACT16 = false, bool ONE = false>
void launch_gemm(int grid, const CUtensorMap& a, const CUtensorMap& b, const GemmArgs& args, cudaStream_t s,
                 const CUtensorMap* a2 = nullptr, const CUtensorMap* b2 = nullptr) {
  if constexpr (MODE == 3) {
    // the fused kernel's down units wait for act tiles that other CTAs produce, so every CTA of
    // the grid must be resident at once: a cooperative launch guarantees it, or fails (with a
    // launch error that the stage's cudaGetLastError check returns) when it cannot be met
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(kGemmThreads);
    cfg.dynamicSmemBytes = gemm_smem_bytes<BN, ST, SPLIT, MODE>();
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaLaunchKernelEx(&cfg, grouped_gemm_kernel<BN, ST, FP8, MODE, SPLIT, ACT16>, a, b, a2 ? *a2 : a,
                       b2 ? *b2 : b, args);
  } else {
    grouped_gemm_kernel<BN, ST, FP8, MODE, SPLIT, ACT16, ONE>
        <<<grid, kGemmThreads, gemm_smem_bytes<BN, ST, SPLIT, MODE, ONE>(), s>>>(a, b, a2 ? *a2 : a, b2 ? *b2 : b,
                                                                             args);
  }
}

// CTAs of the fused (MODE 3) launch: one per SM when that many fit at once (the kernel holds
// one CTA per SM by its shared memory), else as many as can be co-resident; 0 when the device
// cannot launch it cooperatively.
template <bool FP8>
int fused_grid(int num_sms, int device) {
  using P = GemmPair<FP8, kNarrow>;
  if constexpr (!P::fused) {
    return num_sms;
  } else {
    int coop = 0;
    if (cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, device) != cudaSuccess || !coop) {
      cudaGetLastError();
      return 0;
    }
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, grouped_gemm_kernel<P::bn1, P::stf, FP8, 3, true>,
                                                      kGemmThreads, gemm_smem_bytes<P::bn1, P::stf, true, 3>()) !=
        cudaSuccess) {
      cudaGetLastError();
      return 0;
    }
    return std::min(num_sms, per_sm * num_sms);
  }
}

// K split of the tensor-core router: enough units to cover the SMs and stretches of at most
// kRouterMaxSplitChunks chunks, every split non-empty.
void router_ksplit(int T, int H, int E, int sms, int bn, int* ksplit, int* kc_per) {
  const int kchunks = H / 64;
  const int base = ((T + bn - 1) / bn) * ((E + 127) / 128);
  const int min_split = (kchunks + kRouterMaxSplitChunks - 1) / kRouterMaxSplitChunks;
  const int want = std::max(min_split, std::min(kchunks, (sms + base - 1) / base));
  *kc_per = (kchunks + want - 1) / want;
  *ksplit = (kchunks + *kc_per - 1) / *kc_per;
}

void record(afd_ffn_handle* h, int stage, cudaStream_t s) {
  // a failure here surfaces through the cudaGetLastError check that ends each stage
  if (h->n_events > stage && h->events[stage]) cudaEventRecord(h->events[stage], s);
}

// ------------------------------------------------------------------ stages
// Router on the tensor cores (grouped GEMM, MODE 2): logits [T][E] fp32 into h->part, then the
// warp-per-token top-k.  The hidden states' TMA descriptor is encoded per call (host only).
int run_route(afd_ffn_handle* h, const void* hidden, int T, int32_t* idx, float* w, cudaStream_t s) {
  const afd_ffn_cfg& c = h->cfg;
  CUtensorMap tm_h;
  if (!encode_2d(&tm_h, hidden, false, c.H, static_cast<uint64_t>(T), GemmShape<kRouterBN, false, 2>::kBoxRows))
    return AFD_ERR_INVALID_ARG;
  static_assert(GemmShape<kRouterBN, false, 2>::kBoxRows == GemmShape<kRouterBNWide, false, 2>::kBoxRows,
                "router tiles share the hidden-state map");
  const bool wide = T >= kRouterWideT;
  const int bn = wide ? kRouterBNWide : kRouterBN;
  int ksplit = 1, kc_per = 1;
  router_ksplit(T, c.H, c.E, h->num_sms, bn, &ksplit, &kc_per);
  GemmArgs a{};
  a.G = 1;
  a.single_rows = T;
  a.single_mt = (c.E + 127) / 128;
  a.single_total = ((T + bn - 1) / bn) * a.single_mt * ksplit;
  a.kc_per = kc_per;
  a.K = c.H;
  a.a_rows = c.E;
  a.mt_stride = 128;
  a.second_off = c.E;  // plane stride of the [3][E][H] weights
  a.out = h->part;
  a.out_ld = c.E;
  a.err = h->err;
  record(h, 0, s);
  if (wide)
    launch_gemm<kRouterBNWide, kRouterStages, false, 2, false>(std::min(h->num_sms, a.single_total), h->tm_wr, tm_h, a, s);
  else
    launch_gemm<kRouterBN, kRouterStages, false, 2, false>(std::min(h->num_sms, a.single_total), h->tm_wr, tm_h, a, s);
  record(h, 1, s);
  // selection and gate weights from the summed partial logits, a warp per token
  const float* bias = c.has_router_bias ? h->w.router_bias : nullptr;
  launch_router_topk(h->part, ksplit, bias, T, c.E, c.k, idx, w, s);
  AFD_CUDA(h, cudaGetLastError());
  return AFD_OK;
}

int run_permute(afd_ffn_handle* h, const void* hidden, const int32_t* idx, int T, int32_t* counts, int32_t* offsets,
                int32_t* pos, int32_t* src, cudaStream_t s) {
  const afd_ffn_cfg& c = h->cfg;
  const int nchunks = (T + kChunkTokens - 1) / kChunkTokens;
  record(h, 2, s);
  dispatch_count_kernel<<<nchunks, kCountThreads, 0, s>>>(idx, T, c.k, c.E, pos, h->chunk_counts, h->err);
  dispatch_scan_kernel<<<1, kMaxExperts, 0, s>>>(h->chunk_counts, nchunks, c.E, counts, offsets, h->chunk_base);
  record(h, 3, s);
  const __nv_bfloat16* hb = static_cast<const __nv_bfloat16*>(hidden);
  if (h->fp8)
    gather_rows_kernel<true><<<T, 256, 0, s>>>(hb, idx, h->chunk_base, pos, src, T, c.k, c.E, c.H, c.n_shared,
                                               h->xp, h->xscale);
  else
    gather_rows_kernel<false><<<T, 256, 0, s>>>(hb, idx, h->chunk_base, pos, src, T, c.k, c.E, c.H, c.n_shared,
                                                h->xp, h->xscale, h->act16 ? h->f16_bound : 0.f);
  AFD_CUDA(h, cudaGetLastError());
  return AFD_OK;
}

template <bool FP8, int SHAPE>
void run_gemms(afd_ffn_handle* h, int T, cudaStream_t s) {
  using P = GemmPair<FP8, SHAPE>;
  constexpr bool NARROW = SHAPE == kNarrow;
  const int shape = NARROW ? 0 : 1;  // token-row tensor maps: both wide shapes use 64-row boxes
  const afd_ffn_cfg& c = h->cfg;
  const int R = T * c.k + T;
  GemmArgs g1{};
  g1.single_rows = -1;  // grouped: units come from the device schedule
  g1.grp_rows = h->grp_rows;
  g1.grp_base = h->grp_base;
  g1.unit_base = h->ub1;
  g1.G = h->G;
  g1.K = c.H;
  g1.a_rows = 2 * c.I;
  g1.mt_stride = P::gate_rows_per_unit;
  g1.second_off = c.I;
  g1.out = h->act;
  g1.out_ld = c.I;
  g1.lo_rows = h->R_max;
  // decode streams each weight tile once; large micro-batches share it between N tiles
  g1.a_policy = NARROW ? kEvictFirst : kEvictNormal;
  g1.a_scale = h->w.w13_scale;
  g1.b_scale = h->xscale;
  g1.err = h->err;
  if constexpr (P::fused) {
    // one launch: gate/up units then down units, down units gated by the act-tile counters
    GemmArgs f = g1;
    f.unit_base2 = h->ub2;
    f.tile_base = h->tile_base;
    f.tile_done = h->tile_done;
    f.K2 = c.I;
    f.a_rows2 = c.H;
    f.mt_stride2 = 256;
    f.second_off2 = 128;
    f.out2 = h->Y;
    f.out_ld2 = c.H;
    f.mt1 = c.I / 128;
    record(h, 5, s);
    launch_gemm<P::bn1, (P::fused ? P::stf : 1), FP8, 3, true>(h->fused_grid, h->tm_w13, h->tm_xp[shape], f, s,
                                                                &h->tm_w2, &h->tm_act[shape]);
    record(h, 6, s);
    record(h, 7, s);
    return;
  }
  if constexpr (!FP8 && !NARROW && P::bn1 == kAct16BN && P::bn2 == kAct16BN) {
    // (the device schedule was built with P's N tiles, which the f16 kernels share)
    if (h->act16) {  // single-term down GEMM on f16 activations and the f16 copy of W2
      GemmArgs a1 = g1;
      a1.mt_stride = 128;
      record(h, 5, s);
      launch_gemm<kAct16BN, AFD_ACT16_G1_ST, false, 0, false, true>(h->num_sms, h->tm_w13, h->tm_xp[1], a1, s);
      record(h, 6, s);
      GemmArgs a2 = a1;
      a2.unit_base = h->ub2;
      a2.K = c.I;
      a2.a_rows = c.H;
      a2.mt_stride = 256;
      a2.second_off = 128;
      a2.out = h->Y;
      a2.out_ld = c.H;
      record(h, 7, s);
      launch_gemm<kAct16BN, AFD_ACT16_G2_ST, false, 1, false, true>(h->num_sms, h->tm_w2h, h->tm_act16, a2, s);
      return;
    }
  }
  record(h, 5, s);
  const int grid = h->num_sms;
  launch_gemm<P::bn1, P::st1, FP8, 0, false>(grid, h->tm_w13, h->tm_xp[shape], g1, s);
  record(h, 6, s);
  if (FP8)
    quantize_act_kernel<<<(R + 1) / 2, 256, 0, s>>>(static_cast<const float*>(h->act), R, c.I, h->actq, h->ascale);
  GemmArgs g2 = g1;
  g2.unit_base = h->ub2;
  g2.K = c.I;
  g2.a_rows = c.H;
  g2.mt_stride = 256;
  g2.second_off = 128;  // a down unit: output rows h.. and h+128..
  g2.out = h->Y;
  g2.out_ld = c.H;
  g2.a_scale = h->w.w2_scale;
  g2.b_scale = h->ascale;
  record(h, 7, s);
  launch_gemm<P::bn2, P::st2, FP8, 1, P::split>(grid, h->tm_w2, h->tm_act[shape], g2, s);
}

// W8A8 large micro-batches on the one-accumulator GEMMs: gate/up units of 64 interleaved act
// columns, the activation quantisation, then down units of 128 output rows; both with up to
// kOneBN token rows per unit.
void run_gemms_one(afd_ffn_handle* h, int T, cudaStream_t s) {
  const afd_ffn_cfg& c = h->cfg;
  const int R = T * c.k + T;
  GemmArgs g1{};
  g1.single_rows = -1;
  g1.grp_rows = h->grp_rows;
  g1.grp_base = h->grp_base;
  g1.unit_base = h->ub1;
  g1.G = h->G;
  g1.K = c.H;
  g1.a_rows = 2 * c.I;     // scale rows per expert
  g1.mt_stride = 64;       // act columns per unit
  g1.second_off = c.I;     // up row = gate row + I
  g1.out = h->act;         // fp32 SwiGLU rows
  g1.out_ld = c.I;
  g1.a_policy = kEvictNormal;
  g1.a_scale = h->w.w13_scale;
  g1.b_scale = h->xscale;  // hidden row scales
  g1.err = h->err;
  record(h, 5, s);
  launch_gemm<kOneBN, kOneST, true, 0, false, false, true>(h->num_sms, h->tm_w13i, h->tm_xp[1], g1, s);
  record(h, 6, s);
  quantize_act_kernel<<<(R + 1) / 2, 256, 0, s>>>(static_cast<const float*>(h->act), R, c.I, h->actq, h->ascale);
  GemmArgs g2 = g1;
  g2.unit_base = h->ub2;
  g2.K = c.I;
  g2.a_rows = c.H;
  g2.mt_stride = 128;      // output rows per unit
  g2.second_off = 0;
  g2.out = h->Y;
  g2.out_ld = c.H;
  g2.a_scale = h->w.w2_scale;
  g2.b_scale = h->ascale;
  record(h, 7, s);
  launch_gemm<kOneBN, kOneST, true, 1, false, false, true>(h->num_sms, h->tm_w2, h->tm_act[1], g2, s);
}

int run_expert_gemm(afd_ffn_handle* h, const int32_t* offsets, int T, cudaStream_t s) {
  const afd_ffn_cfg& c = h->cfg;
  const bool narrow = use_narrow(h, T);
  const int shape = narrow ? kNarrow : kWide;
  if (!narrow && h->one) {
    record(h, 4, s);
    build_schedule_kernel<<<1, 512, 0, s>>>(offsets, c.E, c.n_shared, T, c.k, kOneBN, kOneBN, c.I / 64, c.H / 128,
                                            h->grp_rows, h->grp_base, h->ub1, h->ub2, h->tile_base, h->tile_done,
                                            h->err);
    run_gemms_one(h, T, s);
    AFD_CUDA(h, cudaGetLastError());
    return AFD_OK;
  }
  int bn1, bn2, gate_rows;
  auto pick = [&](auto p) {
    using P = decltype(p);
    bn1 = P::bn1;
    bn2 = P::bn2;
    gate_rows = P::gate_rows_per_unit;
  };
  if (h->fp8) {
    if (shape == kNarrow) pick(GemmPair<true, kNarrow>{});
    else pick(GemmPair<true, kWide>{});
  } else {
    if (shape == kNarrow) pick(GemmPair<false, kNarrow>{});
    else pick(GemmPair<false, kWide>{});
  }
  record(h, 4, s);
  build_schedule_kernel<<<1, 512, 0, s>>>(offsets, c.E, c.n_shared, T, c.k, bn1, bn2, c.I / gate_rows, c.H / 256,
                                          h->grp_rows, h->grp_base, h->ub1, h->ub2, h->tile_base, h->tile_done,
                                          h->err);
  if (h->fp8) {
    if (shape == kNarrow) run_gemms<true, kNarrow>(h, T, s);
    else run_gemms<true, kWide>(h, T, s);
  } else {
    if (shape == kNarrow) run_gemms<false, kNarrow>(h, T, s);
    else run_gemms<false, kWide>(h, T, s);
  }
  AFD_CUDA(h, cudaGetLastError());
  return AFD_OK;
}

int run_combine(afd_ffn_handle* h, const float* w, const int32_t* pos, int T, void* out, cudaStream_t s) {
  const afd_ffn_cfg& c = h->cfg;
  record(h, 8, s);
  if (h->fp8)  // H is a multiple of 256
    combine8_kernel<<<dim3(static_cast<unsigned>(T), static_cast<unsigned>(combine8_slices(T, c.H))), kCombine8Threads,
                      0, s>>>(reinterpret_cast<const __nv_bfloat16*>(h->Y), nullptr, w, pos, T, c.k, c.H, T * c.k,
                              c.n_shared, static_cast<__nv_bfloat16*>(out), h->err);
  else
    combine_kernel<float><<<dim3(static_cast<unsigned>(T), static_cast<unsigned>(combine_slices(T, c.H))), 256, 0, s>>>(
        h->Y, nullptr, w, pos, T, c.k, c.H, T * c.k, c.n_shared, static_cast<__nv_bfloat16*>(out), h->err);
  record(h, 9, s);
  AFD_CUDA(h, cudaGetLastError());
  return AFD_OK;
}

int validate_cfg(const afd_ffn_cfg* c) {
  if (c->T_max < 1 || c->H < 1 || c->E < 1 || c->k < 1 || c->I < 1) return AFD_ERR_INVALID_ARG;
  if (c->n_shared != 0 && c->n_shared != 1) return AFD_ERR_INVALID_ARG;
  if (c->has_router_bias != 0 && c->has_router_bias != 1) return AFD_ERR_INVALID_ARG;
  if (c->weight_dtype != AFD_DT_BF16 && c->weight_dtype != AFD_DT_FP8_E4M3) return AFD_ERR_INVALID_ARG;
  if (c->act_dtype != c->weight_dtype) return AFD_ERR_UNSUPPORTED;
  if (c->k > c->E) return AFD_ERR_INVALID_ARG;
  if (c->E > kMaxExperts || c->k > 32) return AFD_ERR_UNSUPPORTED;
  if (c->H % 256 != 0 || c->I % 128 != 0) return AFD_ERR_UNSUPPORTED;
  // dispatched rows and per-row offsets must fit int32; TMA row coordinates too
  const long long rows = static_cast<long long>(c->T_max) * (c->k + 1);
  if (rows > (1LL << 30) || static_cast<long long>(c->E + 1) * 2 * c->I > (1LL << 30) ||
      static_cast<long long>(c->E + 1) * c->H > (1LL << 30))
    return AFD_ERR_UNSUPPORTED;
  return AFD_OK;
}

int validate_weights(const afd_ffn_cfg* c, const afd_ffn_weights* w) {
  if (!w->router_w || !w->w13 || !w->w2) return AFD_ERR_INVALID_ARG;
  if (c->has_router_bias && !w->router_bias) return AFD_ERR_INVALID_ARG;
  if (!c->has_router_bias && w->router_bias) return AFD_ERR_INVALID_ARG;
  const bool fp8 = c->weight_dtype == AFD_DT_FP8_E4M3;
  if (fp8 && (!w->w13_scale || !w->w2_scale)) return AFD_ERR_INVALID_ARG;
  if (!fp8 && (w->w13_scale || w->w2_scale)) return AFD_ERR_INVALID_ARG;
  if (!aligned16(w->router_w) || !aligned16(w->w13) || !aligned16(w->w2)) return AFD_ERR_INVALID_ARG;
  return AFD_OK;
}

}  // namespace

// ====================================================================== C ABI
extern "C" {

const char* afd_ffn_strerror(int status) {
  switch (status) {
    case AFD_OK: return "ok";
    case AFD_ERR_INVALID_ARG: return "invalid argument";
    case AFD_ERR_UNSUPPORTED: return "configuration not supported";
    case AFD_ERR_T_TOO_LARGE: return "T exceeds the handle's T_max";
    case AFD_ERR_CUDA: return "CUDA call failed";
    case AFD_ERR_DEVICE_FLAG: return "device skipped invalid data (expert index or position)";
    case AFD_ERR_DEVICE_TIMEOUT: return "a bounded device wait timed out";
    case AFD_ERR_NO_DEVICE: return "no sm_100 CUDA device is current";
    case AFD_ERR_TIMEOUT: return "a bounded host wait timed out";
    case AFD_ERR_STOPPED: return "the FFN service stopped before serving the slot";
    default: return "unknown status";
  }
}

int afd_ffn_last_cuda_error(const afd_ffn_handle* h) { return h ? h->last_cuda_error : g_create_cuda_error; }

int afd_ffn_get_info(const afd_ffn_handle* h, afd_ffn_cfg* cfg, int32_t* device) {
  if (!h) return AFD_ERR_INVALID_ARG;
  if (cfg) *cfg = h->cfg;
  if (device) *device = h->device;
  return AFD_OK;
}

int afd_ffn_create(const afd_ffn_cfg* cfg, const afd_ffn_weights* weights, afd_ffn_handle** out) {
  return afd_ffn_create_ex(cfg, weights, 0u, out);
}

int afd_ffn_create_ex(const afd_ffn_cfg* cfg, const afd_ffn_weights* weights, uint32_t flags,
                      afd_ffn_handle** out) {
  if (!out) return AFD_ERR_INVALID_ARG;
  *out = nullptr;
  if (!cfg || !weights) return AFD_ERR_INVALID_ARG;
  if (flags & ~static_cast<uint32_t>(AFD_CREATE_NO_W2_COPY)) return AFD_ERR_INVALID_ARG;
  int st = validate_cfg(cfg);
  if (st != AFD_OK) return st;
  if ((st = validate_weights(cfg, weights)) != AFD_OK) return st;
  g_create_cuda_error = 0;

  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) { g_create_cuda_error = e; return AFD_ERR_NO_DEVICE; }
  int major = 0, minor = 0, sms = 0;
  AFD_CUDA(nullptr, cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev));
  AFD_CUDA(nullptr, cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev));
  AFD_CUDA(nullptr, cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  if (major != 10 || minor != 0) return AFD_ERR_NO_DEVICE;
  if (!get_encode()) return AFD_ERR_NO_DEVICE;

  afd_ffn_handle* h = new (std::nothrow) afd_ffn_handle();
  if (!h) return AFD_ERR_INVALID_ARG;
  h->cfg = *cfg;
  h->w = *weights;
  h->device = dev;
  h->num_sms = sms;
  h->fp8 = cfg->weight_dtype == AFD_DT_FP8_E4M3;
  h->G = cfg->E + cfg->n_shared;
  h->R_max = cfg->T_max * (cfg->k + 1);

  const afd_ffn_cfg& c = h->cfg;
  size_t part = 0;  // partial router logits [ksplit][T][E], largest over T <= T_max
  for (int T = 1; T <= c.T_max; ++T) {
    int ks, per;
    router_ksplit(T, c.H, c.E, sms, T >= kRouterWideT ? kRouterBNWide : kRouterBN, &ks, &per);
    part = std::max(part, static_cast<size_t>(ks) * T * c.E);
  }
  h->part_floats = part;

  // one allocation, 256-byte aligned pieces
  const size_t R = h->R_max, Tm = c.T_max, wb = h->fp8 ? 1 : 2;
  struct Piece { void** p; size_t bytes; };
  void* act_p = nullptr;
  Piece pieces[] = {
      {reinterpret_cast<void**>(&h->part), part * 4},
      {reinterpret_cast<void**>(&h->idx), Tm * c.k * 4},
      {reinterpret_cast<void**>(&h->wts), Tm * c.k * 4},
      {&h->wr_planes, 3 * static_cast<size_t>(c.E) * c.H * 2},
      {reinterpret_cast<void**>(&h->counts), static_cast<size_t>(c.E) * 4},
      {reinterpret_cast<void**>(&h->offsets), static_cast<size_t>(c.E + 1) * 4},
      {reinterpret_cast<void**>(&h->pos), Tm * c.k * 4},
      {reinterpret_cast<void**>(&h->src), Tm * c.k * 4},
      {reinterpret_cast<void**>(&h->chunk_counts), (Tm + kChunkTokens - 1) / kChunkTokens * c.E * 4},
      {reinterpret_cast<void**>(&h->chunk_base), (Tm + kChunkTokens - 1) / kChunkTokens * c.E * 4},
      {reinterpret_cast<void**>(&h->grp_rows), static_cast<size_t>(h->G) * 4},
      {reinterpret_cast<void**>(&h->grp_base), static_cast<size_t>(h->G) * 4},
      {reinterpret_cast<void**>(&h->ub1), static_cast<size_t>(h->G + 1) * 4},
      {reinterpret_cast<void**>(&h->ub2), static_cast<size_t>(h->G + 1) * 4},
      {reinterpret_cast<void**>(&h->tile_base), static_cast<size_t>(h->G) * 4},
      {reinterpret_cast<void**>(&h->tile_done), static_cast<size_t>(R / 16 + h->G + 1) * 4},
      {reinterpret_cast<void**>(&h->xp), R * c.H * wb},
      {reinterpret_cast<void**>(&h->xscale), R * 4},
      {&act_p, R * c.I * 4},  // fp32 (W8A8) or two bf16 planes (hi, lo)
      {reinterpret_cast<void**>(&h->actq), h->fp8 ? R * c.I : 0},
      {reinterpret_cast<void**>(&h->ascale), R * 4},
      {reinterpret_cast<void**>(&h->Y), R * c.H * 4},
      {reinterpret_cast<void**>(&h->err), 256},
      {&h->hin, Tm * c.H * 2},
      {&h->hout, Tm * c.H * 2},
      {&h->hin2, Tm * c.H * 2},
      {&h->hout2, Tm * c.H * 2},
  };
  size_t total = 0;
  for (auto& p : pieces) total += (p.bytes + 255) & ~size_t(255);
  e = cudaMalloc(&h->ws, total);
  if (e != cudaSuccess) { delete h; return cuda_fail(nullptr, e); }
  e = cudaMemset(h->ws, 0, total);
  if (e != cudaSuccess) { cudaFree(h->ws); delete h; return cuda_fail(nullptr, e); }
  size_t off = 0;
  for (auto& p : pieces) {
    *p.p = p.bytes ? static_cast<uint8_t*>(h->ws) + off : nullptr;
    off += (p.bytes + 255) & ~size_t(255);
  }
  h->act = act_p;

  const uint64_t G = h->G;
  // token-row maps: box heights must match GemmShape<...>::kBoxRows of the kernels using them
  const void* act_src = h->fp8 ? static_cast<const void*>(h->actq) : h->act;
  const uint64_t act_rows = h->fp8 ? R : 2 * R;
  const uint32_t box_xp[2] = {box_rows<kNarrow>(h->fp8, 1), box_rows<kWide>(h->fp8, 1)};
  const uint32_t box_act[2] = {box_rows<kNarrow>(h->fp8, 2), box_rows<kWide>(h->fp8, 2)};

  bool ok = encode_2d(&h->tm_w13, weights->w13, h->fp8, c.H, G * 2 * c.I, 128) &&
            encode_2d(&h->tm_w2, weights->w2, h->fp8, c.I, G * c.H, 128) &&
            encode_2d(&h->tm_xp[0], h->xp, h->fp8, c.H, R, box_xp[0]) &&
            encode_2d(&h->tm_xp[1], h->xp, h->fp8, c.H, R, box_xp[1]) &&
            encode_2d(&h->tm_act[0], act_src, h->fp8, c.I, act_rows, box_act[0]) &&
            encode_2d(&h->tm_act[1], act_src, h->fp8, c.I, act_rows, box_act[1]) &&
            encode_2d(&h->tm_wr, h->wr_planes, false, c.H, 3 * static_cast<uint64_t>(c.E), 128);
  if (!ok) { cudaFree(h->ws); delete h; return AFD_ERR_INVALID_ARG; }
  // bf16 handles that can see large micro-batches keep an f16 copy of W2 for the single-term
  // down GEMM (unless a weight exceeds the f16 range; then the two-term bf16 path stays)
  if (AFD_ACT16 && !h->fp8 && !(flags & AFD_CREATE_NO_W2_COPY) &&
      static_cast<int64_t>(c.T_max) * c.k > 32 * static_cast<int64_t>(c.E)) {
    const size_t n = G * c.H * static_cast<size_t>(c.I);
    e = cudaMalloc(&h->w2h, n * 2);
    if (e != cudaSuccess) { cudaFree(h->ws); delete h; return cuda_fail(nullptr, e); }
    bf16_to_f16_kernel<<<4 * h->num_sms, 256>>>(static_cast<const __nv_bfloat16*>(weights->w2),
                                                static_cast<__half*>(h->w2h), n, h->err);
    int overflow = 0;
    e = cudaGetLastError();
    if (e == cudaSuccess) e = cudaMemcpy(&overflow, h->err, sizeof(int), cudaMemcpyDeviceToHost);
    if (e == cudaSuccess) e = cudaMemset(h->err, 0, sizeof(int));
    if (e != cudaSuccess) { cudaFree(h->w2h); cudaFree(h->ws); delete h; return cuda_fail(nullptr, e); }
    h->act16 = overflow == 0 &&
               encode_2d(&h->tm_w2h, h->w2h, false, c.I, G * c.H, 128) &&
               encode_2d(&h->tm_act16, h->act, false, c.I, R, GemmShape<kAct16BN, false, 1>::kBoxRows);
    if (!h->act16) {
      cudaFree(h->w2h);
      h->w2h = nullptr;
    } else {
      // bound of the SwiGLU output per unit of ||x||^2, for the f16 row scales
      unsigned* c_bits = reinterpret_cast<unsigned*>(h->err) + 1;
      w13_norm_bound_kernel<<<4 * h->num_sms, 256>>>(static_cast<const __nv_bfloat16*>(weights->w13),
                                                     static_cast<int>(G), c.I, c.H, c_bits);
      unsigned bits = 0;
      e = cudaGetLastError();
      if (e == cudaSuccess) e = cudaMemcpy(&bits, c_bits, sizeof(unsigned), cudaMemcpyDeviceToHost);
      if (e == cudaSuccess) e = cudaMemset(c_bits, 0, sizeof(unsigned));
      if (e != cudaSuccess) { cudaFree(h->w2h); cudaFree(h->ws); delete h; return cuda_fail(nullptr, e); }
      float C = 0.f;
      std::memcpy(&C, &bits, sizeof(float));
      // a zero (or NaN) bound still gives every row the scale 1
      h->f16_bound = std::max(2.0f * C / 32768.0f, 1e-30f);
    }
  }
  // large W8A8 micro-batches run the one-accumulator GEMMs, whose gate/up side reads W13 through
  // the interleaved 5-D view
  if (AFD_ONE && h->fp8 && static_cast<int64_t>(c.T_max) * c.k > 32 * static_cast<int64_t>(c.E)) {
    if (!encode_w13_interleaved(&h->tm_w13i, weights->w13, h->fp8, c.H, c.I, G)) {
      if (h->w2h) cudaFree(h->w2h);
      cudaFree(h->ws);
      delete h;
      return AFD_ERR_INVALID_ARG;
    }
    h->one = true;
  }
  e = h->fp8 ? set_all_gemm_attrs<true>() : set_all_gemm_attrs<false>();
  if (e != cudaSuccess) { cudaFree(h->ws); if (h->w2h) cudaFree(h->w2h); delete h; return cuda_fail(nullptr, e); }
  h->fused_grid = h->fp8 ? fused_grid<true>(h->num_sms, dev) : fused_grid<false>(h->num_sms, dev);
  if (h->fused_grid < 1) { cudaFree(h->ws); if (h->w2h) cudaFree(h->w2h); delete h; return AFD_ERR_UNSUPPORTED; }
  router_split_planes_kernel<<<256, 256>>>(weights->router_w, static_cast<size_t>(c.E) * c.H,
                                           static_cast<__nv_bfloat16*>(h->wr_planes));
  e = cudaGetLastError();
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&h->copy_in, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&h->copy_out, cudaStreamNonBlocking);
  for (int i = 0; i < 2 && e == cudaSuccess; ++i) {
    e = cudaEventCreateWithFlags(&h->ev_in[i], cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&h->ev_done[i], cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&h->ev_out[i], cudaEventDisableTiming);
  }
  if (e != cudaSuccess) { afd_ffn_destroy(h); return cuda_fail(nullptr, e); }
  *out = h;
  return AFD_OK;
}

void afd_ffn_destroy(afd_ffn_handle* h) {
  if (!h) return;
  cudaDeviceSynchronize();
  for (int i = 0; i < 2; ++i) {
    if (h->ev_in[i]) cudaEventDestroy(h->ev_in[i]);
    if (h->ev_done[i]) cudaEventDestroy(h->ev_done[i]);
    if (h->ev_out[i]) cudaEventDestroy(h->ev_out[i]);
  }
  if (h->copy_in) cudaStreamDestroy(h->copy_in);
  if (h->copy_out) cudaStreamDestroy(h->copy_out);
  if (h->w2h) cudaFree(h->w2h);
  cudaFree(h->ws);
  delete h;
}

int afd_ffn_route(afd_ffn_handle* h, const void* hidden, int32_t T, int32_t* topk_idx, float* topk_w, void* stream) {
  if (!h) return AFD_ERR_INVALID_ARG;
  int st = check_T(h, T);
  if (st != AFD_OK) return st;
  if (T == 0) return AFD_OK;
  if (!hidden || !topk_idx || !topk_w || !aligned16(hidden)) return AFD_ERR_INVALID_ARG;
  if ((st = check_device(h)) != AFD_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  h->last_stream = s;
  return run_route(h, hidden, T, topk_idx, topk_w, s);
}

int afd_ffn_permute(afd_ffn_handle* h, const void* hidden, const int32_t* topk_idx, int32_t T, int32_t* counts,
                    int32_t* offsets, int32_t* pos, int32_t* src, void* stream) {
  if (!h) return AFD_ERR_INVALID_ARG;
  int st = check_T(h, T);
  if (st != AFD_OK) return st;
  if (!hidden || !topk_idx || !counts || !offsets || !pos || !src || !aligned16(hidden)) return AFD_ERR_INVALID_ARG;
  if ((st = check_device(h)) != AFD_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  h->last_stream = s;
  if (T == 0) {  // no pairs: zero counts and offsets
    AFD_CUDA(h, cudaMemsetAsync(counts, 0, sizeof(int32_t) * h->cfg.E, s));
    AFD_CUDA(h, cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (h->cfg.E + 1), s));
    return AFD_OK;
  }
  return run_permute(h, hidden, topk_idx, T, counts, offsets, pos, src, s);
}

int afd_ffn_expert_gemm(afd_ffn_handle* h, const int32_t* offsets, int32_t T, float* Y, float* Ys, void* stream) {
  if (!h) return AFD_ERR_INVALID_ARG;
  int st = check_T(h, T);
  if (st != AFD_OK) return st;
  if (!offsets) return AFD_ERR_INVALID_ARG;
  if (Ys && h->cfg.n_shared == 0) return AFD_ERR_INVALID_ARG;
  if ((st = check_device(h)) != AFD_OK) return st;
  if (T == 0) return AFD_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  h->last_stream = s;
  if ((st = run_expert_gemm(h, offsets, T, s)) != AFD_OK) return st;
  const size_t H = h->cfg.H, rk = static_cast<size_t>(T) * h->cfg.k;
  if (h->fp8) {  // the W8A8 expert outputs are held as bf16: widen them on the way out
    const __nv_bfloat16* yb = reinterpret_cast<const __nv_bfloat16*>(h->Y);
    if (Y) bf16_to_f32_kernel<<<4 * h->num_sms, 256, 0, s>>>(yb, Y, rk * H);
    if (Ys) bf16_to_f32_kernel<<<4 * h->num_sms, 256, 0, s>>>(yb + rk * H, Ys, static_cast<size_t>(T) * H);
    AFD_CUDA(h, cudaGetLastError());
    return AFD_OK;
  }
  if (Y) AFD_CUDA(h, cudaMemcpyAsync(Y, h->Y, rk * H * 4, cudaMemcpyDeviceToDevice, s));
  if (Ys) AFD_CUDA(h, cudaMemcpyAsync(Ys, h->Y + rk * H, static_cast<size_t>(T) * H * 4, cudaMemcpyDeviceToDevice, s));
  return AFD_OK;
}

int afd_ffn_combine(afd_ffn_handle* h, const float* topk_w, const int32_t* pos, int32_t T, void* out, void* stream) {
  if (!h) return AFD_ERR_INVALID_ARG;
  int st = check_T(h, T);
  if (st != AFD_OK) return st;
  if (T == 0) return AFD_OK;
  if (!topk_w || !pos || !out || !aligned16(out)) return AFD_ERR_INVALID_ARG;
  if ((st = check_device(h)) != AFD_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  h->last_stream = s;
  return run_combine(h, topk_w, pos, T, out, s);
}

int afd_ffn_forward(afd_ffn_handle* h, const void* hidden, int32_t T, void* out, void* stream) {
  if (!h) return AFD_ERR_INVALID_ARG;
  int st = check_T(h, T);
  if (st != AFD_OK) return st;
  if (T == 0) return AFD_OK;
  if (!hidden || !out || !aligned16(hidden) || !aligned16(out)) return AFD_ERR_INVALID_ARG;
  if ((st = check_device(h)) != AFD_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  h->last_stream = s;
  if ((st = run_route(h, hidden, T, h->idx, h->wts, s)) != AFD_OK) return st;
  if ((st = run_permute(h, hidden, h->idx, T, h->counts, h->offsets, h->pos, h->src, s)) != AFD_OK) return st;
  if ((st = run_expert_gemm(h, h->offsets, T, s)) != AFD_OK) return st;
  return run_combine(h, h->wts, h->pos, T, out, s);
}

int afd_ffn_forward_host(afd_ffn_handle* h, const void* hidden_host, int32_t T, void* out_host, void* stream) {
  if (!h) return AFD_ERR_INVALID_ARG;
  int st = check_T(h, T);
  if (st != AFD_OK) return st;
  if (T == 0) return AFD_OK;
  if (!hidden_host || !out_host) return AFD_ERR_INVALID_ARG;
  if ((st = check_device(h)) != AFD_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t bytes = static_cast<size_t>(T) * h->cfg.H * 2;
  AFD_CUDA(h, cudaMemcpyAsync(h->hin, hidden_host, bytes, cudaMemcpyHostToDevice, s));
  if ((st = afd_ffn_forward(h, h->hin, T, h->hout, stream)) != AFD_OK) return st;
  AFD_CUDA(h, cudaMemcpyAsync(out_host, h->hout, bytes, cudaMemcpyDeviceToHost, s));
  AFD_CUDA(h, cudaStreamSynchronize(s));
  return AFD_OK;
}

int afd_ffn_forward_host_batches(afd_ffn_handle* h, const void* const* hidden_host, void* const* out_host,
                                 int32_t n_batches, int32_t T, void* stream) {
  if (!h || n_batches < 0) return AFD_ERR_INVALID_ARG;
  int st = check_T(h, T);
  if (st != AFD_OK) return st;
  if (T == 0 || n_batches == 0) return AFD_OK;
  if (!hidden_host || !out_host) return AFD_ERR_INVALID_ARG;
  for (int i = 0; i < n_batches; ++i)
    if (!hidden_host[i] || !out_host[i]) return AFD_ERR_INVALID_ARG;
  if ((st = check_device(h)) != AFD_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t bytes = static_cast<size_t>(T) * h->cfg.H * 2;
  void* din[2] = {h->hin, h->hin2};
  void* dout[2] = {h->hout, h->hout2};
  // batch i uses staging slot i % 2.  copy_in: H2D of batch i once the layer of batch i-2 has
  // consumed the slot; compute: the layer of batch i once its input landed and the D2H of
  // batch i-2 has drained the output slot; copy_out: D2H of batch i once its layer is done.
  for (int i = 0; i < n_batches; ++i) {
    const int b = i & 1;
    if (i >= 2) AFD_CUDA(h, cudaStreamWaitEvent(h->copy_in, h->ev_done[b], 0));
    AFD_CUDA(h, cudaMemcpyAsync(din[b], hidden_host[i], bytes, cudaMemcpyHostToDevice, h->copy_in));
    AFD_CUDA(h, cudaEventRecord(h->ev_in[b], h->copy_in));
    AFD_CUDA(h, cudaStreamWaitEvent(s, h->ev_in[b], 0));
    if (i >= 2) AFD_CUDA(h, cudaStreamWaitEvent(s, h->ev_out[b], 0));
    if ((st = afd_ffn_forward(h, din[b], T, dout[b], stream)) != AFD_OK) return st;
    AFD_CUDA(h, cudaEventRecord(h->ev_done[b], s));
    AFD_CUDA(h, cudaStreamWaitEvent(h->copy_out, h->ev_done[b], 0));
    AFD_CUDA(h, cudaMemcpyAsync(out_host[i], dout[b], bytes, cudaMemcpyDeviceToHost, h->copy_out));
    AFD_CUDA(h, cudaEventRecord(h->ev_out[b], h->copy_out));
  }
  AFD_CUDA(h, cudaStreamSynchronize(h->copy_out));
  AFD_CUDA(h, cudaStreamSynchronize(s));
  return AFD_OK;
}

int afd_ffn_set_stage_events(afd_ffn_handle* h, void* const* events, int32_t n_events) {
  if (!h || n_events < 0 || n_events > AFD_FFN_NUM_STAGES + 1) return AFD_ERR_INVALID_ARG;
  if (n_events > 0 && !events) return AFD_ERR_INVALID_ARG;
  for (int i = 0; i < n_events; ++i) h->events[i] = static_cast<cudaEvent_t>(events[i]);  // NULL: skipped
  h->n_events = n_events;
  return AFD_OK;
}

int afd_ffn_get_error(afd_ffn_handle* h) {
  if (!h) return AFD_ERR_INVALID_ARG;
  AFD_CUDA(h, cudaStreamSynchronize(h->last_stream));
  int word = 0;
  AFD_CUDA(h, cudaMemcpy(&word, h->err, sizeof(int), cudaMemcpyDeviceToHost));
  AFD_CUDA(h, cudaMemset(h->err, 0, sizeof(int)));
  if (word & kErrTimeout) return AFD_ERR_DEVICE_TIMEOUT;
  if (word) return AFD_ERR_DEVICE_FLAG;
  return AFD_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------- allocation-free router
// Scratch of afd_ffn_route_static: partial router logits.  File-scope device array; host code
// only ever sees its host-side shadow, so the device address is looked up once per device.
static __device__ __align__(256) float g_route_scratch[AFD_FFN_ROUTE_STATIC_SCRATCH_FLOATS];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_route_scratch_mu;
float* g_route_scratch_dev[kMaxDevices] = {};

// Device address of g_route_scratch on the current device (set-up on the first call).
int route_scratch(float** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(nullptr, e);
  if (dev < 0 || dev >= kMaxDevices) return AFD_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_route_scratch_mu);
  if (!g_route_scratch_dev[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_route_scratch);
    if (e != cudaSuccess) return cuda_fail(nullptr, e);
    g_route_scratch_dev[dev] = static_cast<float*>(p);
  }
  *out = g_route_scratch_dev[dev];
  return AFD_OK;
}
}  // namespace

extern "C" int afd_ffn_route_static(const void* hidden, const float* router_w, const float* router_bias,
                                    int32_t T, int32_t H, int32_t E, int32_t k, int32_t* topk_idx,
                                    float* topk_w, void* stream) {
  if (T < 0 || H < kRtK || H % kRtK != 0 || E < 1 || E > kMaxExperts || k < 1 || k > E || k > 32)
    return AFD_ERR_INVALID_ARG;
  if (static_cast<long long>(T) * E > AFD_FFN_ROUTE_STATIC_SCRATCH_FLOATS) return AFD_ERR_UNSUPPORTED;
  if (T == 0) return AFD_OK;
  if (!hidden || !router_w || !topk_idx || !topk_w || !aligned16(hidden) || !aligned16(router_w))
    return AFD_ERR_INVALID_ARG;
  float* part = nullptr;
  int st = route_scratch(&part);
  if (st != AFD_OK) return st;
  int sms = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return cuda_fail(nullptr, e);
  int nsplit = 1, per = 1;
  router_split(T, H, E, sms, &nsplit, &per);
  const long long cap = AFD_FFN_ROUTE_STATIC_SCRATCH_FLOATS / (static_cast<long long>(T) * E);
  if (nsplit > cap) {  // narrow the split of H until the partials fit the scratch
    const int kt = H / kRtK;
    per = (kt + static_cast<int>(cap) - 1) / static_cast<int>(cap);
    nsplit = (kt + per - 1) / per;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  dim3 grid((E + kRtExp - 1) / kRtExp, (T + kRtTok - 1) / kRtTok, nsplit);
  router_logits_kernel<<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(hidden), router_w, part, T, H, E, per);
  launch_router_topk(part, nsplit, router_bias, T, E, k, topk_idx, topk_w, s);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(nullptr, e);
  return AFD_OK;
}

// ---------------------------------------------------------------------- expert parallelism
// Building blocks of an expert-parallel layer whose exchange runs outside the library (the
// dispatch/combine all-to-all of A/F 分离, section 机制): dispatch order and rows without a
// handle, a handle's experts on rows that arrive already grouped by expert, row-block moves,
// and the weighted combine of external expert outputs.  The allocation-free calls share one
// file-scope device error word (indices outside [0, E) and positions out of range are skipped
// and counted there; afd_ffn_rows_error reads and clears it).
static __device__ int g_rows_err;

namespace {
std::mutex g_rows_err_mu;
int* g_rows_err_dev[kMaxDevices] = {};

int rows_err_word(int** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(nullptr, e);
  if (dev < 0 || dev >= kMaxDevices) return AFD_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_rows_err_mu);
  if (!g_rows_err_dev[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_rows_err);
    if (e != cudaSuccess) return cuda_fail(nullptr, e);
    g_rows_err_dev[dev] = static_cast<int*>(p);
  }
  *out = g_rows_err_dev[dev];
  return AFD_OK;
}
}  // namespace

extern "C" int afd_ffn_dispatch_rows(const void* hidden, const int32_t* topk_idx, int32_t T, int32_t k, int32_t E,
                                     int32_t H, int32_t* counts, int32_t* offsets, int32_t* pos, int32_t* src,
                                     void* rows, int32_t* scratch, void* stream) {
  if (T < 0 || k < 1 || k > 32 || E < 1 || E > kMaxExperts || k > E || H < 8 || H % 8 != 0) return AFD_ERR_INVALID_ARG;
  if (!counts || !offsets || !scratch) return AFD_ERR_INVALID_ARG;
  if (T > 0 && (!hidden || !topk_idx || !pos || !src || !rows || !aligned16(hidden) || !aligned16(rows)))
    return AFD_ERR_INVALID_ARG;
  if (static_cast<long long>(T) * k > (1LL << 30)) return AFD_ERR_UNSUPPORTED;
  int* err = nullptr;
  int st = rows_err_word(&err);
  if (st != AFD_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int nchunks = (T + kChunkTokens - 1) / kChunkTokens;
  int32_t* chunk_counts = scratch;
  int32_t* chunk_base = scratch + static_cast<size_t>(nchunks) * E;
  if (T > 0)
    dispatch_count_kernel<<<nchunks, kCountThreads, 0, s>>>(topk_idx, T, k, E, pos, chunk_counts, err);
  dispatch_scan_kernel<<<1, kMaxExperts, 0, s>>>(chunk_counts, nchunks, E, counts, offsets, chunk_base);
  if (T > 0)
    gather_rows_kernel<false><<<T, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(hidden), topk_idx, chunk_base, pos,
                                                src, T, k, E, H, 0, static_cast<uint8_t*>(rows), nullptr);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(nullptr, e);
  return AFD_OK;
}

extern "C" int afd_ffn_dispatch_rows_fp8(const void* hidden, const int32_t* topk_idx, int32_t T, int32_t k, int32_t E,
                                         int32_t H, int32_t with_shared, int32_t* counts, int32_t* offsets,
                                         int32_t* pos, int32_t* src, void* rows, float* row_scale, int32_t* scratch,
                                         void* stream) {
  if (T < 0 || k < 1 || k > 32 || E < 1 || E > kMaxExperts || k > E || H < 16 || H % 16 != 0) return AFD_ERR_INVALID_ARG;
  if (with_shared != 0 && with_shared != 1) return AFD_ERR_INVALID_ARG;
  if (!counts || !offsets || !scratch) return AFD_ERR_INVALID_ARG;
  if (T > 0 && (!hidden || !topk_idx || !pos || !src || !rows || !row_scale || !aligned16(hidden) || !aligned16(rows)))
    return AFD_ERR_INVALID_ARG;
  if (static_cast<long long>(T) * (k + 1) > (1LL << 30)) return AFD_ERR_UNSUPPORTED;
  int* err = nullptr;
  int st = rows_err_word(&err);
  if (st != AFD_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int nchunks = (T + kChunkTokens - 1) / kChunkTokens;
  int32_t* chunk_counts = scratch;
  int32_t* chunk_base = scratch + static_cast<size_t>(nchunks) * E;
  if (T > 0)
    dispatch_count_kernel<<<nchunks, kCountThreads, 0, s>>>(topk_idx, T, k, E, pos, chunk_counts, err);
  dispatch_scan_kernel<<<1, kMaxExperts, 0, s>>>(chunk_counts, nchunks, E, counts, offsets, chunk_base);
  if (T > 0)
    gather_rows_kernel<true><<<T, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(hidden), topk_idx, chunk_base, pos,
                                               src, T, k, E, H, with_shared, static_cast<uint8_t*>(rows), row_scale);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(nullptr, e);
  return AFD_OK;
}

extern "C" int afd_ffn_expert_rows_fp8(afd_ffn_handle* h, const void* rows, const float* row_scale,
                                       const int32_t* counts, int32_t n_rows, void* Y, void* stream) {
  if (!h) return AFD_ERR_INVALID_ARG;
  const afd_ffn_cfg& c = h->cfg;
  if (c.k != 1 || c.n_shared != 0 || !h->fp8) return AFD_ERR_UNSUPPORTED;
  int st = check_T(h, n_rows);
  if (st != AFD_OK) return st;
  if (n_rows == 0) return AFD_OK;
  if (!rows || !row_scale || !counts || !Y || !aligned16(rows) || !aligned16(Y)) return AFD_ERR_INVALID_ARG;
  if ((st = check_device(h)) != AFD_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  h->last_stream = s;
  const size_t H = c.H;
  AFD_CUDA(h, cudaMemcpyAsync(h->xp, rows, static_cast<size_t>(n_rows) * H, cudaMemcpyDeviceToDevice, s));
  AFD_CUDA(h, cudaMemcpyAsync(h->xscale, row_scale, static_cast<size_t>(n_rows) * 4, cudaMemcpyDeviceToDevice, s));
  dispatch_scan_kernel<<<1, kMaxExperts, 0, s>>>(counts, 1, c.E, h->counts, h->offsets, h->chunk_base);
  AFD_CUDA(h, cudaGetLastError());
  if ((st = run_expert_gemm(h, h->offsets, n_rows, s)) != AFD_OK) return st;
  AFD_CUDA(h, cudaMemcpyAsync(Y, h->Y, static_cast<size_t>(n_rows) * H * 2, cudaMemcpyDeviceToDevice, s));
  return AFD_OK;
}

extern "C" int afd_ffn_combine_rows_bf16(const void* Y, const void* Ys, const float* topk_w, const int32_t* pos,
                                         int32_t T, int32_t k, int32_t H, void* out, void* stream) {
  if (T < 0 || k < 1 || k > 32 || H < 4 || H % 4 != 0) return AFD_ERR_INVALID_ARG;
  if (T == 0) return AFD_OK;
  if (!Y || !topk_w || !pos || !out || !aligned16(Y) || !aligned16(out) || (Ys && !aligned16(Ys)))
    return AFD_ERR_INVALID_ARG;
  int* err = nullptr;
  int st = rows_err_word(&err);
  if (st != AFD_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (H % 8 == 0)
    combine8_kernel<<<dim3(static_cast<unsigned>(T), static_cast<unsigned>(combine8_slices(T, H))), kCombine8Threads, 0,
                      s>>>(static_cast<const __nv_bfloat16*>(Y), static_cast<const __nv_bfloat16*>(Ys), topk_w, pos, T,
                           k, H, T * k, Ys ? 1 : 0, static_cast<__nv_bfloat16*>(out), err);
  else
    combine_kernel<__nv_bfloat16><<<dim3(static_cast<unsigned>(T), static_cast<unsigned>(combine_slices(T, H))), 256, 0,
                                    s>>>(static_cast<const __nv_bfloat16*>(Y), static_cast<const __nv_bfloat16*>(Ys),
                                         topk_w, pos, T, k, H, T * k, Ys ? 1 : 0, static_cast<__nv_bfloat16*>(out), err);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(nullptr, e);
  return AFD_OK;
}

extern "C" int afd_ffn_expert_rows(afd_ffn_handle* h, const void* rows, const int32_t* counts, int32_t n_rows,
                                   float* Y, void* stream) {
  if (!h) return AFD_ERR_INVALID_ARG;
  const afd_ffn_cfg& c = h->cfg;
  if (c.k != 1 || c.n_shared != 0 || h->fp8) return AFD_ERR_UNSUPPORTED;
  int st = check_T(h, n_rows);
  if (st != AFD_OK) return st;
  if (n_rows == 0) return AFD_OK;
  if (!rows || !counts || !Y || !aligned16(rows) || !aligned16(Y)) return AFD_ERR_INVALID_ARG;
  if ((st = check_device(h)) != AFD_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  h->last_stream = s;
  const size_t H = c.H;
  AFD_CUDA(h, cudaMemcpyAsync(h->xp, rows, static_cast<size_t>(n_rows) * H * 2, cudaMemcpyDeviceToDevice, s));
  if (h->act16 && !use_narrow(h, n_rows))  // the f16 activations' row scales
    f16_row_scale_kernel<<<n_rows, 256, 0, s>>>(reinterpret_cast<const __nv_bfloat16*>(h->xp), c.H, h->f16_bound,
                                                h->xscale);
  // group offsets from the per-expert counts (one "chunk")
  dispatch_scan_kernel<<<1, kMaxExperts, 0, s>>>(counts, 1, c.E, h->counts, h->offsets, h->chunk_base);
  AFD_CUDA(h, cudaGetLastError());
  if ((st = run_expert_gemm(h, h->offsets, n_rows, s)) != AFD_OK) return st;
  AFD_CUDA(h, cudaMemcpyAsync(Y, h->Y, static_cast<size_t>(n_rows) * H * 4, cudaMemcpyDeviceToDevice, s));
  return AFD_OK;
}

extern "C" int afd_ffn_copy_row_blocks(const void* src, void* dst, const int32_t* blocks, int32_t n_blocks,
                                       int32_t row_bytes, void* stream) {
  if (n_blocks < 0 || row_bytes < 4 || row_bytes % 4 != 0) return AFD_ERR_INVALID_ARG;
  if (n_blocks == 0) return AFD_OK;
  const bool wide = row_bytes % 16 == 0;
  const uintptr_t mis = (reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) & (wide ? 15u : 3u);
  if (!src || !dst || !blocks || mis) return AFD_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const dim3 grid(static_cast<unsigned>(n_blocks), 16);
  if (wide)
    copy_row_blocks_kernel<uint4><<<grid, 256, 0, s>>>(static_cast<const uint4*>(src), static_cast<uint4*>(dst), blocks,
                                                        row_bytes / 16);
  else
    copy_row_blocks_kernel<uint32_t><<<grid, 256, 0, s>>>(static_cast<const uint32_t*>(src),
                                                           static_cast<uint32_t*>(dst), blocks, row_bytes / 4);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(nullptr, e);
  return AFD_OK;
}

extern "C" int afd_ffn_combine_rows(const float* Y, const float* Ys, const float* topk_w, const int32_t* pos,
                                    int32_t T, int32_t k, int32_t H, void* out, void* stream) {
  if (T < 0 || k < 1 || k > 32 || H < 4 || H % 4 != 0) return AFD_ERR_INVALID_ARG;
  if (T == 0) return AFD_OK;
  if (!Y || !topk_w || !pos || !out || !aligned16(Y) || !aligned16(out) || (Ys && !aligned16(Ys)))
    return AFD_ERR_INVALID_ARG;
  int* err = nullptr;
  int st = rows_err_word(&err);
  if (st != AFD_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  combine_kernel<float><<<dim3(static_cast<unsigned>(T), static_cast<unsigned>(combine_slices(T, H))), 256, 0, s>>>(
      Y, Ys, topk_w, pos, T, k, H, T * k, Ys ? 1 : 0, static_cast<__nv_bfloat16*>(out), err);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(nullptr, e);
  return AFD_OK;
}

extern "C" int afd_ffn_rows_error(void) {
  int* err = nullptr;
  int st = rows_err_word(&err);
  if (st != AFD_OK) return st;
  cudaError_t e = cudaDeviceSynchronize();
  int word = 0;
  if (e == cudaSuccess) e = cudaMemcpy(&word, err, sizeof(int), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemset(err, 0, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(nullptr, e);
  return word ? AFD_ERR_DEVICE_FLAG : AFD_OK;
}
