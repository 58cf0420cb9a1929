/*
 * afd_ffn.h -- C ABI of libafd_ffn.so, the FFN-service MoE layer of Attention-FFN
 * Disaggregation on one NVIDIA B200 (sm_100a).
 *
 * What the layer is.  In an A/F split the FFN service receives each layer's post-attention
 * hidden states and returns the layer's FFN output (vLLM AFD Plugin page, section 系統架構,
 * "2. FFN Service": a background loop receives activations, runs compute_ffn_output() and
 * sends the result back).  For an MoE model that output is the routed expert layer: a router
 * picks a few of many experts per token (LLM 推理提速: Attention与FFN分离AFD方, section 一个在
 * 啃带宽，一个在吃算力), the hidden state is dispatched to them, each expert is a large matrix
 * product, and the outputs are combined back per token (A/F 分离, sections 为什么要拆 and 机制).
 *
 * Readings where the pages are silent (the pages print no router or expert formula):
 *   logits  l[t,e]  = sum_h hidden[t,h] * router_w[e,h] (+ router_bias[e])   fp32
 *   idx[t,0..k-1]   = the k largest logits, descending, ties to the lower expert
 *   w[t,j]          = softmax of the selected logits (= renormalised full softmax)
 *   expert e        : y = (silu(x Wg_e^T) * (x Wu_e^T)) W2_e^T,  silu(z) = z / (1 + e^-z)
 *   out[t]          = sum_j w[t,j] * y_{idx[t,j]}(x_t) + y_shared(x_t)      (shared: n_shared = 1)
 * W8A8: each hidden row and each SwiGLU output row is quantised to e4m3 with one fp32 scale
 * (row amax / 448, 1 for an all-zero row, round to nearest even, saturating) before the
 * product that consumes it; weights arrive as e4m3 with one fp32 scale per output channel.
 *
 * Conventions for every entry point below.
 *   - Return value: AFD_OK (0) or a negative AFD_ERR_* status; nothing is thrown.  Checks
 *     that need no device run first and fail immediately (the FFN side fails fast when it is
 *     driven wrongly: Separar Attention de FFN page, section "Ejecutarlo en una sola máquina").
 *   - Every pointer argument is a DEVICE pointer owned by the caller unless stated otherwise.
 *     Weight pointers are borrowed: they must stay valid and unchanged until destroy.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = the legacy default stream) and
 *     returns without a host synchronisation, except where stated.  The calling thread's
 *     current device must be the device the handle was created on.
 *   - One handle owns one device workspace sized for T_max tokens.  Calls on one handle must
 *     not overlap in time (use one stream per handle, or synchronise between streams).
 *   - Data the device finds invalid (an expert index outside [0,E), a position outside the
 *     dispatched range) is skipped and recorded in the handle's device error word; read it
 *     with afd_ffn_get_error.  No kernel traps.
 *   - Layouts are row-major.  bf16 is IEEE bfloat16; e4m3 is the OCP "fn" variant.
 */
#ifndef AFD_FFN_H
#define AFD_FFN_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ---------------------------------------------------------------- */
#define AFD_OK                  0
#define AFD_ERR_INVALID_ARG    (-1)  /* NULL / misaligned pointer, bad size or config field   */
#define AFD_ERR_UNSUPPORTED    (-2)  /* config outside what the kernels implement             */
#define AFD_ERR_T_TOO_LARGE    (-3)  /* T > T_max of the handle                               */
#define AFD_ERR_CUDA           (-4)  /* a CUDA runtime/driver call failed: afd_ffn_last_cuda_error */
#define AFD_ERR_DEVICE_FLAG    (-5)  /* afd_ffn_get_error: kernels skipped invalid data        */
#define AFD_ERR_DEVICE_TIMEOUT (-6)  /* afd_ffn_get_error: a bounded on-device wait gave up    */
#define AFD_ERR_NO_DEVICE      (-7)  /* no sm_100 device current                               */
#define AFD_ERR_TIMEOUT        (-8)  /* a bounded host-side wait gave up                        */
#define AFD_ERR_STOPPED        (-9)  /* the FFN service stopped before it served the slot       */

/* ---- configuration ---------------------------------------------------------------- */
typedef enum { AFD_DT_BF16 = 0, AFD_DT_FP8_E4M3 = 1 } afd_dtype;

typedef struct {
    int32_t T_max;           /* largest micro-batch any call will pass, >= 1                  */
    int32_t H;               /* hidden size, multiple of 256                                  */
    int32_t E;               /* routed experts, 1..256                                        */
    int32_t k;               /* experts per token, 1..min(E, 32)                              */
    int32_t I;               /* expert intermediate size, multiple of 128                     */
    int32_t n_shared;        /* shared experts: 0 or 1                                        */
    int32_t weight_dtype;    /* afd_dtype: AFD_DT_BF16 or AFD_DT_FP8_E4M3                     */
    int32_t act_dtype;       /* afd_dtype: must equal weight_dtype                            */
    int32_t has_router_bias; /* 0 or 1                                                        */
} afd_ffn_cfg;

typedef struct {             /* all DEVICE pointers, 16-byte aligned, borrowed, never written */
    const float *router_w;    /* [E][H] fp32                                                  */
    const float *router_bias; /* [E] fp32, or NULL when has_router_bias == 0                  */
    const void  *w13;         /* [E+n_shared][2I][H] bf16 or e4m3: rows 0..I-1 gate, I..2I-1 up;
                                 the shared expert is index E                                  */
    const void  *w2;          /* [E+n_shared][H][I] bf16 or e4m3 (down projection)            */
    const float *w13_scale;   /* e4m3 only: [E+n_shared][2I] per-output-channel scales         */
    const float *w2_scale;    /* e4m3 only: [E+n_shared][H]                                    */
} afd_ffn_weights;

typedef struct afd_ffn_handle afd_ffn_handle;

/* Create a handle for one MoE layer of the FFN service (vLLM AFD Plugin page, section 系統架構,
 * "2. FFN Service") on the current device: validates cfg and weights (host-side checks come
 * first and touch no device), allocates the workspace for T_max tokens and encodes the TMA
 * descriptors of the weights.  The handle also derives, once, what its kernels read instead of
 * the caller's tensors: the router weights as three bf16 planes (hi + mid + lo = Wr to ~2^-27),
 * and -- for bf16 weights when T_max * k > 32 * E, i.e. when large micro-batches are possible --
 * an f16 copy of W2 ([E+n_shared][H][I], exact for |w| in [2^-14, 65504]; if a weight exceeds
 * 65504 no copy is kept and the two-term bf16 down GEMM is used) together with one pass over W13
 * for the bound max ||wg_i|| ||wu_i|| that sizes the f16 activations' per-row power-of-two
 * scales.  *out receives the handle (NULL on failure).  Synchronous. */
int afd_ffn_create(const afd_ffn_cfg *cfg, const afd_ffn_weights *weights, afd_ffn_handle **out);

/* afd_ffn_create with options.  flags: 0, or AFD_CREATE_NO_W2_COPY -- keep no f16 copy of W2
 * (saves (E+n_shared)*H*I*2 bytes of device memory, 7.5 GB at H=7168, I=2048, E=256+1; large
 * bf16 micro-batches then run the two-term bf16 down GEMM, which multiplies two activation
 * planes and is slower).  Other bits: AFD_ERR_INVALID_ARG. */
#define AFD_CREATE_NO_W2_COPY 1u
int afd_ffn_create_ex(const afd_ffn_cfg *cfg, const afd_ffn_weights *weights, uint32_t flags,
                      afd_ffn_handle **out);

/* Free the workspace and the handle (after synchronising the device).  NULL is a no-op. */
void afd_ffn_destroy(afd_ffn_handle *h);

/* Router, top-k and gate weights: the routing computation the FFN side runs for each token
 * (vLLM AFD Plugin page, section Attention-FFN 解耦的原理), picking a few of the layer's many
 * experts per token (LLM 推理提速: Attention与FFN分离AFD方, section 一个在啃带宽，一个在吃算力).
 * hidden [T][H] bf16 -> topk_idx [T][k] int32 (descending logit order) and topk_w [T][k] fp32
 * (softmax over the selected logits).  0 <= T <= T_max. */
int afd_ffn_route(afd_ffn_handle *h, const void *hidden, int32_t T,
                  int32_t *topk_idx, float *topk_w, void *stream);

/* Dispatch order and dispatched rows: each token's hidden state is sent to the experts it
 * chose (A/F 分离 page, section 机制, the dispatch step).  From topk_idx [T][k]:
 *   counts [E]      rows per expert
 *   offsets[E+1]    exclusive prefix sum of counts (offsets[E] = number of valid pairs)
 *   pos    [T][k]   dispatched row of pair (t,j): expert-major, ascending t inside an expert;
 *                   -1 for a pair whose expert is outside [0,E) (device error word set)
 *   src    [T*k]    token of each dispatched row
 * and fills the handle's internal dispatched-row buffer (hidden rows in pos order, then all
 * T rows for the shared expert; e4m3 + per-row scale in W8A8) used by afd_ffn_expert_gemm. */
int afd_ffn_permute(afd_ffn_handle *h, const void *hidden, const int32_t *topk_idx, int32_t T,
                    int32_t *counts, int32_t *offsets, int32_t *pos, int32_t *src, void *stream);

/* Expert FFNs -- each expert is a large matrix product (A/F 分离 page, section 为什么要拆) --
 * on the rows dispatched by the last afd_ffn_permute of this handle, grouped by
 * `offsets` [E+1] (device).  Writes the handle's internal output rows (fp32; bf16 on the W8A8
 * path); when non-NULL also copies them out as fp32: Y [T*k][H] (row p = the output of
 * dispatched row p, unweighted) and Ys [T][H] (shared expert; must be NULL when n_shared == 0). */
int afd_ffn_expert_gemm(afd_ffn_handle *h, const int32_t *offsets, int32_t T,
                        float *Y, float *Ys, void *stream);

/* Weighted combine of the handle's internal expert outputs, back in token order (A/F 分离
 * page, section 机制, the combine step):
 * out[t] = sum_j topk_w[t][j] * Y[pos[t][j]] + Ys[t], fp32 sum in j order, bf16 out [T][H]. */
int afd_ffn_combine(afd_ffn_handle *h, const float *topk_w, const int32_t *pos, int32_t T,
                    void *out, void *stream);

/* The whole layer, the FFN service's compute_ffn_output() for one micro-batch (vLLM AFD
 * Plugin page, section 系統架構, "2. FFN Service"): hidden [T][H] bf16 -> out [T][H] bf16
 * (route, permute, expert GEMMs, combine).  No host synchronisation, no allocation:
 * capturable in a CUDA graph. */
int afd_ffn_forward(afd_ffn_handle *h, const void *hidden, int32_t T, void *out, void *stream);

/* The whole layer on HOST buffers: copies hidden_host [T][H] bf16 to the device, runs
 * afd_ffn_forward, copies the result to out_host [T][H] bf16, and synchronises `stream`
 * before returning.  Pinned host memory gives the fastest copies. */
int afd_ffn_forward_host(afd_ffn_handle *h, const void *hidden_host, int32_t T, void *out_host,
                         void *stream);

/* The FFN service's loop over a sequence of micro-batches held in HOST memory: for batch i,
 * hidden_host[i] [T][H] bf16 is copied to the device, the layer runs, and the result is copied
 * to out_host[i] [T][H] bf16.  Copies run on two copy streams owned by the handle and overlap
 * the layer of the neighbouring batches (double-buffered device staging), the micro-pipeline of
 * an A/F split in which the period tends to max(compute, transfer) instead of their sum (A/F
 * 分离 page, section 深入推导, 微流水).  Results equal afd_ffn_forward's bit for bit.  `stream`
 * runs the layer; the call synchronises everything it enqueued before returning.  Pinned host
 * buffers are required for the copies to overlap.  0 <= T <= T_max, n_batches >= 0. */
int afd_ffn_forward_host_batches(afd_ffn_handle *h, const void *const *hidden_host,
                                 void *const *out_host, int32_t n_batches, int32_t T, void *stream);

/* Optional stage timing: n_events cudaEvent_t handles (owned by the caller) that
 * afd_ffn_forward records on its stream before each stage and after the last one.  Stages,
 * in order: router logits, top-k, dispatch order, row gather, GEMM schedule, gate/up GEMM,
 * activation quantisation (W8A8 only; empty otherwise), down GEMM, combine -- so
 * AFD_FFN_NUM_STAGES + 1 events, each already created.  A NULL entry skips that boundary (a
 * caller timing one stage passes only the two events around it, so the others add nothing to
 * the stream).  n_events = 0 (events NULL) turns it off. */
#define AFD_FFN_NUM_STAGES 9
int afd_ffn_set_stage_events(afd_ffn_handle *h, void *const *events, int32_t n_events);

/* Synchronise the handle's last stream, return AFD_OK / AFD_ERR_DEVICE_FLAG /
 * AFD_ERR_DEVICE_TIMEOUT from the device error word, and clear it. */
int afd_ffn_get_error(afd_ffn_handle *h);

/* The cudaError_t behind the last AFD_ERR_CUDA of this handle (0 if none; h may be NULL for
 * errors of afd_ffn_create, which are kept per thread). */
int afd_ffn_last_cuda_error(const afd_ffn_handle *h);

/* Static description of a status code. */
const char *afd_ffn_strerror(int status);

/* Router, top-k and gate weights with no handle and no allocation of any kind.
 *
 * This entry point has no counterpart on the pages; it exists for callers that cannot
 * allocate device memory: a serving engine that owns every device byte through its own pool
 * and caps it (a stray cudaMalloc there fails or breaks the engine's accounting), and the
 * per-layer loop of an FFN service, where an allocation can synchronise the device in the
 * middle of a pipelined micro-batch.  afd_ffn_create allocates a workspace, so such callers
 * cannot use afd_ffn_route; this call computes the same routing with the fp32 FMA router
 * (afd_ffn_route runs the router on the tensor cores): the same experts, and gate weights
 * equal to afd_ffn_route's up to the routers' fp32 rounding.
 *
 * Inputs (device, caller-owned, 16-byte aligned): hidden [T][H] bf16, router_w [E][H] fp32,
 * router_bias [E] fp32 or NULL.  Outputs: topk_idx [T][k] int32, topk_w [T][k] fp32.
 * Sizes: 0 <= T, H a multiple of 32, 1 <= E <= 256, 1 <= k <= min(E, 32).
 * Scratch: the partial router logits live in one static device array of
 * AFD_FFN_ROUTE_STATIC_SCRATCH_FLOATS floats (4 MiB) that every GPU loading the library holds
 * until the process exits.  T*E must not exceed it; larger problems return
 * AFD_ERR_UNSUPPORTED before any device work (the split of the reduction over H is narrowed
 * to fit when needed, which changes only the fp32 summation order).
 * The first call on a device looks up the array's device address (cudaGetSymbolAddress with
 * that device current); make that first call before any stream capture on the device.
 * Every call on a device shares the one array: calls that can overlap on the GPU (different
 * streams without ordering between them) race on it and must be serialised by the caller.
 * Nothing in the array needs clearing: each call overwrites every element it reads.
 * The looked-up address is kept for the life of the process: it does not survive a
 * cudaDeviceReset (or any other teardown of the device's primary context), after which this
 * call must not be used on that device.
 * CUDA failures return AFD_ERR_CUDA; the cudaError_t is afd_ffn_last_cuda_error(NULL). */
#define AFD_FFN_ROUTE_STATIC_SCRATCH_FLOATS (1 << 20)
int afd_ffn_route_static(const void *hidden, const float *router_w, const float *router_bias,
                         int32_t T, int32_t H, int32_t E, int32_t k,
                         int32_t *topk_idx, float *topk_w, void *stream);

/* ---- expert parallelism: building blocks ------------------------------------------
 * An expert-parallel layer (experts split in contiguous blocks over ranks, hidden states sent
 * to the experts' ranks and the outputs sent back: the dispatch / combine exchange of the A/F
 * 分离 page, section 机制) runs its exchange outside the library; these calls do the rest.
 * The allocation-free calls (no handle) share one device error word: expert indices outside
 * [0, E) and positions outside the expert rows are skipped and flagged there. */

/* Dispatch order and rows without a handle: for topk_idx [T][k] (device, global expert ids),
 * writes counts [E], offsets [E+1] (exclusive prefix), pos [T][k] (dispatched row of each pair,
 * -1 when skipped), src [T*k] (token of each row) and rows [T*k][H] bf16 = hidden rows in
 * expert-major order, tokens ascending inside an expert -- so experts held in contiguous
 * blocks per rank make the rows rank-major as well.  scratch: int32 [2 * ceil(T/128) * E]
 * (device, caller-owned).  hidden, rows 16-byte aligned; H multiple of 8; 1 <= k <= min(E, 32),
 * E <= 256.  Asynchronous on `stream`. */
int afd_ffn_dispatch_rows(const void *hidden, const int32_t *topk_idx, int32_t T, int32_t k, int32_t E,
                          int32_t H, int32_t *counts, int32_t *offsets, int32_t *pos, int32_t *src,
                          void *rows, int32_t *scratch, void *stream);

/* A handle's experts on rows that arrive grouped by expert: rows [n_rows][H] bf16 (device),
 * counts [E] (device; rows of expert 0 first, then expert 1, ...; sum = n_rows) ->
 * Y [n_rows][H] fp32, row r = the output of row r.  The handle must be bf16 with k == 1 and
 * n_shared == 0 (a rank's expert block, or a replicated shared expert as E = 1);
 * 0 <= n_rows <= T_max.  Asynchronous on `stream`. */
int afd_ffn_expert_rows(afd_ffn_handle *h, const void *rows, const int32_t *counts, int32_t n_rows,
                        float *Y, void *stream);

/* Move blocks of rows: block b copies blocks[3b+2] rows of row_bytes bytes from row blocks[3b]
 * of src to row blocks[3b+1] of dst (blocks: int32 [n_blocks][3], device).  Blocks must not
 * overlap in dst.  row_bytes a multiple of 4 (per-row scales) with src, dst 4-byte aligned, or
 * a multiple of 16 with src, dst 16-byte aligned (moved as 16-byte vectors). */
int afd_ffn_copy_row_blocks(const void *src, void *dst, const int32_t *blocks, int32_t n_blocks,
                            int32_t row_bytes, void *stream);

/* Weighted combine of external expert outputs: out[t] = sum_j topk_w[t][j] * Y[pos[t][j]]
 * (+ Ys[t] when Ys != NULL), fp32 sum in j order with the shared row last, bf16 out [T][H].
 * Y [T*k][H] fp32 in dispatch order, Ys [T][H] fp32 or NULL; pairs with pos < 0 are skipped.
 * H multiple of 4; Y, Ys, out 16-byte aligned. */
int afd_ffn_combine_rows(const float *Y, const float *Ys, const float *topk_w, const int32_t *pos,
                         int32_t T, int32_t k, int32_t H, void *out, void *stream);

/* W8A8 form of the exchange, at the precision the A/F 分离 page counts its bytes in (section
 * 深入推导 / 通信账: the dispatched hidden states travel as FP8).  The rows sent are exactly
 * what the experts consume -- each token's hidden row quantised once to e4m3 with its fp32
 * scale (row amax / 448, 1 for a zero row; round to nearest even, saturating) -- so sending
 * them adds no error; the expert outputs come back as bf16 rows, the W8A8 layer's own output
 * precision for the combine. */

/* afd_ffn_dispatch_rows for the W8A8 path: the same counts, offsets, pos and src, and
 * rows [T*k + with_shared*T][H] e4m3 + row_scale [T*k + with_shared*T] fp32: the quantised
 * hidden rows in expert-major order, then (with_shared = 1) every token's row once, in token
 * order, for a replicated shared expert.  hidden, rows 16-byte aligned; H a multiple of 16;
 * scratch as for afd_ffn_dispatch_rows.  Asynchronous on `stream`. */
int afd_ffn_dispatch_rows_fp8(const void *hidden, const int32_t *topk_idx, int32_t T, int32_t k, int32_t E,
                              int32_t H, int32_t with_shared, int32_t *counts, int32_t *offsets, int32_t *pos,
                              int32_t *src, void *rows, float *row_scale, int32_t *scratch, void *stream);

/* afd_ffn_expert_rows for a W8A8 handle (k == 1, n_shared == 0): rows [n_rows][H] e4m3 with
 * row_scale [n_rows] fp32, grouped by expert as counts [E] says -> Y [n_rows][H] bf16 (the W8A8
 * expert outputs, SwiGLU rows quantised per row before the down projection as in
 * afd_ffn_forward).  0 <= n_rows <= T_max; rows, Y 16-byte aligned.  Asynchronous. */
int afd_ffn_expert_rows_fp8(afd_ffn_handle *h, const void *rows, const float *row_scale, const int32_t *counts,
                            int32_t n_rows, void *Y, void *stream);

/* afd_ffn_combine_rows on bf16 expert outputs: Y [T*k][H] bf16, Ys [T][H] bf16 or NULL; the same
 * fp32 sum in j order with the shared row last, bf16 out [T][H].  H multiple of 4; Y, Ys, out
 * 16-byte aligned. */
int afd_ffn_combine_rows_bf16(const void *Y, const void *Ys, const float *topk_w, const int32_t *pos, int32_t T,
                              int32_t k, int32_t H, void *out, void *stream);

/* Synchronise the device; AFD_ERR_DEVICE_FLAG if an allocation-free call skipped invalid data
 * since the last check (the word is cleared), else AFD_OK. */
int afd_ffn_rows_error(void);

/* Self-check of the device's bounded waits.  One thread waits, through the same bounded wait
 * the GEMM roles use, on an mbarrier that no thread arrives on; the wait must give up after its
 * limit (about 2 s of SM clock) and record the timeout bit, and the kernel then returns.
 * Synchronous (the device is synchronised), on the current device.  Returns
 * AFD_ERR_DEVICE_TIMEOUT when the wait gave up and the bit reached the host (the expected
 * result), AFD_OK if the wait completed, AFD_ERR_CUDA / AFD_ERR_NO_DEVICE on failure.
 * *waited_cycles (may be NULL) receives the SM cycles the wait took. */
int afd_ffn_check_bounded_wait(int64_t *waited_cycles);

/* The configuration and device of a handle (host only; either output may be NULL). */
int afd_ffn_get_info(const afd_ffn_handle *h, afd_ffn_cfg *cfg, int32_t *device);

/* ---- FFN service: mailbox and serving loop ----------------------------------------
 * The FFN side of an A/F split runs a loop per layer: take the activations the attention side
 * sent, run the layer, send the output back (vLLM AFD Plugin page, section 系統架構, "2. FFN
 * Service").  With several micro-batches in flight the attention of one overlaps the FFN of
 * another: the A/F 分离 page (section 深入推导, 微流水) puts the steady-state period at
 * max(t_a, t_f) + t_comm instead of t_a + t_f on one device.  This loop also overlaps the
 * copies with the layer, so with n slots in flight its period is bounded below by
 * max(t_a, t_f, (t_a + t_h2d + t_f + t_d2h) / n).
 *
 * The mailbox is the connector between the two sides on one host: n_slots slots, each an input
 * buffer [T_max][H] bf16 (the hidden states of one micro-batch) and an output buffer of the
 * same shape (the layer's output), both HOST memory owned by the mailbox.  A slot moves
 *     free --post--> posted --take--> taken --complete--> done | failed --post--> ...
 * The producer (attention side) writes the input, posts, later waits and reads the output; the
 * consumer (one thread: the service, or a caller's loop) takes slots in post order and
 * completes them.  Producers on several threads may post distinct slots.  Waits are bounded:
 * they spin for about 20 us, then sleep until the state changes or the time is up; a wait that
 * gives up returns AFD_ERR_TIMEOUT and leaves the slot as it was.  Times are CLOCK_MONOTONIC
 * nanoseconds. */
typedef struct afd_ffn_mailbox afd_ffn_mailbox;
typedef struct afd_ffn_service afd_ffn_service;

#define AFD_MAILBOX_PINNED 1   /* flags: buffers in page-locked memory (needs a CUDA device) */

/* n_slots >= 1, T_max >= 1, H >= 8 and a multiple of 8.  Buffers are 64-byte aligned and
 * zero-filled.  Without AFD_MAILBOX_PINNED they are ordinary host memory (no device needed).
 * AFD_ERR_CUDA when the page-locked allocation fails. */
int afd_ffn_mailbox_create(int32_t n_slots, int32_t T_max, int32_t H, int32_t flags,
                           afd_ffn_mailbox **out);
/* No consumer may run on the mailbox (stop the service first).  NULL is a no-op. */
void afd_ffn_mailbox_destroy(afd_ffn_mailbox *mb);
/* Host pointer of a slot's input / output buffer; NULL for a bad slot. */
void *afd_ffn_mailbox_input(afd_ffn_mailbox *mb, int32_t slot);
void *afd_ffn_mailbox_output(afd_ffn_mailbox *mb, int32_t slot);

/* Producer: hand over the first T rows of the slot's input (0 <= T <= T_max).  The slot must
 * be free, done or failed, else AFD_ERR_INVALID_ARG. */
int afd_ffn_mailbox_post(afd_ffn_mailbox *mb, int32_t slot, int32_t T);
/* Producer: wait up to timeout_us for the posted slot to finish.  AFD_OK once done (the first
 * T rows of the output are valid), the consumer's status once failed (AFD_ERR_STOPPED when the
 * service stopped first), AFD_ERR_TIMEOUT, or AFD_ERR_INVALID_ARG for a slot never posted. */
int afd_ffn_mailbox_wait(afd_ffn_mailbox *mb, int32_t slot, int64_t timeout_us);

/* Consumer (one thread at a time): the oldest posted slot and its T, waiting up to timeout_us;
 * AFD_ERR_TIMEOUT when none was posted in time. */
int afd_ffn_mailbox_take(afd_ffn_mailbox *mb, int32_t *slot, int32_t *T, int64_t timeout_us);
/* Consumer: finish a taken slot: status AFD_OK -> done, a negative status -> failed. */
int afd_ffn_mailbox_complete(afd_ffn_mailbox *mb, int32_t slot, int32_t status);
/* Post / take / complete times of the slot's latest round: times_ns[3], 0 where not reached. */
int afd_ffn_mailbox_times(afd_ffn_mailbox *mb, int32_t slot, int64_t *times_ns);

typedef struct {
  int64_t served;           /* micro-batches completed                                      */
  int32_t status;           /* AFD_OK, or the first failure of the loop or the completer     */
  int32_t device_status;    /* afd_ffn_get_error of the handle when the loop ended           */
  int32_t last_cuda_error;  /* cudaError_t behind an AFD_ERR_CUDA status, else 0             */
  int32_t reserved;
} afd_ffn_service_stats;

/* Start the serving loop on two host threads.  The loop thread takes each slot from mb and
 * enqueues its micro-batch: the input copied to the device, afd_ffn_forward on `stream`, the
 * output copied back.  The copies run on two streams of the service, so with two or more slots
 * in flight the copies of one micro-batch overlap the layer of another.  The completer thread
 * polls the event after each in-flight slot's copy back, in order, and completes the slot as
 * soon as its output has landed.  It keeps one core busy while micro-batches are in flight and
 * sleeps otherwise.  An output that has not landed after 60 s fails its slot with
 * AFD_ERR_TIMEOUT.
 * The handle's H must equal the mailbox's and its T_max must be >= the mailbox's; the calling
 * thread's current device must be the handle's.  While the service runs, the caller makes no
 * other call on h.  After the first failure every later slot fails with the same status. */
int afd_ffn_service_start(afd_ffn_handle *h, afd_ffn_mailbox *mb, void *stream, afd_ffn_service **out);
/* Device timeline of a slot's latest micro-batch, from CUDA events the loop records (the slot
 * must be done; call it before posting the slot again): ms[0] = service start -> H2D start, and
 * from the H2D start: ms[1] H2D end, ms[2] layer start, ms[3] layer end, ms[4] D2H end.
 * AFD_ERR_INVALID_ARG for a slot that is not done. */
int afd_ffn_service_slot_timeline(afd_ffn_service *svc, int32_t slot, float *ms);
/* Stop taking slots, let the ones in flight finish, fail the posted ones with AFD_ERR_STOPPED,
 * release the service and fill *stats (may be NULL).  Returns stats.status. */
int afd_ffn_service_stop(afd_ffn_service *svc, afd_ffn_service_stats *stats);

#ifdef __cplusplus
}
#endif
#endif /* AFD_FFN_H */
