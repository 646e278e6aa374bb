/*
 * tileshare.h -- C ABI of libtileshare.so: the TileShare shared transformer layer
 * for overlapping tiled ViT decoding on B200 (sm_100a).
 *
 * Source of the operations: "TileShare: Training-Free Acceleration of Overlapping
 * Tiled ViT Decoding" (arXiv 2610.32233), cited below as [TileShare] with the
 * figure or table that defines each step.
 *
 * Conventions shared by every call
 *   - Plain C types and pointers only.  "device" pointers are CUDA device memory of
 *     the device current when the plan was created; "host" pointers are ordinary
 *     host memory.  Streams are cudaStream_t values passed as void* (NULL = the
 *     legacy default stream).
 *   - The caller allocates and owns every buffer passed in, including the
 *     workspace.  Compute calls (ts_block_*, ts_decode_stack, ts_quantize_*)
 *     never allocate, never synchronise and only enqueue work on the given stream.
 *   - Every call returns a ts_status.  Arguments are validated on the host before
 *     anything is enqueued; on any error nothing is launched.  No call aborts,
 *     traps or exits.  ts_last_error() gives a one-line reason for the last error
 *     of the calling thread.
 *   - Row-major layouts.  "d" is the model width, "hd" = d / heads, "f" the MLP
 *     width.  All device pointers must be 16-byte aligned.
 *
 * Token layouts (fixed by ts_plan_create)
 *   grid tokens  u = (f * H + y) * W + x for a grid of F x H x W tokens, U = F*H*W.
 *   tiles        T tiles in raster order of their (f, y, x) origins.
 *   window slot  j = (lf * wh + ly) * ww + lx, tile-local raster order, Nw = wf*wh*ww.
 *   registers    R register tokens per tile ([TileShare] Tab. S1: one set per
 *                tile; R = 1, one global token, unless the plan says otherwise).
 *   shared state S [U + T*R, d]: the U grid tokens, then tile t's registers at
 *                rows U + t*R .. U + t*R + R - 1.
 *   per-tile state X [T, N, d], N = Nw + R: rows 0 .. R-1 of tile t are its
 *                registers, row R + j its window slot j.
 */
#ifndef TILESHARE_H
#define TILESHARE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TS_OK = 0,
  TS_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size or geometry     */
  TS_ERR_UNSUPPORTED = 2,   /* valid but not implemented (e.g. head dim != 64)   */
  TS_ERR_WORKSPACE = 3,     /* workspace smaller than ts_workspace_size()        */
  TS_ERR_CUDA = 4,          /* a CUDA runtime/driver call failed                 */
  TS_ERR_DEVICE_CHECK = 5,  /* a kernel's own check failed (ts_device_status)    */
  TS_ERR_TIMEOUT = 6,       /* a kernel's bounded wait ran out (ts_device_status)*/
  TS_ERR_ALLOC = 7          /* ts_plan_create could not allocate                 */
} ts_status;

/* Rule for the blend weights w-bar of overlap tokens. */
typedef enum {
  /* [TileShare] Fig. 2 and abstract: overlap tokens are blended "with the released
     weights".  Read as a separable linear ramp across each overlap band, normalised
     to sum 1 per token. */
  TS_BLEND_LINEAR_RAMP = 0,
  /* Hard stitching ([TileShare] Tab. 2 / Tab. S2 "Hard stitching" baseline; Tab. S11:
     each pixel from its dominant tile), applied to the blend of overlap tokens: each
     token takes its value from one tile, the covering tile with the largest
     linear-ramp weight, the lowest tile index on ties; its CSR row holds that single
     entry with w-bar = 1 (nnz = U). */
  TS_BLEND_HARD_STITCH = 1
} ts_blend_rule;

typedef enum {
  TS_F32 = 0,       /* fp32 states, weights and arithmetic (SIMT kernels)              */
  TS_BF16 = 1,      /* bf16 states/weights, fp32 accumulation (tcgen05 kind::f16)      */
  TS_FP8_E4M3 = 2   /* bf16 states, e4m3 GEMM operands (tcgen05 kind::f8f6f4), bf16
                       attention; weights quantised per output channel, activations
                       per token ([TileShare] Tab. S2 "FP8")                          */
} ts_dtype;

/* Block flavour ([TileShare] Tab. S1 block; Tab. S6 profiles a block with "RMSNorm +
   residual" and a "SwiGLU gate"). */
typedef enum {
  /* pre-LN ViT block: Norm1/Norm2 LayerNorm with gain and bias, MLP
     W_2 GELU(W_1 h + b_1) + b_2 (exact erf GELU) */
  TS_BLOCK_LN_GELU = 0,
  /* Norm1/Norm2 RMSNorm with gain, no bias (ln*_b unused, may be NULL); MLP
     W_2 (silu(W_g h + b_g) * (W_u h + b_u)) + b_2 with silu(z) = z / (1 + e^-z).
     w_1 [2f, d] holds the f gate rows W_g above the f up rows W_u; b_1 [2f] and, for
     e4m3, s_1 [2f] follow the same order. */
  TS_BLOCK_RMS_SWIGLU = 1
} ts_block_kind;

typedef struct ts_plan_s* ts_plan_t;

/* Read-only view of a plan.  Host arrays stay valid until ts_plan_destroy. */
typedef struct {
  int grid[3], win[3], stride[3];  /* (F, H, W), (wf, wh, ww), (sf, sh, sw)          */
  int T, U, Nw, N;                 /* tiles, grid tokens, window slots, Nw + R        */
  int nnz;                         /* CSR entries: T * Nw (ramp), U (hard stitching)  */
  int max_cover;                   /* most tiles covering one token                   */
  int device;                      /* CUDA device holding the plan's device arrays    */
  int run;                         /* attention loads: every aligned group of `run`    */
                                   /* slots (1 + k*run ...) is a run of consecutive    */
                                   /* grid tokens (64, 32, 16 or 8; 0: no such run)    */
  const int* origins;              /* host [T][3] tile origin (f, y, x)               */
  const int* tile_tok;             /* host [T][Nw] grid token of slot j of tile t      */
  const int* slot_pos;             /* host [Nw][3] tile-local (f, y, x) of slot j      */
  const int* tok_ptr;              /* host [U + 1] CSR row pointer over grid tokens    */
  const int* tok_ent;              /* host [nnz] entry t*N + R + j, ascending t        */
  const float* wbar;               /* host [nnz] blend weight of that entry            */
  int R;                           /* register tokens per tile                         */
} ts_plan_desc;

/* Model hyper-parameters ([TileShare] Tab. S1 block; readings in the comments). */
typedef struct {
  int d, heads, mlp;      /* width, heads, MLP width                                  */
  ts_dtype dtype;
  float eps_ln;           /* LayerNorm epsilon (1e-6 in the benchmark workloads)      */
  float eps_qk;           /* QK-RMSNorm epsilon over the head dimension               */
  float rope_base;        /* RoPE base (10000)                                        */
  int rope_dims[3];       /* head-dimension channels rotated by the f, y, x
                             coordinate; sum = hd, each even.  Inside an axis block
                             of D channels, channel j pairs with j + D/2.            */
  ts_block_kind block;    /* block flavour (TS_BLOCK_LN_GELU unless set)              */
} ts_model_desc;

/* One layer's parameters, all device pointers.  Matrices are [out, in] row-major
   (y = x W^T + b).  Matrix element type: float for TS_F32, bf16 for TS_BF16, e4m3
   bytes for TS_FP8_E4M3 (then s_* hold the per-output-channel fp32 scales, see
   ts_quantize_rows_e4m3).  Vectors are always fp32. */
typedef struct {
  const float* ln1_g; const float* ln1_b;    /* [d]                 */
  const void* w_qkv;  const float* b_qkv;    /* [3d, d], [3d]; rows: q | k | v, head h at h*hd */
  const float* q_g;   const float* k_g;      /* [hd] QK-RMSNorm gains              */
  const void* w_o;    const float* b_o;      /* [d, d], [d]          */
  const float* ln2_g; const float* ln2_b;    /* [d]                 */
  const void* w_1;    const float* b_1;      /* [f, d], [f]; [2f, d], [2f] for TS_BLOCK_RMS_SWIGLU */
  const void* w_2;    const float* b_2;      /* [d, f], [d]          */
  const float* s_qkv; const float* s_o;      /* TS_FP8_E4M3 only: [3d], [d] */
  const float* s_1;   const float* s_2;      /* TS_FP8_E4M3 only: [f] ([2f] SwiGLU), [d] */
} ts_layer_weights;

/* ---------------------------------------------------------------------------
 * Plan: tiling of the token grid, tile <-> token index maps and w-bar.
 * [TileShare] abstract (overlapping tiles at deployment resolution) and Fig. 2
 * (overlap tokens stored once, attended in every window, blended with w-bar).
 * Per axis: n = ceil((G - w) / s) + 1 tiles (1 if w == G) at origins
 * min(i*s, G - w).  A 2-D grid is F = wf = sf = 1.
 * Requires 1 <= win <= grid and 1 <= stride <= win per axis.  Allocates host and
 * device memory on the current device (TS_ERR_ALLOC on failure); the plan is
 * immutable afterwards and may be shared between threads and streams.
 * ------------------------------------------------------------------------- */
ts_status ts_plan_create(const int grid[3], const int win[3], const int stride[3],
                         ts_blend_rule rule, ts_plan_t* out);
/* Same plan, host arrays only (no device memory, no CUDA call): for inspecting a
   tiling without a GPU.  Compute calls reject it (TS_ERR_INVALID_ARG); its
   ts_plan_desc reports device = -1. */
ts_status ts_plan_create_host(const int grid[3], const int win[3], const int stride[3],
                              ts_blend_rule rule, ts_plan_t* out);
/* The same two calls for R register tokens per tile, 1 <= registers <= 64
   (TS_ERR_INVALID_ARG otherwise); ts_plan_create and ts_plan_create_host are
   these with registers = 1.  The registers are not rotated by RoPE and attend,
   and are attended by, their own tile only ([TileShare] Tab. S1). */
ts_status ts_plan_create_registers(const int grid[3], const int win[3], const int stride[3],
                                   ts_blend_rule rule, int registers, ts_plan_t* out);
ts_status ts_plan_create_host_registers(const int grid[3], const int win[3], const int stride[3],
                                        ts_blend_rule rule, int registers, ts_plan_t* out);
ts_status ts_plan_info(ts_plan_t plan, ts_plan_desc* out);
void ts_plan_destroy(ts_plan_t plan);

/* Bytes of device workspace needed for this plan and model: with L = 0 (and
   k = 0) by ts_block_tiled and ts_block_shared, with L >= 1 by
   ts_decode_stack(L, k) (which also holds the per-tile and shared states). */
ts_status ts_workspace_size(ts_plan_t plan, const ts_model_desc* model, int L, int k,
                            size_t* bytes);

/* One released (per-tile) layer, in place on X [T, N, d] (device, model dtype; bf16
   for TS_FP8_E4M3).  [TileShare] Tab. S1, "Layer 0" column: every tile keeps its
   own residual stream; Norm1, QKV, QK-RMSNorm, RoPE on tile-local coordinates (the
   registers are not rotated), dense attention over the tile's N rows,
   out-projection, Norm2 and MLP per tile row. */
ts_status ts_block_tiled(ts_plan_t plan, const ts_model_desc* model, const ts_layer_weights* w,
                         void* X, void* workspace, size_t workspace_bytes, void* stream);

/* One TileShare shared layer, in place on S [U + T*R, d] (device).  [TileShare]
   Fig. 2 and Tab. S1 "Layers >= k": Norm1, QKV, QK-RMSNorm, out-projection and MLP
   once per row of S; attention per tile over the rows [registers of t, window
   tokens of t], with RoPE on tile-local coordinates; each grid token's attention
   output is the w-bar weighted sum, in ascending tile order, of its tiles' outputs
   (the only approximate step); each register keeps its own tile's output. */
ts_status ts_block_shared(ts_plan_t plan, const ts_model_desc* model, const ts_layer_weights* w,
                          void* S, void* workspace, size_t workspace_bytes, void* stream);

/* Shared layer without a caller workspace.  The paper has no counterpart: this
   entry point exists for callers that cannot allocate device memory, such as a
   plugin running inside a host application that owns every device buffer
   through its own pool and forbids the plugin from calling cudaMalloc, or code
   working inside a fixed, pre-partitioned memory budget.  It computes exactly
   what ts_block_shared computes (the same kernels, bit for bit), in place on
   S [U + T*R, d], but its scratch (normalised rows, q/k/v, attention outputs,
   blend, MLP hidden) lives in one static device array of
   TS_NOALLOC_SCRATCH_BYTES (32 MiB) instead of a caller workspace.
   - Allocates nothing: no cudaMalloc, cudaFree or allocating library routine.
   - When the array is reserved: the array belongs to the library's device code,
     which the CUDA driver loads into a context on the library's first use there.
     Under lazy module loading (the default of recent CUDA releases) that can be
     the first ts_block_shared_noalloc call itself.  A caller inside a fixed
     budget should make that happen at set-up: any call that launches a library
     kernel or reads its device status, e.g. ts_device_status(), loads the code
     and reserves the 32 MiB in the current context; it is held until the
     context is destroyed or the process exits.
   - Plans and models needing more scratch than the array holds are refused with
     TS_ERR_WORKSPACE before anything is launched (the 48x48-token, d = 512
     workload needs about 26 MB; large grids do not fit and must use
     ts_block_shared).
   - The first call in a CUDA context looks up the array's device address in that
     context (cudaGetSymbolAddress, with the plan's device current) and caches it
     under the context's unique ID, so non-primary contexts and a context
     recreated after cudaDeviceReset get their own lookup; make that first call
     before any stream capture in the context.
   - Every call shares the one array and leaves its contents behind.  No region
     has to start at zero: each is written before it is read within a call.
     Calls that overlap on the GPU (other streams, other threads) race on the
     array and must be serialised by the caller. */
#define TS_NOALLOC_SCRATCH_BYTES (32u << 20)
ts_status ts_block_shared_noalloc(ts_plan_t plan, const ts_model_desc* model, const ts_layer_weights* w,
                                  void* S, void* stream);

/* TileShare-k stack ([TileShare] abstract, Tab. 1): layers 0..k-1 per tile on the
   copies of S0/G0 in every tile, then the per-tile states are merged with w-bar
   (Fig. 3b), then layers k..L-1 shared.  With k = L this is overlapping tiled
   decoding blended with w-bar at the end.  w points to L host-side
   ts_layer_weights structs (whose members are device pointers).
   S0 [U, d] grid tokens and G0 [T*R, d] registers in, out [U, d] grid tokens out
   (device, model dtype).  0 <= k <= L. */
ts_status ts_decode_stack(ts_plan_t plan, const ts_model_desc* model, const ts_layer_weights* w,
                          int L, int k, const void* S0, const void* G0, void* out,
                          void* workspace, size_t workspace_bytes, void* stream);

/* Per-tile copies of the stack input, as ts_decode_stack makes before its first
   per-tile layer: X[t*N + i] = G0[t*R + i], X[t*N + R + j] = S0[grid token of
   slot j of t].  S0 [U, d], G0 [T*R, d], X [T*N, d] (device, model dtype). */
ts_status ts_gather_tiles(ts_plan_t plan, const ts_model_desc* model, const void* S0, const void* G0,
                          void* X, void* stream);

/* Per-row e4m3 quantisation used by TS_FP8_E4M3: scale[r] = max|x[r, :]| / 448
   (1 for an all-zero row), q[r, c] = e4m3(x[r, c] / scale[r]) rounded to nearest
   even and saturated at +-448.  x bf16 [rows, cols] (device), q e4m3 bytes
   [rows, cols] (device), scale fp32 [rows] (device).  Used once on the weight
   matrices (per output channel) before calling the layers. */
ts_status ts_quantize_rows_e4m3(const void* x, int rows, int cols, void* q, float* scale,
                                void* stream);

/* Operations a partially shared layer runs once per token (bit mask). */
typedef enum {
  TS_SHARE_QKV = 1,   /* Norm1, QKV projection, QK-RMSNorm                    */
  TS_SHARE_OUT = 2,   /* out-projection (of the blended attention outputs)     */
  TS_SHARE_MLP = 4    /* Norm2 and MLP                                         */
} ts_shared_op;

/* One layer with per-tile residual streams in which only the operations in
   shared_ops run once per token ([TileShare] Tab. 1 top: from layer k on, each
   tile keeps its own residual stream and only the listed operations are shared;
   attention always runs per tile).  In place on X [T, N, d] as ts_block_tiled.
   A shared operation takes, for each grid token, the w-bar blend of its tiles'
   inputs (each tile's registers keep their own rows) and runs once per token;
   shared q/k/v feed every tile's attention through the tile's rows, and the
   shared out-projection's and MLP's outputs are added to every tile's copy of the
   token.  shared_ops = 0 is ts_block_tiled; from identical per-tile copies, any set
   with TS_SHARE_OUT gives the shared layer's result in every copy.  Workspace as
   for ts_block_tiled (TS_ERR_WORKSPACE if smaller); bits other than the three
   above give TS_ERR_INVALID_ARG. */
ts_status ts_block_partial(ts_plan_t plan, const ts_model_desc* model, const ts_layer_weights* w,
                           unsigned shared_ops, void* X, void* workspace, size_t workspace_bytes, void* stream);

/* Device-side status word of the library on the current device: 0 if no kernel
   check or bounded wait has failed since the last call, else a TS_ERR_* code.
   Synchronises the device and clears the word. */
ts_status ts_device_status(void);

/* Self-test of the kernels' bounded waits (the pages have no counterpart; it checks
   the library's failure reporting).  Launches one thread that waits on an mbarrier
   nothing arrives at, with the kernels' own wait routine and a limit of limit_ns
   (0 < limit_ns <= 1e9).  The wait gives up, the kernel writes done[0] = 1 and
   done[1] = 0 (device int[2], caller-owned) and returns, and the next
   ts_device_status() reports TS_ERR_TIMEOUT; the context stays usable.
   Asynchronous on `stream`. */
ts_status ts_selftest_bounded_wait(long long limit_ns, int* done, void* stream);

/* Kernel trace (tracing subsystem).  Between ts_trace_begin() and ts_trace_end()
   every kernel the library enqueues is bracketed by two CUDA events on its own
   stream and recorded with its algorithmic work (FLOPs of the contraction, bytes
   that must cross HBM at least once).  ts_trace_end() synchronises those events
   and returns one entry per kernel class, in first-seen order; at most
   `capacity` entries are written and *count is the number of classes.  Events
   are taken from a pool made by ts_trace_begin (max_launches events pairs);
   launches beyond it are counted but not timed.  Process-wide, not for
   concurrent use by several threads. */
typedef struct {
  char name[48];      /* kernel class, e.g. "gemm_up", "attention", "blend"      */
  int launches;       /* launches recorded                                       */
  int timed;          /* launches with event timing                              */
  double ms;          /* summed event time of the timed launches                 */
  double flops;       /* summed algorithmic FLOPs of the timed launches          */
  double bytes;       /* summed algorithmic HBM bytes of the timed launches      */
} ts_trace_entry;
ts_status ts_trace_begin(int max_launches);
ts_status ts_trace_end(ts_trace_entry* entries, int capacity, int* count);

/* Kernels enqueued by the library since it was loaded (all devices, all threads). */
long long ts_launch_count(void);

const char* ts_status_string(ts_status s);
const char* ts_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* TILESHARE_H */
