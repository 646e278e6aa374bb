/*
 * tileshare_ops.h -- the individual steps of a layer, exported by libtileshare.so
 * so that each kernel can be checked on its own.  Same conventions as tileshare.h
 * (device pointers, caller-owned buffers, no allocation or synchronisation,
 * ts_status returns, validation before launch).  Sources: [TileShare] =
 * "TileShare: Training-Free Acceleration of Overlapping Tiled ViT Decoding".
 *
 * "rows mode" selects the row set a step works on:
 *   TS_ROWS_SHARED  the U + T*R rows of a shared state S (grid tokens, then registers)
 *   TS_ROWS_TILED   the T * N rows of a per-tile state X
 */
#ifndef TILESHARE_OPS_H
#define TILESHARE_OPS_H

#include "tileshare.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { TS_ROWS_SHARED = 0, TS_ROWS_TILED = 1 } ts_rows_mode;

typedef enum {
  TS_EPI_BIAS = 0,        /* y = x W^T + b                                  */
  TS_EPI_BIAS_GELU = 1,   /* y = GELU(x W^T + b), exact erf GELU            */
  TS_EPI_BIAS_RESID = 2,  /* y += x W^T + b  (y is the residual, in place)  */
  TS_EPI_BIAS_SWIGLU = 3  /* y = silu(x W_g^T + b_g) * (x W_u^T + b_u): W [2N, K]
                             holds the N gate rows above the N up rows, bias and
                             w_scale [2N] likewise; y [rows, N]                   */
} ts_epilogue;

/* Norm1 / Norm2 over the last dimension ([TileShare] Tab. S1 "Norm1"; pre-LN block):
   y[r] = (x[r] - mean) / sqrt(var + eps) * g + b, population variance, eps = eps_ln.
   For TS_BLOCK_RMS_SWIGLU models RMSNorm instead: y[r] = x[r] / sqrt(mean(x[r]^2) +
   eps) * g, and b is unused (may be NULL).
   x, y [rows, d] in the model dtype (bf16 for TS_FP8_E4M3); g, b fp32 [d]. */
ts_status ts_op_layernorm(const ts_model_desc* model, const void* x, int rows,
                          const float* g, const float* b, void* y, void* stream);

/* Linear layer y = x W^T + b with a fused epilogue ([TileShare] Fig. 2: QKV,
   out-projection and MLP once per token).  x [rows, K], W [N, K], y [rows, N], in
   the model dtype (TS_FP8_E4M3: x bf16, W e4m3 with per-row scales w_scale [N];
   x is quantised per row inside the call using `scratch`, which must hold
   rows * K + 4 * rows bytes; scratch is unused otherwise and may be NULL).
   bf16/e4m3 need K % 64 == 0 and N % 64 == 0 (K % 128 for e4m3). */
ts_status ts_op_linear(const ts_model_desc* model, const void* x, int rows, int K,
                       const void* W, const float* w_scale, int N, const float* bias,
                       ts_epilogue epi, void* y, void* scratch, void* stream);

/* Norm1 + QKV projection + QK-RMSNorm + RoPE of the rows of a state ([TileShare]
   Tab. S1: Norm1, QKV, QK-RMSNorm once per token; RoPE on tile coordinates).
   state [rows, d] -> qkv [rows, 3d] (model dtype; bf16 for TS_FP8_E4M3).
   TS_ROWS_TILED rotates q and k of slot j of every tile by its tile-local
   coordinates and leaves rows 0 .. R-1 (the registers) unrotated.  TS_ROWS_SHARED
   rotates grid token u by its grid coordinates and the registers of tile t by
   the tile's origin: attention scores then equal those of tile-local rotation
   exactly (RoPE scores depend on coordinate differences only), so the rotation
   can run once per token.  `scratch` holds, each region 256-byte aligned, the
   normalised rows (rows * d elements of the model dtype), an e4m3 copy
   (rows * d bytes) with per-row scales (4 * rows bytes), and the RoPE cos/sin
   table (8 * (F * D_f + H * D_y + W * D_x) / 2 bytes). */
ts_status ts_op_qkv(ts_plan_t plan, const ts_model_desc* model, const ts_layer_weights* w,
                    ts_rows_mode mode, const void* state, void* qkv, void* scratch, void* stream);

/* Per-tile dense attention ([TileShare] Tab. S1 "Attention (dense, per tile)"; Fig.
   2): for tile t and head h the rows are [registers of t, window slots of t]
   taken from qkv ([U+T*R, 3d] rows for TS_ROWS_SHARED, gathered through the plan's
   index map; [T*N, 3d] for TS_ROWS_TILED); O [T*N, d] (row t*N + s = slot s of
   tile t) = softmax(q k^T / sqrt(hd)) v, no mask.  bf16 needs hd == 64. */
ts_status ts_op_attention(ts_plan_t plan, const ts_model_desc* model, ts_rows_mode mode,
                          const void* qkv, void* O, void* stream);

/* Blend ([TileShare] Fig. 2, Tab. S1 "Blend of attention outputs"; also the merge of
   per-tile states at layer k, Fig. 3b): for the first `rows` rows of the shared
   layout, A[u] = sum over the tiles covering u, in ascending tile order, of
   wbar * P[t*N + R + j] (fp32 sum, one write per token, no atomics) and, for
   rows >= U, A[U + t*R + i] = P[t*N + i].  P [T*N, d], A [rows, d]; rows is U or
   U + T*R. */
ts_status ts_op_merge(ts_plan_t plan, const ts_model_desc* model, const void* P, int rows,
                      void* A, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* TILESHARE_OPS_H */
