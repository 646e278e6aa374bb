"""Oracle: the per-tile layer, the shared layer and the TileShare-k stack.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).  float64 NumPy, no
blocking, fusion or reordering beyond what the pages state.

What the pages fix
    * [TileShare] Tab. S1 (each operation of a block under TileShare):
        - Norm1, QKV projection and QK-RMSNorm run once per token on the shared
          state (exact: identical inputs give identical results);
        - RoPE runs per tile on tile coordinates, as released;
        - attention is dense and per tile, with the tile's own registers (R per
          tile, R14; one global token in the benchmark configurations) that
          attend only to their own tile; keys and values come from the shared
          states;
        - the blend of attention outputs of overlap tokens is the only
          approximation and happens in every shared layer.
    * [TileShare] Fig. 2: out-projection and MLP also run once per token; overlap
      tokens are stored once but attended in every window covering them; their
      attention outputs are blended with w-bar.
    * [TileShare] abstract and Tab. 1: TileShare-k keeps the first k layers per
      tile (each tile its own residual stream), the rest shared.
    * [TileShare] Fig. 3b: the per-tile states can be merged into one state.

Readings taken where the pages are silent
    R4 block: pre-LN ViT block  x += W_o Attn(RoPE(QKnorm(W_qkv LN1(x)))) + b_o;
       x += W_2 GELU(W_1 LN2(x) + b_1) + b_2; LayerNorm and QK-RMSNorm eps 1e-6
       with learnable gain (and LN bias); exact erf GELU; attention scale
       1/sqrt(hd), no mask.  QKV columns: [q | k | v], head h at h*hd.
    R5 the global token is not rotated by RoPE.
    R6 RoPE: the head dimension is split into consecutive blocks of
       rope_dims = (D_f, D_y, D_x) channels for the three axes; inside a block of
       D channels, channel j pairs with j + D/2 (j < D/2) and is rotated by angle
       pos * base^(-2j/D), pos being the integer tile-local coordinate.
    R7 the blend acts on the attention outputs, before the out-projection
       (Fig. 2 says the attention outputs are blended).  Because w-bar sums to 1,
       blending before or after the out-projection and residual is the same map.
    R8 the transition at layer k merges the per-tile states with the same w-bar
       (Fig. 3b); each global token keeps its own tile's state.
    R13 block flavour "rms_swiglu" (Tab. S6 profiles a block with "RMSNorm +
       residual" and a "SwiGLU gate"): Norm1 and Norm2 are RMSNorm with a gain and
       no bias (eps_ln); the MLP is  W_2 (silu(W_g h + b_g) * (W_u h + b_u)) + b_2
       with silu(z) = z / (1 + exp(-z)), where w_1 = [W_g; W_u] stacks the f gate
       rows above the f up rows and b_1 = [b_g; b_u].  Everything else as in R4.
    R12 partial sharing (Tab. 1 top: from layer k on each tile keeps its own
       residual stream and only the listed operations are shared; attention always
       runs per tile): a shared operation takes, for each grid token, the w-bar
       blend of its tiles' inputs (the merge of R8; a tile's global token keeps its
       own row) and runs once per token.  Its result serves every tile covering
       the token: shared q/k/v feed each tile's attention through the tile's rows;
       the shared out-projection's and MLP's outputs are added to every tile's copy
       of the token.
"""

import math
from dataclasses import dataclass

import numpy as np
from scipy.special import erf

from . import fp8 as _fp8


@dataclass(frozen=True)
class Model:
    d: int
    heads: int
    mlp: int
    rope_dims: tuple          # (D_f, D_y, D_x), sum = head dim, each even
    eps_ln: float = 1e-6
    eps_qk: float = 1e-6
    rope_base: float = 10000.0
    fp8: bool = False         # e4m3 GEMMs with per-channel / per-token scales
    block: str = "ln_gelu"    # "ln_gelu" (R4) or "rms_swiglu" (R13)

    @property
    def hd(self):
        return self.d // self.heads


# ---------------------------------------------------------------------------
# elementary operations
# ---------------------------------------------------------------------------

def layer_norm(x, g, b, eps):
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps) * g + b


def rms_norm(x, g, eps):
    return x / np.sqrt((x * x).mean(axis=-1, keepdims=True) + eps) * g


def gelu(x):
    return 0.5 * x * (1.0 + erf(x / math.sqrt(2.0)))


def silu(x):
    """z / (1 + exp(-z)); exp overflows to inf for z < -709, where the quotient is -0."""
    with np.errstate(over="ignore"):
        return x / (1.0 + np.exp(-x))


def block_norm(x, g, b, m):
    """Norm1 / Norm2 of the block: LayerNorm (R4) or RMSNorm without bias (R13)."""
    if m.block == "rms_swiglu":
        return rms_norm(x, g, m.eps_ln)
    return layer_norm(x, g, b, m.eps_ln)


def rope(x, pos, m: Model):
    """Rotate x [n, heads, hd] of rows at integer coordinates pos [n, 3] (R6)."""
    out = x.copy()
    off = 0
    for axis, D in enumerate(m.rope_dims):
        half = D // 2
        for j in range(half):
            theta = m.rope_base ** (-2.0 * j / D)
            ang = pos[:, axis].astype(np.float64) * theta          # [n]
            c = np.cos(ang)[:, None]
            s = np.sin(ang)[:, None]
            a = x[:, :, off + j]
            b = x[:, :, off + j + half]
            out[:, :, off + j] = a * c - b * s
            out[:, :, off + j + half] = a * s + b * c
        off += D
    return out


def linear(x, w, b, m: Model):
    """x @ w.T + b; with m.fp8 the product is the e4m3 scaled GEMM of fp8.scaled_matmul."""
    if m.fp8:
        y = _fp8.scaled_matmul(x, w)
    else:
        y = x @ w.T
    return y + b


def attention(q, k, v):
    """Dense softmax attention of one tile, all heads: q, k, v [n, heads, hd] -> [n, heads*hd].

    Head by head: scores q_j k_j^T / sqrt(hd), a softmax over the keys, then the
    weighted sum of the values.
    """
    n, h, hd = q.shape
    o = np.empty((n, h, hd), dtype=np.float64)
    for j in range(h):
        s = (q[:, j] @ k[:, j].T) / math.sqrt(hd)          # [n, m] scores of head j
        s -= s.max(axis=-1, keepdims=True)
        p = np.exp(s)
        p /= p.sum(axis=-1, keepdims=True)
        o[:, j] = p @ v[:, j]
    return o.reshape(n, h * hd)


# ---------------------------------------------------------------------------
# the pieces of a block
# ---------------------------------------------------------------------------

def qkv_project(x, p, m: Model):
    """Norm1, QKV projection and QK-RMSNorm of rows x [n, d] -> q, k, v [n, heads, hd]."""
    n = x.shape[0]
    h = block_norm(x, p["ln1_g"], p["ln1_b"], m)
    qkv = linear(h, p["w_qkv"], p["b_qkv"], m)
    q = qkv[:, 0 * m.d:1 * m.d].reshape(n, m.heads, m.hd)
    k = qkv[:, 1 * m.d:2 * m.d].reshape(n, m.heads, m.hd)
    v = qkv[:, 2 * m.d:3 * m.d].reshape(n, m.heads, m.hd)
    q = rms_norm(q, p["q_g"], m.eps_qk)
    k = rms_norm(k, p["k_g"], m.eps_qk)
    return q, k, v


def tile_attention(q, k, v, slot_pos, m: Model):
    """Attention of one tile: rows [its R registers, window slot 0..Nw-1].

    RoPE on tile-local coordinates for the window rows only (R5, R6, R14).
    Returns the attention output [N, d] before the out-projection.
    """
    R = q.shape[0] - slot_pos.shape[0]
    q = q.copy()
    k = k.copy()
    q[R:] = rope(q[R:], slot_pos, m)
    k[R:] = rope(k[R:], slot_pos, m)
    return attention(q, k, v)


def mlp_out(x, p, m: Model):
    """W_2 GELU(W_1 LN2(x) + b_1) + b_2 (R4), or the SwiGLU MLP of R13, once per row."""
    h = block_norm(x, p["ln2_g"], p["ln2_b"], m)
    a = linear(h, p["w_1"], p["b_1"], m)
    if m.block == "rms_swiglu":
        h = silu(a[:, :m.mlp]) * a[:, m.mlp:]
    else:
        h = gelu(a)
    return linear(h, p["w_2"], p["b_2"], m)


def mlp_residual(x, p, m: Model):
    """x + W_2 GELU(W_1 LN2(x) + b_1) + b_2, once per row."""
    return x + mlp_out(x, p, m)


# ---------------------------------------------------------------------------
# tile <-> token maps
# ---------------------------------------------------------------------------

def tile_rows(plan, t):
    """Rows of the shared state that tile t attends over: its registers, then its window."""
    U, R = plan.U, plan.R
    return np.concatenate([np.arange(U + t * R, U + (t + 1) * R), plan.tile_tok[t]])


def gather(S, plan):
    """Per-tile copies X [T, N, d] of a shared state S [U + T*R, d]."""
    T, N, U, R = plan.T, plan.N, plan.U, plan.R
    X = np.empty((T, N, S.shape[1]), dtype=S.dtype)
    for t in range(T):
        X[t, :R] = S[U + t * R: U + (t + 1) * R]
        X[t, R:] = S[plan.tile_tok[t]]
    return X


def merge(P, plan):
    """Blend per-tile rows P [T, N, d] into one row per token (Fig. 2, R8).

    S[u] = sum over the tiles t covering u, in ascending t, of w-bar[t, u] *
    P[t, slot of u]; S[U + t*R + i] = P[t, i] (each register keeps its tile's row).
    """
    T, N, U, R = plan.T, plan.N, plan.U, plan.R
    flat = P.reshape(T * N, -1)
    S = np.zeros((U + T * R, P.shape[2]), dtype=np.float64)
    for u in range(U):
        for e in range(plan.tok_ptr[u], plan.tok_ptr[u + 1]):
            S[u] += plan.tok_w[e] * flat[plan.tok_ent[e]]
    for t in range(T):
        S[U + t * R: U + (t + 1) * R] = P[t, :R]
    return S


# ---------------------------------------------------------------------------
# layers and the stack
# ---------------------------------------------------------------------------

def block_tiled(X, p, m: Model, plan):
    """One released (per-tile) layer on per-tile states X [T, N, d] (Tab. S1, layer 0)."""
    out = np.empty_like(X, dtype=np.float64)
    for t in range(X.shape[0]):
        x = X[t].astype(np.float64)
        q, k, v = qkv_project(x, p, m)
        o = tile_attention(q, k, v, plan.slot_pos, m)
        x = x + linear(o, p["w_o"], p["b_o"], m)
        out[t] = mlp_residual(x, p, m)
    return out


def shared_attention_outputs(S, p, m: Model, plan):
    """Per-tile attention outputs O [T, N, d] of a shared layer on S [U + T*R, d].

    Norm1/QKV/QK-norm once per token; then, per tile, the rows of the tile's
    registers and window tokens are taken from the shared q, k, v (Tab. S1).
    """
    T, N = plan.T, plan.N
    q, k, v = qkv_project(S, p, m)
    O = np.empty((T, N, m.d), dtype=np.float64)
    for t in range(T):
        rows = tile_rows(plan, t)
        O[t] = tile_attention(q[rows], k[rows], v[rows], plan.slot_pos, m)
    return O


def block_shared(S, p, m: Model, plan):
    """One TileShare shared layer on the shared state S [U + T*R, d] (Fig. 2, Tab. S1)."""
    S = S.astype(np.float64)
    O = shared_attention_outputs(S, p, m, plan)
    A = merge(O, plan)
    S = S + linear(A, p["w_o"], p["b_o"], m)
    return mlp_residual(S, p, m)


SHARED_OPS = ("qkv", "out", "mlp")


def block_partial(X, p, m: Model, plan, shared):
    """One layer on per-tile states X [T, N, d] in which only the operations named
    in `shared` (of "qkv", "out", "mlp") run once per token (Tab. 1 top, R12).

    "qkv": Norm1, QKV and QK-RMSNorm on the merge of X, then each tile attends over
    its rows of the shared q/k/v (RoPE per tile, as released).  "out": the tiles'
    attention outputs are blended and projected once per token, and the result is
    added to every tile's copy.  "mlp": the MLP runs on the merge of X after the
    attention sublayer, and its output is added to every tile's copy.  Everything
    else runs per tile as in block_tiled.
    """
    shared = set(shared)
    if not shared <= set(SHARED_OPS):
        raise ValueError(f"unknown shared operations {shared - set(SHARED_OPS)}")
    T, N, U = plan.T, plan.N, plan.U
    X = np.asarray(X, np.float64).copy()
    O = np.empty((T, N, m.d), dtype=np.float64)
    if "qkv" in shared:
        q, k, v = qkv_project(merge(X, plan), p, m)
        for t in range(T):
            rows = tile_rows(plan, t)
            O[t] = tile_attention(q[rows], k[rows], v[rows], plan.slot_pos, m)
    else:
        for t in range(T):
            q, k, v = qkv_project(X[t], p, m)
            O[t] = tile_attention(q, k, v, plan.slot_pos, m)
    if "out" in shared:
        X = X + gather(linear(merge(O, plan), p["w_o"], p["b_o"], m), plan)
    else:
        for t in range(T):
            X[t] = X[t] + linear(O[t], p["w_o"], p["b_o"], m)
    if "mlp" in shared:
        X = X + gather(mlp_out(merge(X, plan), p, m), plan)
    else:
        for t in range(T):
            X[t] = mlp_residual(X[t], p, m)
    return X


def decode_stack(S0, G0, layers, m: Model, plan, k: int):
    """TileShare-k: layers 0..k-1 per tile, the rest shared; returns the U token rows.

    S0 [U, d] are the grid tokens entering layer 0, G0 [T*R, d] the registers
    (tile t's register i in row t*R + i).
    With k = L this is overlapping tiled decoding with the tiles blended by w-bar at
    the end (abstract; R8).
    """
    L = len(layers)
    if not 0 <= k <= L:
        raise ValueError("k must lie in [0, L]")
    S = np.concatenate([np.asarray(S0, np.float64), np.asarray(G0, np.float64)], axis=0)
    if k > 0:
        X = gather(S, plan)
        for li in range(k):
            X = block_tiled(X, layers[li], m, plan)
        S = merge(X, plan)
    for li in range(k, L):
        S = block_shared(S, layers[li], m, plan)
    return S[: plan.U]
