"""Pins of the oracle's layers (CPU only).

Each test ties the vectorised float64 oracle to something other than itself:
    * the single-tile case, where both layers reduce to one plain pre-LN ViT block,
      written with torch.nn.functional library routines (RoPE as complex
      multiplication);
    * an explicit scalar-loop restatement on tiny grids (brute force);
    * the exactness statements of the pages: no overlap -> shared == per-tile;
      blending attention outputs before or after the out-projection is the same
      map; identical per-tile states stay identical; k = L is tiled decoding
      blended at the end;
    * RoPE invariants (relative positions, norms).
"""

import dataclasses
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as Fn

from oracle import layers as Lo
from oracle import plan as P
from shared_token_transformer_b200 import workloads as W


def _model(cfg):
    return Lo.Model(cfg.d, cfg.heads, cfg.mlp, cfg.rope_dims, block=cfg.block)


def _setup(cfg, seed=0, affine=True):
    p = P.make_plan(cfg.grid, cfg.win, cfg.stride, registers=cfg.R)
    dr = W.Draw(cfg, p.T, seed=seed, affine=affine)
    S0, G0 = dr.states()
    return p, np.concatenate([S0, G0]), dr.layers()


# ---------------------------------------------------------------------------
# single tile: both layers == a plain pre-LN ViT block from library routines
# ---------------------------------------------------------------------------

def _torch_block(x, prm, m, pos):
    """One pre-LN ViT block; the first len(x) - len(pos) rows (registers) are
    unrotated, the others use positions pos."""
    t = {k: torch.from_numpy(np.asarray(v)) for k, v in prm.items()}
    x = torch.from_numpy(x)
    n, d, h, hd = x.shape[0], m.d, m.heads, m.hd
    R = n - pos.shape[0]
    swiglu = m.block == "rms_swiglu"

    def norm(z, g, b):
        return Fn.rms_norm(z, (d,), g, eps=m.eps_ln) if swiglu else Fn.layer_norm(z, (d,), g, b, eps=m.eps_ln)

    a = norm(x, t["ln1_g"], t["ln1_b"])
    qkv = Fn.linear(a, t["w_qkv"], t["b_qkv"])
    q, k, v = (qkv[:, i * d:(i + 1) * d].reshape(n, h, hd) for i in range(3))
    q = Fn.rms_norm(q, (hd,), t["q_g"], eps=m.eps_qk)
    k = Fn.rms_norm(k, (hd,), t["k_g"], eps=m.eps_qk)

    def rot(z):
        out = z.clone()
        off = 0
        for ax, D in enumerate(m.rope_dims):
            half = D // 2
            if half:
                j = torch.arange(half, dtype=torch.float64)
                ang = torch.from_numpy(pos[:, ax].astype(np.float64))[:, None] * m.rope_base ** (-2 * j / D)
                zc = torch.complex(z[R:, :, off:off + half], z[R:, :, off + half:off + D])
                zr = zc * torch.polar(torch.ones_like(ang), ang)[:, None, :]
                out[R:, :, off:off + half] = zr.real
                out[R:, :, off + half:off + D] = zr.imag
            off += D
        return out

    q, k = rot(q), rot(k)
    o = Fn.scaled_dot_product_attention(q.transpose(0, 1), k.transpose(0, 1), v.transpose(0, 1))
    o = o.transpose(0, 1).reshape(n, d)
    x = x + Fn.linear(o, t["w_o"], t["b_o"])
    a = norm(x, t["ln2_g"], t["ln2_b"])
    up = Fn.linear(a, t["w_1"], t["b_1"])
    if swiglu:
        gate, val = up.chunk(2, dim=-1)          # gate rows first
        hid = Fn.silu(gate) * val
    else:
        hid = Fn.gelu(up)
    x = x + Fn.linear(hid, t["w_2"], t["b_2"])
    return x.numpy()


@pytest.mark.parametrize("block,R", [("ln_gelu", 1), ("rms_swiglu", 1), ("ln_gelu", 4)])
@pytest.mark.parametrize("grid,rope", [((1, 6, 7), (0, 8, 8)), ((2, 3, 4), (4, 6, 6))])
def test_single_tile_equals_library_block(grid, rope, block, R):
    cfg = W.Config("one_tile", grid, grid, grid, 64, 4, 96, "f32", 1, 0, rope, block=block, R=R)
    m = _model(cfg)
    p, S, layers = _setup(cfg)
    assert p.T == 1
    X = Lo.gather(S, p)
    want = _torch_block(X[0].copy(), layers[0], m, p.slot_pos)
    got_tiled = Lo.block_tiled(X, layers[0], m, p)[0]
    np.testing.assert_allclose(got_tiled, want, rtol=0, atol=1e-12)
    got_shared = Lo.block_shared(S, layers[0], m, p)
    np.testing.assert_allclose(Lo.gather(got_shared, p)[0], want, rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------
# brute force: scalar loops on a tiny grid
# ---------------------------------------------------------------------------

def _loop_layer_shared(S, prm, m, p):
    """Shared layer with explicit loops; tiles found by box containment, not CSR."""
    U, T, d, h, hd = p.U, p.T, m.d, m.heads, m.hd
    n = S.shape[0]

    swiglu = m.block == "rms_swiglu"

    def ln(row, g, b):
        if swiglu:                      # RMSNorm: no centring, no bias
            r = math.sqrt(sum(v * v for v in row) / d + m.eps_ln)
            return [row[c] / r * g[c] for c in range(d)]
        mu = sum(row) / d
        var = sum((v - mu) ** 2 for v in row) / d
        return [(row[c] - mu) / math.sqrt(var + m.eps_ln) * g[c] + b[c] for c in range(d)]

    def act(up):
        if swiglu:                      # first half gates the second
            f = len(up) // 2
            return [up[c] / (1 + math.exp(-up[c])) * up[f + c] for c in range(f)]
        return [gelu(z) for z in up]

    def lin(row, w, b):
        return [sum(row[c] * w[o][c] for c in range(len(row))) + b[o] for o in range(len(w))]

    def gelu(z):
        return 0.5 * z * (1 + math.erf(z / math.sqrt(2)))

    def rmsn(vec, g):
        r = math.sqrt(sum(v * v for v in vec) / len(vec) + m.eps_qk)
        return [vec[c] / r * g[c] for c in range(len(vec))]

    def rope_vec(vec, pos):
        out = list(vec)
        off = 0
        for ax, D in enumerate(m.rope_dims):
            for j in range(D // 2):
                ang = pos[ax] * m.rope_base ** (-2.0 * j / D)
                a, b = vec[off + j], vec[off + j + D // 2]
                out[off + j] = a * math.cos(ang) - b * math.sin(ang)
                out[off + j + D // 2] = a * math.sin(ang) + b * math.cos(ang)
            off += D
        return out

    q = [[None] * h for _ in range(n)]
    k = [[None] * h for _ in range(n)]
    v = [[None] * h for _ in range(n)]
    for r in range(n):
        a = lin(ln(list(S[r]), prm["ln1_g"], prm["ln1_b"]), prm["w_qkv"], prm["b_qkv"])
        for hh in range(h):
            q[r][hh] = rmsn(a[hh * hd:(hh + 1) * hd], prm["q_g"])
            k[r][hh] = rmsn(a[d + hh * hd:d + (hh + 1) * hd], prm["k_g"])
            v[r][hh] = a[2 * d + hh * hd:2 * d + (hh + 1) * hd]

    F_, H_, W_ = p.grid
    wf, wh, ww = p.win
    A = [[0.0] * d for _ in range(n)]
    for t in range(T):
        of, oy, ox = (int(c) for c in p.origins[t])
        rows, poss = [U + t * p.R + i for i in range(p.R)], [None] * p.R
        for lf in range(wf):
            for ly in range(wh):
                for lx in range(ww):
                    rows.append(((of + lf) * H_ + (oy + ly)) * W_ + (ox + lx))
                    poss.append((lf, ly, lx))
        for hh in range(h):
            qs = [q[r][hh] if pp is None else rope_vec(q[r][hh], pp) for r, pp in zip(rows, poss)]
            ks = [k[r][hh] if pp is None else rope_vec(k[r][hh], pp) for r, pp in zip(rows, poss)]
            for i, r in enumerate(rows):
                sc = [sum(qs[i][c] * ks[j][c] for c in range(hd)) / math.sqrt(hd) for j in range(len(rows))]
                mx = max(sc)
                ex = [math.exp(s - mx) for s in sc]
                z = sum(ex)
                o = [sum(ex[j] / z * v[rows[j]][hh][c] for j in range(len(rows))) for c in range(hd)]
                if i < p.R:
                    wgt = 1.0
                else:
                    wgt = p.wbar[t, i - p.R]
                for c in range(hd):
                    A[r][hh * hd + c] += wgt * o[c]
    out = np.empty_like(S)
    for r in range(n):
        x = [S[r][c] + y for c, y in enumerate(lin(A[r], prm["w_o"], prm["b_o"]))]
        hid = act(lin(ln(x, prm["ln2_g"], prm["ln2_b"]), prm["w_1"], prm["b_1"]))
        out[r] = [x[c] + y for c, y in enumerate(lin(hid, prm["w_2"], prm["b_2"]))]
    return out


@pytest.mark.parametrize("grid,win,stride,rope,block,R", [
    ((1, 5, 5), (1, 3, 3), (1, 2, 2), (0, 2, 2), "ln_gelu", 1),
    ((2, 4, 5), (2, 3, 3), (1, 1, 2), (2, 2, 4), "ln_gelu", 1),
    ((1, 5, 5), (1, 3, 3), (1, 2, 2), (0, 2, 2), "rms_swiglu", 1),
    ((1, 5, 5), (1, 3, 3), (1, 2, 2), (0, 2, 2), "ln_gelu", 3),
])
def test_shared_layer_brute_force(grid, win, stride, rope, block, R):
    cfg = W.Config("bf", grid, win, stride, 16, 2, 24, "f32", 1, 0, rope, block=block, R=R)
    m = _model(cfg)
    p, S, layers = _setup(cfg, seed=3)
    prm = {k: (v.tolist() if v.ndim == 2 else list(v)) for k, v in layers[0].items()}
    want = _loop_layer_shared(S, prm, m, p)
    got = Lo.block_shared(S, layers[0], m, p)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------
# exactness statements of the pages
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("block,R", [("ln_gelu", 1), ("rms_swiglu", 1), ("ln_gelu", 3)])
def test_no_overlap_shared_equals_tiled(block, R):
    cfg = dataclasses.replace(W.CONFIGS["vit16_nooverlap_fp32"], block=block, R=R)
    m = _model(cfg)
    p, S, layers = _setup(cfg)
    got = Lo.block_shared(S, layers[0], m, p)
    want = Lo.merge(Lo.block_tiled(Lo.gather(S, p), layers[0], m, p), p)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_blend_before_or_after_out_projection():
    # Shared layer == merge of (gathered copies + per-tile attention sub-block), then MLP.
    cfg = W.small_config(grid=(1, 11, 9), win=(1, 6, 5), stride=(1, 4, 2), d=32, heads=2, mlp=48, dtype="f32")
    m = _model(cfg)
    p, S, layers = _setup(cfg, seed=5)
    prm = layers[0]
    X = Lo.gather(S, p)
    Xa = np.empty_like(X)
    for t in range(p.T):
        q, k, v = Lo.qkv_project(X[t], prm, m)
        o = Lo.tile_attention(q, k, v, p.slot_pos, m)
        Xa[t] = X[t] + o @ prm["w_o"].T + prm["b_o"]
    want = Lo.mlp_residual(Lo.merge(Xa, p), prm, m)
    got = Lo.block_shared(S, prm, m, p)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


@pytest.mark.parametrize("R", [1, 3])
def test_identical_per_tile_states_stay_identical(R):
    cfg = dataclasses.replace(W.small_config(grid=(1, 9, 9), win=(1, 5, 5), stride=(1, 2, 2), d=32, heads=2,
                                             mlp=48, dtype="f32"), R=R)
    m = _model(cfg)
    p, S, layers = _setup(cfg, seed=7)
    assert S.shape[0] == p.U + p.T * R
    X = Lo.gather(S, p)
    q, k, v = Lo.qkv_project(S, layers[0], m)
    for t in range(p.T):
        qt, kt, vt = Lo.qkv_project(X[t], layers[0], m)
        rows = np.concatenate([[p.U + t * R + i for i in range(R)], p.tile_tok[t]])
        for a, b in ((qt, q), (kt, k), (vt, v)):
            np.testing.assert_allclose(a, b[rows], rtol=0, atol=1e-14)
    # merging identical copies returns the state itself
    np.testing.assert_allclose(Lo.merge(X, p), S, rtol=0, atol=1e-14)


@pytest.mark.parametrize("block,R", [("ln_gelu", 1), ("rms_swiglu", 1), ("ln_gelu", 2)])
def test_stack_k_equals_L_is_tiled_decoding_blended_at_the_end(block, R):
    cfg = dataclasses.replace(W.small_config(grid=(1, 10, 9), win=(1, 6, 5), stride=(1, 4, 3), d=32, heads=2,
                                             mlp=48, dtype="f32", L=3, k=3, block=block), R=R)
    m = _model(cfg)
    p, S, layers = _setup(cfg, seed=11)
    got = Lo.decode_stack(S[:p.U], S[p.U:], layers, m, p, k=3)
    X = Lo.gather(S, p)
    outs = []
    for t in range(p.T):          # every tile decoded on its own
        x = X[t:t + 1]
        for prm in layers:
            x = Lo.block_tiled(x, prm, m, p)
        outs.append(x[0])
    want = Lo.merge(np.stack(outs), p)[:p.U]
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_stack_k_zero_is_all_shared_and_k_mixes():
    cfg = W.small_config(grid=(1, 8, 8), win=(1, 5, 5), stride=(1, 3, 3), d=32, heads=2, mlp=48,
                         dtype="f32", L=2, k=1)
    m = _model(cfg)
    p, S, layers = _setup(cfg, seed=2)
    got0 = Lo.decode_stack(S[:p.U], S[p.U:], layers, m, p, k=0)
    want0 = Lo.block_shared(Lo.block_shared(S, layers[0], m, p), layers[1], m, p)[:p.U]
    np.testing.assert_allclose(got0, want0, rtol=0, atol=1e-13)
    got1 = Lo.decode_stack(S[:p.U], S[p.U:], layers, m, p, k=1)
    want1 = Lo.block_shared(Lo.merge(Lo.block_tiled(Lo.gather(S, p), layers[0], m, p), p), layers[1], m, p)
    np.testing.assert_allclose(got1, want1[:p.U], rtol=0, atol=1e-13)


# ---------------------------------------------------------------------------
# RoPE invariants and elementary operations
# ---------------------------------------------------------------------------

def test_rope_relative_and_norm_preserving():
    m = Lo.Model(64, 1, 64, (16, 24, 24))
    rng = np.random.default_rng(0)
    q = rng.standard_normal((20, 1, 64))
    k = rng.standard_normal((20, 1, 64))
    pos = rng.integers(0, 40, (20, 3))
    shift = np.array([3, -7, 11])
    s1 = np.einsum("ihc,jhc->ij", Lo.rope(q, pos, m), Lo.rope(k, pos, m))
    s2 = np.einsum("ihc,jhc->ij", Lo.rope(q, pos + shift, m), Lo.rope(k, pos + shift, m))
    np.testing.assert_allclose(s1, s2, rtol=0, atol=1e-11)
    np.testing.assert_allclose(np.linalg.norm(Lo.rope(q, pos, m), axis=-1), np.linalg.norm(q, axis=-1),
                               rtol=1e-14)
    np.testing.assert_array_equal(Lo.rope(q, np.zeros_like(pos), m), q)


def test_elementary_ops_against_library():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((7, 48))
    g = rng.standard_normal(48)
    b = rng.standard_normal(48)
    np.testing.assert_allclose(Lo.layer_norm(x, g, b, 1e-6),
                               Fn.layer_norm(torch.from_numpy(x), (48,), torch.from_numpy(g),
                                             torch.from_numpy(b), eps=1e-6).numpy(), atol=1e-13)
    np.testing.assert_allclose(Lo.gelu(x), Fn.gelu(torch.from_numpy(x)).numpy(), atol=1e-15)
    np.testing.assert_allclose(Lo.rms_norm(x, g, 1e-6),
                               Fn.rms_norm(torch.from_numpy(x), (48,), torch.from_numpy(g), eps=1e-6).numpy(),
                               atol=1e-13)


# ---------------------------------------------------------------------------
# partial sharing (Tab. 1 top, reading R12)
# ---------------------------------------------------------------------------

_PARTIAL_CFG = W.small_config(grid=(2, 9, 11), win=(2, 5, 6), stride=(1, 3, 4), d=32, heads=2, mlp=48,
                              dtype="f32")


def test_partial_sharing_nothing_shared_is_the_per_tile_layer():
    m = _model(_PARTIAL_CFG)
    p, S, layers = _setup(_PARTIAL_CFG, seed=11)
    X = Lo.gather(S, p)
    X = X + 0.1 * np.random.default_rng(1).standard_normal(X.shape)   # tiles disagree on overlap tokens
    np.testing.assert_array_equal(Lo.block_partial(X, layers[0], m, p, ()), Lo.block_tiled(X, layers[0], m, p))


@pytest.mark.parametrize("shared", [("out",), ("qkv", "out"), ("qkv", "out", "mlp"), ("out", "mlp")])
def test_partial_sharing_on_identical_copies_is_the_shared_layer(shared):
    """Tab. 1's footnote: with the out-projection shared, identical per-tile states stay
    identical, so from gathered copies the layer equals the TileShare shared layer
    (every tile holds the shared result for each of its tokens)."""
    m = _model(_PARTIAL_CFG)
    p, S, layers = _setup(_PARTIAL_CFG, seed=12)
    got = Lo.block_partial(Lo.gather(S, p), layers[0], m, p, shared)
    want = Lo.gather(Lo.block_shared(S, layers[0], m, p), p)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_partial_sharing_mlp_only_merges_to_the_shared_layer():
    """MLP only, from identical copies: the tiles' attention outputs differ, but the
    MLP input is their blend, which by linearity of the out-projection is the shared
    layer's state after attention; merging the result gives the shared layer."""
    m = _model(_PARTIAL_CFG)
    p, S, layers = _setup(_PARTIAL_CFG, seed=13)
    X = Lo.block_partial(Lo.gather(S, p), layers[0], m, p, ("mlp",))
    np.testing.assert_allclose(Lo.merge(X, p), Lo.block_shared(S, layers[0], m, p), rtol=0, atol=1e-12)


def test_partial_sharing_qkv_only_from_distinct_copies():
    """QKV only, on per-tile states that disagree: q/k/v come from the merged state and
    are identical for every copy of a token, while the out-projection and MLP stay
    per tile.  Checked against a per-tile loop written out here."""
    m = _model(_PARTIAL_CFG)
    p, S, layers = _setup(_PARTIAL_CFG, seed=14)
    prm = layers[0]
    X = Lo.gather(S, p) + 0.1 * np.random.default_rng(2).standard_normal((p.T, p.N, m.d))
    Sm = Lo.merge(X, p)
    q, k, v = Lo.qkv_project(Sm, prm, m)
    want = np.empty_like(X)
    for t in range(p.T):
        rows = np.concatenate([[p.U + t], p.tile_tok[t]])
        o = Lo.tile_attention(q[rows], k[rows], v[rows], p.slot_pos, m)
        x = X[t] + o @ prm["w_o"].T + prm["b_o"]
        want[t] = Lo.mlp_residual(x, prm, m)
    np.testing.assert_allclose(Lo.block_partial(X, prm, m, p, ("qkv",)), want, rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------
# RMSNorm + SwiGLU block flavour (Tab. S6, reading R13)
# ---------------------------------------------------------------------------

def test_silu_against_library_and_identities():
    from scipy.special import expit
    z = np.concatenate([np.linspace(-40, 40, 801), [-800.0, -1e-300, 0.0, 1e-300, 800.0]])
    np.testing.assert_allclose(Lo.silu(z), z * expit(z), rtol=1e-15, atol=1e-300)
    assert Lo.silu(np.array([0.0]))[0] == 0.0
    # silu(z) - silu(-z) = z (sigmoid(z) + sigmoid(-z) = 1)
    np.testing.assert_allclose(Lo.silu(z[:801]) - Lo.silu(-z[:801]), z[:801], rtol=0, atol=1e-13)


def _swiglu_setup(seed=4):
    cfg = W.small_config(grid=(1, 4, 4), win=(1, 4, 4), stride=(1, 4, 4), d=32, heads=2, mlp=40, dtype="f32",
                         block="rms_swiglu")
    m = _model(cfg)
    dr = W.Draw(cfg, 1, seed=seed, affine=True)
    x = dr.rng.standard_normal((9, cfg.d))
    return cfg, m, dr.layer(), x


def _rms_rows(x, g, eps):
    # RMSNorm through the Euclidean norm: x * sqrt(d) / sqrt(|x|^2 + d eps) * g
    d = x.shape[1]
    return x * math.sqrt(d) / np.sqrt(np.linalg.norm(x, axis=1, keepdims=True) ** 2 + d * eps) * g


def test_swiglu_mlp_odd_part_is_the_gated_product():
    # Negating the gate rows and gate bias: silu(z) - silu(-z) = z, so the difference
    # of the two MLPs is W_2 ((W_g h + b_g) * (W_u h + b_u)); b_2 cancels.  A swapped
    # gate/up split, a dropped bias or a LayerNorm in place of RMSNorm all break it.
    cfg, m, prm, x = _swiglu_setup()
    f = cfg.mlp
    neg = dict(prm)
    neg["w_1"] = prm["w_1"].copy()
    neg["b_1"] = prm["b_1"].copy()
    neg["w_1"][:f] *= -1
    neg["b_1"][:f] *= -1
    h = _rms_rows(x, prm["ln2_g"], m.eps_ln)
    g = h @ prm["w_1"][:f].T + prm["b_1"][:f]
    u = h @ prm["w_1"][f:].T + prm["b_1"][f:]
    want = (g * u) @ prm["w_2"].T
    np.testing.assert_allclose(Lo.mlp_out(x, prm, m) - Lo.mlp_out(x, neg, m), want, rtol=0, atol=1e-13)


def test_swiglu_saturated_gate():
    # W_g = 0: the gate is the constant b_g.  b_g = 60 -> silu = 60 (to 1e-24), the MLP is
    # the linear map 60 W_2 (W_u h + b_u) + b_2;  b_g = -60 -> silu ~ 0, the MLP is b_2.
    cfg, m, prm, x = _swiglu_setup(seed=8)
    f = cfg.mlp
    h = _rms_rows(x, prm["ln2_g"], m.eps_ln)
    for bg, want in ((60.0, 60.0 * (h @ prm["w_1"][f:].T + prm["b_1"][f:]) @ prm["w_2"].T + prm["b_2"]),
                     (-60.0, np.broadcast_to(prm["b_2"], (x.shape[0], cfg.d)))):
        q = dict(prm)
        q["w_1"] = prm["w_1"].copy()
        q["b_1"] = prm["b_1"].copy()
        q["w_1"][:f] = 0.0
        q["b_1"][:f] = bg
        np.testing.assert_allclose(Lo.mlp_out(x, q, m), want, rtol=1e-13, atol=1e-13)


def test_rms_block_norm_is_layer_norm_of_centred_rows():
    # On rows of zero mean, RMSNorm with gain g is LayerNorm with gain g and bias 0.
    m = Lo.Model(48, 2, 64, (0, 12, 12), block="rms_swiglu")
    rng = np.random.default_rng(6)
    x = rng.standard_normal((5, 48))
    x -= x.mean(axis=1, keepdims=True)
    g = rng.standard_normal(48)
    b = rng.standard_normal(48)          # ignored by RMSNorm
    np.testing.assert_allclose(Lo.block_norm(x, g, b, m), Lo.layer_norm(x, g, np.zeros(48), 1e-6), atol=1e-14)
