"""The analytic FLOP model of oracle.flops against the products the oracle's layers
actually carry out (CPU only).

[TileShare] Tab. 1 and Tab. S7 give block FLOPs of shared layers relative to
per-tile layers; oracle.flops restates that count for our shapes (four linear
layers and the two contractions of attention, 2 FLOPs per multiply-add).  Here
every call of oracle.layers.linear and oracle.layers.attention made by a layer or
a stack is intercepted and the FLOPs of its operand shapes are summed:
2 * rows * out * in per linear layer, 2 * n_q * n_k * hd per head for the scores
Q K^T and again for P V.  The totals must equal the closed forms exactly, so a
dropped factor (2 T N^2 d for attention, a missing out-projection, the gate rows of
a SwiGLU MLP) fails here.
"""

import numpy as np
import pytest

from oracle import flops as Fo
from oracle import layers as OL
from oracle import plan as P
from shared_token_transformer_b200 import workloads as W


@pytest.fixture
def count(monkeypatch):
    """Intercept the oracle's linear layers and attention; return the running totals."""
    tot = {"linear": 0, "attention": 0}
    real_linear, real_attention = OL.linear, OL.attention

    def linear(x, w, b, m):
        tot["linear"] += 2 * x.shape[0] * w.shape[0] * w.shape[1]
        return real_linear(x, w, b, m)

    def attention(q, k, v):
        n, h, hd = q.shape
        tot["attention"] += 2 * (2 * n * k.shape[0] * hd * h)     # Q K^T and P V, every head
        return real_attention(q, k, v)

    monkeypatch.setattr(OL, "linear", linear)
    monkeypatch.setattr(OL, "attention", attention)

    def reset():
        tot["linear"] = tot["attention"] = 0
    tot["reset"] = reset
    return tot


def _setup(block="ln_gelu", grid=(1, 11, 13), win=(1, 8, 8), stride=(1, 5, 6), R=1):
    cfg = W.small_config("flops", grid=grid, win=win, stride=stride, d=32, heads=2, mlp=48, dtype="f32", L=3, k=1,
                         block=block)
    op = P.make_plan(cfg.grid, cfg.win, cfg.stride, registers=R)
    dr = W.Draw(cfg, op.T, seed=3, affine=True)
    S0, G0 = dr.states()
    if R > 1:
        G0 = np.random.default_rng(4).standard_normal((op.T * R, cfg.d))
    layers = dr.layers()
    m = OL.Model(cfg.d, cfg.heads, cfg.mlp, cfg.rope_dims, block=block)
    return cfg, op, S0, G0, layers, m


@pytest.mark.parametrize("block", ["ln_gelu", "rms_swiglu"])
def test_layer_flops_equal_the_products_the_oracle_computes(count, block):
    cfg, op, S0, G0, layers, m = _setup(block)
    d, f, gated = cfg.d, cfg.mlp, block == "rms_swiglu"
    T, N, U = op.T, op.N, op.U
    X = OL.gather(np.concatenate([S0, G0]), op)
    OL.block_tiled(X, layers[0], m, op)
    assert count["attention"] == Fo.attention_flops(T, N, d)
    assert count["linear"] == T * N * Fo.linear_flops_per_row(d, f, gated)
    assert count["attention"] + count["linear"] == Fo.tiled_layer_flops(T, N, d, f, gated)
    count["reset"]()
    OL.block_shared(np.concatenate([S0, G0]), layers[0], m, op)
    assert count["attention"] == Fo.attention_flops(T, N, d)
    assert count["linear"] == (U + T) * Fo.linear_flops_per_row(d, f, gated)
    assert count["attention"] + count["linear"] == Fo.shared_layer_flops(U, T, N, d, f, gated)


@pytest.mark.parametrize("shared", [(), ("qkv",), ("out",), ("mlp",), ("qkv", "out"), ("qkv", "mlp"),
                                    ("out", "mlp"), ("qkv", "out", "mlp")], ids=lambda s: "+".join(s) or "none")
def test_partial_layer_flops_equal_the_products_the_oracle_computes(count, shared):
    cfg, op, S0, G0, layers, m = _setup()
    X = OL.gather(np.concatenate([S0, G0]), op)
    OL.block_partial(X, layers[0], m, op, shared)
    assert count["attention"] + count["linear"] == Fo.partial_layer_flops(op.U, op.T, op.N, cfg.d, cfg.mlp, shared)


@pytest.mark.parametrize("k", [0, 1, 3])
def test_stack_flop_ratio_equals_counted_ratio(count, k):
    cfg, op, S0, G0, layers, m = _setup()
    OL.decode_stack(S0, G0, layers, m, op, k)
    stack = count["attention"] + count["linear"]
    count["reset"]()
    OL.decode_stack(S0, G0, layers, m, op, len(layers))           # all per tile
    tiled = count["attention"] + count["linear"]
    want = Fo.stack_flop_ratio(op.U, op.T, op.N, cfg.d, cfg.mlp, len(layers), k)
    assert stack / tiled == pytest.approx(want, rel=1e-15)


def test_counts_follow_the_register_count(count):
    # R register rows per tile: N = Nw + R rows attend in every tile, U + T*R rows are shared
    cfg, op, S0, G0, layers, m = _setup(R=3)
    OL.block_shared(np.concatenate([S0, G0]), layers[0], m, op)
    assert count["attention"] == Fo.attention_flops(op.T, op.N, cfg.d)
    assert count["linear"] == (op.U + op.T * op.R) * Fo.linear_flops_per_row(cfg.d, cfg.mlp)
