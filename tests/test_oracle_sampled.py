"""Pin of the sampled-row oracle used by the full-size GPU tests (CPU only): on
small grids its rows equal the whole oracle shared layer."""

import numpy as np
import pytest

from oracle import layers as OL
from oracle import plan as OP
from shared_token_transformer_b200 import workloads as W

from _sampled import oracle_shared_rows, sample_tokens


@pytest.mark.parametrize("cfg", [
    W.small_config("s2d", grid=(1, 11, 13), win=(1, 8, 8), stride=(1, 5, 6), d=32, heads=2, mlp=48, dtype="f32"),
    W.small_config("s3d", grid=(3, 9, 10), win=(2, 6, 6), stride=(1, 4, 4), d=64, heads=2, mlp=48, dtype="f32"),
], ids=lambda c: c.name)
def test_sampled_rows_equal_full_layer(cfg):
    op = OP.make_plan(cfg.grid, cfg.win, cfg.stride)
    dr = W.Draw(cfg, op.T, seed=9, affine=True)
    S0, G0 = dr.states()
    S = np.concatenate([S0, G0])
    layer = dr.layer()
    om = OL.Model(cfg.d, cfg.heads, cfg.mlp, cfg.rope_dims)
    full = OL.block_shared(S, layer, om, op)
    toks = sample_tokens(op, np.random.default_rng(0), n=12)
    assert len(set(op.coverage[toks].tolist())) >= 2
    rows, got = oracle_shared_rows(S, layer, om, op, toks, [0, op.T - 1])
    np.testing.assert_allclose(got, full[rows], rtol=0, atol=1e-12)
