"""Parity at the full sizes of the benchmark configurations, on sampled rows.

The CUDA path runs a whole shared layer (or per-tile layer) at the configuration's
size, in the launch configuration the benchmark uses.  The float64 oracle then
recomputes only a sample of output rows, one by one, from the same inputs: for a
sampled grid token it needs the q/k/v rows of every tile covering the token, the
attention of the token's query in each of those tiles, the w-bar blend, the
out-projection and the MLP of that row -- all per-row or per-tile steps of
oracle.layers.  Samples cover tokens in 1, 2 and 4 tiles, the grid corners, the
ragged last tiles and the global tokens.  Tolerance as for the stacks: relative
L2 1e-2 (bf16), 3e-2 (e4m3) over the sampled rows, and the worst sampled row of
every coverage class within 1.5 times that.
"""

import numpy as np
import pytest
import torch

from oracle import layers as OL
from oracle import plan as OP
from shared_token_transformer_b200 import binding as B
from shared_token_transformer_b200 import workloads as W

from _gpu import ROW_FACTOR, assert_rows, dev, dev_layer, host, model_desc, oracle_model, rel_l2, row_rel_errors, TORCH_DT
from _sampled import oracle_shared_rows, sample_tokens

pytestmark = pytest.mark.gpu

FULL = ["video44x80_bf16", "video44x80_fp8", "image4k_bf16", "image2k_bf16", "video88x80_st_bf16"]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from shared_token_transformer_b200 import build
    build.build()
    yield
    B.device_status()


def _setup(name, seed=0):
    cfg = W.CONFIGS[name]
    op = OP.make_plan(cfg.grid, cfg.win, cfg.stride)
    dr = W.Draw(cfg, op.T, seed=seed, affine=True)
    S0, G0 = dr.states()
    layer = dr.layer()
    return cfg, op, np.concatenate([S0, G0]), layer


@pytest.mark.parametrize("name", FULL)
def test_shared_layer_full_size_sampled(name):
    cfg, op, S, layer = _setup(name)
    om = oracle_model(cfg)
    plan = B.Plan(cfg.grid, cfg.win, cfg.stride)
    m = model_desc(cfg)
    w = B.layer_weights(dev_layer(cfg, layer))
    dt = TORCH_DT[cfg.dtype]
    Sd = dev(S, dt)
    ws = torch.empty(B.workspace_size(plan, m, 0, 0), dtype=torch.uint8, device="cuda")
    B.block_shared(plan, m, w, Sd, ws)
    got = host(Sd)
    rng = np.random.default_rng(1)
    toks = sample_tokens(op, rng)
    globals_ = [0, op.T - 1]
    rows, want = oracle_shared_rows(S, layer, om, op, toks, globals_)
    tol = 3e-2 if cfg.dtype == "fp8" else 1e-2
    assert rel_l2(got[rows], want) < tol
    assert rel_l2(got[rows] - S[rows], want - S[rows]) < 3 * tol
    assert_rows(got[rows], want, op, "shared", tol, rows=rows)
    plan.close()


@pytest.mark.parametrize("name", FULL)
def test_tiled_layer_full_size_sampled(name):
    cfg, op, S, layer = _setup(name, seed=4)
    om = oracle_model(cfg)
    plan = B.Plan(cfg.grid, cfg.win, cfg.stride)
    m = model_desc(cfg)
    w = B.layer_weights(dev_layer(cfg, layer))
    dt = TORCH_DT[cfg.dtype]
    X = OL.gather(S, op)                                  # [T, N, d]
    Xd = dev(X.reshape(op.T * op.N, -1), dt)
    ws = torch.empty(B.workspace_size(plan, m, 0, 0), dtype=torch.uint8, device="cuda")
    B.block_tiled(plan, m, w, Xd, ws)
    got = host(Xd).reshape(op.T, op.N, -1)
    rng = np.random.default_rng(2)
    for t in sorted({0, op.T - 1, int(rng.integers(op.T))}):
        slots = sorted({0, 1, op.N - 1} | set(rng.integers(1, op.N, 5).tolist()))
        q, k, v = OL.qkv_project(X[t], layer, om)
        q[1:] = OL.rope(q[1:], op.slot_pos, om)
        k[1:] = OL.rope(k[1:], op.slot_pos, om)
        o = OL.attention(q[slots], k, v)
        x = X[t, slots] + OL.linear(o, layer["w_o"], layer["b_o"], om)
        want = OL.mlp_residual(x, layer, om)
        tol = 3e-2 if cfg.dtype == "fp8" else 1e-2
        assert rel_l2(got[t, slots], want) < tol, t
        assert row_rel_errors(got[t, slots], want).max() < ROW_FACTOR * tol, t
    plan.close()
