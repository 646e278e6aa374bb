"""Pins of the oracle's E4M3 rounding, scaled GEMM and FLOP model (CPU only)."""

import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import flops as Fo
from oracle import fp8 as F8
from oracle import plan as P

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_e4m3_codes_exhaustive():
    vals = [F8.decode_e4m3(c) for c in range(256)]
    finite = [v for v in vals if not math.isnan(v)]
    assert len(finite) == 254                      # two NaN codes, no infinities
    assert max(finite) == 448.0 and min(finite) == -448.0
    assert min(v for v in finite if v > 0) == 2.0 ** -9
    for c, v in enumerate(vals):
        if math.isnan(v):
            continue
        assert F8.round_e4m3_scalar(v) == v        # every code is a fixed point
    # library cast decodes the same grid
    codes = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(np.isnan(codes), np.isnan(vals))
    ok = ~np.isnan(codes)
    np.testing.assert_array_equal(codes[ok], np.array(vals)[ok])


def test_e4m3_rounding_against_library_cast():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(20000) * s for s in (1e-3, 0.05, 1, 30, 200)])
    x = x[np.abs(x) < 448]
    grid = np.array(sorted({F8.decode_e4m3(c) for c in range(256) if not math.isnan(F8.decode_e4m3(c))}))
    mids = (grid[1:] + grid[:-1]) / 2                 # exact ties, must round to even
    x = np.concatenate([x, mids[np.abs(mids) < 448]])
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(F8.round_e4m3(x), want)
    assert F8.round_e4m3_scalar(1e6) == 448.0 and F8.round_e4m3_scalar(-500.0) == -448.0


def test_array_rounding_equals_scalar_rounding():
    rng = np.random.default_rng(5)
    x = np.concatenate([rng.standard_normal(3000) * s for s in (1e-4, 3e-3, 0.3, 7, 100, 600)])
    grid = [F8.decode_e4m3(c) for c in range(127)]
    x = np.concatenate([x, grid, -np.array(grid), [(a + b) / 2 for a, b in zip(grid[:-1], grid[1:])]])
    np.testing.assert_array_equal(F8.round_e4m3(x), [F8.round_e4m3_scalar(v) for v in x])


def test_scaled_matmul_exact_on_grid_inputs():
    # rows whose absmax is 448 * 2^e and whose entries lie on the scaled grid quantise exactly
    rng = np.random.default_rng(2)
    grid = np.array([F8.decode_e4m3(c) for c in range(127)])     # non-negative finite codes
    def make(n, K):
        a = rng.choice(grid, (n, K)) * rng.choice([-1, 1], (n, K))
        a[:, 0] = 448.0
        return a * (2.0 ** rng.integers(-8, 4, (n, 1)))
    x, w = make(9, 32), make(5, 32)
    np.testing.assert_allclose(F8.scaled_matmul(x, w), x @ w.T, rtol=1e-15, atol=0)


def test_scaled_matmul_error_bound():
    # relative rounding error of E4M3 is at most 2^-4 per operand
    rng = np.random.default_rng(3)
    x = rng.standard_normal((64, 256))
    w = 0.02 * rng.standard_normal((32, 256))
    got = F8.scaled_matmul(x, w)
    bound = (2 * 2.0 ** -4 + 2.0 ** -8) * (np.abs(x) @ np.abs(w).T)
    assert np.all(np.abs(got - x @ w.T) <= bound)


def test_flop_model_degenerates_and_matches_pages_structure():
    # no overlap: U + T == T * N -> shared layer costs exactly a tiled layer
    p = P.make_plan((1, 16, 16), (1, 8, 8), (1, 8, 8))
    assert Fo.shared_layer_flops(p.U, p.T, p.N, 64, 256) == Fo.tiled_layer_flops(p.T, p.N, 64, 256)
    assert Fo.stack_flop_ratio(p.U, p.T, p.N, 64, 256, 4, 2) == 1.0
    # the pages' savings are additive: all = 1 - sum of single-op savings (Tab. 1 vs Tab. S7)
    with open(os.path.join(GOLDEN, "tab1_flop_ratios.json")) as fh:
        g = json.load(fh)
    for k in ("k4", "k0"):
        r = g[k]
        saved = (1 - r["qkv"]) + (1 - r["out"]) + (1 - r["mlp"])
        assert abs((1 - saved) - r["all"]) <= 0.0015
        assert abs((1 - (1 - r["qkv"]) - (1 - r["out"])) - r["q+o"]) <= 0.0015
    # a shared layer saves exactly the linear work of the duplicated rows
    p = P.make_plan((1, 48, 48), (1, 16, 16), (1, 12, 12))
    d, f = 512, 2048
    diff = Fo.tiled_layer_flops(p.T, p.N, d, f) - Fo.shared_layer_flops(p.U, p.T, p.N, d, f)
    assert diff == (p.T * p.Nw - p.U) * Fo.linear_flops_per_row(d, f)


@pytest.mark.parametrize("gated", [False, True])
def test_partial_sharing_flops(gated):
    # nothing shared is the per-tile layer, everything shared is the shared layer, and the
    # savings of the single operations add up (the structure of Tab. 1 and Tab. S7)
    p = P.make_plan((4, 44, 80), (4, 32, 32), (4, 24, 24))
    U, T, N, d, f = p.U, p.T, p.N, 1536, 6144
    tiled = Fo.tiled_layer_flops(T, N, d, f, gated)
    assert Fo.partial_layer_flops(U, T, N, d, f, (), gated) == tiled
    assert Fo.partial_layer_flops(U, T, N, d, f, ("qkv", "out", "mlp"), gated) == \
        Fo.shared_layer_flops(U, T, N, d, f, gated)
    single = {op: tiled - Fo.partial_layer_flops(U, T, N, d, f, (op,), gated) for op in ("qkv", "out", "mlp")}
    for combo in (("qkv", "out"), ("qkv", "mlp"), ("out", "mlp")):
        assert tiled - Fo.partial_layer_flops(U, T, N, d, f, combo, gated) == sum(single[o] for o in combo)
    # each operation's saving is its per-row FLOPs on the duplicated rows
    dup = T * N - (U + T)
    assert single["qkv"] == 6 * d * d * dup and single["out"] == 2 * d * d * dup
    assert single["mlp"] == 2 * (3 if gated else 2) * d * f * dup
    with pytest.raises(ValueError):
        Fo.partial_layer_flops(U, T, N, d, f, ("attn",))
