"""The per-row bound of the parity tests catches what a whole-tensor norm hides
(CPU only; the mistake is planted in an oracle output, never in the library)."""

import numpy as np
import pytest

from oracle import layers as OL
from oracle import plan as P
from shared_token_transformer_b200 import workloads as W

from _gpu import assert_rows, rel_l2, row_classes


def test_one_wrong_row_passes_the_norm_but_not_the_row_bound():
    cfg = W.CONFIGS["stack48_bf16"]
    op = P.make_plan(cfg.grid, cfg.win, cfg.stride)
    rng = np.random.default_rng(0)
    want = rng.standard_normal((op.U + op.T, 64))
    got = want * (1 + 1e-3 * rng.standard_normal(want.shape))
    four = np.nonzero(op.coverage == 4)[0]
    got[four[7]] *= 1.3                                   # a 4-tile token 30 % off
    assert rel_l2(got, want) < 1e-2                       # invisible in the whole-tensor norm
    with pytest.raises(AssertionError, match="4 tile"):
        assert_rows(got, want, op, "shared", 1e-2)
    got[four[7]] = want[four[7]]
    got[op.U + 3] *= 0.7                                  # a register row 30 % off
    with pytest.raises(AssertionError, match="registers"):
        assert_rows(got, want, op, "shared", 1e-2)


def test_row_classes_cover_every_row_once():
    op = P.make_plan((1, 11, 13), (1, 8, 8), (1, 5, 6), registers=2)
    for layout, n in (("tokens", op.U), ("shared", op.U + op.T * op.R), ("tiled", op.T * op.N)):
        idx = np.concatenate(list(row_classes(op, layout).values()))
        assert np.array_equal(np.sort(idx), np.arange(n)), layout
    tiled = row_classes(op, "tiled")
    assert len(tiled["registers"]) == op.T * op.R
    assert sum(len(v) for k, v in tiled.items() if k != "registers") == op.T * op.Nw
