"""Pins of the oracle's tile plan (CPU only).

The plan is checked against brute-force containment enumeration, the tile counts
stated by the benchmark configurations, and the properties the pages give the blend
weights (a weighted sum normalised per token; a linear ramp across each overlap).
"""

import itertools
import json
import os

import numpy as np
import pytest

from oracle import plan as P

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _axis_props(G, w, s, o):
    assert o[0] == 0 and o[-1] == G - w
    gaps = np.diff(o)
    assert np.all(gaps > 0) and np.all(gaps <= s)
    assert np.all(gaps[:-1] == s)
    # minimal count: one tile fewer cannot reach G - w with steps of at most s
    assert (len(o) - 2) * s < G - w or len(o) == 1


@pytest.mark.parametrize("G", range(1, 13))
def test_axis_origins_properties(G):
    for w in range(1, G + 1):
        for s in range(1, w + 1):
            _axis_props(G, w, s, P.axis_origins(G, w, s))


def _brute_force(grid, win, origins):
    F, H, W = grid
    wf, wh, ww = win
    pairs = {}
    for t, (of, oy, ox) in enumerate(origins):
        for f, y, x in itertools.product(range(F), range(H), range(W)):
            if of <= f < of + wf and oy <= y < oy + wh and ox <= x < ox + ww:
                slot = ((f - of) * wh + (y - oy)) * ww + (x - ox)
                pairs[(t, slot)] = (f * H + y) * W + x
    return pairs


def _small_geometries():
    out = []
    for H in range(1, 10):
        for W in (1, 4, 7, 10):
            for wh in range(1, H + 1):
                for ww in range(1, W + 1):
                    for sh in sorted({1, max(1, wh // 2), wh}):
                        for sw in sorted({1, max(1, ww // 2), ww}):
                            out.append(((1, H, W), (1, wh, ww), (1, sh, sw)))
    out += [((3, 5, 6), (2, 3, 4), (1, 2, 3)), ((4, 6, 6), (4, 4, 4), (4, 2, 2)), ((5, 4, 4), (3, 2, 3), (2, 1, 1))]
    return out


def test_index_maps_match_brute_force():
    for grid, win, stride in _small_geometries():
        p = P.make_plan(grid, win, stride)
        bf = _brute_force(grid, win, p.origins)
        got = {(t, j): int(p.tile_tok[t, j]) for t in range(p.T) for j in range(p.Nw)}
        assert got == bf, (grid, win, stride)
        # CSR: every (tile, slot) containing u, ascending tile index, addressed t*N + 1 + j
        want = {}
        for (t, j), u in sorted(bf.items()):
            want.setdefault(u, []).append(t * p.N + 1 + j)
        for u in range(p.U):
            ents = list(p.tok_ent[p.tok_ptr[u]:p.tok_ptr[u + 1]])
            assert ents == want[u]
            assert p.coverage[u] == len(ents)


def test_wbar_sums_to_one_and_is_positive():
    for grid, win, stride in _small_geometries():
        p = P.make_plan(grid, win, stride)
        assert np.all(p.tok_w > 0)
        sums = np.add.reduceat(p.tok_w, p.tok_ptr[:-1])
        np.testing.assert_allclose(sums, 1.0, rtol=0, atol=1e-15)
        single = p.coverage == 1
        firsts = p.tok_w[p.tok_ptr[:-1]]
        assert np.all(firsts[single] == 1.0)


def test_wbar_mirror_symmetry():
    # a tiling whose last tile lands on the stride grid is symmetric under a flip
    for G, w, s in [(14, 8, 6), (48, 16, 16), (10, 4, 2), (13, 5, 4), (20, 8, 3)]:
        if (G - w) % s:
            continue
        p = P.make_plan((1, 1, G), (1, 1, w), (1, 1, s))
        T = p.T
        for t in range(T):
            np.testing.assert_allclose(p.wbar[t], p.wbar[T - 1 - t][::-1], rtol=0, atol=1e-15)


def test_linear_ramp_across_two_tile_overlap():
    # between two tiles only, the weights cross-fade linearly and already sum to 1
    for G, w, s in [(14, 8, 6), (48, 16, 12), (256, 32, 24), (80, 32, 24), (44, 32, 12)]:
        o = P.axis_origins(G, w, s)
        r = P.axis_ramp(o, w)
        for i in range(len(o) - 1):
            lo, hi = o[i + 1], o[i] + w           # overlap band [lo, hi)
            band = range(lo, hi)
            a = np.array([r[i, g - o[i]] for g in band])
            b = np.array([r[i + 1, g - o[i + 1]] for g in band])
            np.testing.assert_allclose(a + b, 1.0, atol=1e-15)
            if len(band) > 1:
                np.testing.assert_allclose(np.diff(b), 1.0 / (len(band) + 1), atol=1e-15)
                np.testing.assert_allclose(np.diff(a), -1.0 / (len(band) + 1), atol=1e-15)


def test_golden_geometry():
    with open(os.path.join(GOLDEN, "geometry.json")) as fh:
        g = json.load(fh)
    for name in ("vit14_fp32", "stack48_bf16", "image4k_bf16"):
        e = g[name]
        p = P.make_plan(e["grid"], e["win"], e["stride"])
        counts = [len(P.axis_origins(G, w, s)) for G, w, s in zip(e["grid"], e["win"], e["stride"])]
        assert counts == e["tiles"], name
        assert p.T == int(np.prod(e["tiles"]))
        if "overlap_tokens" in e:
            for ax in (1, 2):
                o = P.axis_origins(e["grid"][ax], e["win"][ax], e["stride"][ax])
                assert o[0] + e["win"][ax] - o[1] == e["overlap_tokens"][ax]
    e = g["video_duplicated_share"]
    p = P.make_plan(e["grid"], e["win"], e["stride"])
    assert e["low"] <= P.duplicated_fraction(p) <= e["high"]


def test_single_tile_and_no_overlap_degenerate():
    p = P.make_plan((1, 8, 8), (1, 8, 8), (1, 3, 3))
    assert p.T == 1 and np.all(p.tok_w == 1.0) and p.nnz == 64
    p = P.make_plan((1, 16, 16), (1, 8, 8), (1, 8, 8))
    assert p.T == 4 and np.all(p.coverage == 1) and np.all(p.tok_w == 1.0)


# ---------------------------------------------------------------------------
# hard stitching (reading R11): one tile per token, the largest ramp weight,
# lowest tile index on ties
# ---------------------------------------------------------------------------
def test_hard_stitch_one_entry_of_weight_one():
    for grid, win, stride in _small_geometries():
        p = P.make_plan(grid, win, stride, rule="hard")
        assert np.all(np.diff(p.tok_ptr) == 1) and p.nnz == p.U
        assert np.all(p.tok_w == 1.0)
        # every entry is a (tile, slot) that contains its token
        t = p.tok_ent // p.N
        j = p.tok_ent % p.N - 1
        np.testing.assert_array_equal(p.tile_tok[t, j], np.arange(p.U))


def test_hard_stitch_choice_is_argmax_lowest_tile_on_ties():
    """Recomputed here with a vectorised argmax over the ramp plan's raw weights:
    for each token, the largest raw weight among its tiles, then the lowest tile."""
    for grid, win, stride in _small_geometries()[::7]:
        ramp = P.make_plan(grid, win, stride)
        hard = P.make_plan(grid, win, stride, rule="hard")
        t_all = np.repeat(np.arange(ramp.T), ramp.Nw)
        u_all = ramp.tile_tok.reshape(-1)
        w_all = ramp.wraw.reshape(-1)
        order = np.lexsort((t_all, -w_all, u_all))      # by token, weight descending, tile ascending
        first = order[np.r_[0, np.flatnonzero(np.diff(u_all[order])) + 1]]
        want_t = np.empty(ramp.U, dtype=np.int64)
        want_t[u_all[first]] = t_all[first]
        np.testing.assert_array_equal(hard.tok_ent // hard.N, want_t)


def test_hard_stitch_two_tile_split_point():
    """Two tiles overlapping by o tokens on one axis: at band position i the weights
    are (o - i)/(o + 1) and (i + 1)/(o + 1), so the first tile keeps the positions
    i <= (o - 1)/2 (the tie at odd o goes to the lower tile) and the second the rest."""
    for G, w, s in [(14, 8, 6), (10, 6, 4), (9, 5, 4), (12, 8, 4), (11, 7, 4), (13, 10, 3)]:
        o_list = P.axis_origins(G, w, s)
        assert len(o_list) == 2
        lo, hi = o_list[1], o_list[0] + w
        o = hi - lo
        p = P.make_plan((1, 1, G), (1, 1, w), (1, 1, s), rule="hard")
        chosen = p.tok_ent // p.N
        for g in range(G):
            if g < lo:
                assert chosen[g] == 0
            elif g >= hi:
                assert chosen[g] == 1
            else:
                i = g - lo
                assert chosen[g] == (0 if 2 * i <= o - 1 else 1), (G, w, s, g)


def test_hard_stitch_equals_ramp_without_overlap():
    for grid, win, stride in [((1, 16, 16), (1, 8, 8), (1, 8, 8)), ((2, 6, 9), (1, 3, 3), (1, 3, 3)),
                              ((1, 8, 8), (1, 8, 8), (1, 2, 2))]:
        a = P.make_plan(grid, win, stride)
        b = P.make_plan(grid, win, stride, rule="hard")
        np.testing.assert_array_equal(a.tok_ptr, b.tok_ptr)
        np.testing.assert_array_equal(a.tok_ent, b.tok_ent)
        np.testing.assert_array_equal(a.tok_w, b.tok_w)


@pytest.mark.parametrize("R", [2, 5])
def test_registers_shift_the_entries_only(R):
    """R register tokens per tile (R14): the window slots move to rows R.. of each
    tile's state, so every entry t*N + 1 + j of the one-register plan becomes
    t*(Nw + R) + R + j; weights, tiles and coverage do not change."""
    g, w, st = (2, 9, 11), (2, 5, 6), (1, 3, 4)
    one = P.make_plan(g, w, st)
    p = P.make_plan(g, w, st, registers=R)
    assert p.N == p.Nw + R and p.G == p.T * R
    t, j = np.divmod(one.tok_ent, one.N)
    np.testing.assert_array_equal(p.tok_ent, t * (one.Nw + R) + R + (j - 1))
    np.testing.assert_array_equal(p.tok_ptr, one.tok_ptr)
    np.testing.assert_array_equal(p.tok_w, one.tok_w)
    np.testing.assert_array_equal(p.tile_tok, one.tile_tok)
    with pytest.raises(ValueError):
        P.make_plan(g, w, st, registers=0)
