"""Oracle: overlapping tiling of the token grid and the blend weights w-bar.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

What the pages fix
    * [TileShare] abstract: a fixed-window decoder runs at deployment resolution as
      overlapping tiles; every token of an overlap band is processed by several
      tiles; the overlap token's per-tile results are blended "with the released
      weights".
    * [TileShare] Fig. 2: a token in the overlap of two windows is stored once but
      attended in both windows; its attention outputs are blended with w-bar.

Readings taken where the pages are silent
    R1 tile placement: per axis, n = ceil((G - w) / s) + 1 tiles (1 if w == G), the
       i-th at origin min(i*s, G - w): the last tile sits flush with the far edge,
       no padding.
    R2 w-bar: separable along the axes.  Along one axis a tile whose previous
       neighbour overlaps it by o_p tokens and whose next neighbour overlaps it by
       o_n tokens weighs the token at local position p by
           (p + 1) / (o_p + 1)   if p < o_p            (ramp up)
           (w - p) / (o_n + 1)   if p >= w - o_n       (ramp down)
       (the product of both when the two bands meet) and 1 elsewhere.  A tile's
       weight for a token is the product over axes; w-bar is that weight divided
       by the sum over every tile covering the token, so it sums to 1 per token.
    R3 orders: tiles in raster order of their (f, y, x) origins; window slots in
       tile-local raster order (f, y, x); grid tokens u = (f*H + y)*W + x.  The
       per-tile state of tile t has N = Nw + 1 rows: row 0 is the tile's global
       token, row 1 + j its window slot j.  A (tile, slot) entry is addressed as
       t*N + 1 + j (R registers per tile: see R14).
    R14 registers ([TileShare] Tab. S1: "one set per tile, as released"; in shared
       layers they stay per tile and attend only to their own tile): each tile has
       R register tokens (R = 1: the one global token of the benchmark
       configurations).  The per-tile state has N = Nw + R rows, rows 0 .. R-1 the
       tile's registers and row R + j its window slot j, so an entry is t*N + R + j;
       the shared state has U + T*R rows, tile t's register i at U + t*R + i.
    R11 hard stitching (blend rule "hard"; [TileShare] Tab. 2 and Tab. S2 list a
       "Hard stitching" baseline, Tab. S11 describes it as each pixel taken from its
       dominant tile): applied to the blend of overlap tokens, each token takes its
       value from one tile, the covering tile with the largest unnormalised R2
       weight (the dominant one), the lowest tile index on ties; w-bar is 1 for that
       tile and 0 for the others, and the token's CSR row holds that single entry.
"""

from dataclasses import dataclass, field

import numpy as np


def axis_origins(G: int, w: int, s: int) -> list:
    """Tile origins along one axis of length G, window w, stride s (reading R1)."""
    if not (1 <= w <= G) or not (1 <= s <= w):
        raise ValueError(f"bad axis: G={G} w={w} s={s}")
    if w == G:
        return [0]
    n = -(-(G - w) // s) + 1
    return [min(i * s, G - w) for i in range(n)]


def axis_ramp(origins: list, w: int) -> np.ndarray:
    """Unnormalised per-tile weight at each local position along one axis (R2).

    Returns an array [n_tiles, w] of float64.
    """
    n = len(origins)
    out = np.ones((n, w), dtype=np.float64)
    for i, o in enumerate(origins):
        o_prev = max(origins[i - 1] + w - o, 0) if i > 0 else 0
        o_next = max(o + w - origins[i + 1], 0) if i + 1 < n else 0
        for p in range(w):
            r = 1.0
            if p < o_prev:
                r *= (p + 1) / (o_prev + 1)
            if p >= w - o_next:
                r *= (w - p) / (o_next + 1)
            out[i, p] = r
    return out


@dataclass
class Plan:
    grid: tuple          # (F, H, W) tokens
    win: tuple           # (wf, wh, ww)
    stride: tuple        # (sf, sh, sw)
    origins: np.ndarray  # [T, 3] int64, tile origin (f, y, x)
    tile_tok: np.ndarray  # [T, Nw] int64, grid token of window slot j of tile t
    slot_pos: np.ndarray  # [Nw, 3] int64, tile-local (f, y, x) of window slot j
    wraw: np.ndarray     # [T, Nw] float64, unnormalised weight of slot j of tile t
    wbar: np.ndarray     # [T, Nw] float64, normalised blend weight
    tok_ptr: np.ndarray  # [U + 1] int64, CSR row pointer over grid tokens
    tok_ent: np.ndarray  # [nnz] int64, entry t*N + R + j, ascending t per token
    tok_w: np.ndarray    # [nnz] float64, w-bar of that entry
    coverage: np.ndarray = field(default=None)  # [U] int64, tiles per token
    R: int = 1           # register tokens per tile (R14)

    @property
    def T(self):
        return self.tile_tok.shape[0]

    @property
    def Nw(self):
        return self.tile_tok.shape[1]

    @property
    def N(self):
        return self.Nw + self.R

    @property
    def G(self):
        """Register rows of the shared state, T * R."""
        return self.T * self.R

    @property
    def U(self):
        F, H, W = self.grid
        return F * H * W

    @property
    def nnz(self):
        return int(self.tok_ent.shape[0])


def make_plan(grid, win, stride, rule: str = "ramp", registers: int = 1) -> Plan:
    """Tile plan for a token grid (F, H, W); 2-D grids use F = wf = sf = 1.

    rule "ramp": w-bar of R2 (normalised ramp weights); rule "hard": R11.
    registers: register tokens per tile (R14).
    """
    if rule not in ("ramp", "hard"):
        raise ValueError(f"unknown blend rule {rule!r}")
    if registers < 1:
        raise ValueError("a tile has at least one register token")
    F, H, W = (int(v) for v in grid)
    wf, wh, ww = (int(v) for v in win)
    sf, sh, sw = (int(v) for v in stride)
    of = axis_origins(F, wf, sf)
    oh = axis_origins(H, wh, sh)
    ow = axis_origins(W, ww, sw)
    rf, rh, rw = axis_ramp(of, wf), axis_ramp(oh, wh), axis_ramp(ow, ww)

    Nw = wf * wh * ww
    slot_pos = np.array([(lf, ly, lx) for lf in range(wf) for ly in range(wh) for lx in range(ww)],
                        dtype=np.int64).reshape(Nw, 3)
    tiles = [(i_f, i_h, i_w) for i_f in range(len(of)) for i_h in range(len(oh)) for i_w in range(len(ow))]
    T = len(tiles)
    origins = np.array([(of[a], oh[b], ow[c]) for a, b, c in tiles], dtype=np.int64).reshape(T, 3)
    tile_tok = np.zeros((T, Nw), dtype=np.int64)
    wraw = np.zeros((T, Nw), dtype=np.float64)
    for t, (a, b, c) in enumerate(tiles):
        for j in range(Nw):
            lf, ly, lx = slot_pos[j]
            f, y, x = origins[t, 0] + lf, origins[t, 1] + ly, origins[t, 2] + lx
            tile_tok[t, j] = (f * H + y) * W + x
            wraw[t, j] = rf[a, lf] * rh[b, ly] * rw[c, lx]

    U = F * H * W
    N = Nw + registers
    total = np.zeros(U, dtype=np.float64)
    coverage = np.zeros(U, dtype=np.int64)
    for t in range(T):
        for j in range(Nw):
            total[tile_tok[t, j]] += wraw[t, j]
            coverage[tile_tok[t, j]] += 1
    if np.any(coverage == 0):
        raise ValueError("tiling leaves a token uncovered")
    wbar = wraw / total[tile_tok]
    if rule == "hard":
        # the covering tile with the largest raw weight; strict > keeps the first
        # (lowest) tile on ties, tiles being visited in ascending order
        best_t = np.full(U, -1, dtype=np.int64)
        best_w = np.full(U, -1.0, dtype=np.float64)
        for t in range(T):
            for j in range(Nw):
                u = tile_tok[t, j]
                if wraw[t, j] > best_w[u]:
                    best_w[u] = wraw[t, j]
                    best_t[u] = t
        wbar = np.zeros((T, Nw), dtype=np.float64)
        for t in range(T):
            for j in range(Nw):
                if best_t[tile_tok[t, j]] == t:
                    wbar[t, j] = 1.0

    # CSR over grid tokens; tiles are visited in ascending order, so each token's
    # entries come out in ascending tile index.
    lists = [[] for _ in range(U)]
    for t in range(T):
        for j in range(Nw):
            if rule == "hard" and wbar[t, j] == 0.0:
                continue
            lists[tile_tok[t, j]].append((t * N + registers + j, wbar[t, j]))
    tok_ptr = np.zeros(U + 1, dtype=np.int64)
    for u in range(U):
        tok_ptr[u + 1] = tok_ptr[u] + len(lists[u])
    tok_ent = np.array([e for lst in lists for e, _ in lst], dtype=np.int64)
    tok_w = np.array([wv for lst in lists for _, wv in lst], dtype=np.float64)
    return Plan(grid=(F, H, W), win=(wf, wh, ww), stride=(sf, sh, sw), origins=origins,
                tile_tok=tile_tok, slot_pos=slot_pos, wraw=wraw, wbar=wbar, tok_ptr=tok_ptr,
                tok_ent=tok_ent, tok_w=tok_w, coverage=coverage, R=registers)


def duplicated_fraction(p: Plan) -> float:
    """Share of per-token work that tiled decoding repeats: 1 - U / (T * Nw)."""
    return 1.0 - p.U / (p.T * p.Nw)
