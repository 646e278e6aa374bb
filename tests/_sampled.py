"""Oracle outputs of single rows of a shared layer (test infrastructure).

A shared layer's output row depends only on the q/k/v rows of the tiles that
cover it, so a full-size layer can be checked on a sample of rows: these
helpers recompute such rows with the per-row and per-tile steps of
oracle.layers, in float64.
"""

import numpy as np

from oracle import layers as OL


def sample_tokens(op, rng, n=24):
    cov = op.coverage
    picks = []
    for c in sorted(set(cov.tolist())):
        idx = np.nonzero(cov == c)[0]
        picks += list(rng.choice(idx, size=min(len(idx), n // 3), replace=False))
    picks += [0, op.U - 1]                      # grid corners (last tiles are the ragged ones)
    return sorted(set(int(u) for u in picks))


def oracle_shared_rows(S, layer, om, op, toks, globals_):
    """Rows `toks` (grid tokens) and U + t for t in globals_ of one shared layer."""
    U, N = op.U, op.N
    tok_set = set(toks)
    need_tiles = sorted({t for t in range(op.T) if tok_set & set(op.tile_tok[t].tolist())} | set(globals_))
    rows = sorted({U + t for t in need_tiles} | {int(r) for t in need_tiles for r in op.tile_tok[t]})
    ridx = {r: i for i, r in enumerate(rows)}
    q, k, v = OL.qkv_project(S[rows], layer, om)
    A = {}
    for t in need_tiles:
        trow = [U + t] + [int(r) for r in op.tile_tok[t]]
        sel = [ridx[r] for r in trow]
        qt, kt, vt = q[sel].copy(), k[sel].copy(), v[sel].copy()
        qt[1:] = OL.rope(qt[1:], op.slot_pos, om)
        kt[1:] = OL.rope(kt[1:], op.slot_pos, om)
        want_slots = [s for s, r in enumerate(trow) if (s == 0 and t in globals_) or (s > 0 and r in tok_set)]
        if not want_slots:
            continue
        o = OL.attention(qt[want_slots], kt, vt)
        for s, orow in zip(want_slots, o):
            if s == 0:
                A[U + t] = orow
            else:
                u = trow[s]
                j = s - 1
                A[u] = A.get(u, 0.0) + op.wbar[t, j] * orow
    out_rows = list(toks) + [U + t for t in globals_]
    Am = np.stack([A[r] for r in out_rows])
    x = S[out_rows] + OL.linear(Am, layer["w_o"], layer["b_o"], om)
    return out_rows, OL.mlp_residual(x, layer, om)
