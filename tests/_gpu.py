"""Helpers of the GPU parity tests: device copies of the seeded inputs, the oracle
run on the same inputs, and the error measure used by the tolerances."""

import numpy as np
import torch

from oracle import layers as OL
from oracle import plan as OP
from shared_token_transformer_b200 import binding as B
from shared_token_transformer_b200 import workloads as W

TORCH_DT = {"f32": torch.float32, "bf16": torch.bfloat16, "fp8": torch.bfloat16}
BIG = ("w_qkv", "w_o", "w_1", "w_2")
SCALE = {"w_qkv": "s_qkv", "w_o": "s_o", "w_1": "s_1", "w_2": "s_2"}


def rel_l2(got, want):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    return float(np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-300))


def oracle_model(cfg):
    return OL.Model(cfg.d, cfg.heads, cfg.mlp, cfg.rope_dims, fp8=(cfg.dtype == "fp8"), block=cfg.block)


def model_desc(cfg):
    return B.model_desc(cfg.d, cfg.heads, cfg.mlp, cfg.dtype, cfg.rope_dims, block=cfg.block)


def dev(a, dtype):
    return torch.from_numpy(np.ascontiguousarray(a)).to(device="cuda", dtype=dtype)


def host(t):
    return t.detach().to(torch.float64).cpu().numpy()


def dev_layer(cfg, p):
    """Device tensors of one layer; e4m3 weights quantised on the device, per row."""
    out = {}
    for k, v in p.items():
        if k in BIG:
            t = dev(v, TORCH_DT[cfg.dtype])
            if cfg.dtype == "fp8":
                q = torch.empty(t.shape, dtype=torch.uint8, device="cuda")
                s = torch.empty(t.shape[0], dtype=torch.float32, device="cuda")
                B.quantize_rows_e4m3(t, q, s)
                out[k], out[SCALE[k]] = q, s
            else:
                out[k] = t
        else:
            out[k] = dev(v, torch.float32)
    return out


class Case:
    """Seeded inputs of a configuration, on both sides."""

    def __init__(self, cfg, seed=0, affine=True, L=None, rule="ramp"):
        self.cfg = cfg
        self.oplan = OP.make_plan(cfg.grid, cfg.win, cfg.stride, rule=rule, registers=cfg.R)
        self.plan = B.Plan(cfg.grid, cfg.win, cfg.stride,
                           rule=B.TS_BLEND_HARD_STITCH if rule == "hard" else B.TS_BLEND_LINEAR_RAMP,
                           registers=cfg.R)
        dr = W.Draw(cfg, self.oplan.T, seed=seed, affine=affine)
        self.S0, self.G0 = dr.states()
        self.layers = dr.layers(L)
        self.m = model_desc(cfg)
        self.om = oracle_model(cfg)
        self.dlayers = [dev_layer(cfg, p) for p in self.layers]
        self.wlist = [B.layer_weights(t) for t in self.dlayers]
        self.dt = TORCH_DT[cfg.dtype]

    @property
    def S(self):
        return np.concatenate([self.S0, self.G0])

    def workspace(self, L=0, k=0):
        n = B.workspace_size(self.plan, self.m, L, k)
        return torch.empty(n, dtype=torch.uint8, device="cuda")


# ---------------------------------------------------------------------------
# per-row error bounds
# ---------------------------------------------------------------------------
# A whole-tensor relative L2 error hides a single wrong row: one row of a
# 2,320-row state carries about 1/2,320 of the squared norm.  Every layer and
# stack test therefore also bounds the worst row of each coverage class (grid
# tokens in 1, 2, 4 or 8 tiles, register rows).  The rounding errors of a row
# are sums over d >= 64 independent element errors, so a row's relative error
# stays near the whole tensor's (the largest of 10^5 rows of d = 512 lies about
# 20 % above the mean); ROW_FACTOR leaves room for that spread and for rows whose
# per-token e4m3 scale is set by an outlier, while a row with a wrong blend
# weight, slot or register is off by far more.
ROW_FACTOR = 1.5


def row_rel_errors(got, want):
    """Relative L2 error of every row of [rows, d] arrays."""
    got = np.asarray(got, np.float64).reshape(-1, np.shape(want)[-1])
    want = np.asarray(want, np.float64).reshape(got.shape)
    return np.linalg.norm(got - want, axis=1) / np.maximum(np.linalg.norm(want, axis=1), 1e-300)


def row_classes(op, layout, rows=None):
    """Row indices by coverage class for an output of the given layout:
    "tokens" [U] grid tokens, "shared" [U + T*R] shared state, "tiled" [T*N]
    per-tile state; `rows` restricts a "shared" layout to the listed rows."""
    cov = op.coverage
    if layout == "tiled":
        cls = np.empty(op.T * op.N, dtype=np.int64)
        for t in range(op.T):
            cls[t * op.N: t * op.N + op.R] = 0
            cls[t * op.N + op.R: (t + 1) * op.N] = cov[op.tile_tok[t]]
    else:
        cls = np.concatenate([cov, np.zeros(op.T * op.R, dtype=np.int64)])
        if layout == "tokens":
            cls = cls[: op.U]
        if rows is not None:
            cls = cls[np.asarray(rows)]
    return {("registers" if c == 0 else f"{c} tile(s)"): np.nonzero(cls == c)[0] for c in np.unique(cls)}


def assert_rows(got, want, op, layout, tol, rows=None):
    """Worst row of each coverage class within ROW_FACTOR * tol."""
    err = row_rel_errors(got, want)
    for name, idx in row_classes(op, layout, rows).items():
        if len(idx) == 0:
            continue
        i = idx[np.argmax(err[idx])]
        assert err[i] < ROW_FACTOR * tol, f"{name}: row {i} relative error {err[i]:.3e} (bound {ROW_FACTOR * tol:.1e})"
