"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Op level first (LayerNorm, linear epilogues, QKV + QK-norm + RoPE, gathered
attention, blend), then layers, stacks, determinism and error paths.  Inputs are
the seeded draws of ``workloads`` (with nonzero biases and gains: affine=True);
the oracle consumes the same dtype-rounded values in float64.

Tolerances (relative L2 against the oracle): fp32 path 1e-5 per layer; bf16 path
1e-2 on stack outputs (and per layer); e4m3 path 3e-2.  Layer and stack tests
also bound the worst row of every coverage class (tokens in 1, 2, 4 or 8 tiles,
register rows) by 1.5 times the tolerance (``_gpu.assert_rows``).  Op-level bf16
checks use the rounding of one bf16 store (2^-8 relative per element) as their
scale.
"""

import dataclasses

import numpy as np
import pytest
import torch

from oracle import layers as OL
from shared_token_transformer_b200 import binding as B
from shared_token_transformer_b200 import workloads as W

from _gpu import Case, assert_rows, dev, host, rel_l2

pytestmark = pytest.mark.gpu

SMALL = W.small_config("small_bf16", grid=(1, 11, 13), win=(1, 8, 8), stride=(1, 5, 6), d=256, heads=4, mlp=512,
                       dtype="bf16", L=3, k=1)
RAGGED = W.small_config("ragged_bf16", grid=(1, 40, 37), win=(1, 15, 21), stride=(1, 12, 9), d=256, heads=4,
                        mlp=512, dtype="bf16", L=2, k=1)
VOL = W.small_config("vol_bf16", grid=(3, 12, 14), win=(2, 8, 8), stride=(1, 4, 6), d=256, heads=4, mlp=768,
                     dtype="bf16", L=2, k=1)
SMALL_FP8 = W.small_config("small_fp8", grid=(1, 11, 13), win=(1, 8, 8), stride=(1, 5, 6), d=256, heads=4,
                           mlp=512, dtype="fp8", L=2, k=1)
VIT14 = W.CONFIGS["vit14_fp32"]
# attention load paths: SMALL, VOL and the benchmark windows fetch a 64-slot block as one
# grid box; RUNS16 (48-slot window rows of 16) as 2-D boxes of 16-row runs; WIDE (window
# rows of 128) as grid boxes one row high; RAGGED (rows of 21) through four-row gathers
RUNS16 = W.small_config("runs16_bf16", grid=(1, 9, 40), win=(1, 3, 16), stride=(1, 2, 12), d=256, heads=4,
                        mlp=512, dtype="bf16", L=2, k=1)
WIDE = W.small_config("wide_bf16", grid=(1, 5, 200), win=(1, 2, 128), stride=(1, 1, 72), d=256, heads=4,
                      mlp=512, dtype="bf16", L=2, k=1)


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from shared_token_transformer_b200 import build
    build.build()
    torch.manual_seed(0)
    yield
    B.device_status()


_cases = {}


def case(cfg, **kw):
    key = (cfg.name, tuple(sorted(kw.items())))
    if key not in _cases:
        _cases[key] = Case(cfg, **kw)
    return _cases[key]


# ---------------------------------------------------------------------------
# op level
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("cfg", [SMALL, RAGGED, VIT14], ids=lambda c: c.name)
def test_layernorm(cfg):
    c = case(cfg)
    x = dev(c.S, c.dt)
    y = torch.empty_like(x)
    p = c.layers[0]
    B.op_layernorm(c.m, x, c.dlayers[0]["ln1_g"], c.dlayers[0]["ln1_b"], y)
    want = OL.layer_norm(c.S, p["ln1_g"], p["ln1_b"], 1e-6)
    tol = 1e-6 if cfg.dtype == "f32" else 3e-3
    assert rel_l2(host(y), want) < tol


def test_gelu_epilogue_matches_exact_erf():
    """The GELU epilogue evaluates erf by Abramowitz & Stegun 7.1.26 with the
    approximate reciprocal and exponential: through an identity fp32 linear layer,
    every output must be within 2e-6 of 0.5 x (1 + erf(x / sqrt 2)) (plus fp32
    rounding), over x in [-10, 10] including 0, both signs and the tails."""
    import math
    m = B.model_desc(64, 1, 64, "f32", (0, 32, 32))
    x = np.linspace(-10.0, 10.0, 64 * 64).reshape(64, 64)
    x[0, 0] = 0.0
    xd = torch.tensor(x, dtype=torch.float32, device="cuda")
    W = torch.eye(64, dtype=torch.float32, device="cuda")
    b = torch.zeros(64, dtype=torch.float32, device="cuda")
    y = torch.empty(64, 64, dtype=torch.float32, device="cuda")
    B.op_linear(m, xd, W, b, y, epi=B.TS_EPI_BIAS_GELU)
    got = host(y).astype(np.float64)
    xf = x.astype(np.float32).astype(np.float64)
    want = np.vectorize(lambda v: 0.5 * v * (1.0 + math.erf(v / math.sqrt(2.0))))(xf)
    assert np.max(np.abs(got - want) / np.maximum(1.0, np.abs(want))) < 2e-6


def test_gelu_epilogue_bf16_matches_exact_erf():
    """The bf16 GEMMs' GELU epilogue (Abramowitz & Stegun 7.1.26 on pairs of values
    in packed f32x2 arithmetic): bf16 inputs through an identity weight are exact
    in the fp32 accumulator, so every bf16 output must be exact-erf GELU of its
    input within one bf16 rounding (2^-8 relative to max(1, |GELU|)), over
    [-10, 10] with zero, both signs and the tails, at a size that takes the
    two-SM pair path (2304 rows, 256-wide tiles)."""
    import math
    M = K = N = 256
    x = W.round_to(np.linspace(-10.0, 10.0, 2304 * K).reshape(2304, K), "bf16")
    x[0, 0] = 0.0
    m = B.model_desc(256, 4, 256, "bf16", (0, 32, 32))
    y = torch.empty((2304, N), dtype=torch.bfloat16, device="cuda")
    B.op_linear(m, dev(x, torch.bfloat16), dev(np.eye(N, K), torch.bfloat16), dev(np.zeros(N), torch.float32), y,
                epi=B.TS_EPI_BIAS_GELU)
    want = np.vectorize(lambda v: 0.5 * v * (1.0 + math.erf(v / math.sqrt(2.0))))(x)
    assert np.max(np.abs(host(y) - want) / np.maximum(1.0, np.abs(want))) <= 2.0 ** -8


def test_gelu_epilogue_e4m3_matches_exact_erf():
    """The e4m3 GEMMs' GELU epilogue evaluates erf by Abramowitz & Stegun 7.1.28
    (one approximate reciprocal raised to the 16th power).  Inputs on the e4m3
    grid times a power of two and an identity weight make the scaled product
    exact, so every bf16 output must be exact-erf GELU of its input within one
    bf16 rounding (2^-8 relative to max(1, |GELU|)), over both signs, zero and
    the tails."""
    import math
    from oracle import fp8 as F8
    K = N = 128
    grid = np.array(sorted({F8.decode_e4m3(c) for c in range(127)}))
    rng = np.random.default_rng(9)
    x = rng.choice(grid, (256, K)) * rng.choice([-1.0, 1.0], (256, K)) / 32.0
    x[:, 0] = 448.0 / 32.0                       # row absmax 14: scale 1/32, the row quantises exactly
    x[0, 1:] = 0.0
    w = np.eye(N, K)
    m = B.model_desc(256, 4, 256, "fp8", (0, 32, 32))
    q = torch.empty((N, K), dtype=torch.uint8, device="cuda")
    s = torch.empty(N, dtype=torch.float32, device="cuda")
    B.quantize_rows_e4m3(dev(w, torch.bfloat16), q, s)
    y = torch.empty((256, N), dtype=torch.bfloat16, device="cuda")
    scratch = torch.empty(256 * K + 4 * 256 + 512, dtype=torch.uint8, device="cuda")
    B.op_linear(m, dev(x, torch.bfloat16), q, dev(np.zeros(N), torch.float32), y, epi=B.TS_EPI_BIAS_GELU,
                w_scale=s, scratch=scratch)
    want = np.vectorize(lambda v: 0.5 * v * (1.0 + math.erf(v / math.sqrt(2.0))))(x)
    assert np.max(np.abs(host(y) - want) / np.maximum(1.0, np.abs(want))) <= 2.0 ** -8


# (2320, 2048, 512) and (2320, 512, 512): the 48 x 48 layer's MLP down and out-projection
@pytest.mark.parametrize("M,K,N", [(300, 256, 512), (128, 512, 768), (129, 256, 192), (1, 256, 64), (2320, 512, 1536),
                                   (777, 2048, 512), (2320, 2048, 512), (2320, 512, 512)])
@pytest.mark.parametrize("epi", [B.TS_EPI_BIAS, B.TS_EPI_BIAS_GELU, B.TS_EPI_BIAS_RESID])
def test_linear_bf16(M, K, N, epi):
    rng = np.random.default_rng(M * 7 + N + epi)
    x = W.round_to(rng.standard_normal((M, K)), "bf16")
    w = W.round_to(0.05 * rng.standard_normal((N, K)), "bf16")
    b = W.round_to(0.1 * rng.standard_normal(N), "f32")
    y0 = W.round_to(rng.standard_normal((M, N)), "bf16")
    m = B.model_desc(256, 4, 256, "bf16", (0, 32, 32))
    y = dev(y0, torch.bfloat16)
    B.op_linear(m, dev(x, torch.bfloat16), dev(w, torch.bfloat16), dev(b, torch.float32), y, epi=epi)
    want = x @ w.T + b
    if epi == B.TS_EPI_BIAS_GELU:
        want = OL.gelu(want)
    if epi == B.TS_EPI_BIAS_RESID:
        want = want + y0
    assert rel_l2(host(y), want) < 3e-3


@pytest.mark.parametrize("M,K,N", [(300, 256, 512), (129, 512, 256), (64, 1536, 4608), (300, 1024, 512)])
def test_linear_fp8(M, K, N):
    from oracle import fp8 as F8
    rng = np.random.default_rng(M + K)
    x = W.round_to(rng.standard_normal((M, K)), "bf16")
    w = W.round_to(0.02 * rng.standard_normal((N, K)), "bf16")
    b = W.round_to(0.1 * rng.standard_normal(N), "f32")
    m = B.model_desc(256, 4, 256, "fp8", (0, 32, 32))
    wd = dev(w, torch.bfloat16)
    q = torch.empty((N, K), dtype=torch.uint8, device="cuda")
    s = torch.empty(N, dtype=torch.float32, device="cuda")
    B.quantize_rows_e4m3(wd, q, s)
    # the weight codes equal the oracle's rounding of the same bf16 values
    qo, so = F8.quantize_rows(w)
    got_codes = q.cpu().view(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_allclose(host(s), so, rtol=1e-6)
    assert np.mean(got_codes == qo) > 0.999
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    scratch = torch.empty(M * K + 4 * M + 512, dtype=torch.uint8, device="cuda")
    B.op_linear(m, dev(x, torch.bfloat16), q, dev(b, torch.float32), y, epi=B.TS_EPI_BIAS, w_scale=s,
                scratch=scratch)
    want = F8.scaled_matmul(x, w) + b
    assert rel_l2(host(y), want) < 1e-2


def _qkv_oracle(c, state, rows_pos, unrot):
    """LN1 + QKV + QK-norm (oracle), then RoPE at the given per-row coordinates."""
    p = c.layers[0]
    q, k, v = OL.qkv_project(state, p, c.om)
    rot = ~unrot
    q[rot] = OL.rope(q[rot], rows_pos[rot], c.om)
    k[rot] = OL.rope(k[rot], rows_pos[rot], c.om)
    n = state.shape[0]
    return np.concatenate([q.reshape(n, -1), k.reshape(n, -1), v.reshape(n, -1)], axis=1)


@pytest.mark.parametrize("cfg", [SMALL, VOL, VIT14], ids=lambda c: c.name)
@pytest.mark.parametrize("mode", [B.TS_ROWS_SHARED, B.TS_ROWS_TILED])
def test_qkv_norm_rope(cfg, mode):
    c = case(cfg)
    op = c.oplan
    if mode == B.TS_ROWS_SHARED:
        state = c.S
        F, H, Wd = cfg.grid
        u = np.arange(op.U)
        pos = np.concatenate([np.stack([u // (H * Wd), (u // Wd) % H, u % Wd], 1), op.origins])
        unrot = np.zeros(len(state), bool)
    else:
        state = OL.gather(c.S, op).reshape(op.T * op.N, -1)
        pos = np.tile(np.concatenate([[[0, 0, 0]], op.slot_pos]), (op.T, 1))
        unrot = np.zeros(len(state), bool)
        unrot[::op.N] = True
    want = _qkv_oracle(c, state, pos, unrot)
    qkv = torch.empty((len(state), 3 * cfg.d), dtype=c.dt, device="cuda")
    scratch = torch.empty(len(state) * cfg.d * 6 + 4096, dtype=torch.uint8, device="cuda")
    B.op_qkv(c.plan, c.m, c.wlist[0], mode, dev(state, c.dt), qkv, scratch)
    got = host(qkv)
    tol = 1e-5 if cfg.dtype == "f32" else 8e-3
    for part in range(3):
        sl = slice(part * cfg.d, (part + 1) * cfg.d)
        assert rel_l2(got[:, sl], want[:, sl]) < tol, part


@pytest.mark.parametrize("cfg", [SMALL, RAGGED, VOL, RUNS16, WIDE, VIT14], ids=lambda c: c.name)
@pytest.mark.parametrize("mode", [B.TS_ROWS_SHARED, B.TS_ROWS_TILED])
def test_attention(cfg, mode):
    c = case(cfg)
    op = c.oplan
    rows = op.U + op.T if mode == B.TS_ROWS_SHARED else op.T * op.N
    rng = np.random.default_rng(3)
    qkv = W.round_to(rng.standard_normal((rows, 3 * cfg.d)), cfg.dtype if cfg.dtype != "fp8" else "bf16")
    O = torch.empty((op.T * op.N, cfg.d), dtype=c.dt, device="cuda")
    B.op_attention(c.plan, c.m, mode, dev(qkv, c.dt), O)
    hd = cfg.hd
    want = np.empty((op.T * op.N, cfg.d))
    for t in range(op.T):
        if mode == B.TS_ROWS_SHARED:
            r = np.concatenate([[op.U + t], op.tile_tok[t]])
        else:
            r = t * op.N + np.arange(op.N)
        q = qkv[r, :cfg.d].reshape(op.N, cfg.heads, hd)
        k = qkv[r, cfg.d:2 * cfg.d].reshape(op.N, cfg.heads, hd)
        v = qkv[r, 2 * cfg.d:].reshape(op.N, cfg.heads, hd)
        want[t * op.N:(t + 1) * op.N] = OL.attention(q, k, v)
    tol = 1e-5 if cfg.dtype == "f32" else 1e-2
    got = host(O)
    assert rel_l2(got, want) < tol
    # global-token rows (handled by their own code path) checked separately
    assert rel_l2(got[::op.N], want[::op.N]) < tol


@pytest.mark.parametrize("cfg", [SMALL, RAGGED, VOL, VIT14], ids=lambda c: c.name)
def test_merge(cfg):
    c = case(cfg)
    op = c.oplan
    rng = np.random.default_rng(4)
    P = W.round_to(rng.standard_normal((op.T, op.N, cfg.d)), cfg.dtype if cfg.dtype != "fp8" else "bf16")
    for rows in (op.U, op.U + op.T):
        A = torch.empty((rows, cfg.d), dtype=c.dt, device="cuda")
        B.op_merge(c.plan, c.m, dev(P.reshape(op.T * op.N, -1), c.dt), rows, A)
        want = OL.merge(P, op)[:rows]
        tol = 1e-6 if cfg.dtype == "f32" else 3e-3
        assert rel_l2(host(A), want) < tol


# ---------------------------------------------------------------------------
# layers
# ---------------------------------------------------------------------------
def _tol(cfg):
    return {"f32": 1e-5, "bf16": 1e-2, "fp8": 3e-2}[cfg.dtype]


@pytest.mark.parametrize("cfg", [SMALL, RAGGED, VOL, VIT14, SMALL_FP8], ids=lambda c: c.name)
def test_block_shared(cfg):
    c = case(cfg)
    S_in = c.S
    S = dev(S_in, c.dt)
    ws = c.workspace()
    B.block_shared(c.plan, c.m, c.wlist[0], S, ws)
    want = OL.block_shared(S_in, c.layers[0], c.om, c.oplan)
    got = host(S)
    assert rel_l2(got, want) < _tol(cfg)
    assert rel_l2(got - S_in, want - S_in) < 3 * _tol(cfg)
    assert_rows(got, want, c.oplan, "shared", _tol(cfg))


@pytest.mark.parametrize("cfg", [SMALL, RAGGED, VOL, VIT14, SMALL_FP8], ids=lambda c: c.name)
def test_block_tiled(cfg):
    c = case(cfg)
    X_in = OL.gather(c.S, c.oplan)
    X = dev(X_in.reshape(c.oplan.T * c.oplan.N, -1), c.dt)
    ws = c.workspace()
    B.block_tiled(c.plan, c.m, c.wlist[0], X, ws)
    want = OL.block_tiled(X_in, c.layers[0], c.om, c.oplan).reshape(X.shape)
    got = host(X)
    X_in = X_in.reshape(X.shape)
    assert rel_l2(got, want) < _tol(cfg)
    assert rel_l2(got - X_in, want - X_in) < 3 * _tol(cfg)
    assert_rows(got, want, c.oplan, "tiled", _tol(cfg))


# ---------------------------------------------------------------------------
# stacks
# ---------------------------------------------------------------------------
def _run_stack(c, k):
    op = c.oplan
    L = len(c.wlist)
    out = torch.empty((op.U, c.cfg.d), dtype=c.dt, device="cuda")
    ws = c.workspace(L, k)
    B.decode_stack(c.plan, c.m, c.wlist, k, dev(c.S0, c.dt), dev(c.G0, c.dt), out, ws)
    return out


@pytest.mark.parametrize("cfg,ks", [(SMALL, (0, 1, 3)), (RAGGED, (1,)), (VOL, (0, 2)), (VIT14, (0, 1)),
                                    (SMALL_FP8, (0, 1, 2))], ids=lambda x: getattr(x, "name", str(x)))
def test_decode_stack(cfg, ks):
    c = case(cfg)
    for k in ks:
        got = host(_run_stack(c, k))
        want = OL.decode_stack(c.S0, c.G0, c.layers, c.om, c.oplan, k)
        assert rel_l2(got, want) < _tol(cfg), k
        assert_rows(got, want, c.oplan, "tokens", _tol(cfg))


@pytest.mark.parametrize("cfg", [SMALL, VOL, SMALL_FP8], ids=lambda c: c.name)
def test_hard_stitch_shared_layer_and_stack(cfg):
    """Hard stitching: the plan's CSR has one entry of weight one per token, so the
    blend and the transition copy each token's row from its chosen tile.  A shared
    layer and a stack (k = 1) against the oracle with the same rule."""
    c = case(cfg, rule="hard")
    assert c.plan.nnz == c.plan.U
    S_in = c.S
    S = dev(S_in, c.dt)
    B.block_shared(c.plan, c.m, c.wlist[0], S, c.workspace())
    want = OL.block_shared(S_in, c.layers[0], c.om, c.oplan)
    assert rel_l2(host(S), want) < _tol(cfg)
    assert_rows(host(S), want, c.oplan, "shared", _tol(cfg))
    got = host(_run_stack(c, 1))
    want = OL.decode_stack(c.S0, c.G0, c.layers, c.om, c.oplan, 1)
    assert rel_l2(got, want) < _tol(cfg)
    assert_rows(got, want, c.oplan, "tokens", _tol(cfg))


_SHARE = {"qkv": B.TS_SHARE_QKV, "out": B.TS_SHARE_OUT, "mlp": B.TS_SHARE_MLP}


@pytest.mark.parametrize("cfg", [SMALL, VOL, VIT14, SMALL_FP8], ids=lambda c: c.name)
@pytest.mark.parametrize("shared", [(), ("qkv",), ("out",), ("mlp",), ("qkv", "mlp"), ("qkv", "out", "mlp")],
                         ids=lambda s: "+".join(s) or "none")
def test_block_partial(cfg, shared):
    """Partial sharing against the oracle, from per-tile states that disagree on
    their overlap tokens (gathered copies plus seeded noise)."""
    c = case(cfg)
    op = c.oplan
    X = OL.gather(c.S, op) + 0.1 * np.random.default_rng(21).standard_normal((op.T, op.N, cfg.d))
    X = W.round_to(X, cfg.dtype if cfg.dtype != "fp8" else "bf16")
    Xd = dev(X.reshape(op.T * op.N, cfg.d), c.dt)
    ops = 0
    for s in shared:
        ops |= _SHARE[s]
    B.block_partial(c.plan, c.m, c.wlist[0], ops, Xd, c.workspace())
    want = OL.block_partial(X, c.layers[0], c.om, op, shared)
    got = host(Xd).reshape(op.T, op.N, cfg.d)
    assert rel_l2(got, want) < _tol(cfg)
    assert rel_l2(got - X, want - X) < 3 * _tol(cfg)
    assert_rows(got, want, op, "tiled", _tol(cfg))


# ---------------------------------------------------------------------------
# RMSNorm + SwiGLU block flavour (Tab. S6)
# ---------------------------------------------------------------------------
SMALL_SW = dataclasses.replace(SMALL, name="small_swiglu_bf16", block="rms_swiglu")
VOL_SW = dataclasses.replace(VOL, name="vol_swiglu_bf16", block="rms_swiglu")
VIT14_SW = dataclasses.replace(VIT14, name="vit14_swiglu_fp32", block="rms_swiglu")
SMALL_FP8_SW = dataclasses.replace(SMALL_FP8, name="small_swiglu_fp8", block="rms_swiglu")
_SW = [SMALL_SW, VOL_SW, VIT14_SW, SMALL_FP8_SW]


@pytest.mark.parametrize("cfg", [SMALL_SW, VIT14_SW], ids=lambda c: c.name)
def test_rmsnorm(cfg):
    c = case(cfg)
    x = dev(c.S, c.dt)
    y = torch.empty_like(x)
    B.op_layernorm(c.m, x, c.dlayers[0]["ln1_g"], None, y)
    want = OL.rms_norm(c.S, c.layers[0]["ln1_g"], 1e-6)
    assert rel_l2(host(y), want) < (1e-6 if cfg.dtype == "f32" else 3e-3)


def _swiglu_want(x, w, b):
    n = w.shape[0] // 2
    a = x @ w.T + b
    return OL.silu(a[:, :n]) * a[:, n:]


@pytest.mark.parametrize("M,K,N", [(300, 256, 256), (129, 512, 192), (1, 256, 64), (2320, 512, 2048),
                                   (777, 1024, 320)])
def test_linear_swiglu_bf16(M, K, N):
    rng = np.random.default_rng(M * 3 + N)
    x = W.round_to(rng.standard_normal((M, K)), "bf16")
    w = W.round_to(0.05 * rng.standard_normal((2 * N, K)), "bf16")
    b = W.round_to(0.5 * rng.standard_normal(2 * N), "f32")
    m = B.model_desc(256, 4, 256, "bf16", (0, 32, 32), block="rms_swiglu")
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    B.op_linear(m, dev(x, torch.bfloat16), dev(w, torch.bfloat16), dev(b, torch.float32), y,
                epi=B.TS_EPI_BIAS_SWIGLU)
    assert rel_l2(host(y), _swiglu_want(x, w, b)) < 3e-3


@pytest.mark.parametrize("M,K,N", [(70, 48, 40), (129, 64, 96)])
def test_linear_swiglu_f32(M, K, N):
    rng = np.random.default_rng(M + N)
    x = W.round_to(rng.standard_normal((M, K)), "f32")
    w = W.round_to(0.2 * rng.standard_normal((2 * N, K)), "f32")
    b = W.round_to(0.5 * rng.standard_normal(2 * N), "f32")
    m = B.model_desc(64, 1, 64, "f32", (0, 32, 32), block="rms_swiglu")
    y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    B.op_linear(m, dev(x, torch.float32), dev(w, torch.float32), dev(b, torch.float32), y, epi=B.TS_EPI_BIAS_SWIGLU)
    assert rel_l2(host(y), _swiglu_want(x, w, b)) < 1e-6


def test_linear_swiglu_fp8():
    from oracle import fp8 as F8
    M, K, N = 300, 256, 256
    rng = np.random.default_rng(5)
    x = W.round_to(rng.standard_normal((M, K)), "bf16")
    w = W.round_to(0.02 * rng.standard_normal((2 * N, K)), "bf16")
    b = W.round_to(0.1 * rng.standard_normal(2 * N), "f32")
    m = B.model_desc(256, 4, 256, "fp8", (0, 32, 32), block="rms_swiglu")
    q = torch.empty((2 * N, K), dtype=torch.uint8, device="cuda")
    s = torch.empty(2 * N, dtype=torch.float32, device="cuda")
    B.quantize_rows_e4m3(dev(w, torch.bfloat16), q, s)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    scratch = torch.empty(M * K + 4 * M + 512, dtype=torch.uint8, device="cuda")
    B.op_linear(m, dev(x, torch.bfloat16), q, dev(b, torch.float32), y, epi=B.TS_EPI_BIAS_SWIGLU, w_scale=s,
                scratch=scratch)
    a = F8.scaled_matmul(x, w) + b
    want = OL.silu(a[:, :N]) * a[:, N:]
    assert rel_l2(host(y), want) < 1e-2


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_silu_epilogue_values(dtype):
    """Gate rows = identity, up rows = 0 with bias 1: the layer returns silu(x) itself,
    over x in [-30, 30] with 0 and both tails; fp32 within 2e-6 (relative to
    max(1, |silu|)), bf16 within its output rounding."""
    n = 64
    x = np.linspace(-30.0, 30.0, 128 * n).reshape(128, n)
    x[0, 0] = 0.0
    dt = torch.float32 if dtype == "f32" else torch.bfloat16
    x = W.round_to(x, dtype)
    w = np.concatenate([np.eye(n), np.zeros((n, n))])
    b = np.concatenate([np.zeros(n), np.ones(n)])
    m = B.model_desc(256, 4, 256, dtype, (0, 32, 32), block="rms_swiglu")
    y = torch.empty((128, n), dtype=dt, device="cuda")
    B.op_linear(m, dev(x, dt), dev(w, dt), dev(b, torch.float32), y, epi=B.TS_EPI_BIAS_SWIGLU)
    want = x / (1.0 + np.exp(-x))
    err = np.max(np.abs(host(y) - want) / np.maximum(1.0, np.abs(want)))
    assert err < (2e-6 if dtype == "f32" else 2.0 ** -8)


@pytest.mark.parametrize("cfg", _SW, ids=lambda c: c.name)
def test_swiglu_block_shared_and_tiled(cfg):
    c = case(cfg)
    S_in = c.S
    S = dev(S_in, c.dt)
    B.block_shared(c.plan, c.m, c.wlist[0], S, c.workspace())
    want = OL.block_shared(S_in, c.layers[0], c.om, c.oplan)
    assert rel_l2(host(S), want) < _tol(cfg)
    assert rel_l2(host(S) - S_in, want - S_in) < 3 * _tol(cfg)
    assert_rows(host(S), want, c.oplan, "shared", _tol(cfg))
    X_in = OL.gather(S_in, c.oplan)
    X = dev(X_in.reshape(c.oplan.T * c.oplan.N, -1), c.dt)
    B.block_tiled(c.plan, c.m, c.wlist[0], X, c.workspace())
    want = OL.block_tiled(X_in, c.layers[0], c.om, c.oplan).reshape(X.shape)
    assert rel_l2(host(X), want) < _tol(cfg)
    assert_rows(host(X), want, c.oplan, "tiled", _tol(cfg))


@pytest.mark.parametrize("cfg", _SW, ids=lambda c: c.name)
def test_swiglu_decode_stack(cfg):
    c = case(cfg)
    for k in (0, 1):
        got = host(_run_stack(c, k))
        want = OL.decode_stack(c.S0, c.G0, c.layers, c.om, c.oplan, k)
        assert rel_l2(got, want) < _tol(cfg), k
        assert_rows(got, want, c.oplan, "tokens", _tol(cfg))


@pytest.mark.parametrize("cfg", [SMALL_SW, SMALL_FP8_SW], ids=lambda c: c.name)
@pytest.mark.parametrize("shared", [("mlp",), ("qkv", "out", "mlp")], ids=lambda s: "+".join(s))
def test_swiglu_block_partial(cfg, shared):
    c = case(cfg)
    op = c.oplan
    X = OL.gather(c.S, op) + 0.1 * np.random.default_rng(22).standard_normal((op.T, op.N, cfg.d))
    X = W.round_to(X, cfg.dtype if cfg.dtype != "fp8" else "bf16")
    Xd = dev(X.reshape(op.T * op.N, cfg.d), c.dt)
    ops = 0
    for s_ in shared:
        ops |= _SHARE[s_]
    B.block_partial(c.plan, c.m, c.wlist[0], ops, Xd, c.workspace())
    want = OL.block_partial(X, c.layers[0], c.om, op, shared)
    assert rel_l2(host(Xd).reshape(op.T, op.N, cfg.d), want) < _tol(cfg)
    assert_rows(host(Xd), want, op, "tiled", _tol(cfg))


# ---------------------------------------------------------------------------
# several register tokens per tile (Tab. S1: one set per tile)
# ---------------------------------------------------------------------------
SMALL_R4 = dataclasses.replace(SMALL, name="small_r4_bf16", R=4)
VOL_R2 = dataclasses.replace(VOL, name="vol_r2_bf16", R=2)
VIT14_R3 = dataclasses.replace(VIT14, name="vit14_r3_fp32", R=3)
SMALL_FP8_R2 = dataclasses.replace(SMALL_FP8, name="small_r2_fp8", R=2)
RUNS16_R8 = dataclasses.replace(RUNS16, name="runs16_r8_bf16", R=8)
_REG = [SMALL_R4, VOL_R2, VIT14_R3, SMALL_FP8_R2, RUNS16_R8]


@pytest.mark.parametrize("cfg", _REG, ids=lambda c: c.name)
def test_registers_block_shared_and_tiled(cfg):
    c = case(cfg)
    assert c.plan.R == cfg.R and c.plan.N == c.plan.Nw + cfg.R
    S_in = c.S
    assert S_in.shape[0] == c.oplan.U + c.oplan.T * cfg.R
    S = dev(S_in, c.dt)
    B.block_shared(c.plan, c.m, c.wlist[0], S, c.workspace())
    want = OL.block_shared(S_in, c.layers[0], c.om, c.oplan)
    assert rel_l2(host(S), want) < _tol(cfg)
    assert rel_l2(host(S) - S_in, want - S_in) < 3 * _tol(cfg)
    assert_rows(host(S), want, c.oplan, "shared", _tol(cfg))
    X_in = OL.gather(S_in, c.oplan)
    X = dev(X_in.reshape(c.oplan.T * c.oplan.N, -1), c.dt)
    B.block_tiled(c.plan, c.m, c.wlist[0], X, c.workspace())
    want = OL.block_tiled(X_in, c.layers[0], c.om, c.oplan).reshape(X.shape)
    assert rel_l2(host(X), want) < _tol(cfg)
    assert_rows(host(X), want, c.oplan, "tiled", _tol(cfg))


@pytest.mark.parametrize("cfg", _REG, ids=lambda c: c.name)
def test_registers_decode_stack(cfg):
    c = case(cfg)
    for k in (0, 1):
        got = host(_run_stack(c, k))
        want = OL.decode_stack(c.S0, c.G0, c.layers, c.om, c.oplan, k)
        assert rel_l2(got, want) < _tol(cfg), k
        assert_rows(got, want, c.oplan, "tokens", _tol(cfg))


@pytest.mark.parametrize("cfg", [SMALL_R4, SMALL_FP8_R2], ids=lambda c: c.name)
def test_registers_block_partial(cfg):
    c = case(cfg)
    op = c.oplan
    X = OL.gather(c.S, op) + 0.1 * np.random.default_rng(23).standard_normal((op.T, op.N, cfg.d))
    X = W.round_to(X, cfg.dtype if cfg.dtype != "fp8" else "bf16")
    Xd = dev(X.reshape(op.T * op.N, cfg.d), c.dt)
    B.block_partial(c.plan, c.m, c.wlist[0], B.TS_SHARE_QKV | B.TS_SHARE_OUT | B.TS_SHARE_MLP, Xd, c.workspace())
    want = OL.block_partial(X, c.layers[0], c.om, op, ("qkv", "out", "mlp"))
    assert rel_l2(host(Xd).reshape(op.T, op.N, cfg.d), want) < _tol(cfg)
    assert_rows(host(Xd), want, op, "tiled", _tol(cfg))


def test_block_partial_rejects_unknown_operations():
    c = case(SMALL)
    Xd = torch.zeros((c.oplan.T * c.oplan.N, SMALL.d), dtype=c.dt, device="cuda")
    with pytest.raises(B.TileShareError) as e:
        B.block_partial(c.plan, c.m, c.wlist[0], 8, Xd, c.workspace())
    assert e.value.status == 1


def test_stack48_bf16_full():
    """The benchmark stack (48x48 tokens, d=512, L=8, k=2) against the full oracle."""
    cfg = W.CONFIGS["stack48_bf16"]
    c = case(cfg, affine=False)
    got = host(_run_stack(c, cfg.k))
    want = OL.decode_stack(c.S0, c.G0, c.layers, c.om, c.oplan, cfg.k)
    assert rel_l2(got, want) < 1e-2
    assert_rows(got, want, c.oplan, "tokens", 1e-2)


def test_stack_deterministic():
    c = case(SMALL)
    a = _run_stack(c, 1).clone()
    b = _run_stack(c, 1)
    assert torch.equal(a, b)


@pytest.mark.parametrize("name", ["image2k_bf16", "stack48_bf16"])
def test_attention_bitwise_repeatable(name):
    """The attention kernel's buffers (TMEM S/P, K/V, Q) are recycled under
    barrier control only; repeated launches on the same input at a benchmark
    size must give identical bits (a missed ordering shows up as run-to-run
    differences long before it exceeds a tolerance)."""
    cfg = W.CONFIGS[name]
    plan = B.Plan(cfg.grid, cfg.win, cfg.stride)
    m = B.model_desc(cfg.d, cfg.heads, cfg.mlp, cfg.dtype, cfg.rope_dims)
    gen = torch.Generator(device="cuda").manual_seed(5)
    for mode, rows in ((B.TS_ROWS_SHARED, plan.U + plan.T), (B.TS_ROWS_TILED, plan.T * plan.N)):
        qkv = torch.randn(rows, 3 * cfg.d, device="cuda", generator=gen).to(torch.bfloat16)
        O = [torch.zeros(plan.T * plan.N, cfg.d, device="cuda", dtype=torch.bfloat16) for _ in range(3)]
        for o in O:
            B.op_attention(plan, m, mode, qkv, o)
        torch.cuda.synchronize()
        assert torch.equal(O[0], O[1]) and torch.equal(O[0], O[2])
    plan.close()


# ---------------------------------------------------------------------------
# error paths: refused on the host, nothing written
# ---------------------------------------------------------------------------
def test_bounded_wait_times_out_and_context_survives():
    """A kernel wait that nothing satisfies gives up after its limit (here 2 ms),
    reports TS_ERR_TIMEOUT through ts_device_status, and the context keeps working:
    no trap, no fault, no hang."""
    done = torch.zeros(2, dtype=torch.int32, device="cuda")
    B.selftest_bounded_wait(2_000_000, done)
    with pytest.raises(B.TileShareError) as e:
        B.device_status()
    assert e.value.status == 6
    assert done.tolist() == [1, 0]
    B.device_status()                      # the status word was cleared
    c = case(SMALL)                        # and the library still computes
    S = dev(c.S, c.dt)
    B.block_shared(c.plan, c.m, c.wlist[0], S, c.workspace())
    B.device_status()
    assert torch.isfinite(S.float()).all()


def test_error_paths():
    c = case(SMALL)
    S = dev(c.S, c.dt)
    before = S.clone()
    ws = c.workspace()
    with pytest.raises(B.TileShareError) as e:
        B.block_shared(c.plan, c.m, c.wlist[0], S, ws[:-1024])
    assert e.value.status == 3
    with pytest.raises(B.TileShareError) as e:
        B.block_shared(c.plan, c.m, c.wlist[0], S.view(torch.uint8).flatten()[2:], ws)
    assert e.value.status == 1
    bad = dict(c.dlayers[0])
    bad["w_o"] = None
    with pytest.raises(B.TileShareError) as e:
        B.block_shared(c.plan, c.m, B.layer_weights(bad), S, ws)
    assert e.value.status == 1
    with pytest.raises(B.TileShareError) as e:
        B.decode_stack(c.plan, c.m, c.wlist, 7, dev(c.S0, c.dt), dev(c.G0, c.dt),
                       torch.empty((c.oplan.U, 256), dtype=c.dt, device="cuda"), c.workspace(3, 1))
    assert e.value.status == 1
    torch.cuda.synchronize()
    assert torch.equal(S, before)
