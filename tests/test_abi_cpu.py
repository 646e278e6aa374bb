"""The C-ABI library on the CPU: it loads, exports every declared entry point, its
host planner equals the oracle's plan bit for bit, and bad arguments are refused.
No CUDA compute call is made here."""

import ctypes
import os
import re

import numpy as np
import pytest

from oracle import plan as OP
from shared_token_transformer_b200 import binding as B
from shared_token_transformer_b200 import build as Bd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    Bd.build()


def _declared():
    names = set()
    for h in os.listdir(os.path.join(ROOT, "include")):
        txt = open(os.path.join(ROOT, "include", h)).read()
        names |= set(re.findall(r"^(?:ts_status|void|long long|const char\*)\s+(ts_\w+)\s*\(", txt, re.M))
    return names


def test_exports_every_declared_symbol():
    names = _declared()
    assert len(names) >= 16
    L = ctypes.CDLL(B.LIB_PATH)
    for n in sorted(names):
        assert hasattr(L, n), n
    assert names <= set(B.exported_symbols()), names - set(B.exported_symbols())


GEOMS = [
    ((1, 14, 14), (1, 8, 8), (1, 6, 6)),
    ((1, 16, 16), (1, 8, 8), (1, 8, 8)),
    ((1, 48, 48), (1, 16, 16), (1, 12, 12)),
    ((4, 44, 80), (4, 32, 32), (4, 24, 24)),
    ((1, 128, 128), (1, 32, 32), (1, 24, 24)),
    ((1, 11, 13), (1, 8, 8), (1, 5, 6)),
    ((3, 7, 9), (2, 4, 5), (1, 1, 2)),
    ((1, 20, 9), (1, 8, 3), (1, 3, 1)),
    ((1, 5, 5), (1, 5, 5), (1, 2, 2)),
    ((1, 9, 40), (1, 3, 16), (1, 2, 12)),
    ((1, 5, 200), (1, 2, 128), (1, 1, 72)),
]


@pytest.mark.parametrize("grid,win,stride", GEOMS)
def test_host_planner_bit_exact_against_oracle(grid, win, stride):
    o = OP.make_plan(grid, win, stride)
    p = B.Plan(grid, win, stride, host_only=True)
    try:
        assert (p.T, p.U, p.Nw, p.N, p.nnz) == (o.T, o.U, o.Nw, o.N, o.nnz)
        assert p.device == -1
        np.testing.assert_array_equal(p.origins, o.origins)
        np.testing.assert_array_equal(p.tile_tok, o.tile_tok)
        np.testing.assert_array_equal(p.slot_pos, o.slot_pos)
        np.testing.assert_array_equal(p.tok_ptr, o.tok_ptr)
        np.testing.assert_array_equal(p.tok_ent, o.tok_ent)
        # w-bar: the planner rounds its double weights to float once
        np.testing.assert_array_equal(p.wbar, o.tok_w.astype(np.float32))
        assert p.max_cover == int(o.coverage.max())
    finally:
        p.close()


@pytest.mark.parametrize("R", [2, 5])
def test_host_planner_registers_bit_exact_against_oracle(R):
    grid, win, stride = (2, 9, 11), (2, 5, 6), (1, 3, 4)
    o = OP.make_plan(grid, win, stride, registers=R)
    p = B.Plan(grid, win, stride, host_only=True, registers=R)
    try:
        assert (p.T, p.U, p.Nw, p.N, p.nnz, p.R) == (o.T, o.U, o.Nw, o.N, o.nnz, R)
        np.testing.assert_array_equal(p.tok_ptr, o.tok_ptr)
        np.testing.assert_array_equal(p.tok_ent, o.tok_ent)
        np.testing.assert_array_equal(p.wbar, o.tok_w.astype(np.float32))
    finally:
        p.close()


@pytest.mark.parametrize("R", [0, 65])
def test_plan_rejects_bad_register_count(R):
    with pytest.raises(B.TileShareError):
        B.Plan((1, 8, 8), (1, 4, 4), (1, 2, 2), host_only=True, registers=R)


RUNS = {(1, 48, 48): 16, (4, 44, 80): 32, (1, 128, 128): 32, (1, 11, 13): 8, (3, 7, 9): 0, (1, 20, 9): 0,
        (1, 5, 5): 64, (1, 9, 40): 16, (1, 5, 200): 64}


@pytest.mark.parametrize("grid,win,stride", GEOMS)
def test_plan_run_length(grid, win, stride):
    """Attention loads fetch each run of consecutive grid tokens as one box: the
    planner's run length is the longest of 64, 32, 16, 8 whose aligned slot groups
    are consecutive tokens in every tile (brute force over the oracle's map)."""
    o = OP.make_plan(grid, win, stride)
    want = 0
    for L in (64, 32, 16, 8):
        tt = np.asarray(o.tile_tok)
        j = np.arange(1, o.Nw)
        j = j[j % L != 0]
        if np.all(tt[:, j] == tt[:, j - 1] + 1):
            want = L
            break
    if grid in RUNS:
        assert want == RUNS[grid]
    p = B.Plan(grid, win, stride, host_only=True)
    try:
        assert p.run == want
    finally:
        p.close()


@pytest.mark.parametrize("grid,win,stride", GEOMS)
def test_host_planner_hard_stitch_bit_exact_against_oracle(grid, win, stride):
    o = OP.make_plan(grid, win, stride, rule="hard")
    p = B.Plan(grid, win, stride, host_only=True, rule=B.TS_BLEND_HARD_STITCH)
    try:
        assert (p.T, p.U, p.N, p.nnz) == (o.T, o.U, o.N, o.nnz) and p.nnz == p.U
        np.testing.assert_array_equal(p.tok_ptr, o.tok_ptr)
        np.testing.assert_array_equal(p.tok_ent, o.tok_ent)
        np.testing.assert_array_equal(p.wbar, o.tok_w.astype(np.float32))
    finally:
        p.close()


def test_unknown_blend_rule_rejected():
    with pytest.raises(B.TileShareError) as e:
        B.Plan((1, 8, 8), (1, 4, 4), (1, 2, 2), host_only=True, rule=7)
    assert e.value.status == 1


def test_image4k_plan_counts():
    p = B.Plan((1, 256, 256), (1, 32, 32), (1, 24, 24), host_only=True)
    assert (p.T, p.U, p.N, p.nnz, p.max_cover) == (121, 65536, 1025, 123904, 4)
    p.close()


@pytest.mark.parametrize("grid,win,stride", [
    ((1, 8, 8), (1, 9, 8), (1, 1, 1)),     # window larger than grid
    ((1, 8, 8), (1, 4, 4), (1, 5, 4)),     # stride larger than window
    ((1, 8, 8), (1, 4, 4), (1, 0, 4)),     # zero stride
    ((0, 8, 8), (1, 4, 4), (1, 4, 4)),     # empty axis
])
def test_plan_rejects_bad_geometry(grid, win, stride):
    with pytest.raises(B.TileShareError) as e:
        B.Plan(grid, win, stride, host_only=True)
    assert e.value.status == 1


def test_status_strings_and_workspace_on_host_plan():
    L = B.lib()
    assert L.ts_status_string(0) == b"ok"
    assert L.ts_status_string(3) == b"workspace too small"
    p = B.Plan((1, 48, 48), (1, 16, 16), (1, 12, 12), host_only=True)
    m = B.model_desc(512, 8, 2048, "bf16", (0, 32, 32))
    n0 = B.workspace_size(p, m, 0, 0)
    n8 = B.workspace_size(p, m, 8, 2)
    assert n8 > n0 > 0
    # unsupported head dim on the bf16 path, bad k, bad rope split
    with pytest.raises(B.TileShareError) as e:
        B.workspace_size(p, B.model_desc(512, 4, 2048, "bf16", (0, 64, 64)), 0, 0)
    assert e.value.status == 2
    with pytest.raises(B.TileShareError) as e:
        B.workspace_size(p, m, 4, 5)
    assert e.value.status == 1
    with pytest.raises(B.TileShareError) as e:
        B.workspace_size(p, B.model_desc(512, 8, 2048, "bf16", (0, 30, 32)), 0, 0)
    assert e.value.status == 1
    p.close()


def test_compute_calls_refuse_host_plan():
    # a host-only plan is refused before any launch (device -1 never matches)
    p = B.Plan((1, 14, 14), (1, 8, 8), (1, 6, 6), host_only=True)
    m = B.model_desc(64, 4, 256, "f32", (0, 8, 8))
    w = B.LayerWeights()
    st = B.lib().ts_block_shared(p.handle, ctypes.byref(m), ctypes.byref(w), None, None, 0, None)
    assert st in (1, 4)     # invalid argument (or CUDA unavailable when querying the device)
    p.close()


def test_layer_weights_keep_their_tensors_alive():
    # the struct holds raw pointers; it must also hold the tensors behind them
    import gc
    import weakref

    import torch
    t = torch.zeros(16)
    ref = weakref.ref(t)
    w = B.layer_weights({"w_o": t})
    del t
    gc.collect()
    assert ref() is not None and w.w_o == ref().data_ptr()
    del w
    gc.collect()
    assert ref() is None


def test_host_planner_matches_oracle_on_random_geometries():
    """The C++ planner against the oracle on 60 seeded random geometries (2-D and 3-D,
    both blend rules, 1-4 registers): counts, maps, CSR and w-bar bit-exact."""
    rng = np.random.default_rng(2024)
    for _ in range(60):
        grid = [int(rng.integers(1, 4)), int(rng.integers(1, 19)), int(rng.integers(1, 19))]
        win = [int(rng.integers(1, g + 1)) for g in grid]
        stride = [int(rng.integers(1, w + 1)) for w in win]
        rule = "hard" if rng.random() < 0.3 else "ramp"
        R = int(rng.integers(1, 5))
        o = OP.make_plan(grid, win, stride, rule=rule, registers=R)
        p = B.Plan(grid, win, stride, host_only=True, registers=R,
                   rule=B.TS_BLEND_HARD_STITCH if rule == "hard" else B.TS_BLEND_LINEAR_RAMP)
        try:
            assert (p.T, p.U, p.Nw, p.N, p.nnz, p.R) == (o.T, o.U, o.Nw, o.N, o.nnz, R), (grid, win, stride)
            np.testing.assert_array_equal(p.origins, o.origins)
            np.testing.assert_array_equal(p.tile_tok, o.tile_tok)
            np.testing.assert_array_equal(p.tok_ptr, o.tok_ptr)
            np.testing.assert_array_equal(p.tok_ent, o.tok_ent)
            np.testing.assert_array_equal(p.wbar, o.tok_w.astype(np.float32))
            assert p.max_cover == int(o.coverage.max())
        finally:
            p.close()


def test_plain_c_program_against_the_headers(tmp_path):
    """The headers are plain C: a C11 program compiles against include/, links
    libtileshare.so and uses the host-side calls (no GPU)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    so = B.lib()._name
    exe = str(tmp_path / "abi_host")
    r = subprocess.run([cc, "-std=c11", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                        os.path.join(ROOT, "tests", "c", "abi_host.c"), so, "-o", exe,
                        "-Wl,-rpath," + os.path.dirname(so)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, (r.stdout, r.stderr)
    fields = dict(kv.split("=", 1) for kv in r.stdout.split()[:10])
    o = OP.make_plan((1, 48, 48), (1, 16, 16), (1, 12, 12), registers=2)
    assert (int(fields["T"]), int(fields["U"]), int(fields["N"]), int(fields["R"]), int(fields["nnz"])) == \
        (o.T, o.U, o.N, 2, o.nnz)
    assert fields["device"] == "-1" and int(fields["ws"]) > 0 and fields["bad"] == "1"


@pytest.mark.parametrize("grid,win,stride", [((4, 44, 80), (4, 32, 32), (4, 24, 24)),
                                             ((8, 44, 80), (4, 32, 32), (2, 24, 24)),
                                             ((1, 48, 48), (1, 16, 16), (1, 12, 12)),
                                             ((1, 128, 128), (1, 32, 32), (1, 24, 24))])
def test_host_wbar_sums_to_one_within_one_ulp(grid, win, stride):
    """The planner's fp32 w-bar of each token, summed in fp32 in ascending tile order (the
    blend's order), is 1 within one ulp of 1.0 (2^-23)."""
    p = B.Plan(grid, win, stride, host_only=True)
    try:
        w = p.wbar.astype(np.float32)
        acc = np.zeros(p.U, dtype=np.float32)
        cnt = np.diff(p.tok_ptr)
        for k in range(int(cnt.max())):
            has = cnt > k
            acc[has] = (acc[has] + w[p.tok_ptr[:-1][has] + k]).astype(np.float32)
        assert np.max(np.abs(acc.astype(np.float64) - 1.0)) <= 2.0 ** -23
    finally:
        p.close()
