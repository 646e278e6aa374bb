"""Host-side helpers of bench.py (CPU only): workload selection, FLOP counts, kernel classes
and the source keys of the DRAM-traffic table."""

import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from oracle import flops as Fo  # noqa: E402
from oracle import plan as OP  # noqa: E402


class _Args:
    def __init__(self, config, block=None):
        self.config, self.block = config, block


def test_config_of_block_flavour():
    assert bench.config_of(_Args("stack48_bf16")).block == "ln_gelu"
    c = bench.config_of(_Args("stack48_bf16", "rms_swiglu"))
    assert c.block == "rms_swiglu" and c.d == 512 and c.mlp == 2048


@pytest.mark.parametrize("gated", [False, True])
def test_bench_flops_match_the_oracle_count(gated):
    # the bench's per-layer FLOPs equal the oracle's analytic count for both layer kinds
    p = OP.make_plan((1, 48, 48), (1, 16, 16), (1, 12, 12))
    d, f = 512, 2048
    assert bench.flops_layer(p.T * p.N, p.T, p.N, d, f, gated) == Fo.tiled_layer_flops(p.T, p.N, d, f, gated)
    assert bench.flops_layer(p.U + p.T, p.T, p.N, d, f, gated) == Fo.shared_layer_flops(p.U, p.T, p.N, d, f, gated)


def test_kernel_classes():
    assert bench.kernel_class("attention") == "attention"
    assert bench.kernel_class("gemm_up") == "gemm" and bench.kernel_class("linear") == "gemm"
    assert bench.kernel_class("blend") == "rows" and bench.kernel_class("layernorm") == "rows"


def test_traffic_table_records():
    """Every record of profiles/traffic.json names a traced kernel class, carries positive bytes
    and a source hash of the form kernel_source_sha writes (the bench reports a record only
    while that hash matches the current sources of the class)."""
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as fh:
        tj = json.load(fh)
    shas = {k: bench.kernel_source_sha(k) for k in ("attention", "gemm", "rows")}
    assert len(set(shas.values())) == 3 and all(len(v) == 16 for v in shas.values())
    for cfg, kinds in tj.items():
        if cfg.startswith("_"):
            continue
        for kind, rec in kinds.items():
            assert bench.kernel_class(kind) in shas
            assert rec["traffic_bytes_per_launch"] > 0
            assert len(rec["kernel_source_sha"]) == 16 and int(rec["kernel_source_sha"], 16) >= 0


@pytest.mark.parametrize("ops", [(), ("qkv",), ("out",), ("mlp",), ("qkv", "mlp"), ("qkv", "out", "mlp")])
def test_bench_partial_flops_match_the_oracle_count(ops):
    p = OP.make_plan((4, 44, 80), (4, 32, 32), (4, 24, 24))
    d, f = 1536, 6144
    got = bench.flops_partial(p.U, p.T, p.N, d, f, "qkv" in ops, "out" in ops, "mlp" in ops)
    assert got == Fo.partial_layer_flops(p.U, p.T, p.N, d, f, ops)


def test_config_of_k_override():
    a = _Args("video44x80_fp8")
    a.k = 0
    assert bench.config_of(a).k == 0 and bench.config_of(a).L == 24
    a.k = 25
    with pytest.raises(SystemExit):
        bench.config_of(a)


def test_oracle_sample_covers_the_whole_layer_when_the_budget_allows():
    # with room for everything the sample is the whole layer, piece by piece: every
    # row block and every tile timed once, and no scaling
    cfg = bench.config_of(_Args("vit14_fp32"))
    op, S, layer, om = bench._oracle_inputs(cfg, "ramp")
    sec, what = bench.oracle_layer_sample_seconds(op, S, layer, om, budget_s=1e9, row_block=64)
    assert sec > 0
    assert f"{S.shape[0]} of {S.shape[0]} rows" in what and f"{op.T} of {op.T} tiles" in what
    # a tiny budget still times one row block and one tile
    sec, what = bench.oracle_layer_sample_seconds(op, S, layer, om, budget_s=1e-9, row_block=64)
    assert f"64 of {S.shape[0]} rows" in what and f"1 of {op.T} tiles" in what


def test_oracle_tiled_sample_covers_the_whole_layer_when_the_budget_allows():
    cfg = bench.config_of(_Args("vit14_fp32"))
    op, S, layer, om = bench._oracle_inputs(cfg, "ramp")
    from oracle import layers as OL
    X = OL.gather(S, op)
    sec, what = bench.oracle_tiled_layer_sample_seconds(op, X, layer, om, budget_s=1e9, row_block=64)
    assert sec > 0
    assert f"{op.T * op.N} of {op.T * op.N} tile rows" in what and f"{op.T} of {op.T} tiles" in what
    sec, what = bench.oracle_tiled_layer_sample_seconds(op, X, layer, om, budget_s=1e-9, row_block=64)
    assert f"64 of {op.T * op.N} tile rows" in what and f"1 of {op.T} tiles" in what


def test_cpu_detail_times_both_layers_and_the_stack():
    a = _Args("vit14_fp32")
    a.blend = "ramp"
    cfg = bench.config_of(a)
    res = bench.run_cpu_detail(a, cfg, budget_s=60.0, stack_limit_s=60.0)
    assert res["dtype"] == "f64" and res["cores"] >= 1
    assert res["shared_layer_s"] > 0 and res["tiled_layer_s"] > 0 and res["stack_s"] > 0
    assert res["shared_layer_how"] == "one whole layer" and res["tiled_layer_how"] == "one whole layer"
    res = bench.run_cpu_detail(a, cfg, budget_s=1e-9, stack_limit_s=0.0)
    assert res["shared_layer_how"].startswith("bounded sample") and res["tiled_layer_how"].startswith("bounded sample")
    assert res["stack_s"] is None and "not run" in res["stack_note"]
