#!/usr/bin/env python
"""Benchmark of the TileShare shared layer on B200: unique tokens/s per shared layer.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl tileshare|reference] [--config NAME]

A step is one TileShare-k decode of the configuration's seeded synthetic input
(default: the 4K image, 256x256 tokens, d=1024, L=16, k=4 bf16 stack; --k sets
another k): per-tile copies of the input, k per-tile layers, the merge of the
per-tile states, L-k shared layers and the copy of the output rows.  It runs through the library's public calls,
captured as CUDA graphs (one for the per-tile part, one for the shared part) so
that the shared layers are timed on their own by CUDA events on the launching
stream; L2 is flushed (512 MiB write) before every step, outside the events.

value  = unique tokens per second per shared layer = U * (L - k) * K * N_ranks /
         (max over ranks of the summed shared-part time of the K steps).
e2e    = the same metric through the public call with host buffers: per step one
         independent state, pinned host -> device, one ts_block_shared, device ->
         pinned host; uploads, calls and downloads of successive steps overlap on
         three streams, and the value is steps over the whole run (CUDA events).
roofline  per kernel class from a traced pass (library kernel trace: CUDA events
         around each launch, algorithmic FLOPs / HBM bytes per launch); the
         dominant class (most time) is reported against MEASURED_PEAKS.json: the
         burst bf16 figure when the traced pass lasts under a second, the
         sustained one otherwise (frac_vs_burst and frac_vs_sustained give
         both); fp32 kernels against the FP32 SIMT peak.
cpu_baseline  the float64 CPU oracle's shared layer on the same inputs (rank 0,
         N = 1): whole layers when one fits the budget, else a bounded sample
         (per-token steps on blocks of rows, attention of whole tiles, the whole
         blend) scaled to the layer.  --impl reference times that oracle alone as
         the reference arm, each step a bounded sample of the same kind.
         With --cpu-detail the reference arm times one shared and one per-tile
         oracle layer and the whole stack where it ends within 15 minutes.

Multi-GPU (torchrun): every rank decodes its own image (independent inputs, the
same weights); there is no data-path collective, only a barrier and a max of the
timings.  Scaling is weak.
"""

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "unique tokens/sec per shared layer on 1 B200; % of bf16 tensor/HBM roofline"
UNIT = "unique tokens/s per shared layer"
BIG = ("w_qkv", "w_o", "w_1", "w_2")
SCALE = {"w_qkv": "s_qkv", "w_o": "s_o", "w_1": "s_1", "w_2": "s_2"}
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="tileshare", choices=["tileshare", "reference"])
    ap.add_argument("--config", default="image4k_bf16")
    ap.add_argument("--k", type=int, default=None, help="per-tile layers before the merge (default: the workload's)")
    ap.add_argument("--no-graph", action="store_true", help="launch the calls eagerly instead of CUDA graphs")
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="budget of the CPU oracle baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-detail", action="store_true",
                    help="with --impl reference: the oracle's shared and per-tile layer and whole stack")
    ap.add_argument("--trace-steps", type=int, default=20)
    ap.add_argument("--shared-ops", default=None,
                    help="partial sharing from layer k on: comma list of qkv,out,mlp ('none': nothing shared) run "
                         "once per token on per-tile residual streams; default: the TileShare shared layer")
    ap.add_argument("--blend", default="ramp", choices=["ramp", "hard"],
                    help="blend rule of the plan: normalised linear ramp (default) or hard stitching")
    ap.add_argument("--block", default=None, choices=["ln_gelu", "rms_swiglu"],
                    help="block flavour: the configuration's (pre-LN + GELU) or RMSNorm + SwiGLU (gate and up "
                         "of the configuration's MLP width each)")
    return ap.parse_args()


def config_of(args):
    import dataclasses
    from shared_token_transformer_b200 import workloads as W
    cfg = W.CONFIGS[args.config]
    if args.block is not None and args.block != cfg.block:
        cfg = dataclasses.replace(cfg, block=args.block)
    k = getattr(args, "k", None)
    if k is not None:
        if not 0 <= k <= cfg.L:
            raise SystemExit(f"--k must lie in [0, {cfg.L}]")
        cfg = dataclasses.replace(cfg, k=k)
    return cfg


def workload_config(cfg, args, U, T, N, world):
    """The `config` object of the JSON line (the same for both arms)."""
    return {"workload": f"{cfg.name}: {cfg.note}", "grid": list(cfg.grid), "window": list(cfg.win),
            "stride": list(cfg.stride), "blend": args.blend, "block": cfg.block,
            "shared_ops": args.shared_ops or "TileShare shared layer",
            "L": cfg.L, "k": cfg.k, "unique_tokens": U, "tiles": T, "rows_per_tile": N,
            "l2": "flushed before every step (512 MiB write, outside the timed events)",
            "launch": "eager public calls" if args.no_graph else "CUDA graphs of the public calls",
            "parallelism": f"replicas x{world} (one image per GPU)"}


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------
def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def flops_layer(rows, T, N, d, f, gated=False):
    # QKV + out-projection, MLP up (gate and up rows when gated) and down, attention
    return rows * 2.0 * (4 * d * d + (3 if gated else 2) * d * f) + 4.0 * T * N * N * d


def flops_partial(U, T, N, d, f, qkv, out, mlp, gated=False):
    """A partially shared layer: each shared operation on U + T rows, the others on T * N rows."""
    def rows(shared):
        return U + T if shared else T * N
    return (2.0 * 3 * d * d * rows(qkv) + 2.0 * d * d * rows(out) + (6.0 if gated else 4.0) * d * f * rows(mlp)
            + 4.0 * T * N * N * d)


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples of one GPU while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.samples = []
        self.proc = None
        self.gpu_id = gpu_id
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu_id), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 9:
                self.samples.append((time.time(), parts))

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0, t1):
        inside = [p for t, p in self.samples if t0 - 0.15 <= t <= t1 + 0.15]
        if len(inside) < 3:
            inside = [p for t, p in self.samples if t0 - 1.0 <= t <= t1 + 1.0]
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        mhz, mx = [], []
        for p in inside:
            try:
                mhz.append(float(p[1]))
                mx.append(float(p[2]))
            except ValueError:
                pass
            for n, v in zip(names, p[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(inside)}


# ---------------------------------------------------------------------------
# CPU oracle (the cpu_baseline leg and the reference arm)
# ---------------------------------------------------------------------------
def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:
        pass
    return os.cpu_count()


def _oracle_inputs(cfg, rule):
    from oracle import layers as OL
    from oracle import plan as OP
    from shared_token_transformer_b200 import workloads as W
    op = OP.make_plan(cfg.grid, cfg.win, cfg.stride, rule=rule)
    dr = W.Draw(cfg, op.T, seed=0)
    S0, G0 = dr.states()
    S = np.concatenate([S0, G0])
    layer = dr.layer()
    om = OL.Model(cfg.d, cfg.heads, cfg.mlp, cfg.rope_dims, fp8=(cfg.dtype == "fp8"), block=cfg.block)
    return op, S, layer, om


def oracle_layer_sample_seconds(op, S, layer, om, budget_s, row_block=1024):
    """Seconds of one float64 oracle shared layer, estimated from a bounded sample.

    The layer's work is per-token steps (Norm1, QKV, QK-RMSNorm, out-projection,
    MLP) on its U + T rows, attention of each of its T tiles, and the blend.  Row
    blocks and whole tiles are timed in turn until each kind has used half the
    budget or all of its work; the blend over all tokens is timed once.  Each
    kind's time is scaled by (all its units / units timed).  With a budget large
    enough for the whole layer this is the whole layer, timed piece by piece.
    Returns (seconds, description)."""
    from oracle import layers as OL
    M, T = S.shape[0], op.T
    t_tok = t_att = 0.0
    rows = tiles = 0
    half = budget_s / 2
    while rows < M and (rows == 0 or t_tok < half):
        x = S[rows: rows + row_block]
        t0 = time.perf_counter()
        OL.qkv_project(x, layer, om)
        y = x + OL.linear(x, layer["w_o"], layer["b_o"], om)      # out-projection of a block of rows
        OL.mlp_residual(y, layer, om)
        t_tok += time.perf_counter() - t0
        rows += x.shape[0]
    while tiles < T and (tiles == 0 or t_att < half):
        r = OL.tile_rows(op, tiles)
        q, k, v = OL.qkv_project(S[r], layer, om)                  # untimed: counted with the rows
        t0 = time.perf_counter()
        OL.tile_attention(q, k, v, op.slot_pos, om)
        t_att += time.perf_counter() - t0
        tiles += 1
    O = np.zeros((T, op.N, S.shape[1]))
    t0 = time.perf_counter()
    OL.merge(O, op)
    t_blend = time.perf_counter() - t0
    sec = t_tok * M / rows + t_att * T / tiles + t_blend
    what = (f"per-token steps on {rows} of {M} rows, attention of {tiles} of {T} tiles, the whole blend; "
            f"each scaled by its share of the layer")
    return sec, what


def oracle_tiled_layer_sample_seconds(op, X, layer, om, budget_s, row_block=1024):
    """Seconds of one float64 oracle per-tile layer on X [T, N, d], estimated from a
    bounded sample: per-token steps (Norm1, QKV, QK-RMSNorm, out-projection, MLP) on
    blocks of the T*N tile rows and attention of whole tiles, each timed in turn until
    it has used half the budget or all of its work and scaled by (all its units /
    units timed).  Returns (seconds, description)."""
    from oracle import layers as OL
    T, N = X.shape[0], X.shape[1]
    R = X.reshape(T * N, X.shape[2])
    t_tok = t_att = 0.0
    rows = tiles = 0
    half = budget_s / 2
    while rows < R.shape[0] and (rows == 0 or t_tok < half):
        x = R[rows: rows + row_block]
        t0 = time.perf_counter()
        OL.qkv_project(x, layer, om)
        y = x + OL.linear(x, layer["w_o"], layer["b_o"], om)
        OL.mlp_residual(y, layer, om)
        t_tok += time.perf_counter() - t0
        rows += x.shape[0]
    while tiles < T and (tiles == 0 or t_att < half):
        q, k, v = OL.qkv_project(X[tiles], layer, om)               # untimed: counted with the rows
        t0 = time.perf_counter()
        OL.tile_attention(q, k, v, op.slot_pos, om)
        t_att += time.perf_counter() - t0
        tiles += 1
    sec = t_tok * (T * N) / rows + t_att * T / tiles
    return sec, (f"per-token steps on {rows} of {T * N} tile rows, attention of {tiles} of {T} tiles; "
                 f"each scaled by its share of the layer")


def run_cpu_detail(args, cfg, budget_s=300.0, stack_limit_s=900.0):
    """The reference arm's detailed form (--impl reference --cpu-detail): oracle timings
    of the workload on the host cores, one shared layer and one per-tile layer, whole
    when the estimate fits budget_s, else a bounded sample, and the whole TileShare-k
    stack when its estimate is under stack_limit_s."""
    from oracle import layers as OL
    from shared_token_transformer_b200 import workloads as W
    op, S, layer, om = _oracle_inputs(cfg, args.blend)
    res = {"impl": "reference", "kind": "oracle-detail", "config": cfg.name, "L": cfg.L, "k": cfg.k, "unique_tokens": op.U,
           "tiles": op.T, "rows_per_tile": op.N, "dtype": "f64", "cores": os.cpu_count(),
           "blas_threads": blas_threads(),
           "note": "the oracle computes in float64 by definition; it has no float32 form to time"}
    est, _ = oracle_layer_sample_seconds(op, S, layer, om, min(budget_s, 4.0))
    if est <= budget_s:
        t0 = time.perf_counter()
        OL.block_shared(S, layer, om, op)
        sh, how = time.perf_counter() - t0, "one whole layer"
    else:
        sh, how = oracle_layer_sample_seconds(op, S, layer, om, budget_s)
        how = "bounded sample: " + how
    res.update(shared_layer_s=round(sh, 3), shared_layer_unique_tok_s=round(op.U / sh, 2), shared_layer_how=how)
    X = OL.gather(S, op)
    est, _ = oracle_tiled_layer_sample_seconds(op, X, layer, om, min(budget_s, 4.0))
    if est <= budget_s:
        t0 = time.perf_counter()
        OL.block_tiled(X, layer, om, op)
        ti, how = time.perf_counter() - t0, "one whole layer"
    else:
        ti, how = oracle_tiled_layer_sample_seconds(op, X, layer, om, budget_s)
        how = "bounded sample: " + how
    res.update(tiled_layer_s=round(ti, 3), tiled_layer_how=how)
    est_stack = cfg.k * ti + (cfg.L - cfg.k) * sh
    res["stack_estimate_s"] = round(est_stack, 1)
    if est_stack <= stack_limit_s:
        dr = W.Draw(cfg, op.T, seed=0)
        S0, G0 = dr.states()
        layers = dr.layers()
        t0 = time.perf_counter()
        OL.decode_stack(S0, G0, layers, om, op, cfg.k)
        res["stack_s"] = round(time.perf_counter() - t0, 3)
    else:
        res["stack_s"] = None
        res["stack_note"] = f"not run: estimated {est_stack:.0f} s, above {stack_limit_s:.0f} s"
    return res


def oracle_shared_layer_timing(cfg, budget_s, max_steps, warmup=1, rule="ramp"):
    """Unique tokens/s of the float64 oracle's shared layer on the configuration's
    seeded input: whole layers (block_shared) when one fits the budget, else one
    bounded sample (oracle_layer_sample_seconds).  Returns (rate, steps, sample)."""
    from oracle import layers as OL
    op, S, layer, om = _oracle_inputs(cfg, rule)
    est, what = oracle_layer_sample_seconds(op, S, layer, om, min(budget_s, 4.0))
    if est * (max(1, warmup) + 1) > budget_s:
        sec, what = oracle_layer_sample_seconds(op, S, layer, om, budget_s)
        return op.U / sec, 1, f"one float64 oracle shared layer of {cfg.name}, timed on a bounded sample: {what}"
    for _ in range(warmup):
        OL.block_shared(S, layer, om, op)
    times = []
    t_all = time.perf_counter()
    while len(times) < max(1, max_steps):
        t0 = time.perf_counter()
        OL.block_shared(S, layer, om, op)
        times.append(time.perf_counter() - t0)
        if time.perf_counter() - t_all > budget_s:
            break
    mean = float(np.mean(times))
    return op.U / mean, len(times), f"{len(times)} whole float64 oracle shared layers of {cfg.name} (~{budget_s:.0f} s budget)"


# ---------------------------------------------------------------------------
# tileshare arm
# ---------------------------------------------------------------------------
def run_tileshare(args, rank, world, local):
    import torch
    import torch.distributed as dist

    from shared_token_transformer_b200 import binding as B
    from shared_token_transformer_b200 import build as Bd
    from shared_token_transformer_b200 import workloads as W

    Bd.build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    cfg = config_of(args)
    L, k = cfg.L, cfg.k
    dt = {"f32": torch.float32, "bf16": torch.bfloat16, "fp8": torch.bfloat16}[cfg.dtype]
    num_sms = torch.cuda.get_device_properties(dev).multi_processor_count
    plan = B.Plan(cfg.grid, cfg.win, cfg.stride,
                  rule=B.TS_BLEND_HARD_STITCH if args.blend == "hard" else B.TS_BLEND_LINEAR_RAMP)
    U, T, N, d, f = plan.U, plan.T, plan.N, cfg.d, cfg.mlp
    m = B.model_desc(d, cfg.heads, f, cfg.dtype, cfg.rope_dims, block=cfg.block)

    # seeded inputs: weights from seed 0 (same on every rank); each rank its own image
    dr = W.Draw(cfg, T, seed=0)
    S0, G0 = dr.states()
    if rank > 0:
        S0, G0 = W.Draw(cfg, T, seed=rank).states()

    def todev(a, dtype):
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev, dtype)

    dlayers = []
    for _ in range(L):
        p = dr.layer()
        t = {}
        for key, v in p.items():
            if key in BIG:
                x = todev(v, dt)
                if cfg.dtype == "fp8":
                    q = torch.empty(x.shape, dtype=torch.uint8, device=dev)
                    s = torch.empty(x.shape[0], dtype=torch.float32, device=dev)
                    B.quantize_rows_e4m3(x, q, s)
                    t[key], t[SCALE[key]] = q, s
                else:
                    t[key] = x
            else:
                t[key] = todev(v, torch.float32)
        dlayers.append(t)
    wl = [B.layer_weights(t) for t in dlayers]
    S0d, G0d = todev(S0, dt), todev(G0, dt)
    X = torch.empty((T * N, d), dtype=dt, device=dev)
    S = torch.empty((U + T, d), dtype=dt, device=dev)
    out = torch.empty((U, d), dtype=dt, device=dev)
    ws = torch.empty(B.workspace_size(plan, m, 0, 0), dtype=torch.uint8, device=dev)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)

    share = None
    if args.shared_ops is not None:
        names = [x for x in args.shared_ops.split(",") if x and x != "none"]
        bits = {"qkv": B.TS_SHARE_QKV, "out": B.TS_SHARE_OUT, "mlp": B.TS_SHARE_MLP}
        share = 0
        for x in names:
            share |= bits[x]

    def part_tiled(kk=k):
        if share is not None:
            # partial sharing keeps per-tile states throughout; merged once at the end
            B.gather_tiles(plan, m, S0d, G0d, X)
            for li in range(kk):
                B.block_tiled(plan, m, wl[li], X, ws)
            return
        if kk > 0:
            B.gather_tiles(plan, m, S0d, G0d, X)
            for li in range(kk):
                B.block_tiled(plan, m, wl[li], X, ws)
            if kk < L:
                B.op_merge(plan, m, X, U + T, S)
            else:
                B.op_merge(plan, m, X, U, out)
        else:
            S[:U].copy_(S0d)
            S[U:].copy_(G0d)

    def part_shared():
        for li in range(k, L):
            if share is not None:
                B.block_partial(plan, m, wl[li], share, X, ws)
            else:
                B.block_shared(plan, m, wl[li], S, ws)

    def part_out():
        if share is not None:
            B.op_merge(plan, m, X, U, out)
        elif k < L:
            out.copy_(S[:U])

    # warm-up (eager: configures every kernel), then capture
    for _ in range(max(1, args.warmup)):
        part_tiled()
        part_shared()
        part_out()
    torch.cuda.synchronize()
    use_graph = not args.no_graph
    launches_per_step = None
    if use_graph:
        n0 = B.launch_count()
        g1, g2, g3 = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            with torch.cuda.graph(g1, stream=side):
                part_tiled()
            if k < L:                      # with k = L there is no shared layer to capture
                with torch.cuda.graph(g2, stream=side):
                    part_shared()
            with torch.cuda.graph(g3, stream=side):
                part_out()
        torch.cuda.current_stream().wait_stream(side)
        launches_per_step = B.launch_count() - n0
        run1, run2, run3 = g1.replay, (g2.replay if k < L else (lambda: None)), g3.replay
        for _ in range(max(3, args.warmup)):
            run1(); run2(); run3()
    else:
        run1, run2, run3 = part_tiled, part_shared, part_out
    torch.cuda.synchronize()

    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
    gpu_id = local
    try:
        props = torch.cuda.get_device_properties(dev)
        if getattr(props, "uuid", None) is not None:
            gpu_id = "GPU-" + str(props.uuid)
    except Exception:
        pass
    sampler = ClockSampler(gpu_id)
    sampler.start()
    time.sleep(0.6)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    n_before = B.launch_count()
    t_wall0 = time.time()
    for i in range(K):
        flush.zero_()
        e = evs[i]
        e[0].record()
        run1()
        e[1].record()
        run2()
        e[2].record()
        run3()
        e[3].record()
    torch.cuda.synchronize()
    t_wall1 = time.time()
    if world > 1:
        dist.barrier()
    eager_launches = B.launch_count() - n_before
    t_step = np.array([e[0].elapsed_time(e[3]) for e in evs])
    t_tiled = np.array([e[0].elapsed_time(e[1]) for e in evs])
    t_shared = np.array([e[1].elapsed_time(e[2]) for e in evs])
    shared_total_ms, step_ms, tiled_ms = max_over_ranks([t_shared.sum(), t_step.mean(), t_tiled.mean()], world)
    value = replica_rate(U * (L - k) * K, world, shared_total_ms)
    gpu_launches = launches_per_step * K if use_graph else eager_launches

    # own batched per-tile path on the same input: k = L (all layers per tile, blended at the end)
    Kt = min(K, 100)
    if use_graph:
        gt = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            part_tiled(L)
            with torch.cuda.graph(gt, stream=side):
                part_tiled(L)
        torch.cuda.current_stream().wait_stream(side)
        run_t = gt.replay
    else:
        def run_t():
            part_tiled(L)
    run_t()
    torch.cuda.synchronize()
    tev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(Kt)]
    for i in range(Kt):
        flush.zero_()
        tev[i][0].record()
        run_t()
        tev[i][1].record()
    torch.cuda.synchronize()
    tiled_stack_ms = float(np.mean([a.elapsed_time(b) for a, b in tev]))

    # e2e: one shared layer per step through the public call with pinned host buffers.
    # Steps are independent images: step i's upload, step i-1's layer and step i-2's
    # download overlap on three streams (three device slots, one pinned result
    # buffer per slot); every step still copies its whole state in and its result
    # out.  The value is steps over the whole pipelined run.
    Ke = max(20, min(K, 200))
    if share is not None:
        # partial sharing: the per-tile state [T * N, d] goes in and out
        B.gather_tiles(plan, m, S0d, G0d, X)
        S_host = X.cpu().pin_memory()
    else:
        S_host = torch.cat([S0d, G0d]).cpu().pin_memory()
    NSLOT = 3
    Sd = [torch.empty(tuple(S_host.shape), dtype=dt, device=dev) for _ in range(NSLOT)]
    S_back = [torch.empty_like(S_host).pin_memory() for _ in range(NSLOT)]
    s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()

    def e2e_call(buf):
        if share is not None:
            B.block_partial(plan, m, wl[min(k, L - 1)], share, buf, ws)
        else:
            B.block_shared(plan, m, wl[min(k, L - 1)], buf, ws)

    run_c = [(lambda b=b: e2e_call(Sd[b])) for b in range(NSLOT)]
    if use_graph:
        # one graph per slot for the call, as a caller would replay it
        graphs = []
        for b in range(NSLOT):
            g = torch.cuda.CUDAGraph()
            side.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(side):
                e2e_call(Sd[b])
                with torch.cuda.graph(g, stream=side):
                    e2e_call(Sd[b])
            torch.cuda.current_stream().wait_stream(side)
            graphs.append(g)
        run_c = [g.replay for g in graphs]
    torch.cuda.synchronize()

    def pipeline(n, e_out):
        e_in = [torch.cuda.Event() for _ in range(n)]
        e_cmp = [torch.cuda.Event() for _ in range(n)]
        for i in range(n):
            b = i % NSLOT
            if i >= NSLOT:
                s_in.wait_event(e_out[i - NSLOT])      # the slot's previous result has left
            with torch.cuda.stream(s_in):
                Sd[b].copy_(S_host, non_blocking=True)
            e_in[i].record(s_in)
            s_cmp.wait_event(e_in[i])
            with torch.cuda.stream(s_cmp):
                run_c[b]()
            e_cmp[i].record(s_cmp)
            s_out.wait_event(e_cmp[i])
            with torch.cuda.stream(s_out):
                S_back[b].copy_(Sd[b], non_blocking=True)
            e_out[i].record(s_out)

    pipeline(NSLOT, [torch.cuda.Event() for _ in range(NSLOT)])     # warm-up
    torch.cuda.synchronize()
    main = torch.cuda.current_stream()
    t_e0, t_e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_e0.record(main)
    for st_ in (s_in, s_cmp, s_out):
        st_.wait_stream(main)
    e_done = [torch.cuda.Event(enable_timing=True) for _ in range(Ke)]
    pipeline(Ke, e_done)
    main.wait_stream(s_out)
    t_e1.record(main)
    torch.cuda.synchronize()
    e2e_total = t_e0.elapsed_time(t_e1)
    (e2e_max,) = max_over_ranks([e2e_total], world)
    e2e_value = replica_rate(U * Ke, world, e2e_max)
    gaps = np.array([e_done[i - 1].elapsed_time(e_done[i]) for i in range(1, Ke)])
    e2e_spread = {"steps": int(Ke), "ms_total": round(e2e_total, 4), "ms_per_step": round(e2e_total / Ke, 4),
                  "step_interval_ms_median": round(float(np.median(gaps)), 4),
                  "step_interval_ms_p10": round(float(np.percentile(gaps, 10)), 4),
                  "step_interval_ms_p90": round(float(np.percentile(gaps, 90)), 4)}
    state_bytes = S_host.numel() * S_host.element_size()

    # traced pass: per-kernel times of the same step, eagerly launched
    torch.cuda.synchronize()
    t_tr0 = time.perf_counter()
    B.trace_begin(100000)
    for _ in range(args.trace_steps):
        flush.zero_()
        part_tiled()
        part_shared()
        part_out()
    tr = B.trace_end()
    trace_s = time.perf_counter() - t_tr0
    sampler.stop()
    clocks = sampler.summary(t_wall0, t_wall1)

    pk, pk_src = peaks()
    # a traced pass under a second runs at burst clocks; a longer one settles
    # under the power cap, where the sustained figure applies
    burst = trace_s < 1.0 or "bf16_tflops_sustained" not in pk
    bf16_key = "bf16_tflops" if burst else "bf16_tflops_sustained"
    bf16_peak = pk[bf16_key]
    # fp32 path: SIMT FMA lanes x 2 FLOPs x clock (148 SMs x 128 FP32 lanes)
    f32_peak = num_sms * 128 * 2 * float(pk.get("sm_max_mhz", 1965.0)) * 1e6 / 1e12

    def tensor_peak_of(name):
        # e4m3 GEMMs against the bf16 peak x the nominal e4m3 : bf16 dense ratio;
        # attention computes in bf16 in every configuration
        if cfg.dtype == "f32":
            return f32_peak
        return 2.0 * bf16_peak if cfg.dtype == "fp8" and not name.startswith("attention") else bf16_peak

    def peak_source(name, unit):
        if unit != "TFLOP/s":
            return f"{pk_src} hbm_gbs"
        if cfg.dtype == "f32":
            return f"fp32 SIMT: {num_sms} SMs x 128 lanes x 2 FLOP x {pk.get('sm_max_mhz', 1965.0):.0f} MHz"
        src = f"{pk_src} {bf16_key} (traced pass {trace_s:.2f} s)"
        return src + (" x2 (e4m3:bf16 nominal)" if tensor_peak_of(name) > bf16_peak else "")
    total_ms = sum(v["ms"] for v in tr.values()) or 1.0
    kernels = {}
    for name, v in tr.items():
        if v["timed"] == 0:
            continue
        per = v["ms"] / v["timed"]
        tensor = v["flops"] > 0 and name.startswith(("gemm", "attention", "linear"))
        if tensor:
            ach = v["flops"] / (v["ms"] / 1e3) / 1e12
            frac = ach / tensor_peak_of(name)
            unit = "TFLOP/s"
        else:
            ach = v["bytes"] / (v["ms"] / 1e3) / 1e9
            frac = ach / pk["hbm_gbs"]
            unit = "GB/s"
        kernels[name] = {"launches": v["launches"], "ms_per_launch": round(per, 5),
                         "share": round(v["ms"] / total_ms, 4), "achieved": round(ach, 2), "unit": unit,
                         "frac": round(frac, 4),
                         "flops_per_launch": v["flops"] / v["timed"], "bytes_per_launch": v["bytes"] / v["timed"]}
    dom = max(kernels, key=lambda n: kernels[n]["share"])
    kd = kernels[dom]
    traffic = None
    tpath = os.path.join(ROOT, "profiles", "traffic.json")
    if os.path.exists(tpath):
        with open(tpath) as fh:
            tj = json.load(fh)
        ent = tj.get(args.config, {}).get(dom)
        if ent and ent.get("kernel_source_sha") == kernel_source_sha(kernel_class(dom)):
            traffic = ent.get("traffic_bytes_per_launch")
    bound = ("alu" if cfg.dtype == "f32" else "tensor") if kd["unit"] == "TFLOP/s" else "hbm"
    roofline = {"bound": bound, "kernel": dom, "achieved": kd["achieved"],
                "peak": round(tensor_peak_of(dom) if kd["unit"] == "TFLOP/s" else pk["hbm_gbs"], 1), "unit": kd["unit"],
                "frac": kd["frac"], "traffic": traffic, "peak_source": peak_source(dom, kd["unit"])}
    if kd["unit"] == "TFLOP/s" and cfg.dtype != "f32" and "bf16_tflops_sustained" in pk:
        # both measured bf16 figures, since a traced pass near one second could take either
        scale = tensor_peak_of(dom) / bf16_peak
        roofline["frac_vs_burst"] = round(kd["achieved"] / (scale * pk["bf16_tflops"]), 4)
        roofline["frac_vs_sustained"] = round(kd["achieved"] / (scale * pk["bf16_tflops_sustained"]), 4)

    gated = cfg.block == "rms_swiglu"
    ft = flops_layer(T * N, T, N, d, f, gated)
    fs = flops_layer(U + T, T, N, d, f, gated)
    if share is not None:
        fs = flops_partial(U, T, N, d, f, share & B.TS_SHARE_QKV, share & B.TS_SHARE_OUT, share & B.TS_SHARE_MLP,
                           gated)
    flop_ratio = (k * ft + (L - k) * fs) / (L * ft)
    res = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(step_ms, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": {"bf16": "bf16", "f32": "f32", "fp8": "e4m3"}[cfg.dtype],
        "data": "synthetic (seeded N(0,1) states, N(0,0.02) weights, random init)",
        "config": workload_config(cfg, args, U, T, N, world),
        "shared_layer_ms": round(shared_total_ms / K / max(1, L - k), 5),
        "per_tile_part_ms": round(tiled_ms, 5),
        "tiled_stack_ms": round(tiled_stack_ms, 5),
        "speedup_vs_tiled": round(tiled_stack_ms / step_ms, 4),
        "flop_ratio": round(flop_ratio, 4),
        "speedup_bar": round(0.85 / flop_ratio, 4),
        "e2e": {"value": round(e2e_value, 1), "unit": UNIT, "h2d_bytes_per_step": state_bytes,
                "d2h_bytes_per_step": state_bytes, "spread": e2e_spread,
                "call": ("ts_block_partial" if share is not None else "ts_block_shared") +
                        " on one independent state per step, each copied in from pinned host memory and back; uploads, "
                        "calls and downloads of successive steps overlap on three streams" +
                        (" (the call replayed as a CUDA graph)" if use_graph else "")},
        "gpu_launches": int(gpu_launches),
        **({"note": "k = L: every layer per tile, no shared layer (value 0 by definition)"} if L == k else {}),
        "roofline": roofline,
        "kernels": kernels,
        "clocks": clocks,
    }
    return res, cfg


def max_over_ranks(vals, world):
    """Element-wise maximum over the ranks of a list of floats (the slowest rank's
    times; identity with one rank).  The tensor lives where the process group's
    backend wants it: on the rank's GPU for NCCL, on the host for gloo."""
    if world <= 1:
        return [float(v) for v in vals]
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(v) for v in vals], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.cpu()]


def replica_rate(units_per_rank, world, ms):
    """Whole-job rate of `world` replicas, each processing `units_per_rank` units,
    over the slowest rank's `ms` milliseconds."""
    return units_per_rank * world / (ms / 1e3) if ms > 0 else 0.0


# source files behind each kernel class: its own header, plus the shared device
# helpers and the host code that sets its launches up
_CLASS_SOURCES = {"attention": "attention.cuh", "gemm": "gemm_tc.cuh", "rows": "rowops.cuh"}


def kernel_source_sha(kind=None):
    """Hash of the sources a kernel class is built from (all of csrc/ when kind is None)."""
    import hashlib
    h = hashlib.sha256()
    d = os.path.join(ROOT, "shared_token_transformer_b200", "csrc")
    files = sorted(os.listdir(d))
    if kind is not None:
        files = sorted({"common.cuh", "plan.inl", "tileshare.cu", _CLASS_SOURCES[kind]})
    for fn in files:
        with open(os.path.join(d, fn), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def kernel_class(name):
    """Kernel class of a traced kernel name."""
    if name.startswith("attention"):
        return "attention"
    if name.startswith(("gemm", "linear")):
        return "gemm"
    return "rows"


def run_reference(args, cfg, world):
    """The reference arm: the float64 CPU oracle's shared layer on this arm's
    workload, W untimed and K timed steps, each a whole layer when one fits the
    per-step budget, else a bounded sample of it, so that the run ends within a
    few minutes."""
    from oracle import layers as OL
    op, S, layer, om = _oracle_inputs(cfg, args.blend)
    K, Wm = max(1, args.steps), max(0, args.warmup)
    per = max(1.0, 90.0 / (K + Wm))
    est, what = oracle_layer_sample_seconds(op, S, layer, om, min(per, 4.0))
    whole = est <= per
    times = []
    for i in range(Wm + K):
        if whole:
            t0 = time.perf_counter()
            OL.block_shared(S, layer, om, op)
            sec = time.perf_counter() - t0
        else:
            sec, what = oracle_layer_sample_seconds(op, S, layer, om, per)
        if i >= Wm:
            times.append(sec)
    mean = float(np.mean(times))
    v = op.U / mean
    sample = (f"each step one whole float64 oracle shared layer of {cfg.name}" if whole else
              f"each step one float64 oracle shared layer of {cfg.name} timed on a bounded sample "
              f"(~{per:.0f} s): {what}")
    return {"impl": "reference", "metric": METRIC, "value": round(v, 2), "unit": UNIT, "n_gpus": world,
            "steps": K, "warmup": Wm, "ms_per_step": round(mean * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded, same draws as the tileshare arm)",
            "config": workload_config(cfg, args, op.U, op.T, op.N, world),
            "cpu_baseline": {"value": round(v, 2), "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(v, 2), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    from shared_token_transformer_b200 import workloads as W
    cfg = config_of(args)

    if args.cpu_detail and args.impl != "reference":
        raise SystemExit("--cpu-detail is a form of the reference arm: add --impl reference")
    if args.impl == "reference":
        if rank != 0:
            return
        print(json.dumps(run_cpu_detail(args, cfg) if args.cpu_detail else run_reference(args, cfg, world)))
        return

    import torch.distributed as dist
    if world > 1:
        import datetime
        import torch
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    res, cfg = run_tileshare(args, rank, world, local)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, n, what = oracle_shared_layer_timing(cfg, args.cpu_seconds, 1000, rule=args.blend)
        if args.shared_ops is not None:
            what += "; the oracle's fully shared layer (partial sharing is not timed on the CPU)"
        res["cpu_baseline"] = {"value": round(rate, 2), "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                               "sample": what}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res))


if __name__ == "__main__":
    main()
