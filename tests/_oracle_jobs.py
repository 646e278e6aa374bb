"""Full-size oracle stacks computed in worker processes (test infrastructure).

One float64 oracle stack at a benchmark geometry and width takes minutes of CPU
time, most of it in single-threaded NumPy element-wise passes.  The stack parity
tests therefore hand their oracle runs to a pool of worker processes when pytest
has finished collecting (tests/conftest.py), so that the oracle runs while the
other GPU tests use the device, and each test waits for its own result.

Workers are started with the "spawn" method: they never inherit a CUDA context.
Each worker limits its BLAS threads so that the pool shares the host's cores.
The inputs are the seeded draws of ``workloads`` (seed SEED, affine), the same
draws the GPU side of the test makes.

For e4m3 stacks a second run gives the oracle's own sensitivity to storage
precision ("floor" keys): the same stack with the attention outputs and the
residual state after each layer rounded to bf16, as the kernels store them.
Every e4m3 code is a rounding decision; a perturbation of one bf16 unit moves a
few per cent of the codes by one e4m3 step, and those flips feed the next
quantiser, so two runs that differ only in storage precision drift apart by
about as much as the e4m3 tolerance after two layers.
"""

import concurrent.futures as cf
import multiprocessing as mp
import os

SEED = 0

# test key -> (configuration, layers L, per-tile layers k); reduced depth at the
# full geometry and width of each benchmark workload
JOBS = {
    "image4k_bf16-L2-k1": ("image4k_bf16", 2, 1),
    "video44x80_fp8-L2-k0": ("video44x80_fp8", 2, 0),
    "video44x80_fp8-L2-k1": ("video44x80_fp8", 2, 1),
    "video44x80_fp8-L2-k2": ("video44x80_fp8", 2, 2),
    "video44x80_bf16-L2-k1": ("video44x80_bf16", 2, 1),
    "image2k_bf16-L3-k1": ("image2k_bf16", 3, 1),
}

_pool = None
_threads = 1
_futures = {}


FLOOR = "/floor"


def oracle_stack(name, L, k, threads, bf16_storage=False):
    """decode_stack of the oracle on the seeded inputs of configuration `name`;
    with bf16_storage, attention outputs and layer outputs rounded to bf16."""
    from threadpoolctl import threadpool_limits

    from oracle import layers as OL
    from oracle import plan as OP
    from shared_token_transformer_b200 import workloads as W

    attention, mlp_residual = OL.attention, OL.mlp_residual
    if bf16_storage:
        OL.attention = lambda q, k_, v: W.round_to(attention(q, k_, v), "bf16")
        OL.mlp_residual = lambda x, p, m: W.round_to(mlp_residual(x, p, m), "bf16")
    try:
        with threadpool_limits(limits=threads):
            cfg = W.CONFIGS[name]
            op = OP.make_plan(cfg.grid, cfg.win, cfg.stride, registers=cfg.R)
            dr = W.Draw(cfg, op.T, seed=SEED, affine=True)
            S0, G0 = dr.states()
            layers = dr.layers(L)
            m = OL.Model(cfg.d, cfg.heads, cfg.mlp, cfg.rope_dims, fp8=(cfg.dtype == "fp8"), block=cfg.block)
            return OL.decode_stack(S0, G0, layers, m, op, k)
    finally:
        OL.attention, OL.mlp_residual = attention, mlp_residual     # a worker runs several jobs


def needs_floor(key):
    return JOBS[key][0].endswith("_fp8")


def start(keys):
    """Submit the oracle runs of `keys` (those not yet submitted), in JOBS order,
    with the storage-precision runs of the e4m3 keys after them."""
    global _pool, _threads
    keys = [k for k in JOBS if k in set(keys) and k not in _futures]
    if not keys:
        return
    runs = keys + [k + FLOOR for k in keys if needs_floor(k)]
    if _pool is None:
        cores = os.cpu_count() or 1
        workers = max(1, min(len(runs), cores // 2))
        _threads = max(1, cores // workers)
        _pool = cf.ProcessPoolExecutor(max_workers=workers, mp_context=mp.get_context("spawn"))
    for key in runs:
        base = key[: -len(FLOOR)] if key.endswith(FLOOR) else key
        _futures[key] = _pool.submit(oracle_stack, *JOBS[base], _threads, key.endswith(FLOOR))


def result(key, timeout):
    """The oracle output [U, d] of `key` (or of `key + FLOOR`), waiting at most
    `timeout` seconds."""
    base = key[: -len(FLOOR)] if key.endswith(FLOOR) else key
    if base not in _futures:
        start([base])
    return _futures[key].result(timeout=timeout)


def shutdown():
    if _pool is not None:
        _pool.shutdown(wait=False, cancel_futures=True)
