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


def oracle_stack(name, L, k, threads):
    """decode_stack of the oracle on the seeded inputs of configuration `name`."""
    from threadpoolctl import threadpool_limits

    from oracle import layers as OL
    from oracle import plan as OP
    from shared_token_transformer_b200 import workloads as W

    with threadpool_limits(limits=threads):
        cfg = W.CONFIGS[name]
        op = OP.make_plan(cfg.grid, cfg.win, cfg.stride, registers=cfg.R)
        dr = W.Draw(cfg, op.T, seed=SEED, affine=True)
        S0, G0 = dr.states()
        layers = dr.layers(L)
        m = OL.Model(cfg.d, cfg.heads, cfg.mlp, cfg.rope_dims, fp8=(cfg.dtype == "fp8"), block=cfg.block)
        return OL.decode_stack(S0, G0, layers, m, op, k)


def start(keys):
    """Submit the oracle runs of `keys` (those not yet submitted), in JOBS order."""
    global _pool, _threads
    keys = [k for k in JOBS if k in set(keys) and k not in _futures]
    if not keys:
        return
    if _pool is None:
        cores = os.cpu_count() or 1
        workers = max(1, min(len(JOBS), cores // 2))
        _threads = max(1, cores // workers)
        _pool = cf.ProcessPoolExecutor(max_workers=workers, mp_context=mp.get_context("spawn"))
    for key in keys:
        _futures[key] = _pool.submit(oracle_stack, *JOBS[key], _threads)


def result(key, timeout):
    """The oracle output [U, d] of `key`, waiting at most `timeout` seconds."""
    if key not in _futures:
        start([key])
    return _futures[key].result(timeout=timeout)


def shutdown():
    if _pool is not None:
        _pool.shutdown(wait=False, cancel_futures=True)
