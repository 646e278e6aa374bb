"""TileShare-k stacks at the full geometry and width of the benchmark workloads,
against the whole oracle stack.

ts_decode_stack runs k per-tile layers, the transition merge of the per-tile
states ([TileShare] Fig. 3b) and the remaining shared layers ([TileShare]
abstract, TileShare-k) at the 2K and 4K image sizes and the video size in bf16
and e4m3 (k = 0, 1, 2), with reduced depth so that the float64 oracle finishes
within the test run (it runs in worker processes while the other GPU tests
use the device, see _oracle_jobs).  The whole output is compared with the
oracle's decode_stack on the same seeded inputs (relative L2 1e-2 for bf16,
3e-2 for e4m3), and the worst row of every coverage class within 1.5 times that.
"""

import numpy as np
import pytest
import torch

import _oracle_jobs as J
from shared_token_transformer_b200 import binding as B
from shared_token_transformer_b200 import workloads as W

from _gpu import Case, assert_rows, dev, host, rel_l2

pytestmark = pytest.mark.gpu

TOL = {"bf16": 1e-2, "fp8": 3e-2}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from shared_token_transformer_b200 import build
    build.build()
    yield
    B.device_status()


@pytest.mark.parametrize("job", list(J.JOBS))
def test_decode_stack_full_geometry(job):
    name, L, k = J.JOBS[job]
    cfg = W.CONFIGS[name]
    c = Case(cfg, seed=J.SEED, affine=True, L=L)
    op = c.oplan
    out = torch.empty((op.U, cfg.d), dtype=c.dt, device="cuda")
    ws = c.workspace(L, k)
    B.decode_stack(c.plan, c.m, c.wlist, k, dev(c.S0, c.dt), dev(c.G0, c.dt), out, ws)
    got = host(out)
    del ws, out
    torch.cuda.empty_cache()
    want = J.result(job, timeout=900)
    assert want.shape == got.shape
    tol = TOL[cfg.dtype]
    assert rel_l2(got, want) < tol
    assert_rows(got, want, op, "tokens", tol)
    c.plan.close()
