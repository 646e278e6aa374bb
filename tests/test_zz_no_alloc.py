"""ts_block_shared_noalloc: the shared layer for callers that cannot allocate.

Some callers of this library must not allocate device memory themselves, for
example a plugin inside a host application that owns every device buffer through
its own pool.  For them the library keeps the shared layer's scratch in one
static device array and ts_block_shared_noalloc uses it instead of a caller
workspace.  These tests call it through the C ABI and check its output against
ts_block_shared (with a caller workspace) on two calls in a row.  Both run the
same kernels on the same inputs, with no atomics and 256-byte aligned regions
either way, so the outputs must be identical bit for bit: a scratch region that
overlaps another, or stale contents of the previous call read back, would break
the equality long before it reached a tolerance.  A plan needing more scratch
than the array holds must be refused before anything runs.

The file is named so that pytest collects it last.
"""

import pytest
import torch

from shared_token_transformer_b200 import binding as B
from shared_token_transformer_b200 import workloads as W

from _gpu import Case, dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from shared_token_transformer_b200 import build
    build.build()


@pytest.mark.parametrize("cfg", [
    W.CONFIGS["stack48_bf16"],
    W.CONFIGS["vit14_fp32"],
    W.small_config("noalloc_fp8", grid=(1, 11, 13), win=(1, 8, 8), stride=(1, 5, 6), d=256, heads=4, mlp=512,
                   dtype="fp8", L=2, k=0),
], ids=lambda c: c.name)
def test_noalloc_matches_workspace_path_two_calls_in_a_row(cfg):
    c = Case(cfg, affine=True, L=2)
    S_ref = dev(c.S, c.dt)
    S_na = S_ref.clone()
    ws = c.workspace()
    for call in range(2):
        B.block_shared(c.plan, c.m, c.wlist[call], S_ref, ws)
        B.block_shared_noalloc(c.plan, c.m, c.wlist[call], S_na)
        torch.cuda.synchronize()
        assert torch.equal(S_na, S_ref), call
    B.device_status()
    c.plan.close()


def test_noalloc_refuses_plans_beyond_the_static_scratch():
    plan = B.Plan((1, 256, 256), (1, 32, 32), (1, 24, 24))          # 65,536 tokens, d = 1024
    m = B.model_desc(1024, 16, 4096, "bf16", (0, 32, 32))
    dummy = torch.zeros(1 << 16, dtype=torch.float32, device="cuda")
    w = B.layer_weights({n: dummy for n in ("ln1_g", "ln1_b", "w_qkv", "b_qkv", "q_g", "k_g", "w_o", "b_o",
                                            "ln2_g", "ln2_b", "w_1", "b_1", "w_2", "b_2")})
    S = torch.full((64, 1024), 1.5, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(B.TileShareError) as e:
        B.block_shared_noalloc(plan, m, w, S)
    assert e.value.status == 3
    assert "static" in str(e.value)
    torch.cuda.synchronize()
    assert torch.all(S == 1.5)
    plan.close()
