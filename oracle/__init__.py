"""CPU oracle for the TileShare shared transformer layer.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The product path (``shared_token_transformer_b200``) never imports it
and shares no code, table or helper with it.

The oracle is a plain, slow, obviously correct restatement of what the method
computes, written from

    [TileShare] "TileShare: Training-Free Acceleration of Overlapping Tiled ViT
    Decoding" (arXiv 2610.32233): abstract, Fig. 2, Fig. 3b, Tab. 1, Tab. S1,
    Tab. S6.

in float64 (NumPy), in the order the pages describe the computation.  Where the
pages leave a step open, the reading taken is stated at the function that takes
it.

Modules
    plan    tiling of the token grid, tile<->token index maps, blend weights w-bar
    layers  per-tile layer, shared layer, merge, TileShare-k stack
    fp8     OCP FP8 E4M3 rounding and the per-channel / per-token scaled GEMM
    flops   analytic FLOP count of a tiled and a shared layer

Parity status: every function here is pinned by ``tests/test_oracle_*.py``
against closed forms, brute force, library routines and the exactness
statements of the pages; see the header of each module.
"""

from . import plan, layers, fp8, flops  # noqa: F401
