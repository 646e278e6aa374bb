"""Oracle: analytic FLOP count of a per-tile and a shared layer.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

[TileShare] Tab. 1 and Tab. S7 report block FLOPs of partly or fully shared
layers relative to per-tile layers; Tab. S6 notes that per-token work shrinks
with the token count while attention is unchanged.  Counted here: the four
linear layers (2 FLOPs per multiply-add) and the two attention contractions;
norms, softmax, GELU / SiLU gating and the blend are not counted.

Pinned by tests/test_oracle_flop_count.py: every linear layer and attention call
that the oracle's own layers and stacks make is intercepted and the FLOPs of its
operand shapes are summed; the closed forms below must equal those sums exactly.
"""


def linear_flops_per_row(d: int, f: int, gated: bool = False) -> int:
    """QKV, out-projection, MLP up (2f rows when gated: SwiGLU gate and up) and down."""
    return 2 * (3 * d * d + d * d + (3 if gated else 2) * d * f)


def attention_flops(T: int, N: int, d: int) -> int:
    return 4 * T * N * N * d


def tiled_layer_flops(T: int, N: int, d: int, f: int, gated: bool = False) -> int:
    return T * N * linear_flops_per_row(d, f, gated) + attention_flops(T, N, d)


def shared_layer_flops(U: int, T: int, N: int, d: int, f: int, gated: bool = False) -> int:
    return (U + T) * linear_flops_per_row(d, f, gated) + attention_flops(T, N, d)


def stack_flop_ratio(U: int, T: int, N: int, d: int, f: int, L: int, k: int, gated: bool = False) -> float:
    """FLOPs of TileShare-k over FLOPs of L per-tile layers."""
    tiled = tiled_layer_flops(T, N, d, f, gated)
    shared = shared_layer_flops(U, T, N, d, f, gated)
    return (k * tiled + (L - k) * shared) / (L * tiled)


def partial_layer_flops(U: int, T: int, N: int, d: int, f: int, shared, gated: bool = False) -> int:
    """A partially shared layer (Tab. 1 top, Tab. S7): the operations named in `shared`
    ("qkv", "out", "mlp") run on the U + T shared rows, the others on the T * N tile rows;
    attention is per tile either way."""
    shared = set(shared)
    if not shared <= {"qkv", "out", "mlp"}:
        raise ValueError(f"unknown shared operations {shared}")
    def rows(op):
        return U + T if op in shared else T * N
    return (2 * 3 * d * d * rows("qkv") + 2 * d * d * rows("out") + 2 * (3 if gated else 2) * d * f * rows("mlp")
            + attention_flops(T, N, d))
