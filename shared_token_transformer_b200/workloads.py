"""Synthetic workloads: configuration shapes and seeded input draws.

This module holds no arithmetic of the method (no tiling, no weights of the blend,
no layer math).  It only names the shapes of the benchmark configurations and
draws their inputs, so that the CUDA path, the CPU oracle and the benchmark all
see the same numbers.  Inputs stand in for the decoders' latents and trained
weights, which are not available: states and global tokens ~ N(0, 1), weight
matrices ~ N(0, 0.02), biases 0, norm gains 1, drawn in float64 from
``numpy.random.Generator(PCG64(seed))`` in a fixed order (S0, G0, then per layer
w_qkv, w_o, w_1, w_2) and rounded to the working dtype.  ``affine=True`` adds
nonzero biases and gains (drawn after the matrices of each layer) so that a
dropped bias or gain cannot hide behind zeros and ones.
"""

from dataclasses import dataclass, field

import numpy as np

# ---------------------------------------------------------------------------
# configurations (token grid F x H x W, window, stride, model, stack)
# ---------------------------------------------------------------------------


@dataclass(frozen=True)
class Config:
    name: str
    grid: tuple
    win: tuple
    stride: tuple
    d: int
    heads: int
    mlp: int
    dtype: str            # "f32", "bf16" or "fp8" (e4m3 GEMMs, bf16 activations)
    L: int
    k: int
    rope_dims: tuple      # channels of the head dimension given to the (f, y, x) axes
    note: str = ""
    ks: tuple = field(default=())   # further k values the configuration compares
    R: int = 1                      # register tokens per tile (one global token in the benchmarks)
    block: str = "ln_gelu"          # "ln_gelu" or "rms_swiglu" (MLP up of 2 x mlp rows: gate, then up)

    @property
    def hd(self):
        return self.d // self.heads

    @property
    def U(self):
        return self.grid[0] * self.grid[1] * self.grid[2]


CONFIGS = {
    # single shared ViT block in fp32, 14x14 tokens, 8x8 windows at stride 6 (2x2 tiles)
    "vit14_fp32": Config("vit14_fp32", (1, 14, 14), (1, 8, 8), (1, 6, 6), 64, 4, 256, "f32",
                         L=1, k=0, rope_dims=(0, 8, 8),
                         note="14x14 grid, d=64, 4 heads, MLP 256, window 8 stride 6, fp32"),
    # zero-overlap variant of the same block: stride = window on a 16x16 grid
    "vit16_nooverlap_fp32": Config("vit16_nooverlap_fp32", (1, 16, 16), (1, 8, 8), (1, 8, 8), 64, 4, 256,
                                   "f32", L=1, k=0, rope_dims=(0, 8, 8),
                                   note="16x16 grid, window 8 stride 8 (no overlap), fp32"),
    # stack of 8 layers, 2 per tile, bf16, 48x48 tokens, 16x16 windows at stride 12 (4x4 tiles)
    "stack48_bf16": Config("stack48_bf16", (1, 48, 48), (1, 16, 16), (1, 12, 12), 512, 8, 2048, "bf16",
                           L=8, k=2, rope_dims=(0, 32, 32),
                           note="48x48 grid, d=512, 8 heads, MLP 2048, window 16 stride 12, L=8 k=2, bf16"),
    # video-decoder-scale layer: 4 latent frames of 44x80 tokens, window 4x32x32, spatial stride 24
    "video44x80_bf16": Config("video44x80_bf16", (4, 44, 80), (4, 32, 32), (4, 24, 24), 1536, 24, 6144,
                              "bf16", L=24, k=6, rope_dims=(16, 24, 24),
                              note="4x44x80 grid, d=1536, 24 heads, MLP 6144, window 4x32x32 stride 24, "
                                   "L=24 k=6, bf16"),
    "video44x80_fp8": Config("video44x80_fp8", (4, 44, 80), (4, 32, 32), (4, 24, 24), 1536, 24, 6144,
                             "fp8", L=24, k=6, rope_dims=(16, 24, 24), ks=(0, 4, 6, 24),
                             note="as video44x80_bf16 with e4m3 GEMMs; k in 0, 4, 6, 24"),
    # spatio-temporal tiling: 8 latent frames, windows of 4 frames at temporal stride 2, so tiles
    # overlap in time as well as in space (a token lies in up to 8 tiles)
    "video88x80_st_bf16": Config("video88x80_st_bf16", (8, 44, 80), (4, 32, 32), (2, 24, 24), 1536, 24, 6144,
                                 "bf16", L=24, k=6, rope_dims=(16, 24, 24),
                                 note="8x44x80 grid, d=1536, 24 heads, MLP 6144, window 4x32x32 stride 2x24x24 "
                                      "(temporal overlap), L=24 k=6, bf16"),
    # image-autoencoder-scale decode at 4K (256x256 tokens) and 2K (128x128 tokens)
    "image4k_bf16": Config("image4k_bf16", (1, 256, 256), (1, 32, 32), (1, 24, 24), 1024, 16, 4096, "bf16",
                           L=16, k=4, rope_dims=(0, 32, 32),
                           note="256x256 grid, d=1024, 16 heads, MLP 4096, window 32 stride 24, L=16 k=4"),
    "image2k_bf16": Config("image2k_bf16", (1, 128, 128), (1, 32, 32), (1, 24, 24), 1024, 16, 4096, "bf16",
                           L=16, k=4, rope_dims=(0, 32, 32),
                           note="128x128 grid, d=1024, 16 heads, MLP 4096, window 32 stride 24, L=16 k=4"),
}


def small_config(name="tiny", grid=(1, 11, 13), win=(1, 8, 8), stride=(1, 5, 6), d=128, heads=2, mlp=256,
                 dtype="bf16", L=3, k=1, rope_dims=None, block="ln_gelu"):
    """A reduced configuration for fast parity tests (ragged tiles, several GEMM tiles)."""
    hd = d // heads
    if rope_dims is None:
        rope_dims = (0, hd // 2, hd // 2) if grid[0] == 1 else (hd // 4, 3 * hd // 8, 3 * hd // 8)
    return Config(name, tuple(grid), tuple(win), tuple(stride), d, heads, mlp, dtype, L, k, tuple(rope_dims),
                  block=block)


# ---------------------------------------------------------------------------
# rounding to the working dtype (input preparation only)
# ---------------------------------------------------------------------------

def round_to(a: np.ndarray, dtype: str) -> np.ndarray:
    """Round float64 values to the storage dtype and return them as float64."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))
    if dtype == "f32":
        return t.to(torch.float32).to(torch.float64).numpy()
    if dtype in ("bf16", "fp8"):
        return t.to(torch.bfloat16).to(torch.float64).numpy()
    raise ValueError(dtype)


# ---------------------------------------------------------------------------
# seeded draws
# ---------------------------------------------------------------------------

class Draw:
    """Sequential seeded draws of one configuration (fixed order, see module doc)."""

    def __init__(self, cfg: Config, T: int, seed: int = 0, affine: bool = False):
        self.cfg = cfg
        self.T = T
        self.affine = affine
        self.rng = np.random.Generator(np.random.PCG64(seed))

    def states(self):
        """(S0 [U, d], G0 [T*R, d]) rounded to the working dtype, as float64."""
        c = self.cfg
        S0 = self.rng.standard_normal((c.U, c.d))
        G0 = self.rng.standard_normal((self.T * c.R, c.d))
        return round_to(S0, c.dtype), round_to(G0, c.dtype)

    def layer(self):
        """One layer's parameters (dict of float64 arrays rounded to the working dtype)."""
        c = self.cfg
        d, f, hd = c.d, c.mlp, c.hd
        f1 = 2 * f if c.block == "rms_swiglu" else f     # rows of w_1
        r = self.rng
        p = {
            "w_qkv": 0.02 * r.standard_normal((3 * d, d)),
            "w_o": 0.02 * r.standard_normal((d, d)),
            "w_1": 0.02 * r.standard_normal((f1, d)),
            "w_2": 0.02 * r.standard_normal((d, f)),
        }
        if self.affine:
            p.update({
                "b_qkv": 0.1 * r.standard_normal(3 * d), "b_o": 0.1 * r.standard_normal(d),
                "b_1": 0.1 * r.standard_normal(f1), "b_2": 0.1 * r.standard_normal(d),
                "ln1_g": 1 + 0.2 * r.standard_normal(d), "ln1_b": 0.1 * r.standard_normal(d),
                "ln2_g": 1 + 0.2 * r.standard_normal(d), "ln2_b": 0.1 * r.standard_normal(d),
                "q_g": 1 + 0.2 * r.standard_normal(hd), "k_g": 1 + 0.2 * r.standard_normal(hd),
            })
        else:
            p.update({
                "b_qkv": np.zeros(3 * d), "b_o": np.zeros(d), "b_1": np.zeros(f1), "b_2": np.zeros(d),
                "ln1_g": np.ones(d), "ln1_b": np.zeros(d), "ln2_g": np.ones(d), "ln2_b": np.zeros(d),
                "q_g": np.ones(hd), "k_g": np.ones(hd),
            })
        big = ("w_qkv", "w_o", "w_1", "w_2")
        # matrices in the working dtype; the small vectors are kept in float32
        return {k: round_to(v, c.dtype) if k in big else round_to(v, "f32") for k, v in p.items()}

    def layers(self, L=None):
        return [self.layer() for _ in range(self.cfg.L if L is None else L)]
