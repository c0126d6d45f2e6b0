"""The synthetic workloads: shapes and dtypes only, no arithmetic.

Shapes follow the TERRA page ("TERRA: A Hierarchical Parallel Training and
Memory Orchestration Framework for High-Resolution AI-based Earth Modeling"):
the 1/12 degree GLORYS-based Wenhai workload of the Abstract, the padded
resolution of Table I, and the window / head sizes of Table V, scaled to one
GPU. The data themselves are not on the page and are replaced by seeded
synthetic fields (see ``synth.py``).
"""
from dataclasses import dataclass


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    W: int
    win: int
    shift: int
    heads: int
    head_dim: int
    dtype: str          # "f32" or "bf16"
    seed: int
    note: str = ""
    valid: tuple = None  # (valid_h, valid_w): tokens that carry field data; None = all

    @property
    def Hp(self):
        return -(-self.H // self.win) * self.win

    @property
    def Wp(self):
        return -(-self.W // self.win) * self.win

    @property
    def tokens(self):
        return self.B * self.H * self.W

    @property
    def n_windows(self):
        return self.B * (self.Hp // self.win) * (self.Wp // self.win)

    @property
    def n_bins(self):
        return (2 * self.win - 1) ** 2

    @property
    def grid_shape(self):
        return (self.B, self.H, self.W, self.heads, self.head_dim)

    def flops_fwd_bwd(self):
        """Dense window FLOPs, masked pairs included: 4*N*hd per padded token per
        head forward (QK^T, PV), 8*N*hd backward (dV, dP, dQ, dK); the backward's
        recompute of S is not counted."""
        N = self.win * self.win
        return 12 * N * self.head_dim * self.B * self.Hp * self.Wp * self.heads

    def elem_bytes(self):
        return 4 if self.dtype == "f32" else 2

    def alg_bytes_fwd(self):
        """q, k, v read and o written once each."""
        return 4 * self.tokens * self.heads * self.head_dim * self.elem_bytes()

    def alg_bytes_bwd(self):
        """q, k, v, dO read and dq, dk, dv written once each."""
        return 7 * self.tokens * self.heads * self.head_dim * self.elem_bytes()

    def flops_bwd(self):
        """Dense window FLOPs of the backward alone: 8*N*hd per padded token per
        head (dV, dP, dQ, dK; the recompute of S not counted)."""
        N = self.win * self.win
        return 8 * N * self.head_dim * self.B * self.Hp * self.Wp * self.heads


WORKLOADS = {
    w.name: w for w in (
        Workload("tiny-16x16-w4", 1, 16, 16, 4, 2, 2, 16, "f32", 0,
                 "16x16 grid, 4x4 windows, shift 2, 2 heads x 16, fp32"),
        Workload("ragged-90x180-w8", 1, 90, 180, 8, 4, 4, 32, "bf16", 1,
                 "90x180 grid padded to 96x184, 8x8 windows, shift 4, 4 heads x 32, pad masked"),
        Workload("twelfth-degree-256x544-w8", 1, 256, 544, 8, 4, 16, 64, "bf16", 2,
                 "1/12-degree field 2041x4320 padded to 2048x4352, patch 8 -> 256x544 tokens, "
                 "d=1024 = 16 heads x 64, 8x8 windows, shift 4"),
        Workload("downsampled-128x272-w16", 1, 128, 272, 16, 8, 32, 64, "bf16", 3,
                 "stride-2 stage: 128x272 tokens, d=2048 = 32 heads x 64, 16x16 windows, shift 8"),
        Workload("small-patch-2x512x1088-w8", 2, 512, 1088, 8, 4, 12, 64, "bf16", 4,
                 "patch 4 -> 512x1088 tokens, d=768 = 12 heads x 64, 8x8 windows, shift 4, "
                 "batch 2 (two rollout steps)"),
        Workload("profile-128x544-w8", 1, 128, 544, 8, 4, 16, 64, "bf16", 6,
                 "half of the 1/12-degree token grid (128 x 544 tokens, 16 heads x 64): the "
                 "same kernels on 0.57 GB of inputs, for profiler captures"),
        Workload("table5-256x544-8x128-w8", 1, 256, 544, 8, 4, 8, 128, "bf16", 5,
                 "the 1/12-degree token grid with the 128-channel heads of Table V: "
                 "d=1024 = 8 heads x 128, 8x8 windows, shift 4"),
        Workload("table5-large-256x544-8x128-w32", 1, 256, 544, 32, 16, 8, 128, "bf16", 7,
                 "the 1/12-degree token grid with the window of Table V's largest model: "
                 "32x32 windows (1024 tokens), shift 16, d=1024 = 8 heads x 128"),
    )
}

# The workload the throughput metric is quoted on: the 1/12-degree-shaped grid.
BENCH_WORKLOAD = "twelfth-degree-256x544-w8"
