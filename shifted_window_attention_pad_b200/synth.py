"""Seeded synthetic inputs, shared by the tests, the smoke check and the bench.

Holds no attention arithmetic: it only draws random numbers and rounds them to
the workload's storage type. Draw order per workload: q, k, v, the bias table,
dO, each from one numpy PCG64 stream seeded with the workload seed; q, k, v, dO
~ N(0, 1), bias table ~ N(0, 0.02^2), all drawn as fp32, then q, k, v, dO are
rounded to the storage type (bf16 round-to-nearest-even) while the table stays
fp32.
"""
import numpy as np
import torch


def _bf16_round(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(a).to(torch.bfloat16)


def make_inputs(wl, seed=None, shape_override=None):
    """Returns dict(q, k, v, dout: CPU tensors in the storage dtype [B,H,W,heads,hd];
    table: fp32 CPU tensor [(2w-1)^2, heads])."""
    rng = np.random.Generator(np.random.PCG64(wl.seed if seed is None else seed))
    shape = wl.grid_shape if shape_override is None else shape_override
    out = {}
    for name in ("q", "k", "v"):
        out[name] = rng.standard_normal(shape, dtype=np.float32)
    table = (rng.standard_normal((wl.n_bins, wl.heads), dtype=np.float32) * np.float32(0.02))
    out["dout"] = rng.standard_normal(shape, dtype=np.float32)
    res = {"table": torch.from_numpy(table)}
    for name in ("q", "k", "v", "dout"):
        res[name] = torch.from_numpy(out[name]) if wl.dtype == "f32" else _bf16_round(out[name])
    return res


def as_f64(t: torch.Tensor) -> np.ndarray:
    """Exact widening of a CPU/GPU tensor to a numpy fp64 array."""
    return t.detach().to("cpu").to(torch.float64).numpy()
