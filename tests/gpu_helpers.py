"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
and the fp64 oracle on the same seeded inputs, and the error measures of the
acceptance bar, per tensor:
  fp32 outputs: max|gpu - ref| / max|ref| <= 1e-5;
  bf16 outputs: max over elements of (|gpu - ref| - half a bf16 ulp of ref),
  divided by RMS(ref), <= 2e-2. The half ulp is the output type's own
  rounding: storing the exact fp64 result in bf16 already moves the largest
  values by up to 0.04 RMS on these workloads, so only error beyond the
  storage rounding is charged to the computation."""
import numpy as np
import torch

import oracle
from shifted_window_attention_pad_b200 import binding as sb
from shifted_window_attention_pad_b200.synth import as_f64

F32_TOL = 1e-5
BF16_TOL = 2e-2


def oracle_shape(desc):
    return oracle.Shape(desc.B, desc.H, desc.W, desc.win_h, desc.win_w, desc.shift_h,
                        desc.shift_w, desc.heads, desc.head_dim, desc.valid_h, desc.valid_w)


def run_gpu(desc, inp, want_lse=True, backward=True):
    dev = "cuda"
    q, k, v, do = (inp[n].to(dev) for n in ("q", "k", "v", "dout"))
    T = inp["table"].to(dev)
    ws = sb.new_workspace(desc)
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:-1], dtype=torch.float32, device=dev) if want_lse else None
    sb.swin_wattn_fwd(desc, q, k, v, T, out, lse, ws)
    res = {"o": out, "lse": lse}
    if backward:
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        dT = torch.empty_like(T)
        sb.swin_wattn_bwd(desc, q, k, v, T, do, dq, dk, dv, dT, ws)
        res.update(dq=dq, dk=dk, dv=dv, dT=dT)
    torch.cuda.synchronize()
    assert sb.swin_wattn_poll_status(ws) == 0
    return res


def run_oracle(desc, inp, backward=True):
    s = oracle_shape(desc)
    q, k, v, do, T = (as_f64(inp[n]) for n in ("q", "k", "v", "dout", "table"))
    o, lse = oracle.forward(s, q, k, v, T)
    res = {"o": o, "lse": lse}
    if backward:
        dq, dk, dv, dT = oracle.backward(s, q, k, v, T, do)
        res.update(dq=dq, dk=dk, dv=dv, dT=dT)
    return res


def half_ulp_bf16(x):
    """Half the spacing of bf16 numbers at |x| (8 significant bits)."""
    a = np.abs(x)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, np.ldexp(1.0, (e - 8).astype(np.int64)), 0.0)


def err_bf16(gpu, ref, storage_rounding=True):
    """max(|gpu - ref| - half ulp_bf16(ref)) / RMS(ref) (storage rounding not
    charged); storage_rounding=False gives the raw max|gpu - ref| / RMS(ref)."""
    g = as_f64(gpu) if isinstance(gpu, torch.Tensor) else gpu
    rms = float(np.sqrt(np.mean(ref * ref)))
    d = np.abs(g - ref)
    if storage_rounding:
        d = np.maximum(d - half_ulp_bf16(ref), 0.0)
    return float(np.max(d)) / max(rms, 1e-30)


def err_rms(gpu, ref):
    g = as_f64(gpu) if isinstance(gpu, torch.Tensor) else gpu
    return float(np.sqrt(np.mean((g - ref) ** 2)) / max(np.sqrt(np.mean(ref * ref)), 1e-30))


def err_f32(gpu, ref):
    g = as_f64(gpu) if isinstance(gpu, torch.Tensor) else gpu
    return float(np.max(np.abs(g - ref))) / max(float(np.max(np.abs(ref))), 1e-30)


FP32_OUTPUTS = ("lse", "dT")


# Every comparison of a run, for the table the test session prints at its end
# (the margin of each output against its bar, per case).
RECORDED = []


def compare(gpu, ref, dtype, names=("o", "lse", "dq", "dk", "dv", "dT"), label=None):
    """Returns {name: error} against the workload's bar. lse and dT are stored
    in fp32 on every path, so no storage rounding is discounted for them."""
    errs = _compare(gpu, ref, dtype, names)
    if label is None:
        import os
        label = os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0].split("::")[-1]
    RECORDED.append((label, dtype, errs))
    return errs


def _compare(gpu, ref, dtype, names):
    errs = {}
    for n in names:
        if n in gpu and gpu[n] is not None and n in ref and ref[n] is not None:
            if dtype == "f32":
                errs[n] = err_f32(gpu[n], ref[n])
            else:
                errs[n] = err_bf16(gpu[n], ref[n], storage_rounding=n not in FP32_OUTPUTS)
    return errs
