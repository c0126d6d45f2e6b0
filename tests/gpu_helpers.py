"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
and the fp64 oracle on the same seeded inputs, and the error measures of the
acceptance bar (fp32: max|gpu - ref| / max|ref| <= 1e-5; bf16: max|gpu - ref| /
RMS(ref) <= 2e-2, per tensor)."""
import numpy as np
import torch

import oracle
from shifted_window_attention_pad_b200 import binding as sb
from shifted_window_attention_pad_b200.synth import as_f64

F32_TOL = 1e-5
BF16_TOL = 2e-2


def oracle_shape(desc):
    return oracle.Shape(desc.B, desc.H, desc.W, desc.win_h, desc.win_w, desc.shift_h,
                        desc.shift_w, desc.heads, desc.head_dim)


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


def err_bf16(gpu, ref):
    g = as_f64(gpu) if isinstance(gpu, torch.Tensor) else gpu
    rms = float(np.sqrt(np.mean(ref * ref)))
    return float(np.max(np.abs(g - ref))) / max(rms, 1e-30)


def err_f32(gpu, ref):
    g = as_f64(gpu) if isinstance(gpu, torch.Tensor) else gpu
    return float(np.max(np.abs(g - ref))) / max(float(np.max(np.abs(ref))), 1e-30)


def compare(gpu, ref, dtype, names=("o", "lse", "dq", "dk", "dv", "dT")):
    """Returns {name: error}; lse and dT are fp32 on both paths and use the
    measure of the workload's dtype."""
    f = err_f32 if dtype == "f32" else err_bf16
    errs = {}
    for n in names:
        if n in gpu and gpu[n] is not None and n in ref and ref[n] is not None:
            errs[n] = f(gpu[n], ref[n])
    return errs
