"""swin_wattn_bwd_noalloc: the backward for callers that cannot allocate device
memory (or hand over a workspace) when they run it -- its scratch is a static
array inside the library. It must give the results of swin_wattn_bwd, call
after call, since every call reuses the same scratch. This file sorts last so
that a run stopping at the first failure has already run every other test; it
passes alone in a fresh process as well."""
import ctypes

import pytest
import torch

from shifted_window_attention_pad_b200 import WORKLOADS, binding as sb
from shifted_window_attention_pad_b200.synth import make_inputs

from gpu_helpers import BF16_TOL, compare
from shifted_window_attention_pad_b200.synth import as_f64


def test_noalloc_rejects_what_does_not_fit_its_scratch():
    """Host-side checks only (no CUDA call): a description whose workspace
    exceeds the static scratch, or that the tcgen05 kernels do not take."""
    from shifted_window_attention_pad_b200 import build
    build.build()
    L = sb.lib()
    P = ctypes.c_void_p(1 << 20)
    big = sb.make_desc(1, 16, 16, 8, 4, 1000, 64, "bf16")      # 1000 heads of bias table
    assert sb.swin_wattn_workspace_size(big) > sb.SWIN_NOALLOC_SCRATCH_BYTES
    assert L.swin_wattn_bwd_noalloc(ctypes.byref(big), P, P, P, P, P, P, P, P, P, None) == -3
    generic = sb.desc_for(WORKLOADS["tiny-16x16-w4"])           # fp32: portable kernels
    assert L.swin_wattn_bwd_noalloc(ctypes.byref(generic), P, P, P, P, P, P, P, P, P, None) == -2


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["ragged-90x180-w8", "twelfth-degree-256x544-w8"])
def test_noalloc_backward_matches_workspace_backward_twice(name):
    from shifted_window_attention_pad_b200 import build
    build.build()
    wl = WORKLOADS[name]
    inp = make_inputs(wl)
    d = sb.desc_for(wl)
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "dout"))
    T = inp["table"].cuda()
    ref = sb.backward(d, q, k, v, T, do)                       # workspace entry point
    torch.cuda.synchronize()
    want = {n: as_f64(t) for n, t in zip(("dq", "dk", "dv", "dT"), ref)}
    for call in range(2):                                       # the scratch is reused
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        dT = torch.empty_like(T)
        sb.swin_wattn_bwd_noalloc(d, q, k, v, T, do, dq, dk, dv, dT)
        torch.cuda.synchronize()
        errs = compare({"dq": dq, "dk": dk, "dv": dv, "dT": dT}, want, wl.dtype)
        print(name, "call", call, errs)
        for n, e in errs.items():
            assert e <= BF16_TOL, (name, call, n, e)
