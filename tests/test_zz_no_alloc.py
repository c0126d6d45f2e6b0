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


def _documented_need(heads, bins):
    """Workspace of the tcgen05 kernels as the header states it: a 256-byte
    header, the bias table [heads][bins_pad] fp32 and the bias-gradient sums
    [heads][bins_pad][10] int64, each region rounded up to 256 bytes."""
    bp = (bins + 3) // 4 * 4
    a256 = lambda x: (x + 255) // 256 * 256
    return 256 + a256(heads * bp * 4) + a256(heads * bp * 80)


def test_noalloc_scratch_limit_is_the_documented_layout():
    """The largest head count that fits the static scratch with 8 x 8 windows,
    from the documented layout, fits; one more head is rejected."""
    from shifted_window_attention_pad_b200 import build
    build.build()
    L = sb.lib()
    h = 1
    while _documented_need(h + 1, 225) <= sb.SWIN_NOALLOC_SCRATCH_BYTES:
        h += 1
    for heads, fits in ((h, True), (h + 1, False)):
        d = sb.make_desc(1, 16, 16, 8, 4, heads, 64, "bf16")
        assert sb.swin_wattn_workspace_size(d) == _documented_need(heads, 225)
        assert (sb.swin_wattn_workspace_size(d) <= sb.SWIN_NOALLOC_SCRATCH_BYTES) == fits
    P = ctypes.c_void_p(1 << 20)
    over = sb.make_desc(1, 16, 16, 8, 4, h + 1, 64, "bf16")
    assert L.swin_wattn_bwd_noalloc(ctypes.byref(over), P, P, P, P, P, P, P, P, P, None) == -3


def test_noalloc_checks_pointers_before_queueing_work():
    """A null or misaligned data pointer is rejected on the host (nothing is
    queued on the stream, so no CUDA call is needed to see it)."""
    from shifted_window_attention_pad_b200 import build
    build.build()
    L = sb.lib()
    d = sb.desc_for(WORKLOADS["ragged-90x180-w8"])
    P, bad = ctypes.c_void_p(1 << 20), ctypes.c_void_p((1 << 20) + 8)
    assert L.swin_wattn_bwd_noalloc(ctypes.byref(d), P, P, P, P, P, P, P, P, None, None) == -1
    assert L.swin_wattn_bwd_noalloc(ctypes.byref(d), P, bad, P, P, P, P, P, P, P, None) == -1


def test_noalloc_rejects_what_does_not_fit_its_scratch():
    """Host-side checks only (no CUDA call): a description whose workspace
    exceeds the static scratch, or that the tcgen05 kernels do not take."""
    from shifted_window_attention_pad_b200 import build
    build.build()
    L = sb.lib()
    P = ctypes.c_void_p(1 << 20)
    big = sb.make_desc(1, 16, 16, 8, 4, 1000, 64, "bf16")      # 1000 heads of bias-gradient sums
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
    want = dict(zip(("dq", "dk", "dv", "dT"), ref))
    for call in range(2):                                       # the scratch is reused
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        dT = torch.empty_like(T)
        sb.swin_wattn_bwd_noalloc(d, q, k, v, T, do, dq, dk, dv, dT)
        torch.cuda.synchronize()
        got = {"dq": dq, "dk": dk, "dv": dv, "dT": dT}
        errs = compare(got, {n: as_f64(t) for n, t in want.items()}, wl.dtype)
        print(name, "call", call, errs)
        for n, e in errs.items():
            assert e <= BF16_TOL, (name, call, n, e)
        # same kernels, fixed-order integer dT sums: identical bits
        for n in want:
            assert torch.equal(got[n], want[n]), (name, call, n)
